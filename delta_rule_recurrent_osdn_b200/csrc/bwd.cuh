// bwd.cuh -- the backward pass of the OSDN forward pass (gradients of a loss L with respect to
// q, k, v, beta, r, eta, S_0 and d_0, given dL/do, dL/dS_T and dL/dd_T), in fp32 FMA arithmetic.
//
// The forward pass ("OSDN: Improving Delta Rule with Provable Online Preconditioning in Linear
// Attention", technical summary, sections 2.1-2.3), per (sequence, head), a_t = k_t (.) k_t,
// n_t = ||k_t||^2, s_t = <d_t, a_t>:
//   phase 1:  k~_t = d_t (.) k_t,   d_{t+1} = r_t d_t + eta x_t a_t,   x_t = beta_t (1 - beta_t s_t) / n_t
//   phase 2:  u_t = v_t - S_{t-1} k_t,   S_t = S_{t-1} + beta_t u_t k~_t^T,   o_t = scale S_t q_t
// (x_t = 0 when n_t = 0).  The pages give no backward; this one is the chain rule applied to
// those steps in reverse order:
//   dS_t  = dS_{t+1} - beta_{t+1} g_{t+1} k_{t+1}^T + scale do_t q_t^T,   g_t = dS_t k~_t
//   dv_t  = beta_t g_t,   dbeta_t = <u_t, g_t> + ...,   dk~_t = beta_t dS_t^T u_t,
//   dq_t  = scale S_t^T do_t,   dk_t = -beta_t S_{t-1}^T g_t + dk~_t (.) d_t + 2 k_t (.) da_t,
//   dd_t  = r_t dd_{t+1} - eta beta_t^2 / n_t <a_t, dd_{t+1}> a_t + dk~_t (.) k_t,
//   dr_t  = <dd_{t+1}, d_t>,   deta = sum_t x_t <a_t, dd_{t+1}>,
//   da_t  = eta x_t dd_{t+1} - eta <a_t, dd_{t+1}> (beta_t^2 d_t + x_t) / n_t,
//   dbeta_t += eta <a_t, dd_{t+1}> (1 - 2 beta_t s_t) / n_t.
//
// Kernels (one call of osdn_bwd):
//   1. phase 1 forward (the forward pass's own kernels), which also writes d_t of every token;
//   2. bwd_delta_kernel: one CTA per (sequence, head, 64 value rows).  Rows of S and of dS are
//      independent, so each CTA carries its rows through the chunk-level algebra (32-token chunks,
//      the state S_c at each chunk start, A = K K~^T, T = (I + strict_tril(diag(beta) A))^-1,
//      E = V - K S_c^T, R = diag(beta) E, W = T R, P = tril(Q K~^T), S' = S_c + W^T K~): a forward
//      sweep keeps S_c of every chunk in a workspace; then, chunks in reverse, with dS' the adjoint
//      at the chunk's end,
//        dW = K~ dS'^T + scale P^T dO,  dP = tril(scale dO W^T),  dR = T^T dW,
//        dL = -strict_tril(T^T (dW R^T) T^T),  dv = diag(beta) dR,
//        dq = scale dO S_c + dP K~,  dk~ = W dS' + dP^T Q + (diag(beta) dL)^T K,
//        dk = diag(beta) dL K~ - diag(beta) dR S_c,  dbeta = rowsum(dL . A) + rowsum(dR . E),
//        dS = dS' + scale dO^T Q - (diag(beta) dR)^T K.
//      dv and dS are per row; dq, dk, dk~ and dbeta's phase-2 term sum over all value rows (dP and
//      dL are linear in such sums), so each CTA writes its share;
//   3. bwd_reduce_kernel: the shares added up, elementwise over the batch (dq final);
//      bwd_precond_kernel: one CTA per (sequence, head) runs the phase-1 adjoint recurrence in
//      reverse (one warp; 32-token chunks double-buffered in shared memory by asynchronous copies);
//   4. bwd_sum_kernel: deta, summed over (sequence, head) in a fixed order.
#pragma once

#include "common.cuh"

namespace osdn {

constexpr int BWD_BV = 64;      // value rows per bwd_delta_kernel CTA
constexpr int BWD_C = 32;       // tokens per chunk (state checkpoints, chunk algebra)
constexpr int BWD_THREADS = 256;
// Per chunk and value tile, the forward sweep keeps A = K K~^T, T, E = V - K S_c^T and W for the
// reverse sweep: C x C + C x C + C x BV + C x BV floats.
constexpr int BWD_FW = 2 * BWD_C * BWD_C + 2 * BWD_C * BWD_BV;

template <int DK>
struct BwdSmem {
    static constexpr int KS = DK + 4;          // row strides (floats), multiples of 4, = 4 mod 32
    static constexpr int VS = BWD_BV + 4;
    static constexpr int CS = BWD_C + 4;
    static constexpr int S = 0;                                // [BV][KS] state rows S_c
    static constexpr int DS = S + BWD_BV * KS;                 // [BV][KS] adjoint rows
    static constexpr int K = DS + BWD_BV * KS;                 // [C][KS] keys of the chunk
    static constexpr int KT = K + BWD_C * KS;                  // [C][KS] k~ = d (.) k
    static constexpr int Q = KT + BWD_C * KS;                  // [C][KS] queries
    static constexpr int O = Q + BWD_C * KS;                   // [C][KS] a gradient share, staged
    static constexpr int V = O + BWD_C * KS;                   // [C][VS] v, then E = v - S_c k
    static constexpr int G = V + BWD_C * VS;                   // [C][VS] dL/do
    static constexpr int R = G + BWD_C * VS;                   // [C][VS] R = beta E
    static constexpr int W = R + BWD_C * VS;                   // [C][VS] W = T R
    static constexpr int DW = W + BWD_C * VS;                  // [C][VS] dW
    static constexpr int DR = DW + BWD_C * VS;                 // [C][VS] dR = T^T dW
    static constexpr int DRB = DR + BWD_C * VS;                // [C][VS] beta dR (= dv)
    static constexpr int A = DRB + BWD_C * VS;                 // [C][CS] K K~^T
    static constexpr int P = A + BWD_C * CS;           // [C][CS] tril(Q K~^T)
    static constexpr int TT = P + BWD_C * CS;          // [C][CS] T = (I + L)^-1
    static constexpr int DP = TT + BWD_C * CS;         // [C][CS] dP
    static constexpr int M = DP + BWD_C * CS;          // [C][CS] dW R^T, then dL
    static constexpr int X = M + BWD_C * CS;           // [C][CS] T^T M
    static constexpr int DLB = X + BWD_C * CS;         // [C][CS] beta dL
    static constexpr int BETA = DLB + BWD_C * CS;      // [C]
    static constexpr int floats = BETA + BWD_C;
    static constexpr size_t bytes = sizeof(float) * floats;
};

// Checkpoint slot of chunk ch (0-based, BWD_C tokens) of sequence n starting at row `first`:
// floor(first / C) + ch + n.  Distinct over all (sequence, chunk) pairs of a batch, and below
// ceil(rows / C) + N + 1 (the workspace holds that many).
__device__ __forceinline__ int64_t bwd_slot(int64_t first, int ch, int n) {
    return first / BWD_C + ch + n;
}

// Shared-memory matrix products of the chunk algebra, all 256 threads:
//   C[m][n] (= or +=) alpha * rs[m] * sum_k A(m, k) B(k, n)   (rs optional; tri 1 keeps n <= m,
//   tri 2 keeps n < m), with A(m, k) = A[m lda + k] (NN, NT) or A[k lda + m] (TN) and
//   B(k, n) = B[k ldb + n] (NN, TN) or B[n ldb + k] (NT).  A thread owns TM rows x TN columns of C;
//   NT walks k four at a time with 16-byte loads of both operands.  The columns of a thread are
//   spread over the row (NT: n = tn + j N / TN; NN, TN: groups of four at 4 tn + j N / TN) so the
//   lanes of a warp read consecutive 16-byte pieces.
enum { GEMM_NN = 0, GEMM_TN = 1, GEMM_NT = 2 };

template <int MODE, int TM, int TN>
__device__ __forceinline__ void bwd_gemm(int Mr, int Nc, int Kd, const float* __restrict__ A, int lda,
                                         const float* __restrict__ B, int ldb, float* Cm, int ldc,
                                         float alpha, bool accum, int tri = 0,
                                         const float* __restrict__ rs = nullptr) {
    const int ntn = Nc / TN, ntm = Mr / TM;
    for (int tile = threadIdx.x; tile < ntn * ntm; tile += BWD_THREADS) {
        const int tn = tile % ntn, tm = tile / ntn;
        float acc[TM][TN];
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
            for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;
        if constexpr (MODE == GEMM_NT) {
#pragma unroll 2
            for (int k = 0; k < Kd; k += 4) {
                float4 a[TM], b[TN];
#pragma unroll
                for (int i = 0; i < TM; ++i) a[i] = *reinterpret_cast<const float4*>(A + (tm * TM + i) * lda + k);
#pragma unroll
                for (int j = 0; j < TN; ++j) b[j] = *reinterpret_cast<const float4*>(B + (tn + ntn * j) * ldb + k);
#pragma unroll
                for (int i = 0; i < TM; ++i)
#pragma unroll
                    for (int j = 0; j < TN; ++j) {
                        acc[i][j] = fmaf(a[i].x, b[j].x, acc[i][j]);
                        acc[i][j] = fmaf(a[i].y, b[j].y, acc[i][j]);
                        acc[i][j] = fmaf(a[i].z, b[j].z, acc[i][j]);
                        acc[i][j] = fmaf(a[i].w, b[j].w, acc[i][j]);
                    }
            }
        } else {
#pragma unroll 4
            for (int k = 0; k < Kd; ++k) {
                float a[TM], b[TN];
#pragma unroll
                for (int i = 0; i < TM; ++i)
                    a[i] = MODE == GEMM_NN ? A[(tm * TM + i) * lda + k] : A[k * lda + tm * TM + i];
                if constexpr (TN % 4 == 0) {
#pragma unroll
                    for (int j = 0; j < TN; j += 4) {
                        const float4 v = *reinterpret_cast<const float4*>(B + k * ldb + 4 * tn + ntn * j);
                        b[j] = v.x;
                        b[j + 1] = v.y;
                        b[j + 2] = v.z;
                        b[j + 3] = v.w;
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < TN; ++j) b[j] = B[k * ldb + tn * TN + j];
                }
#pragma unroll
                for (int i = 0; i < TM; ++i)
#pragma unroll
                    for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
            }
        }
#pragma unroll
        for (int i = 0; i < TM; ++i) {
            const int m = tm * TM + i;
            const float sc = alpha * (rs ? rs[m] : 1.f);
#pragma unroll
            for (int j = 0; j < TN; ++j) {
                const int n = MODE == GEMM_NT ? tn + ntn * j
                            : (TN % 4 == 0 ? 4 * tn + ntn * (j & ~3) + (j & 3) : tn * TN + j);
                float v = sc * acc[i][j];
                if ((tri == 1 && n > m) || (tri == 2 && n >= m)) v = 0.f;
                float* c = Cm + m * ldc + n;
                *c = accum ? *c + v : v;
            }
        }
    }
}

template <int DK, typename IO>
__global__ void __launch_bounds__(BWD_THREADS, 1)
bwd_delta_kernel(const IO* __restrict__ q, const IO* __restrict__ k, const IO* __restrict__ v,
                 const float* __restrict__ beta, const float* __restrict__ dall,
                 const float* __restrict__ S0, float scale, const IO* __restrict__ dO,
                 const float* __restrict__ dST, float* __restrict__ dv, float* __restrict__ dS0,
                 float* __restrict__ ws_state, float* __restrict__ ws_fw, float* __restrict__ dq_part,
                 float* __restrict__ dk_part, float* __restrict__ dkt_part,
                 float* __restrict__ dbeta_part, const int32_t* __restrict__ cu, int N, int T,
                 int H, int Dv, int64_t rows) {
    using L = BwdSmem<DK>;
    using tr = io_traits<IO>;
    constexpr int BV = BWD_BV, C = BWD_C, NT = BWD_THREADS, KS = L::KS, VS = L::VS, CS = L::CS;
    constexpr int TNK = DK / 16;  // a thread's columns in the DK-wide products (16 x 16 tiles)
    extern __shared__ float4 bwd_smem4[];
    float* sm = reinterpret_cast<float*>(bwd_smem4);
    float* sS = sm + L::S;
    float* sdS = sm + L::DS;
    float* sK = sm + L::K;
    float* sKt = sm + L::KT;
    float* sQ = sm + L::Q;
    float* sO = sm + L::O;
    float* sV = sm + L::V;
    float* sG = sm + L::G;
    float* sR = sm + L::R;
    float* sW = sm + L::W;
    float* sdW = sm + L::DW;
    float* sdR = sm + L::DR;
    float* sdRb = sm + L::DRB;
    float* sA = sm + L::A;
    float* sP = sm + L::P;
    float* sT = sm + L::TT;
    float* sdP = sm + L::DP;
    float* sM = sm + L::M;
    float* sX = sm + L::X;
    float* sdLb = sm + L::DLB;
    float* sB = sm + L::BETA;

    const int tid = threadIdx.x;
    const int ntile = Dv / BV, vt = blockIdx.x % ntile, nh = blockIdx.x / ntile;
    const int n = nh / H, h = nh - n * H;
    if (n >= N) return;
    int64_t first, count;
    if (!seq_range(cu, n, N, T, first, count)) return;  // uniform over the CTA
    const int c0 = vt * BV;
    const int nchunks = (int)((count + C - 1) / C);
    const int64_t sbase = (int64_t)nh * Dv * DK + (int64_t)c0 * DK;

    // the chunk's tokens (rows past its end are zero, so they contribute nothing); loops unrolled
    // and 4 elements wide so that a thread's loads are all in flight at once
    auto load_chunk = [&](int ch, bool grads) -> int {
        const int64_t row0 = first + (int64_t)ch * C;
        const int Lc = count - (int64_t)ch * C < C ? (int)(count - (int64_t)ch * C) : C;
        const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int it = 0; it < C * DK / 4 / NT; ++it) {
            const int idx = tid + it * NT, t = idx / (DK / 4), c = 4 * (idx - t * (DK / 4));
            float4 kk = z, dd = z, qq = z;
            if (t < Lc) {
                const int64_t o = ((row0 + t) * H + h) * DK + c;
                kk = load4<IO>(k + o);
                dd = __ldg(reinterpret_cast<const float4*>(dall + o));
                if (grads) qq = load4<IO>(q + o);
            }
            *reinterpret_cast<float4*>(sK + t * KS + c) = kk;
            *reinterpret_cast<float4*>(sKt + t * KS + c) =
                make_float4(dd.x * kk.x, dd.y * kk.y, dd.z * kk.z, dd.w * kk.w);
            *reinterpret_cast<float4*>(sQ + t * KS + c) = qq;
        }
#pragma unroll
        for (int it = 0; it < C * BV / 4 / NT; ++it) {
            const int idx = tid + it * NT, t = idx / (BV / 4), r = 4 * (idx - t * (BV / 4));
            float4 vv = z, gg = z;
            if (t < Lc) {
                const int64_t o = ((row0 + t) * H + h) * Dv + c0 + r;
                vv = load4<IO>(v + o);
                if (grads) gg = load4<IO>(dO + o);
            }
            *reinterpret_cast<float4*>(sV + t * VS + r) = vv;
            *reinterpret_cast<float4*>(sG + t * VS + r) = gg;
        }
        if (tid < C) sB[tid] = tid < Lc ? __ldg(beta + (row0 + tid) * H + h) : 0.f;
        return Lc;
    };
    // a BV x DK state tile between global memory (row stride DK) and shared memory (row stride KS)
    auto tile_in = [&](float* dst, const float* src) {
#pragma unroll
        for (int it = 0; it < BV * DK / 4 / NT; ++it) {
            const int idx = tid + it * NT, rr = idx / (DK / 4), c = 4 * (idx - rr * (DK / 4));
            *reinterpret_cast<float4*>(dst + rr * KS + c) =
                src ? __ldg(reinterpret_cast<const float4*>(src + rr * DK + c)) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    auto tile_out = [&](float* dst, const float* src) {
#pragma unroll
        for (int it = 0; it < BV * DK / 4 / NT; ++it) {
            const int idx = tid + it * NT, rr = idx / (DK / 4), c = 4 * (idx - rr * (DK / 4));
            *reinterpret_cast<float4*>(dst + rr * DK + c) = *reinterpret_cast<const float4*>(src + rr * KS + c);
        }
    };
    // T = (I + strict_tril(diag(beta) A))^-1 by columns (thread j < C), then R = beta E, W = T R
    auto wy = [&]() {
        if (tid < C) {
            const int j = tid;
            float x[C];
#pragma unroll
            for (int i = 0; i < C; ++i) x[i] = 0.f;
#pragma unroll
            for (int i = 0; i < C; ++i) {
                if (i < j) continue;
                float acc = i == j ? 1.f : 0.f;
                const float bi = sB[i];
#pragma unroll
                for (int s2 = 0; s2 < i; ++s2) acc = fmaf(-bi * sA[i * CS + s2], x[s2], acc);
                x[i] = acc;
            }
#pragma unroll
            for (int i = 0; i < C; ++i) sT[i * CS + j] = x[i];
        }
        for (int idx = tid; idx < C * BV; idx += NT) {
            const int t = idx / BV, r = idx - t * BV;
            sR[t * VS + r] = sB[t] * sV[t * VS + r];
        }
        __syncthreads();
        bwd_gemm<GEMM_NN, 2, 4>(C, BV, C, sT, CS, sR, VS, sW, VS, 1.f, false);
    };
    // the forward sweep's A, T, E, W of chunk ch <-> the workspace (dense rows)
    auto fw_of = [&](int ch) {
        return ws_fw + ((bwd_slot(first, ch, n) * H + h) * ntile + vt) * (int64_t)BWD_FW;
    };
    auto fw_move = [&](int ch, bool store) {
        float* g = fw_of(ch);
        float* const src[4] = {sA, sT, sV, sW};
        const int ld[4] = {CS, CS, VS, VS}, w4[4] = {C / 4, C / 4, BV / 4, BV / 4};
        int base = 0;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            for (int idx = tid; idx < C * w4[m]; idx += NT) {
                const int t = idx / w4[m], c = 4 * (idx - t * w4[m]);
                float4* gp = reinterpret_cast<float4*>(g + base + t * 4 * w4[m] + c);
                float4* sp = reinterpret_cast<float4*>(src[m] + t * ld[m] + c);
                if (store) *gp = *sp;
                else *sp = *gp;
            }
            base += C * 4 * w4[m];
        }
    };
    auto store_share = [&](float* dst, int ch, int Lc) {  // sO rows t < Lc -> a [rows, H, DK] share
        const int64_t row0 = first + (int64_t)ch * C;
#pragma unroll
        for (int it = 0; it < C * DK / 4 / NT; ++it) {
            const int idx = tid + it * NT, t = idx / (DK / 4), c = 4 * (idx - t * (DK / 4));
            if (t < Lc && OSDN_IN_BOUNDS(row0 + t, rows))
                *reinterpret_cast<float4*>(dst + (((int64_t)vt * rows + row0 + t) * H + h) * DK + c) =
                    *reinterpret_cast<const float4*>(sO + t * KS + c);
        }
    };

    // =========================================================== forward: state at chunk starts
    tile_in(sS, S0 ? S0 + sbase : nullptr);
    for (int ch = 0; ch < nchunks; ++ch) {
        __syncthreads();  // the state rows are settled; the chunk buffers are free
        if (OSDN_IN_BOUNDS(bwd_slot(first, ch, n), (rows + C - 1) / C + N + 1))  // block-uniform
            tile_out(ws_state + (bwd_slot(first, ch, n) * H + h) * (int64_t)Dv * DK + (int64_t)c0 * DK, sS);
        load_chunk(ch, false);
        __syncthreads();
        bwd_gemm<GEMM_NT, 2, 2>(C, C, DK, sK, KS, sKt, KS, sA, CS, 1.f, false);       // A = K K~^T
        bwd_gemm<GEMM_NT, 2, 4>(C, BV, DK, sK, KS, sS, KS, sV, VS, -1.f, true);       // E = V - K S^T
        __syncthreads();
        wy();
        __syncthreads();
        if (OSDN_IN_BOUNDS(bwd_slot(first, ch, n), (rows + C - 1) / C + N + 1))
            fw_move(ch, true);                                                        // keep A, T, E, W
        bwd_gemm<GEMM_TN, 4, TNK>(BV, DK, C, sW, VS, sKt, KS, sS, KS, 1.f, true);     // S += W^T K~
    }

    // =========================================================== reverse over chunks
    tile_in(sdS, dST ? dST + sbase : nullptr);
    for (int ch = nchunks - 1; ch >= 0; --ch) {
        __syncthreads();
        tile_in(sS, ws_state + (bwd_slot(first, ch, n) * H + h) * (int64_t)Dv * DK + (int64_t)c0 * DK);
        const int Lc = load_chunk(ch, true);
        const int64_t row0 = first + (int64_t)ch * C;
        __syncthreads();
        fw_move(ch, false);                                    // A, T, E (over V), W from the forward sweep
        bwd_gemm<GEMM_NT, 2, 2>(C, C, DK, sQ, KS, sKt, KS, sP, CS, 1.f, false, 1);    // P = tril(Q K~^T)
        bwd_gemm<GEMM_NT, 2, 4>(C, BV, DK, sKt, KS, sdS, KS, sdW, VS, 1.f, false);    // dW = K~ dS'^T
        __syncthreads();
        for (int idx = tid; idx < C * BV; idx += NT) {                                // R = beta E
            const int t = idx / BV, r = idx - t * BV;
            sR[t * VS + r] = sB[t] * sV[t * VS + r];
        }
        __syncthreads();
        bwd_gemm<GEMM_TN, 2, 4>(C, BV, C, sP, CS, sG, VS, sdW, VS, scale, true);      // dW += s P^T dO
        bwd_gemm<GEMM_NT, 2, 2>(C, C, BV, sG, VS, sW, VS, sdP, CS, scale, false, 1);  // dP = tril(s dO W^T)
        __syncthreads();
        bwd_gemm<GEMM_TN, 2, 4>(C, BV, C, sT, CS, sdW, VS, sdR, VS, 1.f, false);      // dR = T^T dW
        bwd_gemm<GEMM_NT, 2, 2>(C, C, BV, sdW, VS, sR, VS, sM, CS, 1.f, false);       // M = dW R^T
        bwd_gemm<GEMM_NN, 2, TNK>(C, DK, BV, sG, VS, sS, KS, sO, KS, scale, false);   // dQ = s dO S_c
        __syncthreads();
        bwd_gemm<GEMM_NN, 2, TNK>(C, DK, C, sdP, CS, sKt, KS, sO, KS, 1.f, true);     //   + dP K~
        bwd_gemm<GEMM_TN, 2, 2>(C, C, C, sT, CS, sM, CS, sX, CS, 1.f, false);         // X = T^T M
        for (int idx = tid; idx < C * BV; idx += NT) {                                // beta dR = dv
            const int t = idx / BV, r = idx - t * BV;
            const float x = sB[t] * sdR[t * VS + r];
            sdRb[t * VS + r] = x;
            if (t < Lc && OSDN_IN_BOUNDS(row0 + t, rows)) dv[((row0 + t) * H + h) * Dv + c0 + r] = x;
        }
        __syncthreads();
        store_share(dq_part, ch, Lc);
        bwd_gemm<GEMM_NT, 2, 2>(C, C, C, sX, CS, sT, CS, sM, CS, -1.f, false, 2);     // dL = -stril(X T^T)
        __syncthreads();
        if (tid < C) {  // this share of dbeta: rowsum(dL . A) + rowsum(dR . E)
            const int t = tid;
            float acc = 0.f;
            for (int j = 0; j < t; ++j) acc = fmaf(sM[t * CS + j], sA[t * CS + j], acc);
            for (int r = 0; r < BV; ++r) acc = fmaf(sdR[t * VS + r], sV[t * VS + r], acc);
            if (t < Lc && OSDN_IN_BOUNDS(row0 + t, rows)) dbeta_part[((int64_t)vt * rows + row0 + t) * H + h] = acc;
        }
        for (int idx = tid; idx < C * C; idx += NT) {                                 // beta dL
            const int t = idx / C, j = idx - t * C;
            sdLb[t * CS + j] = sB[t] * sM[t * CS + j];
        }
        bwd_gemm<GEMM_NN, 2, TNK>(C, DK, BV, sW, VS, sdS, KS, sO, KS, 1.f, false);    // dK~ = W dS'
        __syncthreads();
        bwd_gemm<GEMM_TN, 2, TNK>(C, DK, C, sdP, CS, sQ, KS, sO, KS, 1.f, true);      //   + dP^T Q
        __syncthreads();
        bwd_gemm<GEMM_TN, 2, TNK>(C, DK, C, sdLb, CS, sK, KS, sO, KS, 1.f, true);     //   + (beta dL)^T K
        __syncthreads();
        store_share(dkt_part, ch, Lc);
        __syncthreads();
        bwd_gemm<GEMM_NN, 2, TNK>(C, DK, C, sdLb, CS, sKt, KS, sO, KS, 1.f, false);   // dK = beta dL K~
        __syncthreads();
        bwd_gemm<GEMM_NN, 2, TNK>(C, DK, BV, sdRb, VS, sS, KS, sO, KS, -1.f, true);   //   - beta dR S_c
        __syncthreads();
        store_share(dk_part, ch, Lc);
        bwd_gemm<GEMM_TN, 4, TNK>(BV, DK, C, sG, VS, sQ, KS, sdS, KS, scale, true);   // dS += s dO^T Q
        __syncthreads();
        bwd_gemm<GEMM_TN, 4, TNK>(BV, DK, C, sdRb, VS, sK, KS, sdS, KS, -1.f, true);  //    - (beta dR)^T K
    }
    __syncthreads();
    if (dS0) tile_out(dS0 + sbase, sdS);
}

// The value-row shares of bwd_delta_kernel added up, elementwise over the whole batch: dq (the
// final gradient), and dk~, dk's phase-2 term and dbeta's phase-2 term summed into share 0.
__global__ void __launch_bounds__(256)
bwd_reduce_kernel(const float4* __restrict__ dq_part, float4* __restrict__ dk_part,
                  float4* __restrict__ dkt_part, float* __restrict__ dbeta_part, int ntile,
                  int64_t n4, int64_t nb, float4* __restrict__ dq) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
        float4 a = dq_part[i], b = dk_part[i], c = dkt_part[i];
        for (int p = 1; p < ntile; ++p) {
            const float4 x = dq_part[p * n4 + i], y = dk_part[p * n4 + i], z = dkt_part[p * n4 + i];
            a.x += x.x; a.y += x.y; a.z += x.z; a.w += x.w;
            b.x += y.x; b.y += y.y; b.z += y.z; b.w += y.w;
            c.x += z.x; c.y += z.y; c.z += z.z; c.w += z.w;
        }
        dq[i] = a;
        dk_part[i] = b;
        dkt_part[i] = c;
    }
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nb; i += stride) {
        float v = dbeta_part[i];
        for (int p = 1; p < ntile; ++p) v += dbeta_part[p * nb + i];
        dbeta_part[i] = v;
    }
}

// Phase 1 in reverse.  One CTA of 128 threads per (sequence, head), 32-token chunks in reverse
// order, three chunk buffers in turn (two when three do not fit in shared memory):
//   warp 0 runs the adjoint recurrence dd_t = r_t dd_{t+1} - c_t y_t a_t + dk~_t (.) k_t over chunk
//     ch, where y_t = <a_t, dd_{t+1}> is its only reduction, and keeps dd_{t+1} and y_t of every
//     token (c_t = eta beta_t^2 / ||k_t||^2, 0 for a zero key);
//   warps 1-3 meanwhile start fetching chunk ch - 1 (asynchronous copies), turn chunk ch + 1's
//     kept values into dk, dr, dbeta and deta, and then compute chunk ch - 1's per-token
//     scalars, none of which depends on dd: ||k_t||^2, s_t = <d_t, a_t>, x_t, c_t and the dbeta
//     factor.  Every value they read is staged in shared memory, so their per-token loops do not
//     wait on global loads.
template <int DK, typename IO>
struct BwdPrecondSmem {
    static constexpr int KB = DK * (int)sizeof(IO) / 4;  // a token's key row, in 4-byte words
    static constexpr int DKT = 0;                        // [C][DK] dk~
    static constexpr int DK2 = DKT + BWD_C * DK;         // [C][DK] dk, phase-2 term
    static constexpr int D = DK2 + BWD_C * DK;           // [C][DK] d_t
    static constexpr int K = D + BWD_C * DK;             // [C][KB] k_t in the io dtype
    static constexpr int SC = K + BWD_C * KB;            // [7][C] beta, r, dbeta phase-2 term,
                                                         //   1/||k||^2, x, c, dbeta factor
    static constexpr int BUF = SC + 7 * BWD_C;           // one chunk buffer
    static constexpr int NB = 3 * BUF + 2 * BWD_C * DK + 2 * BWD_C + 4 <= 232448 / 4 - 256 ? 3 : 2;
    static constexpr int DD = NB * BUF;                  // [2][C][DK] dd_{t+1}, kept by warp 0
    static constexpr int Y = DD + 2 * BWD_C * DK;        // [2][C] y_t
    static constexpr int ETA = Y + 2 * BWD_C;            // [4] deta shares of warps 1-3
    static constexpr int floats = ETA + 4;
    static constexpr size_t bytes = sizeof(float) * floats;
};

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)),
                 "l"(reinterpret_cast<uint64_t>(gsrc))
                 : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// E consecutive values of a row (E = 4 or 2, starting at a multiple of E) as one 16- or 8-byte
// shared-memory access: lane-strided scalar accesses would meet each bank E times.
template <int E>
__device__ __forceinline__ void row_ld(const float* p, float* x) {
    if constexpr (E == 4) {
        const float4 v = *reinterpret_cast<const float4*>(p);
        x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    } else {
        const float2 v = *reinterpret_cast<const float2*>(p);
        x[0] = v.x; x[1] = v.y;
    }
}
template <int E>
__device__ __forceinline__ void row_st(float* p, const float* x) {
    if constexpr (E == 4) *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
    else *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
}
template <int E, typename IO>
__device__ __forceinline__ void row_ld_io(const IO* p, float* x) {
    if constexpr (sizeof(IO) == 4) {
        row_ld<E>(reinterpret_cast<const float*>(p), x);
    } else if constexpr (E == 4) {
        const uint2 w = *reinterpret_cast<const uint2*>(p);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.y));
        x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
    } else {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w));
        x[0] = a.x; x[1] = a.y;
    }
}

template <int DK, typename IO>
__global__ void __launch_bounds__(128)
bwd_precond_kernel(const IO* __restrict__ k, const float* __restrict__ beta,
                   const float* __restrict__ r, float eta, const float* __restrict__ dall,
                   const float* __restrict__ ddT, const float* __restrict__ dk_sum,
                   const float* __restrict__ dkt_sum, const float* __restrict__ dbeta_sum,
                   float* __restrict__ dk, float* __restrict__ dbeta, float* __restrict__ dr,
                   float* __restrict__ dd0, float* __restrict__ deta_part,
                   const int32_t* __restrict__ cu, int N, int T, int H) {
    using L = BwdPrecondSmem<DK, IO>;
    constexpr int C = BWD_C, E = DK / 32;
    extern __shared__ float4 bwdp_smem4[];
    float* sm = reinterpret_cast<float*>(bwdp_smem4);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nh = blockIdx.x, n = nh / H, h = nh - n * H;
    if (n >= N) return;
    int64_t first, count;
    if (!seq_range(cu, n, N, T, first, count)) return;
    const int nchunks = (int)((count + C - 1) / C);
    auto chunk_len = [&](int ch) -> int {
        const int64_t rem = count - (int64_t)ch * C;
        return rem < C ? (int)rem : C;
    };
    auto buf_of = [&](int ch) { return sm + (ch % L::NB) * L::BUF; };

    // warps 1-3: chunk ch into its buffer (tokens past the chunk's end are not read): copies
    // issued here, the gates held in registers until fetch_finish stores them
    float gb = 0.f, gr = 1.f, gd = 0.f;  // beta, r and the dbeta phase-2 term of token tid - 32
    auto fetch_issue = [&](int ch) {
        float* buf = buf_of(ch);
        const int64_t row0 = first + (int64_t)ch * C;
        const int Lc = chunk_len(ch), i = tid - 32;
        constexpr int P4 = DK / 4, PK = L::KB / 4;  // 16-byte pieces per token row
        for (int idx = i; idx < Lc * (3 * P4 + PK); idx += 96) {
            const int t = idx / (3 * P4 + PK), q = idx - t * (3 * P4 + PK);
            const int64_t o = ((row0 + t) * H + h) * DK;
            if (q < P4) cp_async16(buf + L::DKT + t * DK + 4 * q, dkt_sum + o + 4 * q);
            else if (q < 2 * P4) cp_async16(buf + L::DK2 + t * DK + 4 * (q - P4), dk_sum + o + 4 * (q - P4));
            else if (q < 3 * P4) cp_async16(buf + L::D + t * DK + 4 * (q - 2 * P4), dall + o + 4 * (q - 2 * P4));
            else cp_async16(buf + L::K + t * L::KB + 4 * (q - 3 * P4),
                            reinterpret_cast<const float*>(k + o) + 4 * (q - 3 * P4));
        }
        if (i < Lc) {
            const int64_t th = (row0 + i) * H + h;
            gb = __ldg(beta + th);
            gr = r ? __ldg(r + th) : 1.f;
            gd = dbeta_sum[th];
        }
    };
    // ... then, once the copies have landed, the per-token scalars (one warp per token)
    auto fetch_finish = [&](int ch) {
        float* buf = buf_of(ch);
        const int Lc = chunk_len(ch), i = tid - 32;
        if (i < Lc) {
            buf[L::SC + i] = gb;
            buf[L::SC + C + i] = gr;
            buf[L::SC + 2 * C + i] = gd;
        }
        cp_async_wait_all();
        asm volatile("bar.sync 1, 96;" ::: "memory");  // the chunk is in place for warps 1-3
#pragma unroll 2
        for (int t = warp - 1; t < Lc; t += 3) {
            const IO* krow = reinterpret_cast<const IO*>(buf + L::K + t * L::KB);
            float kk[E], dv[E];
            row_ld_io<E>(krow + lane * E, kk);
            row_ld<E>(buf + L::D + t * DK + lane * E, dv);
            float nk = 0.f, sv = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const float a = kk[e] * kk[e];
                nk += a;
                sv = fmaf(dv[e], a, sv);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                nk += __shfl_xor_sync(0xffffffffu, nk, off);
                sv += __shfl_xor_sync(0xffffffffu, sv, off);
            }
            if (lane == 0) {
                const float bt = buf[L::SC + t];
                const bool ok = nk > 0.f;
                const float inv = ok ? 1.f / nk : 0.f;
                buf[L::SC + 3 * C + t] = inv;
                buf[L::SC + 4 * C + t] = ok ? bt * (1.f - bt * sv) * inv : 0.f;     // x_t
                buf[L::SC + 5 * C + t] = ok ? eta * bt * bt * inv : 0.f;           // c_t
                buf[L::SC + 6 * C + t] = ok ? eta * (1.f - 2.f * bt * sv) * inv : 0.f;
            }
        }
    };
    // warps 1-3: the gradients of chunk ch from dd_{t+1} and y_t (one warp per token)
    float deta_acc = 0.f;
    auto outputs = [&](int ch) {
        const float* buf = buf_of(ch);
        const float* sdd = sm + L::DD + (ch & 1) * C * DK;
        const float* sy = sm + L::Y + (ch & 1) * C;
        const int64_t row0 = first + (int64_t)ch * C;
        const int Lc = chunk_len(ch);
#pragma unroll 2
        for (int t = warp - 1; t < Lc; t += 3) {
            const IO* krow = reinterpret_cast<const IO*>(buf + L::K + t * L::KB);
            const float y = sy[t], bt = buf[L::SC + t], inv = buf[L::SC + 3 * C + t];
            const float xt = buf[L::SC + 4 * C + t];
            const int64_t th = (row0 + t) * H + h;
            if (!OSDN_IN_BOUNDS(row0 + t, cu ? (int64_t)T : (int64_t)N * T)) continue;  // warp-uniform
            float rd = 0.f, g[E], ddv[E], dv[E], kk[E], dk2[E], dkt[E];
            row_ld<E>(sdd + t * DK + lane * E, ddv);
            row_ld<E>(buf + L::D + t * DK + lane * E, dv);
            row_ld_io<E>(krow + lane * E, kk);
            row_ld<E>(buf + L::DK2 + t * DK + lane * E, dk2);
            row_ld<E>(buf + L::DKT + t * DK + lane * E, dkt);
#pragma unroll
            for (int e = 0; e < E; ++e) {
                rd = fmaf(ddv[e], dv[e], rd);
                const float da = inv > 0.f ? eta * xt * ddv[e] - eta * y * (bt * bt * dv[e] + xt) * inv : 0.f;
                g[e] = dk2[e] + dkt[e] * dv[e] + 2.f * kk[e] * da;
            }
            if constexpr (E == 4) {
                *reinterpret_cast<float4*>(dk + th * DK + lane * E) = make_float4(g[0], g[1], g[2], g[3]);
            } else {
#pragma unroll
                for (int e = 0; e < E; ++e) dk[th * DK + lane * E + e] = g[e];
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) rd += __shfl_xor_sync(0xffffffffu, rd, off);
            if (lane == 0) {
                dbeta[th] = buf[L::SC + 2 * C + t] + buf[L::SC + 6 * C + t] * y;
                if (dr) dr[th] = rd;
                deta_acc = fmaf(xt, y, deta_acc);
            }
        }
    };

    float dd[E];
#pragma unroll
    for (int e = 0; e < E; ++e) dd[e] = ddT ? __ldg(ddT + (int64_t)nh * DK + lane * E + e) : 0.f;
    if (warp > 0 && nchunks > 0) {
        fetch_issue(nchunks - 1);
        fetch_finish(nchunks - 1);
    }
    __syncthreads();
    for (int ch = nchunks - 1; ch >= 0; --ch) {
        if (warp == 0) {
            const float* buf = buf_of(ch);
            float* sdd = sm + L::DD + (ch & 1) * C * DK;
            float* sy = sm + L::Y + (ch & 1) * C;
            for (int t = chunk_len(ch) - 1; t >= 0; --t) {
                const IO* krow = reinterpret_cast<const IO*>(buf + L::K + t * L::KB);
                float a[E], kk[E], dkt[E];
                row_ld_io<E>(krow + lane * E, kk);
                row_ld<E>(buf + L::DKT + t * DK + lane * E, dkt);
                row_st<E>(sdd + t * DK + lane * E, dd);  // dd_{t+1}
                float y = 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    a[e] = kk[e] * kk[e];
                    y = fmaf(a[e], dd[e], y);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) y += __shfl_xor_sync(0xffffffffu, y, off);
                if (lane == 0) sy[t] = y;
                const float cy = buf[L::SC + 5 * C + t] * y, rt = buf[L::SC + C + t];
#pragma unroll
                for (int e = 0; e < E; ++e) dd[e] = fmaf(rt, dd[e], fmaf(-cy, a[e], dkt[e] * kk[e]));
            }
        } else if constexpr (L::NB == 3) {  // chunk ch - 1's copies land under chunk ch + 1's outputs
            if (ch > 0) fetch_issue(ch - 1);
            if (ch + 1 < nchunks) outputs(ch + 1);
            if (ch > 0) fetch_finish(ch - 1);
        } else {  // chunks ch + 1 and ch - 1 share a buffer
            if (ch + 1 < nchunks) outputs(ch + 1);
            asm volatile("bar.sync 1, 96;" ::: "memory");
            if (ch > 0) {
                fetch_issue(ch - 1);
                fetch_finish(ch - 1);
            }
        }
        __syncthreads();  // chunk ch's dd and y are kept; chunk ch - 1 has landed
    }
    if (warp > 0 && nchunks > 0) outputs(0);
    if (warp > 0 && lane == 0) sm[L::ETA + warp] = deta_acc;
    __syncthreads();
    if (warp == 0) {
        if (dd0) {
#pragma unroll
            for (int e = 0; e < E; ++e) dd0[(int64_t)nh * DK + lane * E + e] = dd[e];
        }
        if (lane == 0) deta_part[nh] = (sm[L::ETA + 1] + sm[L::ETA + 2]) + sm[L::ETA + 3];  // fixed order
    }
}

// deta = sum of the per-(sequence, head) shares, in a fixed order (one block).
__global__ void __launch_bounds__(256) bwd_sum_kernel(const float* __restrict__ part, int64_t n,
                                                      float* __restrict__ out) {
    __shared__ double red[256];
    double acc = 0.0;
    for (int64_t i = threadIdx.x; i < n; i += 256) acc += (double)part[i];
    red[threadIdx.x] = acc;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) *out = (float)red[0];
}

}  // namespace osdn
