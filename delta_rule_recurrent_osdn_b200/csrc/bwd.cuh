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
//      independent, so each CTA carries its rows: a forward sweep over the sequence (states at
//      every 32-token chunk start kept in a workspace, dq's share of these rows), then chunks in
//      reverse: u_s of the chunk's tokens from the chunk-start state (S_{s-1} = S_c +
//      sum_{j<s} beta_j u_j k~_j^T, a forward substitution with the chunk Gram K K~^T), and a
//      reverse token sweep of dS.  dv is per row; dq, dk, dk~ and dbeta's phase-2 term are sums
//      over all value rows, written as per-CTA shares;
//   3. bwd_precond_kernel: one CTA per (sequence, head): adds the shares and runs the phase-1
//      adjoint recurrence in reverse (one warp, a chunk of tokens staged in shared memory);
//   4. bwd_sum_kernel: deta, summed over (sequence, head) in a fixed order.
#pragma once

#include "common.cuh"

namespace osdn {

constexpr int BWD_BV = 64;      // value rows per bwd_delta_kernel CTA
constexpr int BWD_C = 32;       // tokens per chunk (state checkpoints, staging)
constexpr int BWD_THREADS = 256;

template <int DK>
struct BwdSmem {
    static constexpr int KS = DK + 4;  // row stride (floats): conflict-free row and column walks
    static constexpr int S = 0;                              // [BV][KS] state rows (S_c)
    static constexpr int DS = S + BWD_BV * KS;               // [BV][KS] adjoint rows
    static constexpr int K = DS + BWD_BV * KS;               // [C][KS] keys of the chunk
    static constexpr int KT = K + BWD_C * KS;                // [C][KS] k~ = d (.) k
    static constexpr int Q = KT + BWD_C * KS;                // [C][KS] queries
    static constexpr int U = Q + BWD_C * KS;                 // [C][BV] u_t (this CTA's rows)
    static constexpr int V = U + BWD_C * BWD_BV;             // [C][BV] v_t, then v_t - S_c k_t
    static constexpr int DO = V + BWD_C * BWD_BV;            // [C][BV] dL/do_t (rows)
    static constexpr int A = DO + BWD_C * BWD_BV;            // [C][C + 1] k_s . k~_j
    static constexpr int BETA = A + BWD_C * (BWD_C + 1);     // [C]
    static constexpr int G = BETA + BWD_C;                   // [BV] g_t
    static constexpr int SIG = G + BWD_BV;                   // [C] beta_s <u_s, g_t> (s < t)
    static constexpr int floats = SIG + BWD_C + 4;
    static constexpr size_t bytes = sizeof(float) * floats;
};

// Checkpoint slot of chunk ch (0-based, BWD_C tokens) of sequence n starting at row `first`:
// floor(first / C) + ch + n.  Distinct over all (sequence, chunk) pairs of a batch, and below
// ceil(rows / C) + N + 1 (the workspace holds that many).
__device__ __forceinline__ int64_t bwd_slot(int64_t first, int ch, int n) {
    return first / BWD_C + ch + n;
}

// Row `it` (0 .. BV/NP - 1) of the column-walk part `hp` (0 .. NP - 1): 8-row blocks split into
// NP runs of 8 / NP rows, so the lanes of a warp read distinct banks.
template <int NP>
__device__ __forceinline__ int bwd_row(int it, int hp) {
    constexpr int SPAN = 8 / NP;
    return 8 * (it / SPAN) + SPAN * hp + (it % SPAN);
}

template <int DK, typename IO>
__global__ void __launch_bounds__(BWD_THREADS, 1)
bwd_delta_kernel(const IO* __restrict__ q, const IO* __restrict__ k, const IO* __restrict__ v,
                 const float* __restrict__ beta, const float* __restrict__ dall,
                 const float* __restrict__ S0, float scale, const IO* __restrict__ dO,
                 const float* __restrict__ dST, float* __restrict__ dv, float* __restrict__ dS0,
                 float* __restrict__ ws_state, float* __restrict__ dq_part,
                 float* __restrict__ dk_part, float* __restrict__ dkt_part,
                 float* __restrict__ dbeta_part, const int32_t* __restrict__ cu, int N, int T,
                 int H, int Dv, int64_t rows) {
    using L = BwdSmem<DK>;
    using tr = io_traits<IO>;
    constexpr int BV = BWD_BV, C = BWD_C, NT = BWD_THREADS, KS = L::KS;
    constexpr int NP = NT / DK;   // column walk: DK columns x NP row parts
    constexpr int CP = DK / 4;    // row walk: BV rows x 4 column parts (columns 4 j + part)
    static_assert(NT == 4 * BV && C * 8 == NT, "thread layouts");
    extern __shared__ float4 bwd_smem4[];
    float* sm = reinterpret_cast<float*>(bwd_smem4);
    float* sS = sm + L::S;
    float* sdS = sm + L::DS;
    float* sK = sm + L::K;
    float* sKt = sm + L::KT;
    float* sQ = sm + L::Q;
    float* sU = sm + L::U;
    float* sV = sm + L::V;
    float* sDO = sm + L::DO;
    float* sA = sm + L::A;
    float* sB = sm + L::BETA;
    float* sG = sm + L::G;
    float* sSig = sm + L::SIG;

    const int tid = threadIdx.x;
    const int ntile = Dv / BV, vt = blockIdx.x % ntile, nh = blockIdx.x / ntile;
    const int n = nh / H, h = nh - n * H;
    if (n >= N) return;
    int64_t first, count;
    if (!seq_range(cu, n, N, T, first, count)) return;  // uniform over the CTA
    const int c0 = vt * BV;
    const int nchunks = (int)((count + C - 1) / C);
    const int r1 = tid >> 2, p1 = tid & 3;      // row walk
    const int c2 = tid / NP, hp = tid % NP;     // column walk
    const int64_t sbase = (int64_t)nh * Dv * DK + (int64_t)c0 * DK;

    auto load_chunk = [&](int ch) -> int {
        const int64_t row0 = first + (int64_t)ch * C;
        const int Lc = count - (int64_t)ch * C < C ? (int)(count - (int64_t)ch * C) : C;
        for (int idx = tid; idx < C * DK; idx += NT) {
            const int t = idx / DK, c = idx - t * DK;
            float kk = 0.f, dd = 0.f, qq = 0.f;
            if (t < Lc) {
                const int64_t o = ((row0 + t) * H + h) * DK + c;
                kk = tr::to_f32(k[o]);
                dd = dall[o];
                qq = tr::to_f32(q[o]);
            }
            sK[t * KS + c] = kk;
            sKt[t * KS + c] = dd * kk;
            sQ[t * KS + c] = qq;
        }
        for (int idx = tid; idx < C * BV; idx += NT) {
            const int t = idx / BV, r = idx - t * BV;
            float vv = 0.f, gg = 0.f;
            if (t < Lc) {
                const int64_t o = ((row0 + t) * H + h) * Dv + c0 + r;
                vv = tr::to_f32(v[o]);
                gg = tr::to_f32(dO[o]);
            }
            sV[t * BV + r] = vv;
            sDO[t * BV + r] = gg;
        }
        if (tid < C) sB[tid] = tid < Lc ? __ldg(beta + (row0 + tid) * H + h) : 0.f;
        return Lc;
    };

    // =========================================================== forward sweep
    for (int idx = tid; idx < BV * DK; idx += NT) {
        const int r = idx / DK, c = idx - r * DK;
        sS[r * KS + c] = S0 ? __ldg(S0 + sbase + idx) : 0.f;
    }
    for (int ch = 0; ch < nchunks; ++ch) {
        __syncthreads();  // the state rows are settled; the chunk buffers are free
        {
            float* dst = ws_state + (bwd_slot(first, ch, n) * H + h) * (int64_t)Dv * DK +
                         (int64_t)c0 * DK;
            for (int idx = tid; idx < BV * DK; idx += NT) {
                const int r = idx / DK, c = idx - r * DK;
                dst[idx] = sS[r * KS + c];
            }
        }
        const int Lc = load_chunk(ch);
        __syncthreads();
        for (int t = 0; t < Lc; ++t) {
            {  // u_t = v_t - S_{t-1} k_t on row r1, then S += beta_t u_t k~_t^T (own columns)
                float acc = 0.f;
#pragma unroll 8
                for (int j = 0; j < CP; ++j) acc = fmaf(sS[r1 * KS + 4 * j + p1], sK[t * KS + 4 * j + p1], acc);
                acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                const float bu = sB[t] * (sV[t * BV + r1] - acc);
#pragma unroll 8
                for (int j = 0; j < CP; ++j)
                    sS[r1 * KS + 4 * j + p1] = fmaf(bu, sKt[t * KS + 4 * j + p1], sS[r1 * KS + 4 * j + p1]);
            }
            __syncthreads();
            {  // this CTA's share of dq_t = scale S_t^T do_t
                float acc = 0.f;
#pragma unroll 8
                for (int it = 0; it < BV / NP; ++it) {
                    const int r = bwd_row<NP>(it, hp);
                    acc = fmaf(sS[r * KS + c2], sDO[t * BV + r], acc);
                }
#pragma unroll
                for (int off = 1; off < NP; off <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
                if (hp == 0)
                    dq_part[(((int64_t)vt * rows + first + (int64_t)ch * C + t) * H + h) * DK + c2] =
                        scale * acc;
            }
            __syncthreads();
        }
    }

    // =========================================================== reverse sweep
    for (int idx = tid; idx < BV * DK; idx += NT) {
        const int r = idx / DK, c = idx - r * DK;
        sdS[r * KS + c] = dST ? __ldg(dST + sbase + idx) : 0.f;
    }
    for (int ch = nchunks - 1; ch >= 0; --ch) {
        __syncthreads();
        {
            const float* src = ws_state + (bwd_slot(first, ch, n) * H + h) * (int64_t)Dv * DK +
                               (int64_t)c0 * DK;
            for (int idx = tid; idx < BV * DK; idx += NT) {
                const int r = idx / DK, c = idx - r * DK;
                sS[r * KS + c] = src[idx];
            }
        }
        const int Lc = load_chunk(ch);
        __syncthreads();
        // chunk Gram A[s][j] = k_s . k~_j (j < s) and V' = V - S_c K^T
        for (int idx = tid; idx < C * C; idx += NT) {
            const int s = idx / C, j = idx - s * C;
            float a = 0.f;
            if (j < s && s < Lc) {
#pragma unroll 8
                for (int c = 0; c < DK; ++c) a = fmaf(sK[s * KS + c], sKt[j * KS + c], a);
            }
            sA[s * (C + 1) + j] = a;
        }
        for (int idx = tid; idx < C * BV; idx += NT) {
            const int s = idx / BV, r = idx - s * BV;
            if (s < Lc) {
                float a = 0.f;
#pragma unroll 8
                for (int c = 0; c < DK; ++c) a = fmaf(sS[r * KS + c], sK[s * KS + c], a);
                sV[s * BV + r] -= a;
            }
        }
        __syncthreads();
        // u_s = V'[s] - sum_{j<s} beta_j u_j A[s][j], row by row (the row's 4 lanes share a warp)
        for (int s = 0; s < Lc; ++s) {
            float acc = 0.f;
            for (int j = p1; j < s; j += 4) acc = fmaf(sB[j] * sU[j * BV + r1], sA[s * (C + 1) + j], acc);
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            if (p1 == 0) sU[s * BV + r1] = sV[s * BV + r1] - acc;
            __syncwarp();
        }
        __syncthreads();
        float g_prev = 0.f, b_prev = 0.f;  // token t+1's pending update dS -= beta g k^T (row r1)
        for (int t = Lc - 1; t >= 0; --t) {
            const int64_t row = first + (int64_t)ch * C + t;
            {  // dS_t = dS_{t+1} - beta_{t+1} g_{t+1} k_{t+1}^T + scale do_t q_t^T;  g_t = dS_t k~_t
                const float dor = scale * sDO[t * BV + r1];
                const float bg = (t + 1 < Lc) ? b_prev * g_prev : 0.f;
                const int tn = (t + 1 < Lc) ? t + 1 : t;
                float acc = 0.f;
#pragma unroll 8
                for (int j = 0; j < CP; ++j) {
                    const int c = 4 * j + p1;
                    float x = sdS[r1 * KS + c];
                    x = fmaf(-bg, sK[tn * KS + c], x);
                    x = fmaf(dor, sQ[t * KS + c], x);
                    sdS[r1 * KS + c] = x;
                    acc = fmaf(x, sKt[t * KS + c], acc);
                }
                acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                g_prev = acc;
                b_prev = sB[t];
                if (p1 == 0) {
                    sG[r1] = acc;
                    dv[(row * H + h) * Dv + c0 + r1] = b_prev * acc;
                }
            }
            __syncthreads();
            float a1 = 0.f, a2 = 0.f;  // column walk: sum_r dS[r][c] u_t[r], sum_r S_c[r][c] g[r]
#pragma unroll 8
            for (int it = 0; it < BV / NP; ++it) {
                const int r = bwd_row<NP>(it, hp);
                a1 = fmaf(sdS[r * KS + c2], sU[t * BV + r], a1);
                a2 = fmaf(sS[r * KS + c2], sG[r], a2);
            }
#pragma unroll
            for (int off = 1; off < NP; off <<= 1) {
                a1 += __shfl_xor_sync(0xffffffffu, a1, off);
                a2 += __shfl_xor_sync(0xffffffffu, a2, off);
            }
            {  // <u_s, g_t> over this CTA's rows for s <= t (thread: s = tid / 8, rows q8 + 8 i)
                const int s = tid >> 3, q8 = tid & 7;
                float x = 0.f;
                if (s <= t) {
#pragma unroll
                    for (int i = 0; i < BV / 8; ++i) x = fmaf(sU[s * BV + q8 + 8 * i], sG[q8 + 8 * i], x);
                }
                x += __shfl_xor_sync(0xffffffffu, x, 1);
                x += __shfl_xor_sync(0xffffffffu, x, 2);
                x += __shfl_xor_sync(0xffffffffu, x, 4);
                if (q8 == 0) sSig[s] = s < t ? sB[s] * x : (s == t ? x : 0.f);
            }
            __syncthreads();
            if (hp == 0) {  // S_{t-1}^T g_t = S_c^T g_t + sum_{s<t} k~_s beta_s <u_s, g_t>
                float sk = 0.f;
                for (int s = 0; s < t; ++s) sk = fmaf(sKt[s * KS + c2], sSig[s], sk);
                const int64_t o = (((int64_t)vt * rows + row) * H + h) * DK + c2;
                dkt_part[o] = sB[t] * a1;
                dk_part[o] = -sB[t] * (a2 + sk);
            }
            if (tid == 0) dbeta_part[((int64_t)vt * rows + row) * H + h] = sSig[t];
        }
        if (Lc > 0) {  // token 0's pending update
#pragma unroll 8
            for (int j = 0; j < CP; ++j) {
                const int c = 4 * j + p1;
                sdS[r1 * KS + c] = fmaf(-b_prev * g_prev, sK[c], sdS[r1 * KS + c]);
            }
        }
    }
    __syncthreads();
    if (dS0) {
        for (int idx = tid; idx < BV * DK; idx += NT) {
            const int r = idx / DK, c = idx - r * DK;
            dS0[sbase + idx] = sdS[r * KS + c];
        }
    }
}

// Phase 1 in reverse, with the shares of bwd_delta_kernel added up.  One CTA of 128 threads per
// (sequence, head): all threads stage a chunk of BWD_C tokens (and write dq), warp 0 runs the
// adjoint recurrence over it.
template <int DK>
struct BwdPrecondSmem {
    static constexpr int DKT = 0;                    // [C][DK] dk~ (summed)
    static constexpr int DK2 = DKT + BWD_C * DK;     // [C][DK] dk, phase-2 term (summed)
    static constexpr int D = DK2 + BWD_C * DK;       // [C][DK] d_t
    static constexpr int K = D + BWD_C * DK;         // [C][DK] k_t
    static constexpr int VEC = K + BWD_C * DK;       // [C] beta, r, dbeta phase-2 term
    static constexpr int floats = VEC + 3 * BWD_C;
    static constexpr size_t bytes = sizeof(float) * floats;
};

template <int DK, typename IO>
__global__ void __launch_bounds__(128)
bwd_precond_kernel(const IO* __restrict__ k, const float* __restrict__ beta,
                   const float* __restrict__ r, float eta, const float* __restrict__ dall,
                   const float* __restrict__ ddT, const float* __restrict__ dq_part,
                   const float* __restrict__ dk_part, const float* __restrict__ dkt_part,
                   const float* __restrict__ dbeta_part, int ntile, float* __restrict__ dq,
                   float* __restrict__ dk, float* __restrict__ dbeta, float* __restrict__ dr,
                   float* __restrict__ dd0, float* __restrict__ deta_part,
                   const int32_t* __restrict__ cu, int N, int T, int H, int64_t rows) {
    using L = BwdPrecondSmem<DK>;
    using tr = io_traits<IO>;
    constexpr int C = BWD_C, E = DK / 32;
    extern __shared__ float4 bwdp_smem4[];
    float* sm = reinterpret_cast<float*>(bwdp_smem4);
    float* sDkt = sm + L::DKT;
    float* sDk2 = sm + L::DK2;
    float* sD = sm + L::D;
    float* sK = sm + L::K;
    float* sBeta = sm + L::VEC;
    float* sR = sBeta + C;
    float* sDb = sR + C;
    const int tid = threadIdx.x, lane = tid & 31;
    const int nh = blockIdx.x, n = nh / H, h = nh - n * H;
    if (n >= N) return;
    int64_t first, count;
    if (!seq_range(cu, n, N, T, first, count)) return;
    const int nchunks = (int)((count + C - 1) / C);
    const int64_t part_stride = rows * H * DK;

    float dd[E];
#pragma unroll
    for (int e = 0; e < E; ++e) dd[e] = ddT ? __ldg(ddT + (int64_t)nh * DK + lane * E + e) : 0.f;
    float deta = 0.f;

    for (int ch = nchunks - 1; ch >= 0; --ch) {
        const int64_t row0 = first + (int64_t)ch * C;
        const int Lc = count - (int64_t)ch * C < C ? (int)(count - (int64_t)ch * C) : C;
        __syncthreads();  // warp 0 is done with the previous chunk's tiles
        for (int idx = tid; idx < Lc * DK; idx += 128) {
            const int t = idx / DK, c = idx - t * DK;
            const int64_t o = ((row0 + t) * H + h) * DK + c;
            float skt = 0.f, sk2 = 0.f, sq = 0.f;
            for (int p = 0; p < ntile; ++p) {
                skt += dkt_part[p * part_stride + o];
                sk2 += dk_part[p * part_stride + o];
                sq += dq_part[p * part_stride + o];
            }
            dq[o] = sq;
            sDkt[idx] = skt;
            sDk2[idx] = sk2;
            sD[idx] = dall[o];
            sK[idx] = tr::to_f32(k[o]);
        }
        for (int t = tid; t < Lc; t += 128) {
            const int64_t th = (row0 + t) * H + h;
            sBeta[t] = __ldg(beta + th);
            sR[t] = r ? __ldg(r + th) : 1.f;
            float sb = 0.f;
            for (int p = 0; p < ntile; ++p) sb += dbeta_part[(int64_t)p * rows * H + th];
            sDb[t] = sb;
        }
        __syncthreads();
        if (tid < 32) {
            for (int t = Lc - 1; t >= 0; --t) {
                float kk[E], dv_[E], a[E];
                float nk = 0.f, s = 0.f, y = 0.f, rd = 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    kk[e] = sK[t * DK + lane * E + e];
                    dv_[e] = sD[t * DK + lane * E + e];
                    a[e] = kk[e] * kk[e];
                    nk += a[e];
                    s = fmaf(dv_[e], a[e], s);
                    y = fmaf(a[e], dd[e], y);
                    rd = fmaf(dd[e], dv_[e], rd);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    nk += __shfl_xor_sync(0xffffffffu, nk, off);
                    s += __shfl_xor_sync(0xffffffffu, s, off);
                    y += __shfl_xor_sync(0xffffffffu, y, off);
                    rd += __shfl_xor_sync(0xffffffffu, rd, off);
                }
                const float bt = sBeta[t], rt = sR[t];
                const bool ok = nk > 0.f;
                const float inv = ok ? 1.f / nk : 0.f;
                const float xt = ok ? bt * (1.f - bt * s) * inv : 0.f;
                const int64_t th = (row0 + t) * H + h;
                if (lane == 0) {
                    dbeta[th] = sDb[t] + (ok ? eta * y * (1.f - 2.f * bt * s) * inv : 0.f);
                    if (dr) dr[th] = rd;
                }
                deta = fmaf(xt, y, deta);
                const float cy = ok ? eta * bt * bt * inv * y : 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const float dkt = sDkt[t * DK + lane * E + e];
                    const float da = ok ? eta * xt * dd[e] - eta * y * (bt * bt * dv_[e] + xt) * inv : 0.f;
                    dk[th * DK + lane * E + e] = sDk2[t * DK + lane * E + e] + dkt * dv_[e] + 2.f * kk[e] * da;
                    dd[e] = fmaf(rt, dd[e], fmaf(-cy, a[e], dkt * kk[e]));
                }
            }
        }
    }
    if (tid < 32) {
        if (dd0) {
#pragma unroll
            for (int e = 0; e < E; ++e) dd0[(int64_t)nh * DK + lane * E + e] = dd[e];
        }
        if (lane == 0) deta_part[nh] = deta;
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
