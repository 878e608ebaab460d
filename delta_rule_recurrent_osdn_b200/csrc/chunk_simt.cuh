// chunk_simt.cuh -- phase 2 of the OSDN forward pass in fp32 FMA (SIMT) arithmetic.
//
// The chunkwise-parallel delta rule with write key K~ ("OSDN: Improving Delta Rule with
// Provable Online Preconditioning in Linear Attention", technical summary, section 2.1:
// K~ replaces K in the chunk Gram matrix and in the intra-chunk scores).  Within a chunk of C
// tokens starting from state S_0 (rows = value channels), with W the per-token writes
// (S_t = S_0 + sum_{s<=t} w_s k~_s^T):
//   w_t + beta_t sum_{s<t} (k_t . k~_s) w_s = beta_t (v_t - S_0 k_t)
//     => W = (I + L)^{-1} diag(beta) (V - K S_0^T),   L = strict_tril(diag(beta) K K~^T)
//   o_t = S_0 q_t + sum_{s<=t} (q_t . k~_s) w_s     (scores P = tril(Q K~^T), diagonal kept)
//   S_C = S_0 + W^T K~
// The unit-lower-triangular solve runs as a forward substitution per value column.
//
// One CTA per (sequence, head, block of BV value channels): rows of S are independent, so
// the value split is exact.  Everything lives in shared memory in fp32; this path serves the
// fp32-I/O mode (every product in fp32 FMA), any chunk size in {16, 32, 64}, and gated backbones.
//
// Gated backbones (decay alpha_t of the state's key channels before each write: Gated DeltaNet,
// one factor per token, or Kimi Delta Attention, one per key channel; the gated delta rule of the
// Gated DeltaNet-2 page, section 1, with OSDN's write key):
//   S_t = S_{t-1} D_t + beta_t (v_t - S_{t-1} D_t k_t) k~_t^T,   D_t = Diag(alpha_t).
// With lambda_t = sum of log alpha over the chunk's tokens up to t and Gamma_t = exp(lambda_t),
// the rescaled state S_t Gamma_t^-1 obeys the ungated recurrence with read key Gamma_t k_t,
// write key Gamma_t^-1 k~_t and query Gamma_t q_t, and S_end = S~_L Gamma_L.  Only decay ratios
// between two tokens (<= 1) enter the Gram matrices: Gram[t][j] = sum_i k_ti k~_ji
// exp(lambda_ti - lambda_ji).  They are evaluated as products of per-token factors scaled to a
// reference token in the chunk's middle when every factor stays inside fp32's range (|lambda -
// lambda_ref| < 80 over the chunk), else with one exponential per term.  After the Grams, K, Q
// and K~ are rescaled in place to Gamma K, Gamma Q and (Gamma_L / Gamma) K~ (all factors <= 1),
// and the ungated steps follow, with S decayed by Gamma_L before its update.
#pragma once

#include "common.cuh"

namespace osdn {

template <int DK, int BV, int C>
struct SimtSmem {
    static constexpr int KS = DK + 4;  // padded row stride: conflict-free float4 row reads
    static constexpr int AS = C + 1;
    static constexpr int oK = 0;
    static constexpr int oKt = oK + C * KS;
    static constexpr int oQ = oKt + C * KS;
    static constexpr int oS = oQ + C * KS;
    static constexpr int oV = oS + BV * KS;
    static constexpr int oW = oV + C * BV;
    static constexpr int oQS = oW + C * BV;
    static constexpr int oA = oQS + C * BV;
    static constexpr int oP = oA + C * AS;
    static constexpr int oB = oP + C * AS;
    static constexpr int oLam = oB + C;     // gated only: lambda [C][DK] (prefix of log alpha)
    static constexpr int oRef = oLam + C * DK;  // lambda at the reference token [DK], flag
    static constexpr int floats = oRef + DK + 4;
    static constexpr size_t bytes = sizeof(float) * floats;
};

__device__ __forceinline__ float dot_row(const float* __restrict__ a, const float* __restrict__ b,
                                         int n) {
    float s0 = 0.f, s1 = 0.f;
    for (int i = 0; i < n; i += 4) {
        const float4 x = *reinterpret_cast<const float4*>(a + i);
        const float4 y = *reinterpret_cast<const float4*>(b + i);
        s0 = fmaf(x.x, y.x, s0);
        s1 = fmaf(x.y, y.y, s1);
        s0 = fmaf(x.z, y.z, s0);
        s1 = fmaf(x.w, y.w, s1);
    }
    return s0 + s1;
}

template <int DK, int DV, int BV, int C, typename IO>
__global__ void __launch_bounds__(256)
chunk_fwd_simt_kernel(const IO* __restrict__ q, const IO* __restrict__ k,
                      const IO* __restrict__ kt, const IO* __restrict__ kt_lo,
                      const IO* __restrict__ v,
                      const float* __restrict__ beta, const float* __restrict__ alpha,
                      int alpha_per_channel, float scale, const float* __restrict__ S0,
                      IO* __restrict__ o, float* __restrict__ ST, const int32_t* __restrict__ cu,
                      int N, int T, int H) {
    using L = SimtSmem<DK, BV, C>;
    constexpr int NT = 256;
    constexpr int KS = L::KS, AS = L::AS;
    static_assert(BV == 32 && DV % BV == 0, "column solve assumes 32 value channels per CTA");
    extern __shared__ float4 smem_f4[];
    float* sm = reinterpret_cast<float*>(smem_f4);
    float* sK = sm + L::oK;
    float* sKt = sm + L::oKt;
    float* sQ = sm + L::oQ;
    float* sS = sm + L::oS;
    float* sV = sm + L::oV;
    float* sW = sm + L::oW;
    float* sQS = sm + L::oQS;
    float* sA = sm + L::oA;
    float* sP = sm + L::oP;
    float* sB = sm + L::oB;
    float* sLam = sm + L::oLam;
    float* sRef = sm + L::oRef;

    const int tid = threadIdx.x;
    constexpr int NVT = DV / BV;
    const int vt = blockIdx.x % NVT;
    const int nh = blockIdx.x / NVT;
    const int n = nh / H, h = nh - n * H;
    if (n >= N) return;
    int64_t first, count;
    if (!seq_range(cu, n, N, T, first, count)) return;
    const int c0 = vt * BV;
    const int64_t sbase = ((int64_t)n * H + h) * DV * DK + (int64_t)c0 * DK;

    for (int idx = tid; idx < BV * DK; idx += NT) {
        const int c = idx / DK, i = idx - c * DK;
        sS[c * KS + i] = S0 ? __ldg(S0 + sbase + idx) : 0.f;
    }

    for (int64_t cs = 0; cs < count; cs += C) {
        const int Lc = (count - cs) < C ? (int)(count - cs) : C;
        __syncthreads();  // previous chunk's readers are done
        // ---- load the chunk (rows past the tail are zero, so they write nothing)
        for (int idx = tid; idx < C * (DK / 4); idx += NT) {
            const int t = idx / (DK / 4), i = (idx - t * (DK / 4)) * 4;
            float4 xq = make_float4(0.f, 0.f, 0.f, 0.f), xk = xq, xt = xq;
            if (t < Lc) {
                const int64_t off = ((first + cs + t) * H + h) * DK + i;
                xq = load4<IO>(q + off);
                xk = load4<IO>(k + off);
                xt = load4<IO>(kt + off);
                if (kt_lo) {  // k~ handed over as io-dtype hi + lo terms
                    const float4 xl = load4<IO>(kt_lo + off);
                    xt.x += xl.x;
                    xt.y += xl.y;
                    xt.z += xl.z;
                    xt.w += xl.w;
                }
            }
            *reinterpret_cast<float4*>(sQ + t * KS + i) = xq;
            *reinterpret_cast<float4*>(sK + t * KS + i) = xk;
            *reinterpret_cast<float4*>(sKt + t * KS + i) = xt;
        }
        for (int idx = tid; idx < C * (BV / 2); idx += NT) {
            const int t = idx / (BV / 2), c = (idx - t * (BV / 2)) * 2;
            float2 xv = make_float2(0.f, 0.f);
            if (t < Lc) xv = load2<IO>(v + ((first + cs + t) * H + h) * DV + c0 + c);
            *reinterpret_cast<float2*>(sV + t * BV + c) = xv;
        }
        for (int t = tid; t < C; t += NT) sB[t] = t < Lc ? __ldg(beta + (first + cs + t) * H + h) : 0.f;
        if (alpha) {  // lambda = prefix of log alpha per key channel (alpha = 1 past the end)
            for (int i = tid; i < DK; i += NT) {
                float lam = 0.f;
                for (int t = 0; t < C; ++t) {
                    float a = 1.f;
                    if (t < Lc) {
                        const int64_t th = (first + cs + t) * H + h;
                        a = __ldg(alpha + (alpha_per_channel ? th * DK + i : th));
                    }
                    lam += __logf(a);
                    sLam[t * DK + i] = lam;
                }
                sRef[i] = sLam[(C / 2) * DK + i];
            }
        }
        __syncthreads();
        bool factored = false;  // gated: Gram ratios as products of reference-scaled factors
        if (alpha) {
            bool far = false;
            for (int idx = tid; idx < C * DK; idx += NT) {
                const int i = idx % DK;
                far |= fabsf(sLam[idx] - sRef[i]) >= 80.f;
            }
            factored = !__syncthreads_or(far);
            if (factored) {
                for (int idx = tid; idx < C * DK; idx += NT) {
                    const int t = idx / DK, i = idx - t * DK;
                    const float dl = sLam[idx] - sRef[i];
                    const float up = __expf(dl), dn = __expf(-dl);
                    sK[t * KS + i] *= up;
                    sQ[t * KS + i] *= up;
                    sKt[t * KS + i] *= dn;
                }
                __syncthreads();
            }
        }

        // ---- Gram (strictly lower, beta-scaled rows) and intra-chunk scores (lower incl.)
        for (int idx = tid; idx < C * C; idx += NT) {
            const int t = idx / C, j = idx - t * C;
            float a = 0.f, p = 0.f;
            if (alpha && !factored) {  // one exponential per term: sum_i x_ti k~_ji e^(lam_ti - lam_ji)
                if (j <= t) {
                    const float* lt = sLam + t * DK;
                    const float* lj = sLam + j * DK;
                    for (int i = 0; i < DK; ++i) {
                        const float e = __expf(lt[i] - lj[i]) * sKt[j * KS + i];
                        a = fmaf(sK[t * KS + i], e, a);
                        p = fmaf(sQ[t * KS + i], e, p);
                    }
                    a = j < t ? sB[t] * a : 0.f;
                }
            } else {
                if (j < t) a = sB[t] * dot_row(sK + t * KS, sKt + j * KS, DK);
                if (j <= t) p = dot_row(sQ + t * KS, sKt + j * KS, DK);
            }
            sA[t * AS + j] = a;
            sP[t * AS + j] = p;
        }
        if (alpha) {  // K -> Gamma K, Q -> Gamma Q, K~ -> (Gamma_L / Gamma) K~; S -> S Gamma_L below
            __syncthreads();
            const float* lamL = sLam + (C - 1) * DK;
            for (int idx = tid; idx < C * DK; idx += NT) {
                const int t = idx / DK, i = idx - t * DK;
                const float lam = sLam[idx];
                // factored: K and Q already carry exp(lam - ref), K~ carries exp(ref - lam)
                const float gk = factored ? __expf(sRef[i]) : __expf(lam);
                const float gt = factored ? __expf(lamL[i] - sRef[i]) : __expf(lamL[i] - lam);
                sK[t * KS + i] *= gk;
                sQ[t * KS + i] *= gk;
                sKt[t * KS + i] *= gt;
            }
            __syncthreads();
        }
        // ---- right-hand side beta (V - K S0^T) and the readout Q S0^T
        for (int idx = tid; idx < C * BV; idx += NT) {
            const int t = idx / BV, c = idx - t * BV;
            const float ks = dot_row(sK + t * KS, sS + c * KS, DK);
            const float qs = dot_row(sQ + t * KS, sS + c * KS, DK);
            sW[t * BV + c] = sB[t] * (sV[t * BV + c] - ks);
            sQS[t * BV + c] = qs;
        }
        __syncthreads();

        // ---- forward substitution W[t] -= sum_{j<t} A[t][j] W[j], column by column.
        // Warp w owns columns 4w..4w+3; 8 lanes share one column's sums.
        {
            const int warp = tid >> 5, lane = tid & 31;
            const int c = warp * 4 + (lane >> 3), p = lane & 7;
            for (int t = 1; t < Lc; ++t) {
                float part = 0.f;
                for (int j = p; j < t; j += 8) part = fmaf(sA[t * AS + j], sW[j * BV + c], part);
                part += __shfl_xor_sync(0xffffffffu, part, 1);
                part += __shfl_xor_sync(0xffffffffu, part, 2);
                part += __shfl_xor_sync(0xffffffffu, part, 4);
                if (p == 0) sW[t * BV + c] -= part;
                __syncwarp();
            }
        }
        __syncthreads();

        // ---- outputs o_t = scale (Q S0^T + P W)_t  and state update S += W^T K~
        for (int idx = tid; idx < C * (BV / 2); idx += NT) {
            const int t = idx / (BV / 2), c = (idx - t * (BV / 2)) * 2;
            if (t < Lc) {
                float a0 = sQS[t * BV + c], a1 = sQS[t * BV + c + 1];
                for (int j = 0; j <= t; ++j) {
                    const float pj = sP[t * AS + j];
                    a0 = fmaf(pj, sW[j * BV + c], a0);
                    a1 = fmaf(pj, sW[j * BV + c + 1], a1);
                }
                if (OSDN_IN_BOUNDS(first + cs + t, cu ? (int64_t)T : (int64_t)N * T))
                    store2<IO>(o + ((first + cs + t) * H + h) * DV + c0 + c,
                               make_float2(scale * a0, scale * a1));
            }
        }
        for (int idx = tid; idx < BV * DK; idx += NT) {
            const int c = idx / DK, i = idx - c * DK;
            float acc = 0.f;
            for (int t = 0; t < Lc; ++t) acc = fmaf(sW[t * BV + c], sKt[t * KS + i], acc);
            if (alpha) sS[c * KS + i] *= __expf(sLam[(C - 1) * DK + i]);  // S Gamma_L
            sS[c * KS + i] += acc;
        }
    }
    __syncthreads();
    if (ST) {
        for (int idx = tid; idx < BV * DK; idx += NT) {
            const int c = idx / DK, i = idx - c * DK;
            ST[sbase + idx] = sS[c * KS + i];
        }
    }
}

}  // namespace osdn
