// scan_warp.cuh -- phase 1 of the OSDN forward pass, one warp per (sequence, head).
//
// Preconditioner scan of "OSDN: Improving Delta Rule with Provable Online Preconditioning in
// Linear Attention" (technical summary, section 2.2: two-phase split, closed-form surrogate
// and its gradient; section 2.3: APF retention gate on d).  Per token, with a = k (.) k:
//   k~_t    = d_t (.) k_t
//   d_{t+1} = r_t d_t + eta * beta_t (1 - beta_t <d_t, a_t>) a_t / ||k_t||^2
// (gradient descent on the surrogate; the step is zero when ||k_t|| == 0).
//
// Each lane owns DK/32 consecutive channels of d in registers.  The only cross-lane work per
// token is one butterfly reduction that carries both <d, a> (on the serial chain) and ||k||^2
// (off it).  Keys, gates and retention values are prefetched PF tokens ahead into registers,
// so the loop is bound by the reduction latency, not by HBM.
#pragma once

#include "common.cuh"

namespace osdn {

template <int DK, typename IO>
__global__ void __launch_bounds__(128)
precond_scan_warp_kernel(const IO* __restrict__ k, const float* __restrict__ beta,
                         const float* __restrict__ r, float eta, const float* __restrict__ d0,
                         IO* __restrict__ k_tilde, IO* __restrict__ k_tilde_lo,
                         float* __restrict__ d_all, float* __restrict__ dT, float* __restrict__ rho,
                         const int32_t* __restrict__ cu, int N, int T, int H) {
    static_assert(DK == 64 || DK == 128, "DK");
    constexpr int E = DK / 32;  // consecutive channels per lane
    constexpr int PF = 8;       // prefetch depth in tokens
    const int lane = threadIdx.x & 31;
    const int unit = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (unit >= N * H) return;
    const int n = unit / H, h = unit - n * H;
    int64_t first, count;
    if (!seq_range(cu, n, N, T, first, count)) return;

    float d[E];
    const int64_t dbase = ((int64_t)n * H + h) * DK + lane * E;
#pragma unroll
    for (int e = 0; e < E; ++e) d[e] = d0 ? __ldg(d0 + dbase + e) : 1.0f;

    const int64_t rs = (int64_t)H * DK;  // row stride between tokens
    const IO* kp = k + (first * H + h) * DK + lane * E;
    IO* ktp = k_tilde + (first * H + h) * DK + lane * E;
    IO* klp = k_tilde_lo ? k_tilde_lo + (first * H + h) * DK + lane * E : nullptr;
    const float* bp = beta + first * H + h;
    const float* rp = r ? r + first * H + h : nullptr;

    float kb[PF][E], bb[PF], rb[PF];
    auto fetch = [&](int slot, int64_t t) {
        if (t < count) {
            if constexpr (E == 4) {
                const float4 x = load4<IO>(kp + t * rs);
                kb[slot][0] = x.x; kb[slot][1] = x.y; kb[slot][2] = x.z; kb[slot][3] = x.w;
            } else {
                const float2 x = load2<IO>(kp + t * rs);
                kb[slot][0] = x.x; kb[slot][1] = x.y;
            }
            bb[slot] = __ldg(bp + t * H);
            rb[slot] = rp ? __ldg(rp + t * H) : 1.0f;
        }
    };
#pragma unroll
    for (int p = 0; p < PF; ++p) fetch(p, p);

    for (int64_t t0 = 0; t0 < count; t0 += PF) {
#pragma unroll
        for (int p = 0; p < PF; ++p) {
            const int64_t t = t0 + p;
            if (t < count) {
                float kk[E];
#pragma unroll
                for (int e = 0; e < E; ++e) kk[e] = kb[p][e];
                const float bt = bb[p], rt = rb[p];
                fetch(p, t + PF);

                float a[E], nk = 0.f, s = 0.f, kt[E];
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    a[e] = kk[e] * kk[e];
                    nk += a[e];
                    s = fmaf(d[e], a[e], s);
                    kt[e] = d[e] * kk[e];
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    s += __shfl_xor_sync(0xffffffffu, s, off);
                    nk += __shfl_xor_sync(0xffffffffu, nk, off);
                }
                if constexpr (E == 4)
                    store4<IO>(ktp + t * rs, make_float4(kt[0], kt[1], kt[2], kt[3]));
                else
                    store2<IO>(ktp + t * rs, make_float2(kt[0], kt[1]));
                if (klp) {  // the io rounding's residual: k~ = hi + lo to about 2^-17 in bf16
                    float lo[E];
#pragma unroll
                    for (int e = 0; e < E; ++e)
                        lo[e] = kt[e] - io_traits<IO>::to_f32(io_traits<IO>::from_f32(kt[e]));
                    if constexpr (E == 4)
                        store4<IO>(klp + t * rs, make_float4(lo[0], lo[1], lo[2], lo[3]));
                    else
                        store2<IO>(klp + t * rs, make_float2(lo[0], lo[1]));
                }
                if (rho && lane == 0) rho[(first + t) * H + h] = (1.f - bt * s) * (1.f - bt * s);
                if (d_all) {  // the preconditioner this token wrote with
                    float* dp = d_all + ((first + t) * H + h) * DK + lane * E;
#pragma unroll
                    for (int e = 0; e < E; ++e) dp[e] = d[e];
                }
                const float coef = nk > 0.f ? eta * bt * (1.0f - bt * s) / nk : 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e) d[e] = fmaf(rt, d[e], coef * a[e]);
            }
        }
    }
    if (dT) {
#pragma unroll
        for (int e = 0; e < E; ++e) dT[dbase + e] = d[e];
    }
}

}  // namespace osdn
