// rho_geomean.cuh -- q_geo, the geometric mean of the residual-contraction ratios of one
// (sequence, head): q_geo = exp(mean_t log rho_t).
//
// "OSDN: Improving Delta Rule with Provable Online Preconditioning in Linear Attention",
// technical summary: section 3 (Theorem 5.2) bounds the product of the token-local residual
// ratios rho_t = f_t(S_t) / f_t(S_{t-1}); the experiments (section 4.3) report their geometric
// mean q_geo.  rho comes from osdn_precond_scan / osdn_fwd (rho_t = (1 - beta_t <d_t, k_t^2>)^2).
#pragma once

#include "common.cuh"

namespace osdn {

constexpr int GEOMEAN_THREADS = 256;

// One CTA per (sequence, head).  Logs in fp32, their sum in fp64.  A ratio of 0 gives
// log 0 = -inf and q_geo = 0; a sequence without tokens gets 1 (the empty product).
__global__ void __launch_bounds__(GEOMEAN_THREADS)
rho_geomean_kernel(const float* __restrict__ rho, const int32_t* __restrict__ cu, int N, int T,
                   int H, float* __restrict__ q_geo) {
    __shared__ double part[GEOMEAN_THREADS / 32];
    const int n = blockIdx.x / H, h = blockIdx.x - n * H;
    if (n >= N) return;
    int64_t first, count;
    if (!seq_range(cu, n, N, T, first, count)) return;  // uniform over the CTA
    double acc = 0.0;
    for (int64_t t = threadIdx.x; t < count; t += GEOMEAN_THREADS)
        acc += (double)__logf(__ldg(rho + (first + t) * H + h));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double s = 0.0;
#pragma unroll
        for (int w = 0; w < GEOMEAN_THREADS / 32; ++w) s += part[w];
        q_geo[(int64_t)n * H + h] = count > 0 ? (float)exp(s / (double)count) : 1.0f;
    }
}

}  // namespace osdn
