// step.cuh -- one recurrent OSDN step per (sequence, head): the decode path.
//
// "OSDN: Improving Delta Rule with Provable Online Preconditioning in Linear Attention",
// technical summary, sections 2.1-2.3, applied to a single token with the state carried in
// HBM.  With a = k (.) k, nk = ||k||^2, s = <d, a>:
//   k~ = d (.) k,   u = v - S k,   S <- S + beta u k~^T,   o = scale * S q,
//   d  <- r d + eta beta (1 - beta s) a / nk   (0 when nk = 0),
// and optionally the residual-contraction ratio (1 - beta s)^2 of the write (section 3).
// On a gated backbone (Gated DeltaNet: one decay factor per token and head; Kimi Delta
// Attention: one per key channel) the state's key channels first decay, S <- S Diag(alpha), and
// the step above runs on the decayed state: the gated delta rule of the Gated DeltaNet-2 page
// (section 1) with OSDN's write key; the preconditioner is unchanged.
// The step reads and writes the fp32 state once (Dv x Dk x 4 bytes each way) and a few hundred
// bytes of token data: it is bound by HBM bandwidth.
//
// One CTA of Dv / 8 warps per (sequence, head).  Warp w owns the 8 state rows (value channels)
// w, w + Dv/8, ...; lane l holds key channels [4l, 4l + 4) (Dk = 128) or [2l, 2l + 2) (Dk = 64).
// Every row load is issued before the first use, so each warp keeps 8 row loads in flight.
// Plain cached accesses: a decode batch's states (64 KB per head) can stay in L2 between steps.
#pragma once

#include "common.cuh"

namespace osdn {

// Threads per CTA for a value dimension DV: one warp per 8 state rows.
constexpr int step_threads(int DV) { return DV * 4; }

template <int N> struct vecf;
template <> struct vecf<4> {
    using T = float4;
    static __device__ __forceinline__ void load(const float* p, float* x) {
        const float4 v = *reinterpret_cast<const float4*>(p);
        x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    }
    static __device__ __forceinline__ void store(float* p, const float* x) {
        *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
    }
};
template <> struct vecf<2> {
    using T = float2;
    static __device__ __forceinline__ void load(const float* p, float* x) {
        const float2 v = *reinterpret_cast<const float2*>(p);
        x[0] = v.x; x[1] = v.y;
    }
    static __device__ __forceinline__ void store(float* p, const float* x) {
        *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
    }
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

template <int DK, int DV, typename IO>
__global__ void __launch_bounds__(DV * 4)
osdn_step_kernel(const IO* __restrict__ q, const IO* __restrict__ k, const IO* __restrict__ v,
                 const float* __restrict__ beta, const float* __restrict__ r, float eta,
                 float scale, float* __restrict__ S, float* __restrict__ d, IO* __restrict__ o,
                 IO* __restrict__ k_tilde, float* __restrict__ rho, const float* __restrict__ alpha,
                 int alpha_per_channel, int NH) {
    constexpr int PL = DK / 32;             // key channels per lane
    constexpr int NW = DV / 8;              // warps
    constexpr int ROWS = 8;                 // state rows per warp
    using tr = io_traits<IO>;
    const int nh = blockIdx.x;
    if (nh >= NH) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float* Sh = S + (int64_t)nh * DV * DK;
    // state rows first: the bulk of the traffic, in flight while the token data arrives
    float srow[ROWS][PL];
#pragma unroll
    for (int i = 0; i < ROWS; ++i) vecf<PL>::load(Sh + (int64_t)(warp + NW * i) * DK + PL * lane, srow[i]);
    float kk[PL], qq[PL], dd[PL];
#pragma unroll
    for (int j = 0; j < PL; ++j) {
        kk[j] = tr::to_f32(k[(int64_t)nh * DK + PL * lane + j]);
        qq[j] = tr::to_f32(q[(int64_t)nh * DK + PL * lane + j]);
        dd[j] = d[(int64_t)nh * DK + PL * lane + j];
    }
    const float bt = beta[nh];
    if (alpha) {  // decay of the key channels, before the write
        float av[PL];
#pragma unroll
        for (int j = 0; j < PL; ++j)
            av[j] = alpha_per_channel ? alpha[(int64_t)nh * DK + PL * lane + j] : alpha[nh];
#pragma unroll
        for (int i = 0; i < ROWS; ++i)
#pragma unroll
            for (int j = 0; j < PL; ++j) srow[i][j] *= av[j];
    }
    float kt[PL], nk = 0.f, sa = 0.f;
#pragma unroll
    for (int j = 0; j < PL; ++j) {
        const float a = kk[j] * kk[j];
        kt[j] = dd[j] * kk[j];
        nk += a;
        sa = fmaf(dd[j], a, sa);
    }
    // u_i = v_i - S_i k, S_i += beta u_i k~, o_i = scale S_i q  (row i = warp + NW i)
#pragma unroll
    for (int i = 0; i < ROWS; ++i) {
        float sk = 0.f;
#pragma unroll
        for (int j = 0; j < PL; ++j) sk = fmaf(srow[i][j], kk[j], sk);
        sk = warp_sum(sk);
        const int row = warp + NW * i;
        const float u = bt * (tr::to_f32(v[(int64_t)nh * DV + row]) - sk);
        float sq = 0.f;
#pragma unroll
        for (int j = 0; j < PL; ++j) {
            srow[i][j] = fmaf(u, kt[j], srow[i][j]);
            sq = fmaf(srow[i][j], qq[j], sq);
        }
        vecf<PL>::store(Sh + (int64_t)row * DK + PL * lane, srow[i]);
        sq = warp_sum(sq);
        if (lane == 0) o[(int64_t)nh * DV + row] = tr::from_f32(scale * sq);
    }
    __syncthreads();  // every warp has read d before it is overwritten
    if (warp == 0) {
        nk = warp_sum(nk);
        sa = warp_sum(sa);
        const float rt = r ? r[nh] : 1.f;
        const float g = nk > 0.f ? eta * bt * (1.f - bt * sa) / nk : 0.f;
        if (rho && lane == 0) rho[nh] = (1.f - bt * sa) * (1.f - bt * sa);
#pragma unroll
        for (int j = 0; j < PL; ++j) {
            if (k_tilde) k_tilde[(int64_t)nh * DK + PL * lane + j] = tr::from_f32(kt[j]);
            d[(int64_t)nh * DK + PL * lane + j] = fmaf(rt, dd[j], g * kk[j] * kk[j]);
        }
    }
}

}  // namespace osdn
