// chunk_prep.cuh -- the WY factor of every phase-2 chunk, computed for all chunks at once.
//
// The chunkwise delta rule with write key K~ ("OSDN: Improving Delta Rule with Provable Online
// Preconditioning in Linear Attention", technical summary, section 2.1) needs, per chunk of 64
// tokens with rows K, K~ and gates beta,
//   T = (I + strict_tril(diag(beta) K K~^T))^-1,
// which does not depend on the state.  wy_prep_kernel computes it for every chunk in parallel:
// K K~^T by bf16 MMAs (both operands are exact bf16 -- K~ as one term, or as the hi + lo terms
// phase 1 hands over inside osdn_fwd -- so the fp32 accumulation is the only rounding), the
// inverse by tril_inverse_64_g128.  The sequential kernel (chunk_tc.cuh) then only reads T.
//
// Hand-off through the output buffer o, which the sequential kernel writes only after reading
// T: each 128-value (256-byte) row of o for a head holds two 128-byte slices, and row t of a
// chunk's slices receives row t of T split into bf16 terms, T = hi + lo -- hi in slice 0, lo in
// slice 1 -- already laid out as a 128-byte-swizzled K-major MMA operand (16-byte group g of
// row t at group position g ^ (t mod 8)).  The sequential kernel loads both slices with TMA
// straight into its operand tiles.  A chunk of Lc < 64 tokens has Lc rows of o, so only rows
// t < Lc are written; the reader completes the tile with identity rows.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "tc_ptx.cuh"
#include "tril_inverse.cuh"
#include "chunk_walk.cuh"

namespace osdn {

struct WyPrepSmem {
    static constexpr uint32_t K = 0;            // bf16 K tile: 2 K-blocks x (64 rows x 128 B)
    static constexpr uint32_t KT = 16384;       // bf16 K~ tile (hi term), same layout
    static constexpr uint32_t KTLO = 32768;     // bf16 K~ lo term (when handed over), same layout
    static constexpr uint32_t SL = 49152;       // fp32 L, then T in place (tsw)
    static constexpr uint32_t BETA = 65536;     // 64 floats
    static constexpr uint32_t BAR = BETA + 256;
    static constexpr uint32_t TMEM_SLOT = BAR + 16;
    static constexpr uint32_t TOTAL = TMEM_SLOT + 16;
    static constexpr size_t BYTES = TOTAL + 1024;
};
constexpr int WY_PREP_CTAS_PER_SM = 3;

// Persistent grid of 128-thread CTAs walking the batch's chunks (ChunkWalk).  o_f32 is the
// output buffer [rows, H, Dv] (bf16) seen as floats; Dv = 128.
__global__ void __launch_bounds__(128, WY_PREP_CTAS_PER_SM)
wy_prep_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_kt,
               const __grid_constant__ CUtensorMap tm_ktlo, int has_lo,
               const float* __restrict__ beta, float* __restrict__ o_f32, int Dv,
               const int32_t* __restrict__ cu, int N, int T, int H, int64_t rows,
               long long limit_ns) {
    using L = WyPrepSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_align1024(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5;
    ChunkWalk walk;
    walk.init(cu, N, T, H, rows);
    if (!walk.next()) return;  // uniform over the CTA

    uint64_t* tma_bar = reinterpret_cast<uint64_t*>(smem + L::BAR);
    uint64_t* mma_bar = tma_bar + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::TMEM_SLOT);
    uint8_t* sK = smem + L::K;
    uint8_t* sKT = smem + L::KT;
    uint8_t* sKTLO = smem + L::KTLO;
    float* sL = reinterpret_cast<float*>(smem + L::SL);
    float* sBeta = reinterpret_cast<float*>(smem + L::BETA);

    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, 64);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(tma_bar, 1);
        mbar_init(mma_bar, 1);
        tc::fence_mbar_init();
        tc::prefetch_tmap(&tm_k);
        tc::prefetch_tmap(&tm_kt);
        if (has_lo) tc::prefetch_tmap(&tm_ktlo);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tlane = static_cast<uint32_t>(warp * 32) << 16;

    auto issue_load = [&](int64_t row, int hh) {
        tc::mbar_expect_tx(tma_bar, has_lo ? 49152 : 32768);
        tc::tma_load_3d(sK, &tm_k, 0, hh, (int)row, tma_bar);
        tc::tma_load_3d(sK + 8192, &tm_k, 64, hh, (int)row, tma_bar);
        tc::tma_load_3d(sKT, &tm_kt, 0, hh, (int)row, tma_bar);
        tc::tma_load_3d(sKT + 8192, &tm_kt, 64, hh, (int)row, tma_bar);
        if (has_lo) {
            tc::tma_load_3d(sKTLO, &tm_ktlo, 0, hh, (int)row, tma_bar);
            tc::tma_load_3d(sKTLO + 8192, &tm_ktlo, 64, hh, (int)row, tma_bar);
        }
    };
    auto load_beta = [&](int64_t row, int Lc, int hh) {
        return tid < Lc ? __ldg(beta + (row + tid) * H + hh) : 0.f;
    };
    if (tid == 0) issue_load(walk.row0, walk.h);
    float bnext = tid < 64 ? load_beta(walk.row0, walk.Lc, walk.h) : 0.f;
    bool tma_pend = tid == 0, mma_pend = false, fail = false, more = true;
    uint32_t tph = 0, mph = 0;
    // M = 128 over the K tile: rows 64..127 of the operand view are the next 64 rows of shared
    // memory (finite data), whose products land in TMEM lanes 64..127 and are never read
    constexpr uint32_t ID_G = tc::idesc(1, 0, 0, 128, 64);
    const int half_f = Dv / 2;

#pragma unroll 1
    while (more) {
        const int64_t row0 = walk.row0;
        const int Lc = walk.Lc, h = walk.h;
        if (tid < 64) sBeta[tid] = bnext;
        const bool got = mbar_wait_bounded(tma_bar, tph, limit_ns);
        if (__syncthreads_or(!got)) {
            fail = true;
            break;
        }
        tph ^= 1u;
        tma_pend = false;
        if (tid == 0) {
            tc::fence_after_sync();
            const uint32_t aK = smem_u32(sK), aKT = smem_u32(sKT), aKTLO = smem_u32(sKTLO);
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const uint32_t o = (s >> 2) * 8192u + (s & 3) * 32u;
                tc::mma_bf16(tmem, tc::sw128_desc(aK + o, 16, 1024), tc::sw128_desc(aKT + o, 16, 1024),
                             ID_G, s > 0);
            }
            if (has_lo) {  // K K~^T = K K~_hi^T + K K~_lo^T
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    const uint32_t o = (s >> 2) * 8192u + (s & 3) * 32u;
                    tc::mma_bf16(tmem, tc::sw128_desc(aK + o, 16, 1024),
                                 tc::sw128_desc(aKTLO + o, 16, 1024), ID_G, 1);
                }
            }
            tc::mma_commit(mma_bar);
            mma_pend = true;
        }
        more = walk.next();  // uniform: every thread walks the same items
        if (more && tid < 64) bnext = load_beta(walk.row0, walk.Lc, walk.h);
        const bool mdone = mbar_wait_bounded(mma_bar, mph, limit_ns);
        if (__syncthreads_or(!mdone)) {
            fail = true;
            break;
        }
        mph ^= 1u;
        mma_pend = false;
        tc::fence_after_sync();
        if (tid == 0 && more) {  // the tiles have been consumed by the MMA: fetch the next chunk's
            issue_load(walk.row0, walk.h);
            tma_pend = true;
        }
        // ---- L[t][j] = beta_t (K K~^T)[t][j] for j < t (lanes 0..63 = rows)
        if (warp < 2) {
            const float bt = sBeta[tid];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float g[16];
                tc::tmem_ld16(tmem + tlane + 16 * q, g);
                tc::tmem_ld_wait();
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const int j = 16 * q + 4 * v;
                    tsw_st4(sL, tid, 4 * q + v,
                            make_float4(j < tid ? bt * g[4 * v] : 0.f, j + 1 < tid ? bt * g[4 * v + 1] : 0.f,
                                        j + 2 < tid ? bt * g[4 * v + 2] : 0.f,
                                        j + 3 < tid ? bt * g[4 * v + 3] : 0.f));
                }
            }
        }
        tc::fence_before_sync();
        __syncthreads();
        tril_inverse_64_g128(sL, tid, 1);  // T over L
        // ---- T rows t < Lc as bf16 hi / lo operand rows (thread: row tid mod 64, half tid / 64 of
        //      its 16-byte groups), into the chunk's o rows
        {
            const int r = tid & 63, g0 = 4 * (tid >> 6);
            if (r < Lc && OSDN_IN_BOUNDS(row0 + r, rows)) {
                uint8_t* orow = reinterpret_cast<uint8_t*>(o_f32 + ((row0 + r) * H + h) * half_f);
#pragma unroll
                for (int g = g0; g < g0 + 4; ++g) {
                    uint32_t hw[4], lw[4];
                    // columns 8 g .. 8 g + 7 as two 16-byte loads (the lanes of a warp, on
                    // consecutive rows, meet each bank at most four times: the minimum for 512 B)
                    const float4 va = tsw_ld4(sL, r, 2 * g), vb = tsw_ld4(sL, r, 2 * g + 1);
                    const float tv[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int c = 8 * g + 2 * e;
                        const float a = c < r ? tv[2 * e] : (c == r ? 1.f : 0.f);
                        const float b = c + 1 < r ? tv[2 * e + 1] : (c + 1 == r ? 1.f : 0.f);
                        const __nv_bfloat162 hb = __floats2bfloat162_rn(a, b);
                        const float2 hf = __bfloat1622float2(hb);
                        const float2 ld = __ffma2_rn(hf, make_float2(-1.f, -1.f), make_float2(a, b));
                        const __nv_bfloat162 lb = __floats2bfloat162_rn(ld.x, ld.y);
                        hw[e] = *reinterpret_cast<const uint32_t*>(&hb);
                        lw[e] = *reinterpret_cast<const uint32_t*>(&lb);
                    }
                    const int pos = (g ^ (r & 7)) << 4;
                    *reinterpret_cast<uint4*>(orow + pos) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                    *reinterpret_cast<uint4*>(orow + 128 + pos) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
                }
            }
        }
        __syncthreads();  // sL is rewritten by the next chunk
    }
    if (fail && tid == 0) {
        if (tma_pend) mbar_wait_bounded(tma_bar, tph, limit_ns);
        if (mma_pend) mbar_wait_bounded(mma_bar, mph, limit_ns);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 64);
}

}  // namespace osdn
