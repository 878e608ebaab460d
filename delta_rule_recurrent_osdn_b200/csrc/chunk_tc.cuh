// chunk_tc.cuh -- phase 2 of the OSDN forward pass on the sm_100a tensor cores (bf16 I/O).
//
// The chunkwise delta rule with write key K~ ("OSDN: Improving Delta Rule with Provable Online
// Preconditioning in Linear Attention", technical summary, section 2.1: K~ replaces K in the
// chunk Gram matrix and in the intra-chunk scores).  Per chunk of C = 64 tokens, state S_0
// (value rows), this CTA's 64 value channels:
//   G = K K~^T,  P = tril(Q K~^T)                 one bf16 MMA, A = [K; Q] (M = 128)
//   T = (I + strict_tril(diag(beta) G))^-1        fp32 blocked solve in shared memory
//   R = diag(beta) (V - K S_0^T)                  A = [K; Q], B = S_0^T  (rows 64..127: Q S_0^T)
//   W = T R                                       A = Z = [T; P], B = R
//   O = Q S_0^T + P W                             A = Z, B = W, accumulated onto Q S_0^T
//   S_C^T = S_0^T + K~^T W                        A = K~^T (MN-major view of the K~ tile)
//
// Precision.  Every computed MMA operand x is split into two bf16 terms, x = hi + lo (about 16
// significant bits).  A product of an exact bf16 input (K, Q, K~) with a computed operand takes
// two MMAs (hi, lo); a product of two computed operands ([T; P] with R or W) takes three
// (hi*hi + hi*lo + lo*hi).  In a CPU emulation of this chunk algorithm against the oracle, plain
// bf16 operands gave 1.5-2.5% max/rms error on o and S_T for the 340M and 1.3B workloads, and
// single-term tf32 products 0.25-0.46%; the split scheme is at the fp32 rounding level.
//
// Layout.  One CTA per (sequence, head, 64 value channels), 128 threads: thread t owns tensor
// memory lane t.  Accumulators in tensor memory (fp32, 128 lanes): S^T (lanes = key channel),
// D1 = [K S^T; Q S^T] then O, D2 = [W; P R], DG = [G; P].  Operand tiles in shared memory use
// the 128-byte swizzle that TMA writes; the K~ tile serves as the K-major B operand of the Gram
// MMA and as the MN-major A operand of the state update.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace osdn {

struct TcSmem {
    static constexpr uint32_t STAGE = 57344;          // [K;Q] 32K | K~ 16K | V 8K
    static constexpr uint32_t KQ = 0, KT = 32768, V = 49152;
    // bf16 [T; P] hi and lo, K-major, 128 rows x 128 B each.  While T is being solved it is
    // held in fp32 in rows 0..63 of both tiles (the bytes of z_off(r < 64, c)).
    static constexpr uint32_t ZHI = 2 * STAGE;
    static constexpr uint32_t ZLO = ZHI + 16384;
    static constexpr uint32_t SHI = ZLO + 16384;      // bf16 S^T hi, 128 rows x 128 B
    static constexpr uint32_t SLO = SHI + 16384;
    static constexpr uint32_t RHI = SLO + 16384;      // bf16 R hi / lo, 64 rows x 128 B
    static constexpr uint32_t RLO = RHI + 8192;
    static constexpr uint32_t WHI = RLO + 8192;       // bf16 W hi / lo, 64 rows x 128 B
    static constexpr uint32_t WLO = WHI + 8192;
    static constexpr uint32_t SOLVE = RHI;            // fp32 L and M scratch (64 x 65 each)
    static constexpr uint32_t SOLVE_END = SOLVE + 2 * 64 * 65 * 4;
    static constexpr uint32_t BAR = SOLVE_END;        // 3 mbarriers
    static constexpr uint32_t TMEM_SLOT = BAR + 32;
    static constexpr uint32_t TOTAL = TMEM_SLOT + 16;
    static constexpr size_t BYTES = TOTAL + 1024;     // + alignment slack
};
static_assert(TcSmem::SOLVE_END >= TcSmem::WLO + 8192, "solve scratch overlays R/W tiles");
static_assert(TcSmem::BYTES <= 232448, "shared memory");

constexpr uint32_t TC_COL_S = 0, TC_COL_D1 = 64, TC_COL_D2 = 128, TC_COL_G = 192;
constexpr uint32_t TC_TMEM_COLS = 256;

// fp32 element (r, c), r < 64, of T while it is being solved: 32 fp32 per 128-byte row, the
// two 32-column halves in the hi and lo tiles.
__device__ __forceinline__ uint32_t z_off(uint32_t r, uint32_t c) {
    return (c >> 5) * 16384u + tc::sw128_off(r, (c & 31u) >> 2) + (c & 3u) * 4u;
}

// Split a 64-value fp32 row into bf16 hi + lo and write both rows (128 B each, swizzled).
__device__ __forceinline__ void st_row_split_bf16(uint8_t* hi, uint8_t* lo, uint32_t row,
                                                  const float* x) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        uint32_t h[4], l[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float a = x[8 * j + 2 * e], b = x[8 * j + 2 * e + 1];
            const __nv_bfloat162 ha = __floats2bfloat162_rn(a, b);
            const float2 hf = __bfloat1622float2(ha);
            const __nv_bfloat162 la = __floats2bfloat162_rn(a - hf.x, b - hf.y);
            h[e] = *reinterpret_cast<const uint32_t*>(&ha);
            l[e] = *reinterpret_cast<const uint32_t*>(&la);
        }
        const uint32_t off = tc::sw128_off(row, j);
        *reinterpret_cast<uint4*>(hi + off) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4*>(lo + off) = make_uint4(l[0], l[1], l[2], l[3]);
    }
}

// T = (I + L)^-1 for a strictly lower 64x64 L (fp32, stride 65), written into rows 0..63 of the
// [T; P] tile.  Diagonal 16x16 blocks by forward substitution, then the off-diagonal blocks by
// distance from the diagonal: T_IJ = -T_II * sum_{m=J}^{I-1} L_Im T_mJ.
__device__ __forceinline__ void solve_unit_lower_64(const float* sL, float* sM, uint8_t* Z,
                                                    int tid) {
    auto T_at = [&](int r, int c) -> float& {
        return *reinterpret_cast<float*>(Z + z_off((uint32_t)r, (uint32_t)c));
    };
    if (tid < 64) {
        const int b = tid >> 4, col = tid & 15, o = 16 * b;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc = 0.f;
#pragma unroll
            for (int m = 0; m < r; ++m)
                if (m >= col) acc = fmaf(sL[(o + r) * 65 + o + m], x[m], acc);
            x[r] = r < col ? 0.f : (r == col ? 1.f : -acc);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) T_at(o + r, o + col) = x[r];
    } else {
        // zero the blocks above the block diagonal: (row block I, column block J > I)
        for (int idx = tid - 64; idx < 64 * 64; idx += 64) {
            const int r = idx >> 6, c = idx & 63;
            if ((c >> 4) > (r >> 4)) T_at(r, c) = 0.f;
        }
    }
    __syncthreads();
#pragma unroll 1
    for (int d = 1; d < 4; ++d) {
        const int nblk = 4 - d;  // blocks (I, I-d) for I = d..3
        for (int idx = tid; idx < nblk * 256; idx += 128) {
            const int I = d + (idx >> 8), J = I - d, r = (idx >> 4) & 15, c = idx & 15;
            float acc = 0.f;
            for (int m = J; m < I; ++m)
#pragma unroll
                for (int l = 0; l < 16; ++l)
                    acc = fmaf(sL[(16 * I + r) * 65 + 16 * m + l], T_at(16 * m + l, 16 * J + c), acc);
            sM[(16 * I + r) * 65 + 16 * J + c] = acc;
        }
        __syncthreads();
        for (int idx = tid; idx < nblk * 256; idx += 128) {
            const int I = d + (idx >> 8), J = I - d, r = (idx >> 4) & 15, c = idx & 15;
            float acc = 0.f;
#pragma unroll
            for (int k = 0; k < 16; ++k)
                acc = fmaf(T_at(16 * I + r, 16 * I + k), sM[(16 * I + k) * 65 + 16 * J + c], acc);
            T_at(16 * I + r, 16 * J + c) = -acc;
        }
        __syncthreads();
    }
}

// D (+)= [T; P] X over K = 64 tokens, as hi*hi + hi*lo + lo*hi: A = the K-major [T; P] tiles
// (z[0] = hi, z[1] = lo), B = the MN-major 64 x 64 tiles of X (x[0] = hi, x[1] = lo).
__device__ __forceinline__ void mma_split3(uint32_t d_tmem, const uint32_t* z, const uint32_t* x,
                                           uint32_t id, bool accumulate) {
    const int pairs[3][2] = {{0, 0}, {0, 1}, {1, 0}};
#pragma unroll
    for (int p = 0; p < 3; ++p)
#pragma unroll
        for (int s = 0; s < 4; ++s)
            tc::mma_bf16(d_tmem, tc::sw128_desc(z[pairs[p][0]] + s * 32, 16, 1024),
                         tc::sw128_desc(x[pairs[p][1]] + s * 2048, 8192, 1024), id,
                         (accumulate || p > 0 || s > 0) ? 1u : 0u);
}

template <int DV>
__global__ void __launch_bounds__(128, 1)
chunk_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_kt, const __grid_constant__ CUtensorMap tm_v,
                    const float* __restrict__ beta, float scale, const float* __restrict__ S0,
                    __nv_bfloat16* __restrict__ o, float* __restrict__ ST,
                    const int32_t* __restrict__ cu, int N, int T, int H, long long limit_ns) {
    constexpr int DK = 128, BV = 64, C = 64, NVT = DV / BV;
    using L = TcSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    const int tid = threadIdx.x, warp = tid >> 5;
    const int vt = blockIdx.x % NVT, nh = blockIdx.x / NVT;
    const int n = nh / H, h = nh - n * H;
    if (n >= N) return;
    int64_t first, count;
    if (!seq_range(cu, n, N, T, first, count)) return;  // uniform over the CTA
    const int c0 = vt * BV;
    const int64_t sbase = ((int64_t)n * H + h) * DV * DK + (int64_t)c0 * DK;

    uint64_t* tma_bar = reinterpret_cast<uint64_t*>(smem + L::BAR);
    uint64_t* mma_bar = tma_bar + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::TMEM_SLOT);
    uint8_t* Z = smem + L::ZHI;  // fp32 T during the solve (rows 0..63 of ZHI and ZLO)
    uint8_t* ZHI = smem + L::ZHI;
    uint8_t* ZLO = smem + L::ZLO;
    uint8_t* SHI = smem + L::SHI;
    uint8_t* SLO = smem + L::SLO;
    uint8_t* RHI = smem + L::RHI;
    uint8_t* RLO = smem + L::RLO;
    uint8_t* WHI = smem + L::WHI;
    uint8_t* WLO = smem + L::WLO;
    float* sL = reinterpret_cast<float*>(smem + L::SOLVE);
    float* sM = sL + 64 * 65;

    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, TC_TMEM_COLS);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&tma_bar[0], 1);
        mbar_init(&tma_bar[1], 1);
        mbar_init(mma_bar, 1);
        tc::fence_mbar_init();
        tc::prefetch_tmap(&tm_q);
        tc::prefetch_tmap(&tm_k);
        tc::prefetch_tmap(&tm_kt);
        tc::prefetch_tmap(&tm_v);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t t_S = tmem + lane + TC_COL_S, t_D1 = tmem + lane + TC_COL_D1;
    const uint32_t t_D2 = tmem + lane + TC_COL_D2, t_G = tmem + lane + TC_COL_G;

    // ---- initial state: S^T lane i = key channel i, columns = this CTA's value channels
    {
        float s[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = S0 ? __ldg(S0 + sbase + (int64_t)c * DK + tid) : 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) tc::tmem_st16(t_S + 16 * q, s + 16 * q);
        tc::tmem_st_wait();
        st_row_split_bf16(SHI, SLO, tid, s);
    }

    const int nchunks = (int)((count + C - 1) / C);
    auto issue_loads = [&](int chunk, int stage) {
        uint8_t* st = smem + stage * L::STAGE;
        const int row = (int)(first + (int64_t)chunk * C);
        tc::mbar_expect_tx(&tma_bar[stage], L::STAGE);
        tc::tma_load_3d(st + L::KQ + 0, &tm_k, 0, h, row, &tma_bar[stage]);
        tc::tma_load_3d(st + L::KQ + 8192, &tm_q, 0, h, row, &tma_bar[stage]);
        tc::tma_load_3d(st + L::KQ + 16384, &tm_k, 64, h, row, &tma_bar[stage]);
        tc::tma_load_3d(st + L::KQ + 24576, &tm_q, 64, h, row, &tma_bar[stage]);
        tc::tma_load_3d(st + L::KT + 0, &tm_kt, 0, h, row, &tma_bar[stage]);
        tc::tma_load_3d(st + L::KT + 8192, &tm_kt, 64, h, row, &tma_bar[stage]);
        tc::tma_load_3d(st + L::V, &tm_v, c0, h, row, &tma_bar[stage]);
    };
    // Async work thread 0 has in flight (parity of the pending TMA phase per stage, -1: none;
    // whether an MMA commit is pending), drained on the error path before leaving.
    int tma_pend[2] = {-1, -1};
    bool mma_pend = false;
    uint32_t mma_phase = 0;
    bool fail = false;
    if (tid == 0 && nchunks > 0) {
        issue_loads(0, 0);
        tma_pend[0] = 0;
    }
    tc::fence_async_smem();
    tc::fence_before_sync();
    __syncthreads();

    auto wait_mma = [&]() {
        if (mbar_wait_bounded(mma_bar, mma_phase, limit_ns)) {
            mma_phase ^= 1u;
            mma_pend = false;
        } else {
            fail = true;
        }
        tc::fence_after_sync();
    };
    auto commit = [&]() {
        tc::mma_commit(mma_bar);
        mma_pend = true;
    };
    // Barrier that also agrees, across the CTA, on whether any thread saw a failed wait.
    auto sync_failed = [&]() -> bool {
        tc::fence_before_sync();
        const bool any = __syncthreads_or(fail) != 0;
        fail = any;
        return any;
    };
    constexpr uint32_t ID_G = tc::idesc(1, 0, 0, 128, 64);   // [K;Q] x K~^T
    constexpr uint32_t ID_1 = tc::idesc(1, 0, 1, 128, 64);   // [K;Q] x S^T
    constexpr uint32_t ID_Z = tc::idesc(1, 0, 1, 128, 64);   // [T;P] x (R | W)
    constexpr uint32_t ID_3 = tc::idesc(1, 1, 1, 128, 64);   // K~^T x W

#pragma unroll 1
    for (int ch = 0; ch < nchunks; ++ch) {
        const int stage = ch & 1;
        uint8_t* st = smem + stage * L::STAGE;
        const uint32_t aKQ = smem_u32(st + L::KQ), aKT = smem_u32(st + L::KT);
        const uint32_t aZ[2] = {smem_u32(ZHI), smem_u32(ZLO)};
        const uint32_t aR[2] = {smem_u32(RHI), smem_u32(RLO)};
        const uint32_t aW[2] = {smem_u32(WHI), smem_u32(WLO)};
        const int64_t cs = (int64_t)ch * C;
        const int Lc = (count - cs) < C ? (int)(count - cs) : C;
        const float bt = (tid < Lc) ? __ldg(beta + (first + cs + tid) * H + h) : 0.f;
        if (tid == 0 && ch + 1 < nchunks) {
            issue_loads(ch + 1, stage ^ 1);
            tma_pend[stage ^ 1] = ((ch + 1) >> 1) & 1;
        }
        if (mbar_wait_bounded(&tma_bar[stage], (uint32_t)(ch >> 1) & 1u, limit_ns))
            tma_pend[stage] = -1;
        else
            fail = true;
        if (sync_failed()) break;

        // ---- Gram and scores: DG = [K; Q] K~^T
        if (tid == 0) {
            tc::fence_after_sync();
#pragma unroll
            for (int s = 0; s < 8; ++s)
                tc::mma_bf16(tmem + TC_COL_G,
                             tc::sw128_desc(aKQ + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024),
                             tc::sw128_desc(aKT + (s >> 2) * 8192 + (s & 3) * 32, 16, 1024), ID_G,
                             s > 0);
            commit();
        }
        wait_mma();
        {
            float g[64];
            tc::tmem_ld64(t_G, g);
            if (tid < 64) {
#pragma unroll
                for (int j = 0; j < 64; ++j) sL[tid * 65 + j] = j < tid ? bt * g[j] : 0.f;
            } else {
                const int r = tid - 64;
#pragma unroll
                for (int j = 0; j < 64; ++j) g[j] = j <= r ? g[j] : 0.f;
                st_row_split_bf16(ZHI, ZLO, tid, g);  // P rows 64..127
            }
        }
        if (sync_failed()) break;
        solve_unit_lower_64(sL, sM, Z, tid);  // ends with __syncthreads
        {
            float x[64];
            if (tid < 64) {
#pragma unroll
                for (int j = 0; j < 64; ++j) x[j] = *reinterpret_cast<const float*>(Z + z_off(tid, j));
            }
            __syncthreads();  // every fp32 row is read before the bf16 rows overwrite it
            if (tid < 64) st_row_split_bf16(ZHI, ZLO, tid, x);  // T rows 0..63
        }
        tc::fence_async_smem();
        if (sync_failed()) break;

        // ---- D1 = [K; Q] S^T  (two bf16 terms of S^T)
        if (tid == 0) {
            tc::fence_after_sync();
            const uint32_t parts[2] = {smem_u32(SHI), smem_u32(SLO)};
#pragma unroll
            for (int p = 0; p < 2; ++p)
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    tc::mma_bf16(tmem + TC_COL_D1,
                                 tc::sw128_desc(aKQ + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024),
                                 tc::sw128_desc(parts[p] + s * 2048, 8192, 1024), ID_1,
                                 (p | s) != 0);
            commit();
        }
        wait_mma();
        if (tid < 64) {  // warps 0-1: R = beta (V - K S^T) for token rows 0..63
            float y[64], r[64];
            tc::tmem_ld64(t_D1, y);
            const uint8_t* vtile = st + L::V;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint4 raw = *reinterpret_cast<const uint4*>(vtile + tc::sw128_off(tid, j));
                const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 vv =
                        __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[e]));
                    r[8 * j + 2 * e] = bt * (vv.x - y[8 * j + 2 * e]);
                    r[8 * j + 2 * e + 1] = bt * (vv.y - y[8 * j + 2 * e + 1]);
                }
            }
            st_row_split_bf16(RHI, RLO, tid, r);
        }
        tc::fence_async_smem();
        if (sync_failed()) break;

        // ---- D2 = [T; P] R  (three split terms; rows 0..63 hold W)
        if (tid == 0) {
            tc::fence_after_sync();
            mma_split3(tmem + TC_COL_D2, aZ, aR, ID_Z, false);
            commit();
        }
        wait_mma();
        if (tid < 64) {
            float w[64];
            tc::tmem_ld64(t_D2, w);
            st_row_split_bf16(WHI, WLO, tid, w);
        }
        tc::fence_async_smem();
        if (sync_failed()) break;

        // ---- S^T += K~^T W (two terms of W);  D1 += [T; P] W (three terms; rows 64..127: O)
        if (tid == 0) {
            tc::fence_after_sync();
#pragma unroll
            for (int p = 0; p < 2; ++p)
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    tc::mma_bf16(tmem + TC_COL_S, tc::sw128_desc(aKT + s * 2048, 8192, 1024),
                                 tc::sw128_desc(aW[p] + s * 2048, 8192, 1024), ID_3, 1);
            mma_split3(tmem + TC_COL_D1, aZ, aW, ID_Z, true);
            commit();
        }
        wait_mma();
        if (tid >= 64) {  // warps 2-3: o rows of this chunk
            float x[64];
            tc::tmem_ld64(t_D1, x);
            const int r = tid - 64;
            if (r < Lc) {
                __nv_bfloat16* orow = o + ((first + cs + r) * H + h) * DV + c0;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint32_t pk[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const __nv_bfloat162 b2 = __floats2bfloat162_rn(
                            scale * x[8 * j + 2 * e], scale * x[8 * j + 2 * e + 1]);
                        pk[e] = *reinterpret_cast<const uint32_t*>(&b2);
                    }
                    *reinterpret_cast<uint4*>(orow + 8 * j) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
        }
        {
            float x[64];
            tc::tmem_ld64(t_S, x);
            st_row_split_bf16(SHI, SLO, tid, x);
        }
        tc::fence_async_smem();
        if (sync_failed()) break;
    }

    if (fail) {
        // error path: let this CTA's own copies and MMAs finish (bounded) before leaving
        if (tid == 0) {
            for (int s = 0; s < 2; ++s)
                if (tma_pend[s] >= 0) mbar_wait_bounded(&tma_bar[s], (uint32_t)tma_pend[s], limit_ns);
            if (mma_pend) mbar_wait_bounded(mma_bar, mma_phase, limit_ns);
        }
    } else if (ST) {
        float s[64];
        tc::tmem_ld64(t_S, s);
#pragma unroll
        for (int c = 0; c < 64; ++c) ST[sbase + (int64_t)c * DK + tid] = s[c];
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, TC_TMEM_COLS);
}

}  // namespace osdn
