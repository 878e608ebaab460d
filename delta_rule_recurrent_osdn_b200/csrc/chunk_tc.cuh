// chunk_tc.cuh -- phase 2 of the OSDN forward pass on the sm_100a tensor cores (bf16 I/O, d_k = 128).
//
// The chunkwise delta rule with write key K~ ("OSDN: Improving Delta Rule with Provable Online
// Preconditioning in Linear Attention", technical summary, section 2.1: K~ replaces K in the
// chunk Gram matrix and in the intra-chunk scores).  Per chunk of C = 64 tokens, state S_0
// (value rows), this CTA's 64 value channels:
//   P = tril(Q K~^T)                              one bf16 MMA, A = [K; Q] (M = 128)
//   T = (I + strict_tril(diag(beta) K K~^T))^-1   computed for all chunks beforehand by
//                                                 wy_prep_kernel (chunk_prep.cuh), read here
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
// Warp roles (one CTA per (sequence, head, 64 value channels), 288 threads):
//   chain    warps 0-3: the state-dependent MMA chain of chunk c and its epilogues (thread t owns
//            tensor-memory lane t);
//   prep     warps 4-7: chunk c+1's [T; P] operand tiles (T unpacked from the copy the
//            pre-kernel left in this CTA's slice of the chunk's o rows, P from a Gram MMA),
//            overlapping chunk c's chain;
//   producer warp 8: TMA loads of the chunk tiles into a 2-stage ring (no multicast).
// Handshakes are mbarriers: zt_* / zp_* for the T and P halves of the [T; P] tiles (W = T R
// uses only the T rows, the outputs only the P rows, so each half is refilled as soon as its
// last reader is done; the other half's rows only reach accumulator lanes nobody reads),
// stage_empty for the ring.
// Every wait is bounded and followed by a group-wide vote, so a role that gives up (recording
// OSDN_ERR_DEVICE_TIMEOUT) leaves its loop as a whole group and no named barrier is left waiting.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "tc_ptx.cuh"
#include "tril_inverse.cuh"

namespace osdn {

struct TcSmem {
    static constexpr uint32_t STAGE = 65536;          // [K;Q] 32K | K~ 16K | V 8K | packed T 8K
    static constexpr uint32_t KQ = 0, KT = 32768, V = 49152, TP = 57344;
    static constexpr uint32_t ZHI = 2 * STAGE;        // bf16 [T; P] hi / lo, K-major, 128 x 128 B
    static constexpr uint32_t ZLO = ZHI + 16384;
    static constexpr uint32_t SHI = ZLO + 16384;      // bf16 S^T hi / lo, MN-major, 128 x 128 B
    static constexpr uint32_t SLO = SHI + 16384;
    static constexpr uint32_t RHI = SLO + 16384;      // bf16 R then W, hi / lo, 64 x 128 B
    static constexpr uint32_t RLO = RHI + 8192;
    static constexpr uint32_t BAR = RLO + 8192;
    static constexpr uint32_t TMEM_SLOT = BAR + 128;
    static constexpr uint32_t TOTAL = TMEM_SLOT + 16;
    static constexpr size_t BYTES = TOTAL + 1024;     // + alignment slack
};
static_assert(TcSmem::BYTES <= 232448, "shared memory");

// Tensor-memory columns: S, D1 (double-buffered: a chunk's outputs are read during the next
// chunk), D2, the prep's Gram.
constexpr uint32_t TC_COL_S = 0, TC_COL_D1 = 64, TC_COL_D2 = 192, TC_COL_G = 256;
constexpr uint32_t TC_TMEM_COLS = 512;
constexpr int TC_THREADS = 288;

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
__global__ void __launch_bounds__(TC_THREADS, 1)
chunk_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_kt, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_tp,
                    const float* __restrict__ beta, float scale, const float* __restrict__ S0,
                    __nv_bfloat16* __restrict__ o, float* __restrict__ ST,
                    const int32_t* __restrict__ cu, int N, int T, int H, long long limit_ns) {
    constexpr int DK = 128, BV = 64, C = 64, NVT = DV / BV;
    using L = TcSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_align1024(smem_raw);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int vt = blockIdx.x % NVT, nh = blockIdx.x / NVT;
    const int n = nh / H, h = nh - n * H;
    if (n >= N) return;
    int64_t first, count;
    if (!seq_range(cu, n, N, T, first, count)) return;  // uniform over the CTA
    const int c0 = vt * BV;
    const int64_t sbase = ((int64_t)n * H + h) * DV * DK + (int64_t)c0 * DK;
    const int nchunks = (int)((count + C - 1) / C);

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR);
    uint64_t* tma_full = bars + 0;     // [2]
    uint64_t* stage_empty = bars + 2;  // [2], two arrivals: chain and prep
    uint64_t* zt_full = bars + 4;      // T rows of [T; P] written
    uint64_t* zt_empty = bars + 5;     // T rows free (W computed)
    uint64_t* zp_full = bars + 9;      // P rows written
    uint64_t* zp_empty = bars + 10;    // P rows free (outputs computed)
    uint64_t* w_ready = bars + 11;     // W of the chunk written (the output MMAs may start)
    uint64_t* mma_c = bars + 6;        // chain MMAs on the state's path
    uint64_t* mma_p = bars + 7;        // prep MMAs
    uint64_t* mma_o = bars + 8;        // chain MMAs of the outputs
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::TMEM_SLOT);
    uint8_t* ZHI = smem + L::ZHI;
    uint8_t* ZLO = smem + L::ZLO;
    uint8_t* SHI = smem + L::SHI;
    uint8_t* SLO = smem + L::SLO;
    uint8_t* RHI = smem + L::RHI;
    uint8_t* RLO = smem + L::RLO;

    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, TC_TMEM_COLS);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&tma_full[0], 1);
        mbar_init(&tma_full[1], 1);
        mbar_init(&stage_empty[0], 2);
        mbar_init(&stage_empty[1], 2);
        mbar_init(zt_full, 1);
        mbar_init(zt_empty, 1);
        mbar_init(zp_full, 1);
        mbar_init(zp_empty, 1);
        mbar_init(w_ready, 1);
        mbar_init(mma_c, 1);
        mbar_init(mma_p, 1);
        mbar_init(mma_o, 1);
        tc::fence_mbar_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (tid == 0) {  // the [T; P] tiles start out free
        mbar_arrive(zt_empty);
        mbar_arrive(zp_empty);
    }
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane = static_cast<uint32_t>((warp & 3) * 32) << 16;
    auto chunk_len = [&](int ch) -> int {
        const int64_t rem = count - (int64_t)ch * C;
        return rem < C ? (int)rem : C;
    };

    if (warp == 8) {
        // =========================================================== producer
        // Lane 0 loads the chunk tiles into the 2-stage ring and issues each chunk's output
        // MMAs (D1 += [T; P] W) once the chain has published W, so that the chain warps go
        // straight on to the state split.
        if ((tid & 31) == 0) {
            tc::prefetch_tmap(&tm_q);
            tc::prefetch_tmap(&tm_k);
            tc::prefetch_tmap(&tm_kt);
            tc::prefetch_tmap(&tm_v);
            tc::prefetch_tmap(&tm_tp);
            constexpr uint32_t ID_O = tc::idesc(1, 0, 1, 128, 64);
            const uint32_t aZ[2] = {smem_u32(ZHI), smem_u32(ZLO)};
            const uint32_t aR[2] = {smem_u32(RHI), smem_u32(RLO)};
            int pend[2] = {-1, -1};
            int o_issued = 0;
            auto load = [&](int ch) {
                const int s = ch & 1;
                uint8_t* st = smem + s * L::STAGE;
                const int row = (int)(first + (int64_t)ch * C);
                tc::mbar_expect_tx(&tma_full[s], L::STAGE);
                tc::tma_load_3d(st + L::KQ + 0, &tm_k, 0, h, row, &tma_full[s]);
                tc::tma_load_3d(st + L::KQ + 8192, &tm_q, 0, h, row, &tma_full[s]);
                tc::tma_load_3d(st + L::KQ + 16384, &tm_k, 64, h, row, &tma_full[s]);
                tc::tma_load_3d(st + L::KQ + 24576, &tm_q, 64, h, row, &tma_full[s]);
                tc::tma_load_3d(st + L::KT + 0, &tm_kt, 0, h, row, &tma_full[s]);
                tc::tma_load_3d(st + L::KT + 8192, &tm_kt, 64, h, row, &tma_full[s]);
                tc::tma_load_3d(st + L::V, &tm_v, c0, h, row, &tma_full[s]);
                tc::tma_load_3d(st + L::TP, &tm_tp, 32 * vt, h, row, &tma_full[s]);
                pend[s] = (ch >> 1) & 1;
            };
            for (int ch = 0; ch < nchunks && ch < 2; ++ch) load(ch);
            for (int ch = 0; ch < nchunks; ++ch) {
                if (!mbar_wait_bounded(w_ready, (uint32_t)ch & 1u, limit_ns)) break;
                tc::fence_after_sync();
                mma_split3(tmem + TC_COL_D1 + 64 * (ch & 1), aZ, aR, ID_O, true);
                tc::mma_commit(mma_o);
                ++o_issued;
                if (ch + 2 < nchunks) {  // chunk ch's stage, once both roles released it
                    if (!mbar_wait_bounded(&stage_empty[ch & 1], (uint32_t)(ch >> 1) & 1u, limit_ns)) break;
                    load(ch + 2);
                }
            }
            // let this CTA's own copies and MMAs land before the block can leave
            for (int s = 0; s < 2; ++s)
                if (pend[s] >= 0) mbar_wait_bounded(&tma_full[s], (uint32_t)pend[s], limit_ns);
            if (o_issued > 0) mbar_wait_bounded(mma_o, (uint32_t)(o_issued - 1) & 1u, limit_ns);
        }
    } else if (warp >= 4) {
        // =========================================================== prep
        const int t = tid - 128;  // 0..127 = tensor-memory lane
        const bool leader = t == 0;
        constexpr uint32_t ID_G = tc::idesc(1, 0, 0, 128, 64);
        bool pend = false;
        uint32_t mphase = 0;
        for (int ch = 0; ch < nchunks; ++ch) {
            const int s = ch & 1;
            if (group_any(2, 128, !mbar_wait_bounded(&tma_full[s], (uint32_t)(ch >> 1) & 1u, limit_ns))) break;
            uint8_t* st = smem + s * L::STAGE;
            if (leader) {
                const uint32_t aKQ = smem_u32(st + L::KQ), aKT = smem_u32(st + L::KT);
                tc::fence_after_sync();
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    tc::mma_bf16(tmem + TC_COL_G, tc::sw128_desc(aKQ + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024),
                                 tc::sw128_desc(aKT + (k >> 2) * 8192 + (k & 3) * 32, 16, 1024), ID_G, k > 0);
                tc::mma_commit(mma_p);
                pend = true;
            }
            // row t of T from the packed strictly-lower copy (unit diagonal; identity rows past
            // the chunk's end), while the Gram runs
            float x[64];
            if (t < 64) {
                const float* tp = reinterpret_cast<const float*>(st + L::TP);
                const int base = t * (t - 1) / 2;
                const bool in = t < chunk_len(ch);
#pragma unroll
                for (int j = 0; j < 64; ++j) x[j] = (in && j < t) ? tp[base + j] : (j == t ? 1.f : 0.f);
            }
            if (group_any(2, 128, !mbar_wait_bounded(mma_p, mphase, limit_ns))) break;
            mphase ^= 1u;
            pend = false;
            tc::fence_after_sync();
            if (leader) mbar_arrive(&stage_empty[s]);  // the prep's last use of the stage
            if (t >= 64) {  // P row t - 64 = tril(Q K~^T)
                tc::tmem_ld64(tmem + lane + TC_COL_G, x);
                const int r = t - 64;
#pragma unroll
                for (int j = 0; j < 64; ++j) x[j] = j <= r ? x[j] : 0.f;
            }
            // rows 0..63 (T) by warps 4-5 and rows 64..127 (P) by warps 6-7, each half as soon
            // as the chain is done with its previous contents
            const int half = t >> 6, hbar = 3 + half;
            bool bad = group_any(hbar, 64, !mbar_wait_bounded(half ? zp_empty : zt_empty,
                                                              (uint32_t)ch & 1u, limit_ns));
            if (!bad) {
                st_row_split_bf16(ZHI, ZLO, t, x);
                tc::fence_async_smem();
            }
            group_bar(hbar, 64);
            if (!bad && (t & 63) == 0) mbar_arrive(half ? zp_full : zt_full);
            if (group_any(2, 128, bad)) break;
        }
        if (leader && pend) mbar_wait_bounded(mma_p, mphase, limit_ns);
    } else {
        // =========================================================== chain
        // Per chunk c: D1[c&1] = [K;Q] S^T -> R -> W -> S^T += K~^T W (the state's path), and
        // D1[c&1] += [T;P] W for the outputs, committed apart so the state split does not wait for
        // them; chunk c's output rows are read and stored by warps 2-3 during chunk c+1's R step,
        // when only warps 0-1 have work.
        const int t = tid;  // 0..127 = tensor-memory lane
        const bool leader = t == 0;
        const uint32_t t_S = tmem + lane + TC_COL_S, t_D2 = tmem + lane + TC_COL_D2;
        constexpr uint32_t ID_1 = tc::idesc(1, 0, 1, 128, 64);  // [K;Q] x S^T and [T;P] x (R | W)
        constexpr uint32_t ID_3 = tc::idesc(1, 1, 1, 128, 64);  // K~^T x W
        const uint32_t aZ[2] = {smem_u32(ZHI), smem_u32(ZLO)};
        const uint32_t aR[2] = {smem_u32(RHI), smem_u32(RLO)};
        const uint32_t aS[2] = {smem_u32(SHI), smem_u32(SLO)};
        bool pend = false;
        uint32_t mphase = 0, ophase = 0;
        bool ok = true;
        auto mma_wait = [&]() -> bool {
            if (group_any(1, 128, !mbar_wait_bounded(mma_c, mphase, limit_ns))) return false;
            mphase ^= 1u;
            pend = false;
            tc::fence_after_sync();
            return true;
        };
        // o rows of chunk pc from D1[pc & 1] (warps 2-3: lanes 64..127 = the chunk's tokens)
        auto store_o = [&](int pc) {
            const int r = t - 64;
            float x[64];
            tc::tmem_ld64(tmem + lane + TC_COL_D1 + 64 * (pc & 1), x);
            if (r < chunk_len(pc)) {
                __nv_bfloat16* orow = o + ((first + (int64_t)pc * C + r) * H + h) * DV + c0;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint32_t pk[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const __nv_bfloat162 b2 = __floats2bfloat162_rn(scale * x[8 * j + 2 * e],
                                                                        scale * x[8 * j + 2 * e + 1]);
                        pk[e] = *reinterpret_cast<const uint32_t*>(&b2);
                    }
                    *reinterpret_cast<uint4*>(orow + 8 * j) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
        };
        // initial state: S^T lane i = key channel i, columns = this CTA's value channels
        {
            float s0[64];
#pragma unroll
            for (int c = 0; c < 64; ++c) s0[c] = S0 ? __ldg(S0 + sbase + (int64_t)c * DK + t) : 0.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) tc::tmem_st16(t_S + 16 * q, s0 + 16 * q);
            tc::tmem_st_wait();
            st_row_split_bf16(SHI, SLO, t, s0);
            tc::fence_async_smem();
            tc::fence_before_sync();
            group_bar(1, 128);
        }
        float bnext = (t < 64 && nchunks > 0 && t < chunk_len(0)) ? __ldg(beta + (first + t) * H + h) : 0.f;
        for (int ch = 0; ch < nchunks && ok; ++ch) {
            const int s = ch & 1;
            const int64_t cs = (int64_t)ch * C;
            const uint32_t t_D1 = tmem + lane + TC_COL_D1 + 64 * s;
            const float bt = bnext;
            if (t < 64 && ch + 1 < nchunks)
                bnext = t < chunk_len(ch + 1) ? __ldg(beta + (first + cs + C + t) * H + h) : 0.f;
            uint8_t* st = smem + s * L::STAGE;
            const uint32_t aKQ = smem_u32(st + L::KQ), aKT = smem_u32(st + L::KT);
            if (group_any(1, 128, !mbar_wait_bounded(&tma_full[s], (uint32_t)(ch >> 1) & 1u, limit_ns))) {
                ok = false;
                break;
            }
            // ---- D1 = [K; Q] S^T  (two terms of S^T)
            if (leader) {
                tc::fence_after_sync();
#pragma unroll
                for (int p = 0; p < 2; ++p)
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        tc::mma_bf16(tmem + TC_COL_D1 + 64 * s,
                                     tc::sw128_desc(aKQ + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024),
                                     tc::sw128_desc(aS[p] + k * 2048, 8192, 1024), ID_1, (p | k) != 0);
                tc::mma_commit(mma_c);
                pend = true;
            }
            if (!mma_wait()) { ok = false; break; }
            if (t < 64) {  // R = beta (V - K S^T), token rows 0..63
                float y[64];
                tc::tmem_ld64(t_D1, y);
                const uint8_t* vtile = st + L::V;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint4 raw = *reinterpret_cast<const uint4*>(vtile + tc::sw128_off(t, j));
                    const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 vv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[e]));
                        y[8 * j + 2 * e] = bt * (vv.x - y[8 * j + 2 * e]);
                        y[8 * j + 2 * e + 1] = bt * (vv.y - y[8 * j + 2 * e + 1]);
                    }
                }
                st_row_split_bf16(RHI, RLO, t, y);
            }
            tc::fence_async_smem();
            tc::fence_before_sync();
            if (group_any(1, 128, !mbar_wait_bounded(zt_full, (uint32_t)ch & 1u, limit_ns))) {
                ok = false;
                break;
            }
            // ---- D2 = [T; P] R  (rows 0..63: W)
            if (leader) {
                tc::fence_after_sync();
                mma_split3(tmem + TC_COL_D2, aZ, aR, ID_1, false);
                tc::mma_commit(mma_c);
                pend = true;
            }
            if (!mma_wait()) { ok = false; break; }
            if (leader) mbar_arrive(zt_empty);  // the T rows have been used
            if (t < 64) {
                float w[64];
                tc::tmem_ld64(t_D2, w);
                st_row_split_bf16(RHI, RLO, t, w);  // R is consumed: W takes its tiles
            } else if (ch > 0) {
                store_o(ch - 1);  // its output MMAs completed before this chunk's R
            }
            tc::fence_async_smem();
            tc::fence_before_sync();
            if (group_any(1, 128, !mbar_wait_bounded(zp_full, (uint32_t)ch & 1u, limit_ns))) {
                ok = false;
                break;
            }
            if (leader) mbar_arrive(w_ready);  // the producer warp issues the output MMAs
            // ---- S^T += K~^T W (two terms of W); the outputs' D1 += [T; P] W is issued by the
            //      producer warp and completes on the output barrier
            if (leader) {
                tc::fence_after_sync();
#pragma unroll
                for (int p = 0; p < 2; ++p)
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc::mma_bf16(tmem + TC_COL_S, tc::sw128_desc(aKT + k * 2048, 8192, 1024),
                                     tc::sw128_desc(aR[p] + k * 2048, 8192, 1024), ID_3, 1);
                tc::mma_commit(mma_c);
                pend = true;
            }
            if (!mma_wait()) { ok = false; break; }
            {
                float x[64];
                tc::tmem_ld64(t_S, x);
                st_row_split_bf16(SHI, SLO, t, x);
            }
            // the output MMAs read the P rows, this chunk's tiles and W: wait for them before
            // releasing those, and before the next chunk's R overwrites W
            if (group_any(1, 128, !mbar_wait_bounded(mma_o, ophase, limit_ns))) {
                ok = false;
                break;
            }
            ophase ^= 1u;
            tc::fence_after_sync();
            if (leader) {
                mbar_arrive(zp_empty);         // the P rows have been used
                mbar_arrive(&stage_empty[s]);  // and this chunk's tiles
            }
            tc::fence_async_smem();
            tc::fence_before_sync();
            group_bar(1, 128);
        }
        if (ok && nchunks > 0 && t >= 64) store_o(nchunks - 1);
        if (ok && ST) {
            float s1[64];
            tc::tmem_ld64(t_S, s1);
#pragma unroll
            for (int c = 0; c < 64; ++c) ST[sbase + (int64_t)c * DK + t] = s1[c];
        }
        if (leader && pend) mbar_wait_bounded(mma_c, mphase, limit_ns);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, TC_TMEM_COLS);
}

}  // namespace osdn
