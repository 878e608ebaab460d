// chunk_tc.cuh -- phase 2 of the OSDN forward pass on the sm_100a tensor cores (bf16 I/O, d_k = 128).
//
// The chunkwise delta rule with write key K~ ("OSDN: Improving Delta Rule with Provable Online
// Preconditioning in Linear Attention", technical summary, section 2.1: K~ replaces K in the
// chunk Gram matrix and in the intra-chunk scores).  Per chunk c of C = 64 tokens with state S_c
// at its start (value rows), for this CTA's 64 value channels:
//   T_c = (I + strict_tril(diag(beta) K_c K~_c^T))^-1   computed for all chunks beforehand by
//                                                       wy_prep_kernel (chunk_prep.cuh), read here
//   R_c = diag(beta) (V_c - K_c S_c^T)
//   W_c = T_c R_c
//   O_c = Q_c S_c^T + P_c W_c,  P_c = tril(Q_c K~_c^T)
//   S_{c+1}^T = S_c^T + K~_c^T W_c
//
// Lookahead form.  Because K_{c+1} S_{c+1}^T = K_{c+1} S_c^T + (K_{c+1} K~_c^T) W_c, the product
// that starts chunk c+1 is assembled from the state one chunk earlier and from W_c:
//   D1_{c+1}  = [K_{c+1}; Q_c] S_c^T        A = the ring stage's [K; Q] tile (M = 128)
//   D1_{c+1} += [X_{c+1}; P_c] W_c          X_{c+1} = K_{c+1} K~_c^T
// after which rows 0..63 of D1_{c+1} are K_{c+1} S_{c+1}^T and rows 64..127 are O_c.  One Gram
// MMA, A = [K_{c+1}; Q_c] and B = K~_c, gives X_{c+1} and (masked) P_c together.  The chain's
// critical path per chunk is R split -> W = T R -> W split -> D1 += [X; P] W: two operand splits
// and two MMA groups.  The state update S += K~^T W, the state's split and the next
// [K; Q] S^T product run beside it, one chunk ahead of their use.  (A thread that issues MMAs
// stalls while the tensor pipe accepts them, so who issues what is part of the schedule.)
//
// Precision.  Every computed MMA operand x is split into two bf16 terms, x = hi + lo with
// |x - hi - lo| <= 2^-16 |x| (split2_bf16: Veltkamp head, truncated residual).  A product of an
// exact bf16 input (K, Q, K~) with a computed operand takes two MMAs (hi, lo); a product of two
// computed operands ([T; .] or [X; P] with R or W) takes three (hi*hi + hi*lo + lo*hi).  In a
// CPU emulation of this chunk algorithm against the oracle, plain bf16 operands gave 1.5-2.5%
// max/rms error on o and S_T for the 340M and 1.3B workloads, and single-term tf32 products
// 0.25-0.46%; the split scheme's own error, at the 2^-16 level per operand, lies far below the
// bf16 rounding of the inputs and outputs.
//
// Warp roles (one CTA per (sequence, head, 64 value channels), 288 threads):
//   chain    warps 0-3: R, W = T R, the [X; P] W product and the output rows (thread t owns
//            tensor-memory lane t); its leader issues only the two MMA groups the chain waits on;
//   prep     warps 4-7: the state's split, the [X; P] operand from the Gram (split in place in
//            tensor memory), identity rows in the T tiles of a short last chunk (the pre-kernel leaves T split into bf16 hi / lo operand
//            rows in the chunk's o rows; they reach the ring stage by TMA);
//   producer warp 8: TMA loads into a 2-stage ring (no multicast) and the MMAs off the critical
//            path (Gram, S += K~^T W, the next [K; Q] S^T).  Ring stage i holds [K_i; Q_{i-1}],
//            K~_{i-1} (one bf16 term, or hi and lo), V_i and the T_i tiles, for i = 0 .. n (n chunks).
// The head's two value-tile CTAs run as a 2-CTA cluster: each loads T hi and lo from both
// 128-byte slices of the o rows, and each overwrites its own slice with outputs, so a CTA stores
// O_c only after its sibling has loaded stage c (a counter in its shared memory that the
// sibling's producer raises through distributed shared memory).
// Handshakes are mbarriers; every wait is bounded and followed by a group-wide vote, so a role
// that gives up (recording OSDN_ERR_DEVICE_TIMEOUT) leaves its loop as a whole group and no named
// barrier is left waiting.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "tc_ptx.cuh"
#include "tril_inverse.cuh"

namespace osdn {

struct TcSmem {
    // ring stage: [K;Q] 32K | K~ hi 16K | K~ lo 16K | V 8K | T hi 8K | T lo 8K.  W = T R reads A
    // as the 64 rows before each T tile followed by the tile ([V; T hi] and [T hi; T lo]), so W
    // lands in accumulator lanes 64..127 and the rows in front, which stay unchanged while that
    // MMA runs, reach only lanes 0..63, which nobody reads.  The K~ lo tile is loaded only when
    // phase 1 hands K~ over as two bf16 terms.
    static constexpr uint32_t STAGE = 90112;
    static constexpr uint32_t KQ = 0, KT = 32768, KTLO = 49152, V = 65536, THI = 73728, TLO = 81920;
    static constexpr uint32_t SHI = 2 * STAGE;        // bf16 S^T hi / lo, MN-major, 128 x 128 B
    static constexpr uint32_t SLO = SHI + 16384;
    static constexpr uint32_t RHI = SLO + 16384;      // bf16 R (then W) hi / lo, 64 x 128 B
    static constexpr uint32_t RLO = RHI + 8192;
    static constexpr uint32_t BAR = RLO + 8192;
    static constexpr uint32_t TMEM_SLOT = BAR + 128;
    static constexpr uint32_t TOTAL = TMEM_SLOT + 16;
    static constexpr size_t BYTES = TOTAL + 1024;     // + alignment slack
};
static_assert(TcSmem::BYTES <= 232448, "shared memory");

// Tensor-memory columns: S; D1 (two buffers: chunk c+1's product is assembled while chunk c is
// read), D2 and the prep's Gram.  D1 and D2 are 128 columns wide: their MMAs take the hi and lo
// terms of the right-hand operand side by side (N = 128), and a reader sums the two halves.  The
// Gram's 64 fp32 columns are read by the prep role and then overwritten with the [X; P] operand
// of the chain's last MMA, as packed bf16 pairs: the hi term in columns G..G+31, the lo term in
// G+32..G+63 (the next Gram is issued only after that MMA has completed).
constexpr uint32_t TC_COL_S = 0, TC_COL_D1 = 64, TC_COL_D2 = 320, TC_COL_G = 448;
constexpr uint32_t TC_TMEM_COLS = 512;
constexpr int TC_THREADS = 288;

// Two fp32 values as bf16 MMA operand terms, x = hi + lo with about 16 significant bits: hi is
// the 8-significant-bit head of x by Veltkamp's splitting (t = (2^16 + 1) x, hi = t - (t - x),
// exactly representable in bf16, so its bf16 bits are the upper half of its fp32 bits); lo =
// x - hi is exact in fp32 and keeps its upper half, so |x - hi - lo| <= 2^-16 |x|.  Two-wide fp32
// arithmetic and byte permutes only.  Returns the packed bf16x2 words (a in the low half).
__device__ __forceinline__ void split2_bf16(float a, float b, uint32_t& hi, uint32_t& lo) {
    const float2 sig = make_float2(65537.f, 65537.f), m1 = make_float2(-1.f, -1.f);
    const float2 xv = make_float2(a, b);
    const float2 tv = __fmul2_rn(sig, xv);
    const float2 hv = __ffma2_rn(__ffma2_rn(xv, m1, tv), m1, tv);
    const float2 lv = __ffma2_rn(hv, m1, xv);
    hi = __byte_perm(__float_as_uint(hv.x), __float_as_uint(hv.y), 0x7632);
    lo = __byte_perm(__float_as_uint(lv.x), __float_as_uint(lv.y), 0x7632);
}

// Split a 64-value fp32 row into bf16 hi + lo (split2_bf16) and write both rows (128 B each,
// swizzled).
__device__ __forceinline__ void st_row_split_bf16(uint8_t* hi, uint8_t* lo, uint32_t row,
                                                  const float* x) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        uint32_t h[4], l[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) split2_bf16(x[8 * j + 2 * e], x[8 * j + 2 * e + 1], h[e], l[e]);
        const uint32_t off = tc::sw128_off(row, j);
        *reinterpret_cast<uint4*>(hi + off) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4*>(lo + off) = make_uint4(l[0], l[1], l[2], l[3]);
    }
}

// D (+)= Z X over K = 64 tokens as Z_hi [X_hi | X_lo] (N = 128, columns 0..127 of D) + Z_lo X_hi
// (columns 0..63): A = the K-major 128-row tiles of Z (z[0] = hi, z[1] = lo), B = the MN-major
// 64 x 64 tiles of X with X_lo 8 KB after X_hi.  The two column halves of D sum to the product.
__device__ __forceinline__ void mma_split3(uint32_t d_tmem, const uint32_t* z, uint32_t x_hi,
                                           bool accumulate) {
    constexpr uint32_t ID_W = tc::idesc(1, 0, 1, 128, 128), ID_N = tc::idesc(1, 0, 1, 128, 64);
    // rolled: issue is paced by the tensor pipe, and the roles share the instruction cache
#pragma unroll 1
    for (int i = 0; i < 8; ++i) {
        const int s = i & 3, lo = i >> 2;
        tc::mma_bf16(d_tmem, tc::sw128_desc(z[lo] + s * 32, 16, 1024),
                     tc::sw128_desc(x_hi + s * 2048, 8192, 1024), lo ? ID_N : ID_W,
                     (accumulate || i > 0) ? 1u : 0u);
    }
}

// The same product with Z = [X; P] read from tensor memory: z_tmem holds Z_hi in its first 32
// columns and Z_lo in the next 32 (two bf16 per column, K = 16 tokens per 8 columns).
__device__ __forceinline__ void mma_split3_ts(uint32_t d_tmem, uint32_t z_tmem, uint32_t x_hi,
                                              bool accumulate) {
    constexpr uint32_t ID_W = tc::idesc(1, 0, 1, 128, 128), ID_N = tc::idesc(1, 0, 1, 128, 64);
#pragma unroll 1
    for (int i = 0; i < 8; ++i) {
        const int s = i & 3, lo = i >> 2;
        tc::mma_bf16_ts(d_tmem, z_tmem + 32 * lo + 8 * s, tc::sw128_desc(x_hi + s * 2048, 8192, 1024),
                        lo ? ID_N : ID_W, (accumulate || i > 0) ? 1u : 0u);
    }
}

// D = A [S_hi | S_lo]^T over K = 128 key channels (N = 128, the halves of D sum to A S^T): A = a
// ring stage's K-major [K; Q] tile (two 64-channel blocks 16 KB apart), B = the MN-major S^T
// tiles with the lo term 16 KB after the hi term.
__device__ __forceinline__ void mma_kq_state(uint32_t d_tmem, uint32_t a_kq, uint32_t s_hi) {
    constexpr uint32_t ID_W = tc::idesc(1, 0, 1, 128, 128);
#pragma unroll 1
    for (int k = 0; k < 8; ++k)
        tc::mma_bf16(d_tmem, tc::sw128_desc(a_kq + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024),
                     tc::sw128_desc(s_hi + k * 2048, 16384, 1024), ID_W, k != 0);
}

// x[c] = D[c] + D[64 + c], c < 64: this thread's lane of a 128-column accumulator.
__device__ __forceinline__ void tmem_ld64_sum(uint32_t taddr, float* x) {
    tc::tmem_ld16(taddr + 0, x + 0);
    tc::tmem_ld16(taddr + 16, x + 16);
    tc::tmem_ld16(taddr + 32, x + 32);
    tc::tmem_ld16(taddr + 48, x + 48);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float t[32];
        tc::tmem_ld16(taddr + 64 + 32 * h, t);
        tc::tmem_ld16(taddr + 80 + 32 * h, t + 16);
        tc::tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
            const float2 s = __fadd2_rn(make_float2(x[32 * h + c], x[32 * h + c + 1]), make_float2(t[c], t[c + 1]));
            x[32 * h + c] = s.x;
            x[32 * h + c + 1] = s.y;
        }
    }
}

template <int DV>
__global__ void __launch_bounds__(TC_THREADS, 1)
chunk_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_kt, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_tp, const __grid_constant__ CUtensorMap tm_ktlo,
                    int has_lo, const float* __restrict__ beta, float scale, const float* __restrict__ S0,
                    __nv_bfloat16* __restrict__ o, float* __restrict__ ST,
                    const int32_t* __restrict__ cu, int N, int T, int H, long long limit_ns) {
    constexpr int DK = 128, BV = 64, C = 64, NVT = DV / BV;
    static_assert(DV == 128, "the T hand-off uses the two 128-byte slices of a 256-byte o row");
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
    [[maybe_unused]] const int64_t rows_all = cu ? (int64_t)T : (int64_t)N * T;  // debug-bounds checks

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR);
    uint64_t* tma_full = bars + 0;     // [2] ring stage landed
    uint64_t* stage_empty = bars + 2;  // [2] two arrivals: chain (W = T R done) and prep (Gram done)
    uint64_t* zt_full = bars + 4;      // [2] the stage's T tiles complete (identity rows past the
                                       // end); one per ring slot, so the prep cannot run a phase
                                       // ahead of a stage the chain has not released
    uint64_t* mma_c = bars + 6;        // W = T R
    uint64_t* mma_p = bars + 7;        // the prep's Gram
    uint64_t* mma_crit = bars + 8;     // D1 += [X; P] W (and everything the chain issued before)
    uint64_t* mma_s = bars + 9;        // S^T += K~^T W
    uint64_t* zxp_full = bars + 10;    // [X; P] tiles written
    uint64_t* d1a_done = bars + 11;    // D1 = [K; Q] S^T of the next chunk
    uint64_t* s_ready = bars + 12;     // the state's split written
    uint64_t* w_done = bars + 13;      // W split written
    uint64_t* o_free = bars + 14;      // a chunk's output rows read out of D1
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::TMEM_SLOT);
    // ring stages the sibling CTA (the head's other value tile) has loaded, written by the sibling
    uint32_t* peer_loaded = tmem_slot + 2;

    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, TC_TMEM_COLS);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&tma_full[0], 1);
        mbar_init(&tma_full[1], 1);
        mbar_init(&stage_empty[0], 2);
        mbar_init(&stage_empty[1], 2);
        mbar_init(&zt_full[0], 1);
        mbar_init(&zt_full[1], 1);
        mbar_init(mma_c, 1);
        mbar_init(mma_p, 1);
        mbar_init(mma_crit, 1);
        mbar_init(mma_s, 1);
        mbar_init(zxp_full, 1);
        mbar_init(d1a_done, 1);
        mbar_init(s_ready, 1);
        mbar_init(w_done, 1);
        mbar_init(o_free, 1);
        *peer_loaded = 0;
        tc::fence_mbar_init();
    }
    tc::fence_before_sync();
    tc::cluster_sync();  // both CTAs of the pair initialised before either writes to the other
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane = static_cast<uint32_t>((warp & 3) * 32) << 16;
    auto chunk_len = [&](int ch) -> int {
        const int64_t rem = count - (int64_t)ch * C;
        return rem < C ? (int)rem : C;
    };
    auto stage = [&](int i) { return smem + (i & 1) * L::STAGE; };
    constexpr uint32_t ID_3 = tc::idesc(1, 1, 1, 128, 64);  // K~^T x W
    constexpr uint32_t ID_G = tc::idesc(1, 0, 0, 128, 64);  // [K; Q] x K~^T
    const uint32_t aS[2] = {smem_u32(smem + L::SHI), smem_u32(smem + L::SLO)};
    const uint32_t aR[2] = {smem_u32(smem + L::RHI), smem_u32(smem + L::RLO)};

    if (warp == 8) {
        // =========================================================== producer
        // Lane 0 runs the ring's TMA loads and issues every MMA off the chain's critical path,
        // each once its inputs are ready (a thread that issues MMAs stalls while the tensor pipe
        // takes them, so the chain's own threads issue only the two groups they wait for):
        //   S^T += K~_{j-1}^T W_{j-1}       after D1_j += [X_j; P_{j-1}] W_{j-1} completed
        //   Gram [K_{j+1}; Q_j] K~_j^T      when stage j+1 has landed
        //   D1_{j+1} = [K_{j+1}; Q_j] S_j^T once the prep has split S_j
        if ((tid & 31) == 0 && nchunks > 0) {
            tc::prefetch_tmap(&tm_q);
            tc::prefetch_tmap(&tm_k);
            tc::prefetch_tmap(&tm_kt);
            tc::prefetch_tmap(&tm_v);
            tc::prefetch_tmap(&tm_tp);
            if (has_lo) tc::prefetch_tmap(&tm_ktlo);
            int pend[2] = {-1, -1};
            uint64_t* last_bar = nullptr;  // this thread's most recent MMA commit
            uint32_t last_par = 0;
            // stage i: K_i, V_i and the T_i tiles from the chunk's rows; Q_{i-1} and K~_{i-1} from
            // the 64 rows before (a negative row reads the fill value; rows past the end are unused)
            auto load = [&](int i) {
                const int s = i & 1;
                uint8_t* st = stage(i);
                const int row = (int)(first + (int64_t)i * C), prow = row - C;
                tc::mbar_expect_tx(&tma_full[s], has_lo ? L::STAGE : L::STAGE - 16384u);
                tc::tma_load_3d(st + L::KQ + 0, &tm_k, 0, h, row, &tma_full[s]);
                tc::tma_load_3d(st + L::KQ + 8192, &tm_q, 0, h, prow, &tma_full[s]);
                tc::tma_load_3d(st + L::KQ + 16384, &tm_k, 64, h, row, &tma_full[s]);
                tc::tma_load_3d(st + L::KQ + 24576, &tm_q, 64, h, prow, &tma_full[s]);
                tc::tma_load_3d(st + L::KT + 0, &tm_kt, 0, h, prow, &tma_full[s]);
                tc::tma_load_3d(st + L::KT + 8192, &tm_kt, 64, h, prow, &tma_full[s]);
                if (has_lo) {
                    tc::tma_load_3d(st + L::KTLO + 0, &tm_ktlo, 0, h, prow, &tma_full[s]);
                    tc::tma_load_3d(st + L::KTLO + 8192, &tm_ktlo, 64, h, prow, &tma_full[s]);
                }
                tc::tma_load_3d(st + L::V, &tm_v, c0, h, row, &tma_full[s]);
                tc::tma_load_3d(st + L::THI, &tm_tp, 0, h, row, &tma_full[s]);
                tc::tma_load_3d(st + L::TLO, &tm_tp, 32, h, row, &tma_full[s]);
                pend[s] = (i >> 1) & 1;
            };
            auto state_update = [&](int jj) {  // S^T += K~_jj^T W_jj (K~_jj sits in stage jj+1)
                const uint32_t aKT = smem_u32(stage(jj + 1) + L::KT);
#pragma unroll
                for (int p = 0; p < 2; ++p)
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc::mma_bf16(tmem + TC_COL_S, tc::sw128_desc(aKT + k * 2048, 8192, 1024),
                                     tc::sw128_desc(aR[p] + k * 2048, 8192, 1024), ID_3, 1);
                if (has_lo) {  // + K~_lo^T W_hi
                    const uint32_t aKL = smem_u32(stage(jj + 1) + L::KTLO);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc::mma_bf16(tmem + TC_COL_S, tc::sw128_desc(aKL + k * 2048, 8192, 1024),
                                     tc::sw128_desc(aR[0] + k * 2048, 8192, 1024), ID_3, 1);
                }
                tc::mma_commit(mma_s);
                last_bar = mma_s;
                last_par = (uint32_t)jj & 1u;
            };
            // stage i loaded (its T tiles read from both CTAs' output slices): tell the sibling
            const uint32_t peer_ctr = tc::cluster_map(smem_u32(peer_loaded), tc::cluster_rank() ^ 1u);
            load(0);
            load(1);
            bool ok = mbar_wait_bounded(&tma_full[0], 0u, limit_ns);
            if (ok) tc::st_cluster_release(peer_ctr, 1u);
            for (int j = 0; j < nchunks && ok; ++j) {
                const int i = j + 1;
                if (j > 0) {
                    if (!(ok = mbar_wait_bounded(mma_crit, (uint32_t)(j - 1) & 1u, limit_ns))) break;
                    tc::fence_after_sync();
                    state_update(j - 1);
                }
                if (!(ok = mbar_wait_bounded(&tma_full[i & 1], (uint32_t)(i >> 1) & 1u, limit_ns))) break;
                tc::st_cluster_release(peer_ctr, (uint32_t)i + 1u);
                {
                    const uint32_t aKQ = smem_u32(stage(i) + L::KQ), aKT = smem_u32(stage(i) + L::KT);
                    const int nk = has_lo ? 16 : 8;  // K~ = hi (+ lo): the lo term accumulates
#pragma unroll 1
                    for (int k = 0; k < nk; ++k)
                        tc::mma_bf16(tmem + TC_COL_G, tc::sw128_desc(aKQ + ((k >> 2) & 1) * 16384 + (k & 3) * 32, 16, 1024),
                                     tc::sw128_desc(aKT + (k >> 3) * (L::KTLO - L::KT) + ((k >> 2) & 1) * 8192 + (k & 3) * 32, 16, 1024),
                                     ID_G, k > 0);
                    tc::mma_commit(mma_p);
                    last_bar = mma_p;
                    last_par = (uint32_t)j & 1u;
                }
                if (j > 0) {  // (the chain issued D1_0 and D1_1); the buffer's O_{j-1} has been read
                    if (!(ok = mbar_wait_bounded(s_ready, (uint32_t)(j - 1) & 1u, limit_ns) &&
                               mbar_wait_bounded(o_free, (uint32_t)(j - 1) & 1u, limit_ns)))
                        break;
                    tc::fence_after_sync();
                    mma_kq_state(tmem + TC_COL_D1 + 128 * (i & 1), smem_u32(stage(i) + L::KQ), aS[0]);
                    tc::mma_commit(d1a_done);
                    last_bar = d1a_done;
                    last_par = (uint32_t)j & 1u;
                }
                if (j + 2 <= nchunks) {  // stage j+2 once both roles are done with stage j
                    if (!(ok = mbar_wait_bounded(&stage_empty[j & 1], (uint32_t)(j >> 1) & 1u, limit_ns))) break;
                    load(j + 2);
                }
            }
            if (ok && mbar_wait_bounded(mma_crit, (uint32_t)(nchunks - 1) & 1u, limit_ns)) {
                tc::fence_after_sync();
                state_update(nchunks - 1);
            }
            // let this CTA's own copies and MMAs land before the block can leave
            for (int s = 0; s < 2; ++s)
                if (pend[s] >= 0) mbar_wait_bounded(&tma_full[s], (uint32_t)pend[s], limit_ns);
            if (last_bar) mbar_wait_bounded(last_bar, last_par, limit_ns);
        }
    } else if (warp >= 4) {
        // =========================================================== prep
        // Iteration j: the split of S_j once S^T += K~_{j-1}^T W_{j-1} has landed; [X_{j+1}; P_j]
        // from the Gram; the T tiles of stage j+1 completed for a short chunk.
        const int t = tid - 128;  // 0..127 = tensor-memory lane
        const bool leader = t == 0;
        bool bad = false;
        auto finish_T = [&](int i) {  // rows past a short chunk's end: identity (hi), zero (lo)
            const int len = chunk_len(i);
            if (len < C && t >= len && t < C) {
                uint8_t* st = stage(i);
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    uint32_t w[4] = {0u, 0u, 0u, 0u};
                    if ((t >> 3) == g) w[(t & 7) >> 1] = (t & 1) ? 0x3f800000u : 0x00003f80u;  // bf16 1.0
                    const uint32_t off = tc::sw128_off((uint32_t)t, (uint32_t)g);
                    *reinterpret_cast<uint4*>(st + L::THI + off) = make_uint4(w[0], w[1], w[2], w[3]);
                    *reinterpret_cast<uint4*>(st + L::TLO + off) = make_uint4(0u, 0u, 0u, 0u);
                }
                tc::fence_async_smem();
            }
            group_bar(2, 128);
            if (leader) {
                mbar_arrive(&zt_full[i & 1]);
                mbar_arrive(&stage_empty[i & 1]);  // the prep's last use of stage i
            }
        };
        if (nchunks > 0) {
            bad = group_any(2, 128, !mbar_wait_bounded(&tma_full[0], 0u, limit_ns));
            if (!bad) finish_T(0);
        }
        for (int j = 0; j < nchunks && !bad; ++j) {
            const int i = j + 1;
            // job 0 (j > 0): split S_j once S^T += K~_{j-1}^T W_{j-1} has landed (its previous split
            // was last read by D1_j, already complete); job 1: [X_{j+1}; P_j] from the Gram (lanes
            // 0..63: X_{j+1} = K_{j+1} K~_j^T; lanes 64..127: P_j = tril(Q_j K~_j^T)), whose tiles'
            // previous contents were last read by D1_j += [X_j; P_{j-1}] W_{j-1}, which the state
            // update waited for.  One code body for both (the roles share the instruction cache).
#pragma unroll 1
            for (int job = j > 0 ? 0 : 1; job < 2; ++job) {
                uint64_t* bar = job ? mma_p : mma_s;
                if (group_any(2, 128, !mbar_wait_bounded(bar, (uint32_t)(job ? j : j - 1) & 1u, limit_ns))) {
                    bad = true;
                    break;
                }
                tc::fence_after_sync();
                float x[64];
                tc::tmem_ld64(tmem + lane + (job ? TC_COL_G : TC_COL_S), x);
                if (job) {  // [X; P] split into the Gram's own columns (the chain's MMA reads it there)
                    if (t >= 64) {
                        const int r = t - 64;
#pragma unroll
                        for (int c = 0; c < 64; ++c) x[c] = c <= r ? x[c] : 0.f;
                    }
                    uint32_t hw[32], lw[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) split2_bf16(x[2 * c], x[2 * c + 1], hw[c], lw[c]);
                    const uint32_t tg = tmem + lane + TC_COL_G;
                    tc::tmem_st16(tg + 0, reinterpret_cast<const float*>(hw));
                    tc::tmem_st16(tg + 16, reinterpret_cast<const float*>(hw + 16));
                    tc::tmem_st16(tg + 32, reinterpret_cast<const float*>(lw));
                    tc::tmem_st16(tg + 48, reinterpret_cast<const float*>(lw + 16));
                    tc::tmem_st_wait();
                } else {
                    st_row_split_bf16(smem + L::SHI, smem + L::SLO, t, x);
                    tc::fence_async_smem();
                }
                tc::fence_before_sync();
                group_bar(2, 128);
                if (leader) mbar_arrive(job ? zxp_full : s_ready);
            }
            if (bad) break;
            if (i < nchunks) {  // once stage i's copies have landed
                if (group_any(2, 128, !mbar_wait_bounded(&tma_full[i & 1], (uint32_t)(i >> 1) & 1u, limit_ns))) {
                    bad = true;
                    break;
                }
                finish_T(i);
            }
        }
    } else {
        // =========================================================== chain
        // Warps 0-1 (lanes 0..63, the chunk's token rows of D1): per chunk j, R_j from D1_j, the
        // MMA W_j = T_j R_j, then D1_{j+1} += [X_{j+1}; P_j] W_j once warps 2-3 have split W_j.
        // Warps 2-3 (lanes 64..127): the split of W_j (lanes 64..127 of D2) and the output rows
        // O_j (lanes 64..127 of D1_{j+1}).  The two halves meet only through mbarriers.
        const int t = tid;  // 0..127 = tensor-memory lane
        const bool lower = t < 64, leader = t == 0 || t == 64;
        const int gbar = lower ? 1 : 3;  // each half's own named barrier
        const uint32_t t_S = tmem + lane + TC_COL_S, t_D2 = tmem + lane + TC_COL_D2;
        bool ok = true;
        uint64_t* last_bar = nullptr;  // the lower leader's most recent commit
        uint32_t last_par = 0;
        auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
            return !group_any(gbar, 64, !mbar_wait_bounded(bar, parity, limit_ns));
        };
        // two barriers, one vote
        auto wait_all2 = [&](uint64_t* b0, uint32_t p0, uint64_t* b1, uint32_t p1) -> bool {
            const bool got = mbar_wait_bounded(b0, p0, limit_ns) && mbar_wait_bounded(b1, p1, limit_ns);
            return !group_any(gbar, 64, !got);
        };
        // initial state: S^T lane i = key channel i, columns = this CTA's value channels
        {
            float s0[64];
#pragma unroll
            for (int c = 0; c < 64; ++c) s0[c] = S0 ? __ldg(S0 + sbase + (int64_t)c * DK + t) : 0.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) tc::tmem_st16(t_S + 16 * q, s0 + 16 * q);
            tc::tmem_st_wait();
            st_row_split_bf16(smem + L::SHI, smem + L::SLO, t, s0);
            tc::fence_async_smem();
            tc::fence_before_sync();
        }
        group_bar(1, 128);  // both halves' rows of the state split are written
        if (lower) {
            if (nchunks > 0) {  // D1_0 = [K_0; .] S_0^T and D1_1 = [K_1; Q_0] S_0^T
                ok = wait_all(&tma_full[0], 0u) && wait_all(&tma_full[1], 0u);
                if (ok && leader) {
                    tc::fence_after_sync();
                    mma_kq_state(tmem + TC_COL_D1, smem_u32(stage(0) + L::KQ), aS[0]);
                    mma_kq_state(tmem + TC_COL_D1 + 128, smem_u32(stage(1) + L::KQ), aS[0]);
                    tc::mma_commit(d1a_done);
                    last_bar = d1a_done;
                    last_par = 0;
                }
            }
            float bnext = (nchunks > 0 && t < chunk_len(0)) ? __ldg(beta + (first + t) * H + h) : 0.f;
            for (int j = 0; j < nchunks && ok; ++j) {
                const int s = j & 1;
                const float bt = bnext;
                if (j + 1 < nchunks)
                    bnext = t < chunk_len(j + 1) ? __ldg(beta + (first + (int64_t)(j + 1) * C + t) * H + h) : 0.f;
                // D1_j complete (D1_0 alone, else [X_j; P_{j-1}] W_{j-1} on top of it), V_j landed
                if (!wait_all2(j == 0 ? d1a_done : mma_crit, (uint32_t)(j == 0 ? 0 : j - 1) & 1u,
                               &tma_full[s], (uint32_t)(j >> 1) & 1u)) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                float y[64];  // R = beta (V - K S^T), token row t
                tmem_ld64_sum(tmem + lane + TC_COL_D1 + 128 * s, y);
                const uint8_t* vtile = stage(j) + L::V;
                const float2 bt2 = make_float2(bt, bt), m1 = make_float2(-1.f, -1.f);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const uint4 raw = *reinterpret_cast<const uint4*>(vtile + tc::sw128_off(t, q));
                    const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 vv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[e]));
                        // beta (v - y): the fma with -1 rounds v - y once, as a subtraction does
                        const float2 d = __ffma2_rn(make_float2(y[8 * q + 2 * e], y[8 * q + 2 * e + 1]), m1, vv);
                        const float2 yy = __fmul2_rn(bt2, d);
                        y[8 * q + 2 * e] = yy.x;
                        y[8 * q + 2 * e + 1] = yy.y;
                    }
                }
                // W_{j-1} (the R tiles' previous contents) has been read by the state update
                if (j > 0 && !wait_all(mma_s, (uint32_t)(j - 1) & 1u)) {
                    ok = false;
                    break;
                }
                st_row_split_bf16(smem + L::RHI, smem + L::RLO, t, y);
                tc::fence_async_smem();
                tc::fence_before_sync();
                if (!wait_all(&zt_full[s], (uint32_t)(j >> 1) & 1u)) {
                    ok = false;
                    break;
                }
                if (leader) {
                    // [V; T hi] and [T hi; T lo]: the stage's T tiles preceded by 64 stable rows
                    const uint32_t aT[2] = {smem_u32(stage(j) + L::THI) - 8192u, smem_u32(stage(j) + L::TLO) - 8192u};
                    tc::fence_after_sync();
                    mma_split3(tmem + TC_COL_D2, aT, aR[0], false);  // lanes 64..127: W
                    tc::mma_commit(mma_c);
                    last_bar = mma_c;
                    last_par = (uint32_t)j & 1u;
                }
                // W_j split by warps 2-3, [X_{j+1}; P_j] written, D1_{j+1} = [K_{j+1}; Q_j] S_j^T complete
                const bool got = mbar_wait_bounded(w_done, (uint32_t)j & 1u, limit_ns) &&
                                 mbar_wait_bounded(zxp_full, (uint32_t)j & 1u, limit_ns) &&
                                 mbar_wait_bounded(d1a_done, (uint32_t)j & 1u, limit_ns);
                if (group_any(gbar, 64, !got)) {
                    ok = false;
                    break;
                }
                if (leader) {
                    tc::fence_after_sync();
                    mma_split3_ts(tmem + TC_COL_D1 + 128 * ((j + 1) & 1), tmem + TC_COL_G, aR[0], true);
                    tc::mma_commit(mma_crit);
                    last_bar = mma_crit;
                    last_par = (uint32_t)j & 1u;
                }
            }
        } else {
            const int r = t - 64;  // row of W and of the output
            for (int j = 0; j < nchunks && ok; ++j) {
                // ---- W_j = lanes 64..127 of D2, into the R tiles (R_j has been consumed)
                if (!wait_all(mma_c, (uint32_t)j & 1u)) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                if (leader) mbar_arrive(&stage_empty[j & 1]);  // the chain's last use of stage j
                {
                    float w[64];
                    tmem_ld64_sum(t_D2, w);
                    st_row_split_bf16(smem + L::RHI, smem + L::RLO, r, w);
                    tc::fence_async_smem();
                }
                tc::fence_before_sync();
                group_bar(3, 64);
                if (leader) mbar_arrive(w_done);
                // ---- O_j = lanes 64..127 of D1_{j+1} once D1_{j+1} += [X_{j+1}; P_j] W_j landed and
                //      the sibling CTA has loaded stage j (it reads T_j from this CTA's slice of o)
                if (!wait_all(mma_crit, (uint32_t)j & 1u) ||
                    group_any(3, 64, leader && !tc::wait_counter(smem_u32(peer_loaded), (uint32_t)j + 1u, limit_ns))) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                float x[64];
                tmem_ld64_sum(tmem + lane + TC_COL_D1 + 128 * ((j + 1) & 1), x);
                if (r < chunk_len(j) && OSDN_IN_BOUNDS(first + (int64_t)j * C + r, rows_all)) {
                    __nv_bfloat16* orow = o + ((first + (int64_t)j * C + r) * H + h) * DV + c0;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        uint32_t pk[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 sx = __fmul2_rn(make_float2(scale, scale),
                                                         make_float2(x[8 * q + 2 * e], x[8 * q + 2 * e + 1]));
                            const __nv_bfloat162 b2 = __floats2bfloat162_rn(sx.x, sx.y);
                            pk[e] = *reinterpret_cast<const uint32_t*>(&b2);
                        }
                        *reinterpret_cast<uint4*>(orow + 8 * q) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    }
                }
                tc::fence_before_sync();
                group_bar(3, 64);
                if (leader) mbar_arrive(o_free);  // D1_{j+1}'s output rows have been read
            }
        }
        // final state: both halves once the last state update has landed
        if (ok && nchunks > 0) ok = wait_all(mma_s, (uint32_t)(nchunks - 1) & 1u);
        if (ok && ST) {
            tc::fence_after_sync();
            float s1[64];
            tc::tmem_ld64(t_S, s1);
#pragma unroll
            for (int c = 0; c < 64; ++c)
                if (OSDN_IN_BOUNDS(sbase + (int64_t)c * DK + t, (int64_t)N * H * DV * DK))
                    ST[sbase + (int64_t)c * DK + t] = s1[c];
        }
        if (!ok && lower && leader && last_bar) mbar_wait_bounded(last_bar, last_par, limit_ns);
    }
    tc::fence_before_sync();
    tc::cluster_sync();  // neither CTA leaves while the other may still write its counter
    if (warp == 0) tc::tmem_dealloc(tmem, TC_TMEM_COLS);
}

}  // namespace osdn
