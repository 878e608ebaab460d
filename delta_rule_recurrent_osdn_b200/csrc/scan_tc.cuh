// scan_tc.cuh -- phase 1 of the OSDN forward pass (bf16 I/O, d_k = 128) as two kernels.
//
// The preconditioner recurrence ("OSDN: Improving Delta Rule with Provable Online
// Preconditioning in Linear Attention", technical summary, sections 2.2 and 2.3; section 2.3
// notes that the APF update keeps the recurrence affine) is, with a_t = k_t (.) k_t,
// e_t = eta beta_t / ||k_t||^2 (0 when k_t = 0) and x_t = e_t (1 - beta_t <d_t, a_t>):
//   d_{t+1} = r_t d_t + x_t a_t,     k~_t = d_t (.) k_t.
// Within a chunk of C = 64 tokens starting from d_0, with R_t = prod_{i<t} r_i and
// Gamma_tj = prod_{j<i<t} r_i:
//   <d_t, a_t> = R_t <d_0, a_t> + sum_{j<t} Gamma_tj <a_j, a_t> x_j, hence
//   (I + L_d) x = b,  b = e (.) (1 - beta (.) R (.) A d_0),  L_d[t][j] = e_t beta_t Gamma_tj <a_t, a_j>,
//   d_C = R_C d_0 + A^T (g (.) x),  g_j = Gamma_Cj.
// L_d and T_d = (I + L_d)^-1 do not depend on d_0, so they are computed for every chunk at once
// by precond_prep_kernel; what remains sequential across chunks is three matrix-vector products
// per chunk (p = A d_0, x = T_d b, d_C), done by precond_chain_kernel, whose other warps emit
// k~ for each chunk by the token recurrence above while the next chunk's products run.
//
// Hand-off without extra memory: for d_k = 128 in bf16, one chunk's k~ rows (64 tokens x 256 B)
// are exactly the size of its fp32 64 x 64 T_d.  The prep kernel writes T_d into the k~ buffer,
// at the chunk's own rows; the chain kernel loads it (TMA) before it overwrites those rows with
// k~.  Row t of T_d is stored with the 16-byte groups permuted as in the tsw layout
// (tril_inverse.cuh), so a straight copy into shared memory is ready for conflict-free reads.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "tc_ptx.cuh"
#include "tril_inverse.cuh"
#include "chunk_walk.cuh"

namespace osdn {

constexpr int SCAN_C = kChunk;

// Gate prefix quantities of one chunk, computed by one warp (lane l: tokens 2l and 2l + 1).
// r is 1 and beta 0 for tokens past the chunk's end.  Gamma_tj = sg[t] sg1[j] exp(lr[t] - lr1[j]).
struct GatePrefix {
    float lr0, lr1_0, lr_1, lr1_1;  // lr and lr1 of tokens 2l, 2l + 1
    float sg0, sg1_0, sg_1, sg1_1;
    float lrC, sgC;                 // over the whole chunk
};

__device__ __forceinline__ GatePrefix gate_prefix(float r0, float r1, int lane) {
    const float l0 = __logf(fmaxf(fabsf(r0), 1e-30f)), l1 = __logf(fmaxf(fabsf(r1), 1e-30f));
    const int n0 = r0 < 0.f, n1 = r1 < 0.f;
    float ps = l0 + l1;
    int pn = n0 + n1;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float ys = __shfl_up_sync(0xffffffffu, ps, off);
        const int yn = __shfl_up_sync(0xffffffffu, pn, off);
        if (lane >= off) {
            ps += ys;
            pn += yn;
        }
    }
    GatePrefix g;
    const float ex = ps - (l0 + l1);
    const int en = pn - (n0 + n1);
    g.lr0 = ex;
    g.lr_1 = ex + l0;
    g.lr1_0 = ex + l0;
    g.lr1_1 = ex + l0 + l1;
    g.sg0 = (en & 1) ? -1.f : 1.f;
    g.sg_1 = ((en + n0) & 1) ? -1.f : 1.f;
    g.sg1_0 = g.sg_1;
    g.sg1_1 = ((en + n0 + n1) & 1) ? -1.f : 1.f;
    g.lrC = __shfl_sync(0xffffffffu, ps, 31);
    g.sgC = (__shfl_sync(0xffffffffu, pn, 31) & 1) ? -1.f : 1.f;
    return g;
}

// ===================================================================== prep: T_d per chunk

struct ScanPrepSmem {
    static constexpr uint32_t K = 0;              // bf16 k tile: 2 K-blocks x (64 rows x 128 B)
    static constexpr uint32_t A = 16384;          // bf16 [a_hi; a_lo] per K-block, 2 x 16 KB
    static constexpr uint32_t SL = A;             // fp32 L_d, then T_d (tsw), over A after the Gram
    static constexpr uint32_t ST = A + 16384;     // fp32 scratch (tsw), over A
    static constexpr uint32_t VEC = A + 32768;    // c, lr, lr1, sg, sg1, R, Rinv, e (8 x 64) + flag
    static constexpr uint32_t BAR = VEC + 8 * 256 + 16;
    static constexpr uint32_t TMEM_SLOT = BAR + 16;
    static constexpr uint32_t TOTAL = TMEM_SLOT + 16;
    static constexpr size_t BYTES = TOTAL + 1024;
};
constexpr int SCAN_PREP_CTAS_PER_SM = 4;

// Persistent grid (one to three CTAs per SM) of 128 threads walking the batch's chunks with
// ChunkWalk.  td_out is the k~ buffer seen as fp32 rows of 64 values.
__global__ void __launch_bounds__(128, SCAN_PREP_CTAS_PER_SM)
precond_prep_kernel(const __grid_constant__ CUtensorMap tm_k, const float* __restrict__ beta,
                    const float* __restrict__ r, float eta, float* __restrict__ td_out,
                    const int32_t* __restrict__ cu, int N, int T, int H, int64_t rows,
                    long long limit_ns) {
    using L = ScanPrepSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_align1024(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    ChunkWalk walk;
    walk.init(cu, N, T, H, rows);
    if (!walk.next()) return;  // uniform over the CTA

    uint64_t* tma_bar = reinterpret_cast<uint64_t*>(smem + L::BAR);
    uint64_t* mma_bar = tma_bar + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::TMEM_SLOT);
    uint8_t* sK = smem + L::K;
    uint8_t* sA = smem + L::A;
    float* sL = reinterpret_cast<float*>(smem + L::SL);
    float* sT = reinterpret_cast<float*>(smem + L::ST);
    float* vc = reinterpret_cast<float*>(smem + L::VEC);
    float* vlr = vc + 64;
    float* vlr1 = vc + 128;
    float* vsg = vc + 192;
    float* vsg1 = vc + 256;
    float* vR = vc + 320;     // sg e^lr
    float* vRi = vc + 384;    // sg1 e^-lr1
    float* ve = vc + 448;     // e = eta beta / ||k||^2 (0 for a zero key or past the end)
    int* vsafe = reinterpret_cast<int*>(vc + 512);

    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, 128);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(tma_bar, 1);
        mbar_init(mma_bar, 1);
        tc::fence_mbar_init();
        tc::prefetch_tmap(&tm_k);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tlane = static_cast<uint32_t>(warp * 32) << 16;

    auto issue_load = [&](int64_t row, int hh) {
        tc::mbar_expect_tx(tma_bar, 16384);
        tc::tma_load_3d(sK, &tm_k, 0, hh, (int)row, tma_bar);
        tc::tma_load_3d(sK + 8192, &tm_k, 64, hh, (int)row, tma_bar);
    };
    if (tid == 0) issue_load(walk.row0, walk.h);
    bool tma_pend = tid == 0, mma_pend = false, fail = false, more = true;
    uint32_t tph = 0, mph = 0;
    constexpr uint32_t ID_G = tc::idesc(1, 0, 0, 128, 64);

#pragma unroll 1
    while (more) {
        const int64_t row0 = walk.row0;
        const int Lc = walk.Lc, h = walk.h;
        const bool got = mbar_wait_bounded(tma_bar, tph, limit_ns);
        if (__syncthreads_or(!got)) {
            fail = true;
            break;
        }
        tph ^= 1u;
        tma_pend = false;
        // ---- a = k (.) k split into bf16 hi + lo rows; e and c = e beta per token.
        //      Thread: row t = 16 warp + (lane & 15), K-block = lane >> 4.
        {
            const int t = 16 * warp + (lane & 15), blk = lane >> 4;
            const bool valid = t < Lc;
            float nk = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t off = blk * 8192u + tc::sw128_off(t, j);
                uint4 raw = *reinterpret_cast<const uint4*>(sK + off);
                if (!valid) raw = make_uint4(0u, 0u, 0u, 0u);  // rows past the chunk's end: a = 0
                const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 kk = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[e]));
                    const float2 a = __fmul2_rn(kk, kk);
                    nk += a.x + a.y;
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(a.x, a.y);
                    const float2 hf = __bfloat1622float2(h2);
                    const float2 ld = __ffma2_rn(hf, make_float2(-1.f, -1.f), a);  // a - hi, exact
                    const __nv_bfloat162 l2 = __floats2bfloat162_rn(ld.x, ld.y);
                    hi[e] = *reinterpret_cast<const uint32_t*>(&h2);
                    lo[e] = *reinterpret_cast<const uint32_t*>(&l2);
                }
                const uint32_t aoff = blk * 16384u + tc::sw128_off(t, j);
                *reinterpret_cast<uint4*>(sA + aoff) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4*>(sA + aoff + 8192u) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
            nk += __shfl_xor_sync(0xffffffffu, nk, 16);
            if (blk == 0) {
                const float bt = valid ? __ldg(beta + (row0 + t) * H + h) : 0.f;
                const float e = nk > 0.f ? eta * bt / nk : 0.f;
                vc[t] = e * bt;
                ve[t] = e;
            }
        }
        if (warp == 3) {  // prefix of log|r| over the chunk
            const int t0 = 2 * lane;
            const float r0 = (r && t0 < Lc) ? __ldg(r + (row0 + t0) * H + h) : 1.f;
            const float r1 = (r && t0 + 1 < Lc) ? __ldg(r + (row0 + t0 + 1) * H + h) : 1.f;
            const GatePrefix g = gate_prefix(r0, r1, lane);
            vlr[t0] = g.lr0;
            vlr[t0 + 1] = g.lr_1;
            vlr1[t0] = g.lr1_0;
            vlr1[t0 + 1] = g.lr1_1;
            vsg[t0] = g.sg0;
            vsg[t0 + 1] = g.sg_1;
            vsg1[t0] = g.sg1_0;
            vsg1[t0 + 1] = g.sg1_1;
            // Gamma_tj = (sg_t e^lr_t) (sg1_j e^-lr1_j) when every prefix is within +-80 (both
            // factors then stay inside the fp32 range); otherwise one exponential per entry
            const float mx = fmaxf(fmaxf(fabsf(g.lr0), fabsf(g.lr_1)), fmaxf(fabsf(g.lr1_0), fabsf(g.lr1_1)));
            const bool safe = __all_sync(0xffffffffu, mx < 80.f);
            vR[t0] = g.sg0 * __expf(g.lr0);
            vR[t0 + 1] = g.sg_1 * __expf(g.lr_1);
            vRi[t0] = g.sg1_0 * __expf(-g.lr1_0);
            vRi[t0 + 1] = g.sg1_1 * __expf(-g.lr1_1);
            if (lane == 0) *vsafe = safe ? 1 : 0;
        }
        tc::fence_async_smem();
        tc::fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            tc::fence_after_sync();
            // Gram: cols 0..63 = [a_hi; a_lo] a_hi^T, cols 64..127 = [a_hi; a_lo] a_lo^T
            const uint32_t aA = smem_u32(sA);
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const uint32_t o = (s >> 2) * 16384u + (s & 3) * 32u;
                tc::mma_bf16(tmem + 0, tc::sw128_desc(aA + o, 16, 1024), tc::sw128_desc(aA + o, 16, 1024),
                             ID_G, s > 0);
                tc::mma_bf16(tmem + 64, tc::sw128_desc(aA + o, 16, 1024),
                             tc::sw128_desc(aA + o + 8192, 16, 1024), ID_G, s > 0);
            }
            tc::mma_commit(mma_bar);
            mma_pend = true;
        }
        more = walk.next();  // uniform: every thread walks the same items
        if (tid == 0 && more) {  // the key tile has been read: fetch the next chunk's
            tc::fence_async_smem();
            issue_load(walk.row0, walk.h);
            tma_pend = true;
        }
        const bool mdone = mbar_wait_bounded(mma_bar, mph, limit_ns);
        if (__syncthreads_or(!mdone)) {
            fail = true;
            break;
        }
        mph ^= 1u;
        mma_pend = false;
        tc::fence_after_sync();
        // ---- G = hi hi^T + hi lo^T (lanes 0..63) + lo hi^T (lanes 64..127, added through sT)
        {
            float* dst = warp < 2 ? sL : sT;
            const int row = warp < 2 ? tid : tid - 64;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float g0[16], g1[16];
                tc::tmem_ld16(tmem + tlane + 16 * q, g0);
                if (warp < 2) tc::tmem_ld16(tmem + tlane + 64 + 16 * q, g1);
                tc::tmem_ld_wait();
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    float4 o;
                    o.x = g0[4 * v] + (warp < 2 ? g1[4 * v] : 0.f);
                    o.y = g0[4 * v + 1] + (warp < 2 ? g1[4 * v + 1] : 0.f);
                    o.z = g0[4 * v + 2] + (warp < 2 ? g1[4 * v + 2] : 0.f);
                    o.w = g0[4 * v + 3] + (warp < 2 ? g1[4 * v + 3] : 0.f);
                    tsw_st4(dst, row, 4 * q + v, o);
                }
            }
        }
        tc::fence_before_sync();
        __syncthreads();
        // ---- L_d[t][j] = c_t Gamma_tj G_tj for j < t; thread: row t = tid & 63, 32 columns
        {
            const int t = tid & 63, g0 = 8 * (tid >> 6);
            const float ct = vc[t], lrt = vlr[t], sgt = vsg[t];
            const bool safe = *vsafe != 0;  // uniform over the CTA
            const float cr = ct * vR[t];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 a = tsw_ld4(sL, t, g0 + q), b = tsw_ld4(sT, t, g0 + q);
                const float gs[4] = {a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w};
                float o[4];
                if (safe) {
                    const float4 ri = *reinterpret_cast<const float4*>(vRi + 4 * (g0 + q));
                    const float rv[4] = {ri.x, ri.y, ri.z, ri.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        o[e] = 4 * (g0 + q) + e < t ? cr * rv[e] * gs[e] : 0.f;
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = 4 * (g0 + q) + e;
                        o[e] = j < t ? ct * sgt * vsg1[j] * __expf(lrt - vlr1[j]) * gs[e] : 0.f;
                    }
                }
                tsw_st4(sL, t, g0 + q, make_float4(o[0], o[1], o[2], o[3]));
            }
        }
        __syncthreads();
        tril_inverse_64_g128(sL, tid, 1);  // T_d over L_d
        // e_t rides in the tile's upper-right block (rows 0-1, columns 32-63), which holds only
        // scratch of the inverse: the chain kernel reads it there instead of recomputing ||k_t||
        if (tid < 64) sL[tsw(tid >> 5, 32 + (tid & 31))] = ve[tid];
        __syncthreads();
        // ---- rows t < Lc of T_d (tsw order kept) to the chunk's rows of the k~ buffer; 16 lanes
        //      per row, so a warp reads two whole rows (no bank conflicts) and writes them whole
#pragma unroll
        for (int it = 0; it < 8; ++it) {
            const int idx = it * 128 + tid, t = idx >> 4, piece = idx & 15;
            if (t < Lc && OSDN_IN_BOUNDS(row0 + t, rows))
                reinterpret_cast<float4*>(td_out + ((row0 + t) * H + h) * 64)[piece] =
                    reinterpret_cast<const float4*>(sL + t * 64)[piece];
        }
        __syncthreads();  // sT and sL lie over the next chunk's a tiles
    }
    if (fail && tid == 0) {
        if (tma_pend) mbar_wait_bounded(tma_bar, tph, limit_ns);
        if (mma_pend) mbar_wait_bounded(mma_bar, mph, limit_ns);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 128);
}

// ===================================================================== chain: d across chunks

struct ScanChainSmem {
    // rank 0 (the chain)
    static constexpr uint32_t KT = 0;                 // 3 x bf16 k tiles (16 KB, SW128)
    static constexpr uint32_t TD = 3 * 16384;         // 3 x fp32 T_d tiles (16 KB, tsw rows)
    // rank 1 (the k~ token pass): a deeper key ring, staging tiles per writer group
    static constexpr int NS1 = 5;                     // key ring slots
    static constexpr int NG = 4;                      // writer groups
    static constexpr uint32_t KT1 = 0;                // NS1 x bf16 k tiles
    static constexpr uint32_t HI = NS1 * 16384;       // NG x bf16 k~ hi staging tile (SW128)
    static constexpr uint32_t LO = HI + NG * 16384;   // NG x bf16 k~ lo staging tile (SW128)
    static constexpr uint32_t RV = LO + NG * 16384;   // NS1 x r of the chunk [64]
    static constexpr uint32_t XR = RV + NS1 * 256;    // NG x x of a chunk [64], from rank 0
    static constexpr uint32_t DR = XR + NG * 256;     // NG x chunk-start d [128], from rank 0
    // rank 0
    static constexpr uint32_t VEC = DR + NG * 512;    // 3 x {R, g, r, beta, R_C, e, beta R}
    static constexpr uint32_t VECB = 2048;
    static constexpr uint32_t D = VEC + 3 * VECB;     // 3 x d at chunk start [128]
    static constexpr uint32_t X = D + 3 * 512;        // 3 x x [64]
    static constexpr uint32_t GX = X + 3 * 256;       // g (.) x [64]
    static constexpr uint32_t BV = GX + 256;          // b [64]
    static constexpr uint32_t XW = BV + 256;          // NG x the writer groups' copy of x [64]
    static constexpr uint32_t BAR = XW + NG * 256;    // 29 mbarriers
    static constexpr uint32_t FAIL = BAR + 29 * 8;    // rank 0: the loader's failure flag
    static constexpr uint32_t TOTAL = FAIL + 16;
    static constexpr size_t BYTES = TOTAL + 1024;
};
static_assert(ScanChainSmem::BYTES <= 232448, "shared memory");
// rank 0: warps 0-7 the chain's products, 8 the chain's per-chunk inputs, 9 the forwarder and
// refills; rank 1: warps 0-7 the k~ output (four groups of two warps), 8 loads
constexpr int SCAN_CHAIN_THREADS = 320;

// One 2-CTA cluster per (sequence, head).  Rank 0 runs the chain (warps 0-7), a loader (warp 8:
// waits for each chunk's k and T_d tiles, writes the gate vectors, e_t and beta_t R_t, then meets
// the chain at a named barrier, so the chain threads never wait on an mbarrier) and a forwarder
// (warp 9: refills the ring slot the chain has finished with, copies x and the chunk-start d of
// each chunk into rank 1's shared memory and arrives on rank 1's barrier, release / acquire at
// cluster scope); rank 1 runs the k~ token pass (warps 0-7) and its own loads (warp 8: k tiles,
// r).  The token pass gets an SM of its own.  Rank 1's writers copy x out and arrive back on
// rank 0 before their token pass.  The two CTAs of a cluster are co-scheduled, so these
// cross-CTA waits are safe (and bounded like every other).  td_in is the k~ buffer holding the
// prep kernel's T_d tiles.
// k_tilde receives k~ rounded to bf16 (hi); with kLo, k_tilde_lo receives the rounding residual
// bf16(k~ - hi), so that hi + lo carries k~ to about 2^-17 of its size.  With kD, d_all
// ([B,T,H,Dk] fp32) receives d_t, the preconditioner each token writes with.  (Compile-time
// options: the token pass is issue-bound, and the forward pass needs neither check.)
template <bool kLo, bool kD>
__global__ void __launch_bounds__(SCAN_CHAIN_THREADS, 1)
precond_chain_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_td,
                     const __grid_constant__ CUtensorMap tm_kto, const __grid_constant__ CUtensorMap tm_ktlo,
                     const float* __restrict__ beta, const float* __restrict__ r, float eta,
                     const float* __restrict__ d0, __nv_bfloat16* __restrict__ k_tilde,
                     __nv_bfloat16* __restrict__ k_tilde_lo, float* __restrict__ d_all,
                     float* __restrict__ dT, float* __restrict__ rho,
                     const int32_t* __restrict__ cu, int N, int T, int H, long long limit_ns) {
    constexpr int C = SCAN_C, DK = 128;
    using L = ScanChainSmem;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_align1024(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = tc::cluster_rank();  // 0: the chain, 1: the k~ token pass
    const int pair = blockIdx.x >> 1;
    const int n = pair / H, h = pair - n * H;
    if (n >= N) return;  // uniform over the cluster
    int64_t first, count;
    if (!seq_range(cu, n, N, T, first, count)) return;  // uniform over the cluster
    const int nchunks = (int)((count + C - 1) / C);
    const int64_t dbase = ((int64_t)n * H + h) * DK;
    [[maybe_unused]] const int64_t rows_all = cu ? (int64_t)T : (int64_t)N * T;  // debug-bounds checks

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR);
    uint64_t* full = bars;         // [5] TMA: k tile (+ T_d tile on rank 0, whose ring has 3 slots)
    uint64_t* vready = bars + 5;   // [5] rank 1: r of the chunk (32 arrivals)
    uint64_t* kempty = bars + 10;  // [5] rank 1: slot released by the chunk's writer group (64)
    // x and d cross to rank 1 through NG receive slots: a writer group is at most NG chunks
    // ahead of the forwarder, so a slot's barrier is never waited on two phases early
    uint64_t* xready = bars + 15;  // [NG] rank 1: x and d of a chunk, from rank 0's forwarder (32)
    uint64_t* outdone = bars + 19; // [NG] rank 0: rank 1's writer group has copied x / d (64)
    uint64_t* fwdin = bars + 23;   // [3] rank 0: x and d of a chunk in local memory, the chain
                                   //     done with the slot (256)
    uint64_t* fwdout = bars + 26;  // [3] rank 0: the forwarder has sent them (32)
    float* sD = reinterpret_cast<float*>(smem + L::D);
    float* sX = reinterpret_cast<float*>(smem + L::X);
    float* sGX = reinterpret_cast<float*>(smem + L::GX);
    float* sB = reinterpret_cast<float*>(smem + L::BV);
    auto vecs = [&](int s) { return reinterpret_cast<float*>(smem + L::VEC + s * L::VECB); };
    auto chunk_len = [&](int c) -> int {
        const int64_t rem = count - (int64_t)c * C;
        return rem < C ? (int)rem : C;
    };

    if (tid == 0) {
        for (int s = 0; s < L::NS1; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&vready[s], 32);
            mbar_init(&kempty[s], 64);
        }
        for (int s = 0; s < L::NG; ++s) {
            mbar_init(&xready[s], 32);
            mbar_init(&outdone[s], 64);
        }
        for (int s = 0; s < 3; ++s) {
            mbar_init(&fwdin[s], 256);
            mbar_init(&fwdout[s], 32);
        }
        tc::fence_mbar_init();
    }
    if (tid < DK) sD[tid] = d0 ? __ldg(d0 + dbase + tid) : 1.0f;
    if (tid == 0) *reinterpret_cast<int*>(smem + L::FAIL) = 0;
    tc::fence_before_sync();
    tc::cluster_sync();  // both CTAs initialised before either touches the other
    // rank 0's view of rank 1's x / d buffers and barriers, and rank 1's of rank 0's
    const uint32_t peer_x = tc::cluster_map(smem_u32(smem + L::XR), 1u);
    const uint32_t peer_d = tc::cluster_map(smem_u32(smem + L::DR), 1u);
    const uint32_t peer_xready = tc::cluster_map(smem_u32(xready), 1u);
    const uint32_t peer_outdone = tc::cluster_map(smem_u32(outdone), 0u);

    if (warp == 8 && rank == 1) {
        // =============================================== rank 1: k tiles and r for the token pass
        if (lane == 0) tc::prefetch_tmap(&tm_k);
        constexpr int NS = L::NS1;
        int last_issued = -1;
        bool fail = false;
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % NS;
            if (c >= NS && !mbar_wait_bounded(&kempty[s], (uint32_t)(c / NS - 1) & 1u, limit_ns)) {
                fail = true;
                break;
            }
            const int64_t row0 = first + (int64_t)c * C;
            if (lane == 0) {
                uint8_t* kt = smem + L::KT1 + s * 16384;
                tc::mbar_expect_tx(&full[s], 16384);
                tc::tma_load_3d(kt, &tm_k, 0, h, (int)row0, &full[s]);
                tc::tma_load_3d(kt + 8192, &tm_k, 64, h, (int)row0, &full[s]);
            }
            last_issued = c;
            const int Lc = chunk_len(c), t0 = 2 * lane;
            float* rv = reinterpret_cast<float*>(smem + L::RV + s * 256);
            rv[t0] = (r && t0 < Lc) ? __ldg(r + (row0 + t0) * H + h) : 1.f;
            rv[t0 + 1] = (r && t0 + 1 < Lc) ? __ldg(r + (row0 + t0 + 1) * H + h) : 1.f;
            mbar_arrive(&vready[s]);
        }
        if (fail && lane == 0 && last_issued >= 0) {  // let the loads in flight land
            for (int c = last_issued > NS - 1 ? last_issued - (NS - 1) : 0; c <= last_issued; ++c)
                mbar_wait_bounded(&full[c % NS], (uint32_t)(c / NS) & 1u, limit_ns);
        }
    } else if (warp == 8) {
        // =============================================== rank 0: the chain's per-chunk inputs
        // For chunk c, once its tiles have landed and the forwarder has sent chunk c - 2 (whose
        // d slot the chain overwrites in chunk c): the gate vectors, e_t = eta beta_t / ||k_t||^2
        // (computed by the prep kernel, carried in the T_d tile) and beta_t R_t, then the
        // chain's barrier.  Every wait of the chain's inputs happens
        // here, one chunk ahead, so the chain threads never wait on an mbarrier; a wait that runs
        // out sets the failure flag before the barrier, and the chain leaves at that chunk.
        volatile int* fail_flag = reinterpret_cast<volatile int*>(smem + L::FAIL);
        float nr0 = 1.f, nr1 = 1.f, nb0 = 0.f, nb1 = 0.f;
        auto fetch_gates = [&](int c) {
            const int64_t row0 = first + (int64_t)c * C;
            const int Lc = chunk_len(c), t0 = 2 * lane;
            const bool v0 = t0 < Lc, v1 = t0 + 1 < Lc;
            nr0 = (r && v0) ? __ldg(r + (row0 + t0) * H + h) : 1.f;
            nr1 = (r && v1) ? __ldg(r + (row0 + t0 + 1) * H + h) : 1.f;
            nb0 = v0 ? __ldg(beta + (row0 + t0) * H + h) : 0.f;
            nb1 = v1 ? __ldg(beta + (row0 + t0 + 1) * H + h) : 0.f;
        };
        if (nchunks > 0) fetch_gates(0);
        for (int c = 0; c < nchunks; ++c) {
            const int s = c % 3;
            bool got = mbar_wait_bounded(&full[s], (uint32_t)(c / 3) & 1u, limit_ns);
            if (got && c >= 2)
                got = mbar_wait_bounded(&fwdout[(c - 2) % 3], (uint32_t)((c - 2) / 3) & 1u, limit_ns);
            if (__any_sync(0xffffffffu, !got)) {
                if (lane == 0) *fail_flag = 1;
                __threadfence_block();
                group_bar(1, 288);  // the chain reads the flag and leaves
                break;
            }
            const int Lc = chunk_len(c), t0 = 2 * lane;
            const float r0 = nr0, r1 = nr1, b0 = nb0, b1 = nb1;
            if (c + 1 < nchunks) fetch_gates(c + 1);
            const GatePrefix g = gate_prefix(r0, r1, lane);
            float* vv = vecs(s);  // R | g | r | beta | R_C | e | beta R
            const float R0 = g.sg0 * __expf(g.lr0), R1 = g.sg_1 * __expf(g.lr_1);
            vv[t0] = R0;
            vv[t0 + 1] = R1;
            vv[64 + t0] = g.sgC * g.sg1_0 * __expf(g.lrC - g.lr1_0);
            vv[64 + t0 + 1] = g.sgC * g.sg1_1 * __expf(g.lrC - g.lr1_1);
            vv[128 + t0] = r0;
            vv[128 + t0 + 1] = r1;
            vv[192 + t0] = b0;
            vv[192 + t0 + 1] = b1;
            if (lane == 0) vv[256] = g.sgC * __expf(g.lrC);
            {  // e_t from the T_d tile's spare block (written there by the prep kernel)
                const float* td = reinterpret_cast<const float*>(smem + L::TD + s * 16384);
                vv[320 + t0] = t0 < Lc ? td[tsw(t0 >> 5, 32 + (t0 & 31))] : 0.f;
                vv[320 + t0 + 1] = t0 + 1 < Lc ? td[tsw((t0 + 1) >> 5, 32 + ((t0 + 1) & 31))] : 0.f;
                vv[384 + t0] = b0 * R0;
                vv[384 + t0 + 1] = b1 * R1;
            }
            __threadfence_block();
            group_bar(1, 288);  // chunk c's inputs are in place; the chain starts it
        }
    } else if (warp < 8 && rank == 0) {
        // =============================================== p = A d, x = T_d b, next d
        // Per chunk: the loader's barrier (its inputs are in place), then three steps separated
        // by the chain's own barrier; every operand that does not depend on the chain's values
        // (the key and T_d tiles, the gate vectors) is read before the first step.
        const volatile int* fail_flag = reinterpret_cast<const volatile int*>(smem + L::FAIL);
        const int u = tid;
        const int t = 8 * warp + (lane & 7), qd = lane >> 3;  // step 1/2 roles: token, channel quarter
        const int cp = u >> 2, par = u & 3;  // step 3 role: channel pair, token quarter
        const int cblk = cp >> 5, cj = (cp & 31) >> 2, cpe = 2 * (cp & 3);
        bool ok = true;
        for (int c = 0; c < nchunks; ++c) {
            group_bar(1, 288);
            if (*fail_flag) {
                ok = false;
                break;
            }
            const int s = c % 3;
            const int Lc = chunk_len(c);
            const uint8_t* kt = smem + L::KT + s * 16384;
            const float* td = reinterpret_cast<const float*>(smem + L::TD + s * 16384);
            const float* vv = vecs(s);
            const float* d = sD + (c % 3) * 128;
            uint4 k1[4];   // step 1: token t, channels 32 qd .. 32 qd + 31
            float4 tv[4];  // step 2: T_d[t][16 qd .. 16 qd + 15]
            uint32_t k3[C / 4];  // step 3: channels 2 cp, 2 cp + 1 of the tokens 8 m + 2 par + {0, 1}
#pragma unroll
            for (int j = 0; j < 4; ++j)
                k1[j] = *reinterpret_cast<const uint4*>(kt + (qd >> 1) * 8192u + tc::sw128_off(t, 4 * (qd & 1) + j));
#pragma unroll
            for (int q = 0; q < 4; ++q) tv[q] = tsw_ld4(td, t, 4 * qd + q);
            {
                const uint8_t* col = kt + cblk * 8192u + cpe * 2;
#pragma unroll
                for (int jj = 0; jj < C / 4; ++jj) {
                    const int j = 8 * (jj >> 1) + 2 * par + (jj & 1);
                    k3[jj] = *reinterpret_cast<const uint32_t*>(col + tc::sw128_off(j, cj));
                }
            }
            const float e_t = vv[320 + t], hR_t = vv[384 + t], g_t = vv[64 + t], rc = vv[256];
            // ---- step 1: p_t = <a_t, d>, b_t = e_t (1 - beta_t R_t p_t)
            float bRp = 0.f;  // kept for the residual ratio of step 2
            {
                float2 pa = make_float2(0.f, 0.f), pb = make_float2(0.f, 0.f);  // channel pairs
#pragma unroll
                for (int j = 0; j < 4; ++j) {  // channels 32 qd + 8 j .. + 7
                    const uint32_t w4[4] = {k1[j].x, k1[j].y, k1[j].z, k1[j].w};
                    const float4 da = *reinterpret_cast<const float4*>(d + 32 * qd + 8 * j);
                    const float4 db = *reinterpret_cast<const float4*>(d + 32 * qd + 8 * j + 4);
                    const float2 dv[4] = {make_float2(da.x, da.y), make_float2(da.z, da.w),
                                          make_float2(db.x, db.y), make_float2(db.z, db.w)};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 kk = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[e]));
                        if (e & 1) pb = __ffma2_rn(__fmul2_rn(kk, kk), dv[e], pb);
                        else pa = __ffma2_rn(__fmul2_rn(kk, kk), dv[e], pa);
                    }
                }
                float p = (pa.x + pb.x) + (pa.y + pb.y);
                p += __shfl_xor_sync(0xffffffffu, p, 8);
                p += __shfl_xor_sync(0xffffffffu, p, 16);
                if (qd == 0) {
                    bRp = hR_t * p;
                    sB[t] = e_t * (1.f - bRp);
                }
            }
            group_bar(5, 256);
            // ---- step 2: x_t = sum_{j <= t} T_d[t][j] b_j
            {
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int g = 4 * qd + q;
                    const float4 bv = *reinterpret_cast<const float4*>(sB + 4 * g);
                    const int j = 4 * g;
                    acc[q] = fmaf(j <= t ? tv[q].x : 0.f, bv.x, acc[q]);
                    acc[q] = fmaf(j + 1 <= t ? tv[q].y : 0.f, bv.y, acc[q]);
                    acc[q] = fmaf(j + 2 <= t ? tv[q].z : 0.f, bv.z, acc[q]);
                    acc[q] = fmaf(j + 3 <= t ? tv[q].w : 0.f, bv.w, acc[q]);
                }
                float xs = (acc[0] + acc[1]) + (acc[2] + acc[3]);
                xs += __shfl_xor_sync(0xffffffffu, xs, 8);
                xs += __shfl_xor_sync(0xffffffffu, xs, 16);
                if (qd == 0) {
                    const float x = t < Lc ? xs : 0.f;
                    sX[(c % 3) * 64 + t] = x;
                    sGX[t] = g_t * x;
                    // residual-contraction ratio (1 - beta s)^2: x = e (1 - beta s) when e != 0;
                    // else d_t = R_t d_0 on this token's row, so beta s = beta R p
                    if (rho && t < Lc && OSDN_IN_BOUNDS(first + (int64_t)c * C + t, rows_all)) {
                        const float gr = e_t != 0.f ? x / e_t : 1.f - bRp;
                        rho[(first + (int64_t)c * C + t) * H + h] = gr * gr;
                    }
                }
            }
            group_bar(5, 256);
            // ---- step 3: d_C[i] = R_C d[i] + sum_j g_j x_j a_j[i]; thread: channels 2cp, 2cp + 1
            //      over the tokens j = 8 m + 2 par + {0, 1} -- the four parts read rows of distinct
            //      swizzle phases, so the lanes read disjoint banks -- summed by shuffles
            {
                float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};  // the channel pair
#pragma unroll
                for (int jj = 0; jj < C / 4; ++jj) {
                    const int j = 8 * (jj >> 1) + 2 * par + (jj & 1);
                    const float2 kv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&k3[jj]));
                    const float gx = sGX[j];
                    acc[jj & 1] = __ffma2_rn(make_float2(gx, gx), __fmul2_rn(kv, kv), acc[jj & 1]);
                }
                float acc0 = acc[0].x + acc[1].x, acc1 = acc[0].y + acc[1].y;
                acc0 += __shfl_xor_sync(0xffffffffu, acc0, 1);
                acc1 += __shfl_xor_sync(0xffffffffu, acc1, 1);
                acc0 += __shfl_xor_sync(0xffffffffu, acc0, 2);
                acc1 += __shfl_xor_sync(0xffffffffu, acc1, 2);
                if (par == 0) {
                    const float2 dv = *reinterpret_cast<const float2*>(d + 2 * cp);
                    const float2 dn = make_float2(fmaf(rc, dv.x, acc0), fmaf(rc, dv.y, acc1));
                    *reinterpret_cast<float2*>(sD + ((c + 1) % 3) * 128 + 2 * cp) = dn;
                }
            }
            // x_c and d_c are in sX, sD and this thread is done with the slot: the forwarder sends
            // them and refills the slot
            mbar_arrive(&fwdin[c % 3]);
        }
        group_bar(5, 256);  // the last chunk's d is complete
        if (ok && dT && u < DK && OSDN_IN_BOUNDS(dbase + u, (int64_t)N * H * DK))
            dT[dbase + u] = sD[(nchunks % 3) * 128 + u];
    } else if (warp == 9 && rank == 0) {
        // =============================================== forwarder: x_c, d_c to rank 1; refills
        // Once the chain is done with chunk c (fwdin): the refill of its ring slot with chunk
        // c + 3; then chunk c's x and chunk-start d go into receive slot c % NG of rank 1 once
        // rank 1's writer of chunk c - NG has copied that slot out; the chain may then overwrite
        // its local copies (fwdout).
        int last_issued = -1;
        auto issue = [&](int c) {
            const int s = c % 3;
            const int64_t row0 = first + (int64_t)c * C;
            if (lane == 0) {
                uint8_t* kt = smem + L::KT + s * 16384;
                tc::mbar_expect_tx(&full[s], 32768);
                tc::tma_load_3d(kt, &tm_k, 0, h, (int)row0, &full[s]);
                tc::tma_load_3d(kt + 8192, &tm_k, 64, h, (int)row0, &full[s]);
                tc::tma_load_3d(smem + L::TD + s * 16384, &tm_td, 0, h, (int)row0, &full[s]);
            }
            last_issued = c;
        };
        if (lane == 0) {
            tc::prefetch_tmap(&tm_k);
            tc::prefetch_tmap(&tm_td);
        }
        for (int c = 0; c < 3 && c < nchunks; ++c) issue(c);
        for (int c = 0; c < nchunks; ++c) {
            const int k = c % 3;
            bool got = mbar_wait_bounded(&fwdin[k], (uint32_t)(c / 3) & 1u, limit_ns);
            if (__any_sync(0xffffffffu, !got)) break;
            if (c + 3 < nchunks) issue(c + 3);
            const int m = c % L::NG;  // rank 1's receive slot
            if (c >= L::NG)
                got = tc::mbar_wait_cluster(&outdone[m], (uint32_t)(c / L::NG - 1) & 1u, limit_ns);
            if (__any_sync(0xffffffffu, !got)) break;
            {
                const float2 xv = *reinterpret_cast<const float2*>(sX + k * 64 + 2 * lane);
                tc::st_cluster_v2f32(peer_x + 4u * (uint32_t)(m * 64 + 2 * lane), xv.x, xv.y);
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int e = 2 * lane + 64 * q;
                    const float2 dv = *reinterpret_cast<const float2*>(sD + k * 128 + e);
                    tc::st_cluster_v2f32(peer_d + 4u * (uint32_t)(m * 128 + e), dv.x, dv.y);
                }
            }
            mbar_arrive(&fwdout[k]);                                // local copies are free
            tc::mbar_arrive_cluster(peer_xready + 8u * (uint32_t)m);  // rank 1 may read them
        }
        // let the copies in flight land (the last one issued into each slot): on the normal
        // path the loader has waited for all of them already
        if (lane == 0 && last_issued >= 0) {
            for (int c = last_issued > 2 ? last_issued - 2 : 0; c <= last_issued; ++c)
                mbar_wait_bounded(&full[c % 3], (uint32_t)(c / 3) & 1u, limit_ns);
        }
    } else if (warp < 8 && rank == 1) {
        // =============================================== k~ = d (.) k, token by token
        // Four groups of 64 threads take every fourth chunk (group g: chunks c = g, g + 4, ...),
        // so each has four chunk periods for its token pass and stores; a thread carries the
        // key-channel pair (2 jj, 2 jj + 1): packed bf16x2 conversions and 4-byte stores.
        constexpr int NS = L::NS1, NG = L::NG;
        const int i = tid, g = i >> 6, jj = i & 63;
        const int blk = jj >> 5, cj = (jj & 31) >> 2, ce = 2 * (jj & 3);  // channel 2 jj in the tile
        const int gbar = 2 + g;  // the group's named barrier
        uint8_t* lo_stage = smem + L::LO + g * 16384;
        for (int c = g; c < nchunks; c += NG) {
            const int s = c % NS;
            const uint32_t ph = (uint32_t)(c / NS) & 1u;
            // the slot's previous chunk (another group's) released first: then its full and vready
            // barriers are at most one phase behind this chunk, and the parity waits are exact
            const bool got = (c < NS || mbar_wait_bounded(&kempty[s], (uint32_t)(c / NS - 1) & 1u, limit_ns)) &&
                             mbar_wait_bounded(&full[s], ph, limit_ns) &&
                             mbar_wait_bounded(&vready[s], ph, limit_ns) &&
                             tc::mbar_wait_cluster(&xready[c % NG], (uint32_t)(c / NG) & 1u, limit_ns);
            if (group_any(gbar, 64, !got)) break;
            const int Lc = chunk_len(c);
            const uint8_t* col = smem + L::KT1 + s * 16384 + blk * 8192u + ce * 2;
            // copy x and this pair's d out of the slot rank 0's forwarder fills, and free it
            float* xv = reinterpret_cast<float*>(smem + L::XW + g * 256);
            const int m = c % NG;  // the receive slot rank 0's forwarder filled
            xv[jj] = reinterpret_cast<const float*>(smem + L::XR)[m * 64 + jj];
            float2 dd = reinterpret_cast<const float2*>(smem + L::DR)[m * 64 + jj];
            group_bar(gbar, 64);
            tc::mbar_arrive_cluster(peer_outdone + 8u * (uint32_t)m);
            const float* rv = reinterpret_cast<const float*>(smem + L::RV + s * 256);
            // k~ goes to the group's staging tiles in the key tile's swizzled layout, then to
            // global memory as whole tiles or 16-byte row pieces: scattered 2-byte stores would
            // cost about three times the whole token pass
            uint8_t* stage = smem + L::HI + g * 16384;
            uint8_t* ocol = stage + blk * 8192u + ce * 2;
            uint8_t* lcol = lo_stage + blk * 8192u + ce * 2;
            float* drow = kD ? d_all + ((first + (int64_t)c * C) * H + h) * DK + 2 * jj : nullptr;
#pragma unroll 1
            for (int t0 = 0; t0 < Lc; t0 += 16) {
                float2 kv[16];
                float xt[16], rt[16];
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    const uint32_t w = *reinterpret_cast<const uint32_t*>(col + tc::sw128_off(t0 + u, cj));
                    kv[u] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w));
                    xt[u] = xv[t0 + u];
                    rt[u] = rv[t0 + u];
                }
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                    if (kD && t0 + u < Lc && OSDN_IN_BOUNDS(first + (int64_t)c * C + t0 + u, rows_all))
                        *reinterpret_cast<float2*>(drow + (int64_t)(t0 + u) * H * DK) = dd;
                    const float2 kt = __fmul2_rn(dd, kv[u]);
                    const __nv_bfloat162 hb = __floats2bfloat162_rn(kt.x, kt.y);
                    *reinterpret_cast<__nv_bfloat162*>(ocol + tc::sw128_off(t0 + u, cj)) = hb;
                    if (kLo) {
                        const float2 hf = __bfloat1622float2(hb);
                        *reinterpret_cast<__nv_bfloat162*>(lcol + tc::sw128_off(t0 + u, cj)) =
                            __floats2bfloat162_rn(kt.x - hf.x, kt.y - hf.y);
                    }
                    const float2 a = __fmul2_rn(kv[u], kv[u]);
                    dd = __ffma2_rn(make_float2(rt[u], rt[u]), dd, __fmul2_rn(make_float2(xt[u], xt[u]), a));
                }
            }
            // a whole chunk leaves by TMA stores (64 rows x 64 channels per box); a short one, whose
            // box would reach the next sequence's rows, by 16-byte row pieces
            const bool bulk = Lc == C;
            if (bulk) tc::fence_async_smem();
            group_bar(gbar, 64);
            if (bulk) {
                if (jj == 0 && OSDN_IN_BOUNDS(first + (int64_t)c * C + C - 1, rows_all)) {
                    const int row0 = (int)(first + (int64_t)c * C);
                    tc::tma_store_3d(&tm_kto, stage, 0, h, row0);
                    tc::tma_store_3d(&tm_kto, stage + 8192, 64, h, row0);
                    if (kLo) {
                        tc::tma_store_3d(&tm_ktlo, lo_stage, 0, h, row0);
                        tc::tma_store_3d(&tm_ktlo, lo_stage + 8192, 64, h, row0);
                    }
                    tc::bulk_commit();
                    tc::bulk_wait_read_all();  // the staging tiles may be reused
                }
            } else {  // 64 rows x 16 pieces of 16 bytes per tile: piece jj & 15, rows (jj >> 4) + 4 q
                const int piece = jj & 15, blk16 = piece >> 3, j16 = piece & 7;
                const int64_t off = ((first + (int64_t)c * C) * H + h) * DK + 8 * piece;
                const int64_t rs = (int64_t)H * DK;
#pragma unroll 4
                for (int q = 0; q < 16; ++q) {
                    const int row = (jj >> 4) + 4 * q;
                    if (row < Lc && OSDN_IN_BOUNDS(first + (int64_t)c * C + row, rows_all)) {
                        const uint32_t so = blk16 * 8192u + tc::sw128_off(row, j16);
                        *reinterpret_cast<uint4*>(k_tilde + off + row * rs) =
                            *reinterpret_cast<const uint4*>(stage + so);
                        if (kLo)
                            *reinterpret_cast<uint4*>(k_tilde_lo + off + row * rs) =
                                *reinterpret_cast<const uint4*>(lo_stage + so);
                    }
                }
            }
            group_bar(gbar, 64);  // the group's staging tiles and x copy are read out
            mbar_arrive(&kempty[s]);
        }
        if (jj == 0) tc::bulk_wait_all();  // this thread's stores are complete
    }
    tc::fence_before_sync();
    tc::cluster_sync();  // neither CTA leaves while the other may still write to it
}

}  // namespace osdn
