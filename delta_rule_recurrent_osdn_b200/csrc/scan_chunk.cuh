// scan_chunk.cuh -- phase 1 of the OSDN forward pass in chunk-parallel form (bf16 I/O, d_k = 128).
//
// The preconditioner recurrence ("OSDN: Improving Delta Rule with Provable Online
// Preconditioning in Linear Attention", technical summary, sections 2.2 and 2.3; section 2.3
// notes that the APF update keeps the recurrence affine) is, with a_t = k_t (.) k_t,
// e_t = eta beta_t / ||k_t||^2 (0 when k_t = 0) and x_t = e_t (1 - beta_t <d_t, a_t>):
//   d_{t+1} = r_t d_t + x_t a_t,     k~_t = d_t (.) k_t.
// Within a chunk of C = 64 tokens starting from d_0, with R_t = prod_{i<t} r_i and
// Gamma_tj = prod_{j<i<t} r_i:
//   <d_t, a_t> = R_t <d_0, a_t> + sum_{j<t} Gamma_tj <a_j, a_t> x_j, hence
//   (I + L_d) x = b,  b = e (.) (1 - beta (.) R (.) A d_0),  L_d[t][j] = e_t beta_t Gamma_tj <a_t, a_j>.
// L_d is strictly lower triangular (nilpotent), so the fixed-point iteration x <- b - L_d x is
// exact after at most C - 1 steps; it stops earlier once an iteration changes no entry by more
// than 2^-22 of the largest, which on unit-norm keys takes about three steps (the entries of
// L_d are of order eta beta^2 <a_t, a_j> / ||k_t||^2).  Then one pass over the chunk's tokens
// per key channel (d <- r d + x a) emits k~ and leaves d for the next chunk.
//
// Per chunk, the parts that do not depend on d_0 -- the Gram A A^T (two M = 128 bf16 MMAs on the
// stacked [a_hi; a_lo] split of a, giving hi hi^T + lo hi^T + hi lo^T), Gamma (from prefix sums
// of log |r| and a sign parity) and L_d -- are prepared for chunk c+1 while chunk c's serial
// chain runs: the Gram MMA is issued before the chain and read after it.
//
// One CTA of 256 threads per (sequence, head); keys arrive by TMA in a 3-stage ring.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace osdn {

struct ScanSmem {
    static constexpr int S = 65;                           // fp32 matrix row stride
    static constexpr uint32_t KSTAGE = 16384;              // bf16 k tile: 2 blocks of 64 x 128 B
    static constexpr uint32_t K0 = 0;                      // 3 stages
    static constexpr uint32_t A = 3 * KSTAGE;              // bf16 [a_hi; a_lo], 2 K-blocks x 16 KB
    static constexpr uint32_t MATB = 64 * S * 4;
    static constexpr uint32_t G1 = A + 32768, G2 = G1 + MATB, G3 = G2 + MATB;  // Gram parts
    static constexpr uint32_t LD = G3 + MATB;              // L_d
    // per-chunk vectors (3 buffers, 64 floats each field)
    static constexpr int NVEC = 9;                         // beta r e c R lr lr1 sg sg1
    static constexpr uint32_t VEC = LD + MATB;
    static constexpr uint32_t VECB = NVEC * 256;
    static constexpr uint32_t XS = VEC + 3 * VECB;         // x ping-pong 2 x 64
    static constexpr uint32_t VB = XS + 512;               // b (64)
    static constexpr uint32_t VD = VB + 256;               // d (128)
    static constexpr uint32_t RED = VD + 512;              // 2 x 2 x 2 floats of reductions
    static constexpr uint32_t BAR = RED + 64;              // 4 mbarriers
    static constexpr uint32_t TMEM_SLOT = BAR + 32;
    static constexpr uint32_t TOTAL = TMEM_SLOT + 16;
    static constexpr size_t BYTES = TOTAL + 1024;
};
static_assert(ScanSmem::BYTES <= 232448, "shared memory");

struct ScanVec {
    float *beta, *r, *e, *c, *R, *lr, *lr1, *sg, *sg1;
    __device__ ScanVec(uint8_t* base) {
        float* f = reinterpret_cast<float*>(base);
        beta = f; r = f + 64; e = f + 128; c = f + 192; R = f + 256; lr = f + 320;
        lr1 = f + 384; sg = f + 448; sg1 = f + 512;
    }
};

__device__ __forceinline__ void named_bar_64(int id) {
    asm volatile("bar.sync %0, 64;" ::"r"(id) : "memory");
}

__global__ void __launch_bounds__(256, 1)
precond_scan_chunk_kernel(const __grid_constant__ CUtensorMap tm_k, const float* __restrict__ beta,
                          const float* __restrict__ r, float eta, const float* __restrict__ d0,
                          __nv_bfloat16* __restrict__ k_tilde, float* __restrict__ dT,
                          const int32_t* __restrict__ cu, int N, int T, int H, long long limit_ns) {
    constexpr int C = 64, DK = 128;
    using L = ScanSmem;
    constexpr int S = L::S;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lanei = tid & 31;
    const int n = blockIdx.x / H, h = blockIdx.x - n * H;
    if (n >= N) return;
    int64_t first, count;
    if (!seq_range(cu, n, N, T, first, count)) return;  // uniform over the CTA

    uint64_t* tma_bar = reinterpret_cast<uint64_t*>(smem + L::BAR);  // 3
    uint64_t* mma_bar = tma_bar + 3;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::TMEM_SLOT);
    uint8_t* sAt = smem + L::A;
    float* sG1 = reinterpret_cast<float*>(smem + L::G1);
    float* sG2 = reinterpret_cast<float*>(smem + L::G2);
    float* sG3 = reinterpret_cast<float*>(smem + L::G3);
    float* sL = reinterpret_cast<float*>(smem + L::LD);
    float* xs = reinterpret_cast<float*>(smem + L::XS);
    float* vb = reinterpret_cast<float*>(smem + L::VB);
    float* vd = reinterpret_cast<float*>(smem + L::VD);
    float* red = reinterpret_cast<float*>(smem + L::RED);
    auto vec = [&](int chunk) { return ScanVec(smem + L::VEC + (chunk % 3) * L::VECB); };
    auto ktile = [&](int chunk) -> const uint8_t* { return smem + L::K0 + (chunk % 3) * L::KSTAGE; };

    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, 128);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        for (int s = 0; s < 3; ++s) mbar_init(&tma_bar[s], 1);
        mbar_init(mma_bar, 1);
        tc::fence_mbar_init();
        tc::prefetch_tmap(&tm_k);
    }
    const int64_t dbase = ((int64_t)n * H + h) * DK;
    if (tid < DK) vd[tid] = d0 ? __ldg(d0 + dbase + tid) : 1.0f;

    const int nchunks = (int)((count + C - 1) / C);
    auto chunk_len = [&](int chunk) -> int {
        const int64_t rem = count - (int64_t)chunk * C;
        return rem < C ? (int)rem : C;
    };
    // beta and r of a chunk into its vector buffer (threads t < 64); tail tokens: beta 0, r 1
    auto load_gates = [&](int chunk, int t) {
        ScanVec v = vec(chunk);
        const bool valid = t < chunk_len(chunk);
        const int64_t g = (first + (int64_t)chunk * C + t) * H + h;
        v.beta[t] = valid ? __ldg(beta + g) : 0.f;
        v.r[t] = (valid && r) ? __ldg(r + g) : 1.f;
    };
    if (tid < C) {
        if (nchunks > 0) load_gates(0, tid);
        if (nchunks > 1) load_gates(1, tid);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tlane = static_cast<uint32_t>((warp & 3) * 32) << 16;

    int tma_pend[3] = {-1, -1, -1};
    bool mma_pend = false, fail = false;
    uint32_t mma_phase = 0;
    auto issue_load = [&](int chunk) {
        const int s = chunk % 3;
        uint8_t* dst = smem + L::K0 + s * L::KSTAGE;
        const int row = (int)(first + (int64_t)chunk * C);
        tc::mbar_expect_tx(&tma_bar[s], L::KSTAGE);
        tc::tma_load_3d(dst, &tm_k, 0, h, row, &tma_bar[s]);
        tc::tma_load_3d(dst + 8192, &tm_k, 64, h, row, &tma_bar[s]);
        tma_pend[s] = (chunk / 3) & 1;
    };
    if (tid == 0) {
        if (nchunks > 0) issue_load(0);
        if (nchunks > 1) issue_load(1);
    }
    auto sync_failed = [&]() -> bool {
        tc::fence_before_sync();
        const bool any = __syncthreads_or(fail) != 0;
        fail = any;
        return any;
    };
    constexpr uint32_t ID_G = tc::idesc(1, 0, 0, 128, 64);

    // ---- front half of a chunk's preparation: a tiles, e, e*beta, log-prefix of r; Gram MMA
    auto prep_front = [&](int chunk) {
        const int s = chunk % 3;
        if (mbar_wait_bounded(&tma_bar[s], (uint32_t)(chunk / 3) & 1u, limit_ns))
            tma_pend[s] = -1;
        else
            fail = true;
        if (sync_failed()) return;
        const uint8_t* kt = ktile(chunk);
        ScanVec v = vec(chunk);
        const int Lc = chunk_len(chunk);
        {
            const int t = tid >> 2, q = tid & 3, blk = q >> 1;
            const bool valid = t < Lc;
            float nk = 0.f;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int j = (q & 1) * 4 + jj;
                const uint32_t off = tc::sw128_off(t, j);
                const uint4 raw = *reinterpret_cast<const uint4*>(kt + blk * 8192u + off);
                const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 kk = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[e]));
                    const float a0 = valid ? kk.x * kk.x : 0.f, a1 = valid ? kk.y * kk.y : 0.f;
                    nk += a0 + a1;
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(a0, a1);
                    const float2 hf = __bfloat1622float2(h2);
                    const __nv_bfloat162 l2 = __floats2bfloat162_rn(a0 - hf.x, a1 - hf.y);
                    hi[e] = *reinterpret_cast<const uint32_t*>(&h2);
                    lo[e] = *reinterpret_cast<const uint32_t*>(&l2);
                }
                // rows t (hi) and 64 + t (lo) of K-block blk; same swizzle phase (t & 7)
                *reinterpret_cast<uint4*>(sAt + blk * 16384u + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4*>(sAt + blk * 16384u + 8192u + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
            nk += __shfl_xor_sync(0xffffffffu, nk, 1);
            nk += __shfl_xor_sync(0xffffffffu, nk, 2);
            if (q == 0) {
                const float e = nk > 0.f ? eta * v.beta[t] / nk : 0.f;
                v.e[t] = e;
                v.c[t] = e * v.beta[t];
            }
        }
        if (warp == 7) {
            // prefix sums over the chunk of log|r| and of the count of negative r (sign parity)
            const int t0 = 2 * lanei;
            const float r0 = v.r[t0], r1 = v.r[t0 + 1];
            const float l0 = __logf(fmaxf(fabsf(r0), 1e-30f)), l1 = __logf(fmaxf(fabsf(r1), 1e-30f));
            const int n0 = r0 < 0.f, n1 = r1 < 0.f;
            float ps = l0 + l1;
            int pn = n0 + n1;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float ys = __shfl_up_sync(0xffffffffu, ps, off);
                const int yn = __shfl_up_sync(0xffffffffu, pn, off);
                if (lanei >= off) {
                    ps += ys;
                    pn += yn;
                }
            }
            const float ex = ps - (l0 + l1);  // sum over tokens before t0
            const int en = pn - (n0 + n1);
            v.lr[t0] = ex;
            v.lr[t0 + 1] = ex + l0;
            v.lr1[t0] = ex + l0;
            v.lr1[t0 + 1] = ex + l0 + l1;
            v.sg[t0] = (en & 1) ? -1.f : 1.f;
            v.sg[t0 + 1] = ((en + n0) & 1) ? -1.f : 1.f;
            v.sg1[t0] = v.sg[t0 + 1];
            v.sg1[t0 + 1] = ((en + n0 + n1) & 1) ? -1.f : 1.f;
            v.R[t0] = v.sg[t0] * __expf(ex);
            v.R[t0 + 1] = v.sg[t0 + 1] * __expf(ex + l0);
        }
        tc::fence_async_smem();
        if (sync_failed()) return;
        if (tid == 0) {
            tc::fence_after_sync();
            const uint32_t aA = smem_u32(sAt);
#pragma unroll
            for (int st = 0; st < 8; ++st) {
                const uint32_t blk = (st >> 2) * 16384u + (st & 3) * 32u;
                tc::mma_bf16(tmem + 0, tc::sw128_desc(aA + blk, 16, 1024), tc::sw128_desc(aA + blk, 16, 1024),
                             ID_G, st > 0);
                tc::mma_bf16(tmem + 64, tc::sw128_desc(aA + blk, 16, 1024),
                             tc::sw128_desc(aA + blk + 8192, 16, 1024), ID_G, st > 0);
            }
            tc::mma_commit(mma_bar);
            mma_pend = true;
        }
    };

    // ---- back half: L_d = diag(e beta) (Gamma (.) G), G = hi hi^T + lo hi^T + hi lo^T
    auto prep_back = [&](int chunk) {
        if (mbar_wait_bounded(mma_bar, mma_phase, limit_ns)) {
            mma_phase ^= 1u;
            mma_pend = false;
        } else {
            fail = true;
        }
        tc::fence_after_sync();
        if (warp < 6) {
            float g[64];
            tc::tmem_ld64(tmem + tlane + (warp < 4 ? 0u : 64u), g);
            float* dst = warp < 2 ? sG1 : (warp < 4 ? sG2 : sG3);
            const int t = warp < 4 ? (tid & 63) : tid - 128;
#pragma unroll
            for (int j = 0; j < 64; ++j) dst[t * S + j] = g[j];
        }
        if (sync_failed()) return;
        ScanVec v = vec(chunk);
        const int t = tid >> 2, q = tid & 3;
        const float ct = v.c[t], lrt = v.lr[t], sgt = v.sg[t];
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
            const int j = 16 * q + jj;
            float val = 0.f;
            if (j < t) {
                const float gam = sgt * v.sg1[j] * __expf(lrt - v.lr1[j]);
                val = ct * gam * (sG1[t * S + j] + sG2[t * S + j] + sG3[t * S + j]);
            }
            sL[t * S + j] = val;
        }
        __syncthreads();
    };

    if (nchunks > 0) {
        prep_front(0);
        if (!fail) prep_back(0);
    }

#pragma unroll 1
    for (int ch = 0; ch < nchunks && !fail; ++ch) {
        const int Lc = chunk_len(ch);
        const bool more = ch + 1 < nchunks;
        if (more) {
            if (tid == 0 && ch + 2 < nchunks) issue_load(ch + 2);
            prep_front(ch + 1);  // issues the Gram MMA of the next chunk
            if (fail) break;
        }
        const uint8_t* kt = ktile(ch);
        ScanVec v = vec(ch);
        // ---- p = A d0 and b = e (1 - beta R p)
        {
            const int t = tid >> 2, q = tid & 3, blk = q >> 1;
            float acc = 0.f;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int j = (q & 1) * 4 + jj;
                const uint4 raw = *reinterpret_cast<const uint4*>(kt + blk * 8192u + tc::sw128_off(t, j));
                const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
                const int i0 = blk * 64 + j * 8;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 kk = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[e]));
                    acc = fmaf(kk.x * kk.x, vd[i0 + 2 * e], acc);
                    acc = fmaf(kk.y * kk.y, vd[i0 + 2 * e + 1], acc);
                }
            }
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            if (q == 0) vb[t] = (t < Lc) ? v.e[t] * (1.f - v.beta[t] * v.R[t] * acc) : 0.f;
        }
        __syncthreads();
        // ---- x = (I + L_d)^-1 b by x <- b - L_d x (warps 0-1, one row per thread)
        if (tid < 64) {
            const int t = tid;
            const float bt = vb[t];
            xs[t] = bt;
            named_bar_64(1);
            int cur = 0;
            for (int m = 1;; ++m) {
                const float* xc = xs + cur * 64;
                float acc0 = bt, acc1 = 0.f;
#pragma unroll
                for (int j = 0; j < 64; j += 2) {
                    if (j < t) acc0 = fmaf(-sL[t * S + j], xc[j], acc0);
                    if (j + 1 < t) acc1 = fmaf(-sL[t * S + j + 1], xc[j + 1], acc1);
                }
                const float xn = acc0 + acc1;
                float dm = fabsf(xn - xc[t]), xm = fabsf(xn);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    dm = fmaxf(dm, __shfl_xor_sync(0xffffffffu, dm, off));
                    xm = fmaxf(xm, __shfl_xor_sync(0xffffffffu, xm, off));
                }
                float* rb = red + (m & 1) * 4;
                if (lanei == 0) {
                    rb[2 * warp] = dm;
                    rb[2 * warp + 1] = xm;
                }
                xs[(cur ^ 1) * 64 + t] = xn;
                named_bar_64(1);
                cur ^= 1;
                const float dmax = fmaxf(rb[0], rb[2]), xmax = fmaxf(rb[1], rb[3]);
                if (dmax <= 2.384185791015625e-7f * xmax || m >= Lc - 1) break;  // 2^-22
            }
            xs[128 + t] = xs[cur * 64 + t];  // the result, past the ping-pong pair (vb area)
        }
        __syncthreads();
        // ---- one pass over the tokens per key channel: k~ = d k, d <- r d + x k^2;
        //      meanwhile threads 128.. fetch the gates of chunk ch + 2
        if (tid < DK) {
            const int i = tid, blk = i >> 6, j = (i & 63) >> 3, e = i & 7;
            const float* xv = xs + 128;
            float dd = vd[i];
            __nv_bfloat16* out = k_tilde + ((first + (int64_t)ch * C) * H + h) * DK + i;
            const int64_t rs = (int64_t)H * DK;
            for (int t0 = 0; t0 < Lc; t0 += 8) {
                float kk[8], xt[8], rt[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    kk[u] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
                        kt + blk * 8192u + tc::sw128_off(t0 + u, j) + e * 2));
                    xt[u] = xv[t0 + u];
                    rt[u] = v.r[t0 + u];
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    if (t0 + u < Lc) {
                        out[(t0 + u) * rs] = __float2bfloat16_rn(dd * kk[u]);
                        dd = fmaf(rt[u], dd, xt[u] * kk[u] * kk[u]);
                    }
                }
            }
            vd[i] = dd;
        } else if (tid >= 192 && ch + 2 < nchunks) {
            load_gates(ch + 2, tid - 192);
        }
        if (more && !fail) {
            if (sync_failed()) break;
            prep_back(ch + 1);
        } else {
            if (sync_failed()) break;
        }
    }

    if (fail) {
        if (tid == 0) {
            for (int s = 0; s < 3; ++s)
                if (tma_pend[s] >= 0) mbar_wait_bounded(&tma_bar[s], (uint32_t)tma_pend[s], limit_ns);
            if (mma_pend) mbar_wait_bounded(mma_bar, mma_phase, limit_ns);
        }
    } else if (dT && tid < DK) {
        dT[dbase + tid] = vd[tid];
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 128);
}

}  // namespace osdn
