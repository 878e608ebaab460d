// tril_inverse.cuh -- T = (I + L)^-1 for a strictly lower-triangular 64x64 fp32 matrix L, computed
// in shared memory by a group of 128 threads.
//
// The chunked DeltaNet forward pass needs this WY factor once per 64-token chunk, with
// L = strict_tril(diag(beta) K K~^T) (the UT-transform solve of the chunkwise DeltaNet
// algorithm).  Blocked algorithm, all in fp32:
//   A. the four diagonal 16x16 blocks by forward substitution (one column per thread);
//   B. 16x16 level, (I, J) = (1, 0) and (3, 2):  X = L_IJ T_JJ,  T_IJ = -T_II X;
//   C. 32x32 level on the 2x2 grid of 32x32 blocks:  X = L_10 T_00,  T_10 = -T_11 X.
// Each thread keeps one column of the right-hand factor in registers and produces 4 (level B)
// or 8 (level C) outputs of that column, reading the left factor's rows as broadcast 16-byte
// loads, so a product step is a few dozen shared loads per thread rather than two per FMA.
//
// Matrix layout ("tsw"): row stride 64 floats, the 16-byte group g of row r stored at group
// position g ^ (r & 15).  A thread that writes its own row as 16 float4 stores, a warp that
// reads one row (broadcast) and a warp that reads 32 consecutive columns of one row are all
// free of bank conflicts.
#pragma once

namespace osdn {

// Word offset of element (r, c) of a 64x64 fp32 matrix in the swizzled layout.
__device__ __forceinline__ int tsw(int r, int c) {
    return r * 64 + ((((c >> 2) ^ r) & 15) << 2) + (c & 3);
}

__device__ __forceinline__ float4 tsw_ld4(const float* m, int r, int g) {
    return *reinterpret_cast<const float4*>(m + r * 64 + (((g ^ r) & 15) << 2));
}

__device__ __forceinline__ void tsw_st4(float* m, int r, int g, float4 v) {
    *reinterpret_cast<float4*>(m + r * 64 + (((g ^ r) & 15) << 2)) = v;
}

__device__ __forceinline__ void group_bar(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Named-barrier synchronization of a thread group that also returns whether any member passed
// `pred` = true (used to leave a loop together when a bounded wait ran out).
__device__ __forceinline__ bool group_any(int id, int nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, %2, %3, q;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

// Load row r, columns [c0, c0 + 4*NG) of a swizzled matrix into x (c0 a multiple of 4).
template <int NG>
__device__ __forceinline__ void tsw_row(const float* m, int r, int c0, float* x) {
#pragma unroll
    for (int g = 0; g < NG; ++g) {
        const float4 v = tsw_ld4(m, r, (c0 >> 2) + g);
        x[4 * g] = v.x;
        x[4 * g + 1] = v.y;
        x[4 * g + 2] = v.z;
        x[4 * g + 3] = v.w;
    }
}

// Packed dot product: acc += m[r][c0 .. c0 + 4 NG) . col2[0 .. 2 NG), with col2[i] holding the
// column entries c0 + 2i and c0 + 2i + 1, as two-wide fp32 FMAs (two partial sums).
template <int NG>
__device__ __forceinline__ float2 tsw_dot2(const float* m, int r, int c0, const float2* col2,
                                           float2 acc) {
#pragma unroll
    for (int g = 0; g < NG; ++g) {
        const float4 v = tsw_ld4(m, r, (c0 >> 2) + g);
        acc = __ffma2_rn(make_float2(v.x, v.y), col2[2 * g], acc);
        acc = __ffma2_rn(make_float2(v.z, v.w), col2[2 * g + 1], acc);
    }
    return acc;
}

// In place.  On entry M holds L in the swizzled layout (only its strictly lower triangle is
// read); on return it holds T on and below the diagonal, and the entries above the diagonal hold
// scratch values, so a reader masks them (T is lower triangular with a unit diagonal).  Every
// block of L is read before the block of T that replaces it is written: the diagonal blocks
// through registers and a barrier, the off-diagonal blocks one level later.
// Called by all 128 threads t = 0..127 of a group synchronizing on named barrier `bar_id`;
// returns synchronized.
__device__ __forceinline__ void tril_inverse_64_g128(float* __restrict__ M, int t, int bar_id) {
    constexpr int NT = 128;
    const float* sL = M;
    float* sT = M;
    // ---- A. diagonal blocks: column `col` of block b, x[r] = [r == col] - sum_{m<r} L_rm x[m]
    {
        const int o = 16 * ((t & 63) >> 4), col = t & 15;
        float2 xp[8];  // x[2i], x[2i + 1]; zero until computed (their L factor is zeroed too,
                       // but 0 * an uninitialized NaN would still be NaN)
#pragma unroll
        for (int i = 0; i < 8; ++i) xp[i] = make_float2(0.f, 0.f);
        if (t < 64) {
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float2 acc2 = make_float2(0.f, 0.f);
#pragma unroll
                for (int g = 0; 4 * g < r; ++g) {
                    const float4 v = tsw_ld4(sL, o + r, (o >> 2) + g);
                    // x[m] == 0 for m < col, so no per-lane bound is needed; terms m >= r are
                    // excluded by zeroing their L factor
                    const int m = 4 * g;
                    const float2 l0 = make_float2(m < r ? v.x : 0.f, m + 1 < r ? v.y : 0.f);
                    const float2 l1 = make_float2(m + 2 < r ? v.z : 0.f, m + 3 < r ? v.w : 0.f);
                    acc2 = __ffma2_rn(l0, xp[2 * g], acc2);
                    acc2 = __ffma2_rn(l1, xp[2 * g + 1], acc2);
                }
                const float xr = r == col ? 1.f : (r < col ? 0.f : -(acc2.x + acc2.y));
                if (r & 1) xp[r >> 1].y = xr; else xp[r >> 1] = make_float2(xr, 0.f);
            }
        }
        group_bar(bar_id, NT);  // the diagonal blocks of L are read
        if (t < 64) {
#pragma unroll
            for (int r = 0; r < 16; ++r) sT[tsw(o + r, o + col)] = (r & 1) ? xp[r >> 1].y : xp[r >> 1].x;
        }
    }
    group_bar(bar_id, NT);
    // ---- B. 16x16 level; thread: block pair (t >> 6), column c, rows 4*rq .. 4*rq + 3
    {
        const int I = (t >> 6) ? 3 : 1, J = I - 1, c = t & 15, rq = (t >> 4) & 3;
        float2 col2[8];
#pragma unroll
        for (int m = 0; m < 8; ++m)  // T_JJ[:, c]
            col2[m] = make_float2(sT[tsw(16 * J + 2 * m, 16 * J + c)], sT[tsw(16 * J + 2 * m + 1, 16 * J + c)]);
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {  // X = L_IJ T_JJ, kept in the free block (J, I)
            const int r = 4 * rq + rr;
            const float2 acc = tsw_dot2<4>(sL, 16 * I + r, 16 * J, col2, make_float2(0.f, 0.f));
            sT[tsw(16 * J + r, 16 * I + c)] = acc.x + acc.y;
        }
        group_bar(bar_id, NT);
#pragma unroll
        for (int m = 0; m < 8; ++m)  // X[:, c]
            col2[m] = make_float2(sT[tsw(16 * J + 2 * m, 16 * I + c)], sT[tsw(16 * J + 2 * m + 1, 16 * I + c)]);
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {  // T_IJ = -T_II X  (T_II[r][m] == 0 for m > r)
            const int r = 4 * rq + rr;
            const float2 acc = tsw_dot2<4>(sT, 16 * I + r, 16 * I, col2, make_float2(0.f, 0.f));
            sT[tsw(16 * I + r, 16 * J + c)] = -(acc.x + acc.y);
        }
    }
    group_bar(bar_id, NT);
    // ---- C. 32x32 level; thread: column c, rows 8*rq .. 8*rq + 7 (rq = warp of the group)
    {
        const int c = t & 31, rq = t >> 5;
        float2 col2[16];
#pragma unroll
        for (int m = 0; m < 16; ++m) {  // T_00[:, c]; block (0, 1) holds scratch, so mask m < c
            const float v0 = sT[tsw(2 * m, c)], v1 = sT[tsw(2 * m + 1, c)];
            col2[m] = make_float2(2 * m >= c ? v0 : 0.f, 2 * m + 1 >= c ? v1 : 0.f);
        }
        float2 acc[8];
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) acc[rr] = make_float2(0.f, 0.f);
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // X = L_10 T_00, kept in the free block (0, 1) of 32x32
#pragma unroll
            for (int rr = 0; rr < 8; ++rr)
                acc[rr] = tsw_dot2<4>(sL, 32 + 8 * rq + rr, 16 * h, col2 + 8 * h, acc[rr]);
        }
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) sT[tsw(8 * rq + rr, 32 + c)] = acc[rr].x + acc[rr].y;
        group_bar(bar_id, NT);
        // T_10 = -T_11 X.  T_11 is lower triangular, so warp rq (rows 8 rq .. 8 rq + 7 of T_11)
        // needs only its first 8 (rq + 1) terms (which also keeps warps 0-1 away from the
        // level-B scratch in columns 48..63 of rows 32..47).
        const int mlen = 8 * (rq + 1);
#pragma unroll
        for (int m = 0; m < 16; ++m)
            if (2 * m < mlen) col2[m] = make_float2(sT[tsw(2 * m, 32 + c)], sT[tsw(2 * m + 1, 32 + c)]);
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) acc[rr] = make_float2(0.f, 0.f);
#pragma unroll
        for (int q = 0; q < 4; ++q) {  // 8-term slices, taken while below the warp's bound
            if (8 * q < mlen) {
#pragma unroll
                for (int rr = 0; rr < 8; ++rr)
                    acc[rr] = tsw_dot2<2>(sT, 32 + 8 * rq + rr, 32 + 8 * q, col2 + 4 * q, acc[rr]);
            }
        }
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) sT[tsw(32 + 8 * rq + rr, c)] = -(acc[rr].x + acc[rr].y);
    }
    group_bar(bar_id, NT);
}

}  // namespace osdn
