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
        float x[16];
        if (t < 64) {
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float lr[16];
#pragma unroll
                for (int g = 0; 4 * g < r; ++g) {
                    const float4 v = tsw_ld4(sL, o + r, (o >> 2) + g);
                    lr[4 * g] = v.x;
                    lr[4 * g + 1] = v.y;
                    lr[4 * g + 2] = v.z;
                    lr[4 * g + 3] = v.w;
                }
                float acc = 0.f;  // x[m] == 0 for m < col, so no per-lane bound is needed
#pragma unroll
                for (int m = 0; m < r; ++m) acc = fmaf(-lr[m], x[m], acc);
                x[r] = r == col ? 1.f : (r < col ? 0.f : acc);
            }
        }
        group_bar(bar_id, NT);  // the diagonal blocks of L are read
        if (t < 64) {
#pragma unroll
            for (int r = 0; r < 16; ++r) sT[tsw(o + r, o + col)] = x[r];
        }
    }
    group_bar(bar_id, NT);
    // ---- B. 16x16 level; thread: block pair (t >> 6), column c, rows 4*rq .. 4*rq + 3
    {
        const int I = (t >> 6) ? 3 : 1, J = I - 1, c = t & 15, rq = (t >> 4) & 3;
        float col[16];
#pragma unroll
        for (int m = 0; m < 16; ++m) col[m] = sT[tsw(16 * J + m, 16 * J + c)];  // T_JJ[:, c]
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {  // X = L_IJ T_JJ, kept in the free block (J, I)
            const int r = 4 * rq + rr;
            float lr[16];
            tsw_row<4>(sL, 16 * I + r, 16 * J, lr);
            float acc = 0.f;
#pragma unroll
            for (int m = 0; m < 16; ++m) acc = fmaf(lr[m], col[m], acc);
            sT[tsw(16 * J + r, 16 * I + c)] = acc;
        }
        group_bar(bar_id, NT);
#pragma unroll
        for (int m = 0; m < 16; ++m) col[m] = sT[tsw(16 * J + m, 16 * I + c)];  // X[:, c]
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {  // T_IJ = -T_II X  (T_II[r][m] == 0 for m > r)
            const int r = 4 * rq + rr;
            float tr[16];
            tsw_row<4>(sT, 16 * I + r, 16 * I, tr);
            float acc = 0.f;
#pragma unroll
            for (int m = 0; m < 16; ++m) acc = fmaf(-tr[m], col[m], acc);
            sT[tsw(16 * I + r, 16 * J + c)] = acc;
        }
    }
    group_bar(bar_id, NT);
    // ---- C. 32x32 level; thread: column c, rows 8*rq .. 8*rq + 7 (rq = warp of the group)
    {
        const int c = t & 31, rq = t >> 5;
        float col[32];
#pragma unroll
        for (int m = 0; m < 32; ++m) {  // T_00[:, c]; block (0, 1) holds scratch, so mask m < c
            const float v = sT[tsw(m, c)];
            col[m] = m >= c ? v : 0.f;
        }
        float acc[8];
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) acc[rr] = 0.f;
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // X = L_10 T_00, kept in the free block (0, 1) of 32x32
#pragma unroll
            for (int rr = 0; rr < 8; ++rr) {
                float lr[16];
                tsw_row<4>(sL, 32 + 8 * rq + rr, 16 * h, lr);
#pragma unroll
                for (int m = 0; m < 16; ++m) acc[rr] = fmaf(lr[m], col[16 * h + m], acc[rr]);
            }
        }
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) sT[tsw(8 * rq + rr, 32 + c)] = acc[rr];
        group_bar(bar_id, NT);
        // T_10 = -T_11 X.  T_11 is lower triangular, so warp rq (rows 8 rq .. 8 rq + 7 of T_11)
        // needs only its first 8 (rq + 1) terms (which also keeps warps 0-1 away from the
        // level-B scratch in columns 48..63 of rows 32..47).
        const int mlen = 8 * (rq + 1);
#pragma unroll
        for (int m = 0; m < 32; ++m)
            if (m < mlen) col[m] = sT[tsw(m, 32 + c)];  // X[:, c]
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) acc[rr] = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {  // 8-term slices, taken while below the warp's bound
            if (8 * q < mlen) {
#pragma unroll
                for (int rr = 0; rr < 8; ++rr) {
                    float tr[8];
                    tsw_row<2>(sT, 32 + 8 * rq + rr, 32 + 8 * q, tr);
#pragma unroll
                    for (int m = 0; m < 8; ++m) acc[rr] = fmaf(-tr[m], col[8 * q + m], acc[rr]);
                }
            }
        }
#pragma unroll
        for (int rr = 0; rr < 8; ++rr) sT[tsw(32 + 8 * rq + rr, c)] = acc[rr];
    }
    group_bar(bar_id, NT);
}

}  // namespace osdn
