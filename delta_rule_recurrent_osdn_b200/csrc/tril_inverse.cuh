// tril_inverse.cuh -- (I + L)^-1 for a strictly lower-triangular 64x64 fp32 matrix L, computed by
// 256 threads in shared memory.
//
// Both phases of the chunked forward pass need this inverse once per 64-token chunk: phase 2 for
// the WY factor T = (I + strict_tril(diag(beta) K K~^T))^-1 (the (I + T)^-1 solve the Gated
// DeltaNet-2 summary names for the same building block), phase 1 for the analogous factor of
// the preconditioner recurrence.  Blocked algorithm, all in fp32:
//   1. the four diagonal 16x16 blocks by forward substitution (one column per thread);
//   2. 16x16 level: T_IJ = -T_II (L_IJ T_JJ) for (I, J) = (1, 0), (3, 2);
//   3. 32x32 level: T_[10] = -T_[11] (L_[10] T_[00]) on the 2x2 grid of 32x32 blocks.
// Matrices use row stride 65 (conflict-free row and column walks).
#pragma once

namespace osdn {

constexpr int kTrilStride = 65;

// sL: L (only the strictly lower part is read).  sT: receives T (all 64x64 entries written).
// sX: 64x65 fp32 scratch.  Must be called by all 256 threads of the block; ends synchronized.
__device__ __forceinline__ void tril_inverse_64(const float* __restrict__ sL, float* __restrict__ sT,
                                                float* __restrict__ sX, int tid) {
    constexpr int S = kTrilStride;
    // ---- 1. diagonal blocks; other threads clear everything above the block diagonal
    if (tid < 64) {
        const int b = tid >> 4, col = tid & 15, o = 16 * b;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc = 0.f;
#pragma unroll
            for (int m = 0; m < r; ++m)
                if (m >= col) acc = fmaf(sL[(o + r) * S + o + m], x[m], acc);
            x[r] = r < col ? 0.f : (r == col ? 1.f : -acc);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) sT[(o + r) * S + o + col] = x[r];
    } else {
        for (int idx = tid - 64; idx < 64 * 64; idx += 192) {
            const int r = idx >> 6, c = idx & 63;
            if ((c >> 4) > (r >> 4)) sT[r * S + c] = 0.f;
        }
    }
    __syncthreads();
    // ---- 2. 16x16 level, blocks (1,0) and (3,2): X = L_IJ T_JJ (T_JJ lower: m >= c).  Loops are
    //      fully unrolled with the triangular bound as a predicate so the loads pipeline.
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int idx = tid + 256 * k;
        const int I = (idx >> 8) ? 3 : 1, J = I - 1, r = (idx >> 4) & 15, c = idx & 15;
        const float* lrow = sL + (16 * I + r) * S + 16 * J;
        const float* tcol = sT + (16 * J) * S + 16 * J + c;
        float acc = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m)
            if (m >= c) acc = fmaf(lrow[m], tcol[m * S], acc);
        sX[(16 * I + r) * S + 16 * J + c] = acc;
    }
    __syncthreads();
    //      T_IJ = -T_II X (T_II lower: m <= r)
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int idx = tid + 256 * k;
        const int I = (idx >> 8) ? 3 : 1, J = I - 1, r = (idx >> 4) & 15, c = idx & 15;
        const float* trow = sT + (16 * I + r) * S + 16 * I;
        const float* xcol = sX + (16 * I) * S + 16 * J + c;
        float acc = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m)
            if (m <= r) acc = fmaf(trow[m], xcol[m * S], acc);
        sT[(16 * I + r) * S + 16 * J + c] = -acc;
    }
    __syncthreads();
    // ---- 3. 32x32 level: X = L[32:64, 0:32] T[0:32, 0:32]  (T lower: m >= c)
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int idx = tid + 256 * k, r = idx >> 5, c = idx & 31;
        const float* lrow = sL + (32 + r) * S;
        const float* tcol = sT + c;
        float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
        for (int m = 0; m < 32; m += 2) {
            if (m >= c) acc0 = fmaf(lrow[m], tcol[m * S], acc0);
            if (m + 1 >= c) acc1 = fmaf(lrow[m + 1], tcol[(m + 1) * S], acc1);
        }
        sX[(32 + r) * S + c] = acc0 + acc1;
    }
    __syncthreads();
    //      T[32:64, 0:32] = -T[32:64, 32:64] X   (m <= r)
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int idx = tid + 256 * k, r = idx >> 5, c = idx & 31;
        const float* trow = sT + (32 + r) * S + 32;
        const float* xcol = sX + 32 * S + c;
        float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
        for (int m = 0; m < 32; m += 2) {
            if (m <= r) acc0 = fmaf(trow[m], xcol[m * S], acc0);
            if (m + 1 <= r) acc1 = fmaf(trow[m + 1], xcol[(m + 1) * S], acc1);
        }
        sT[(32 + r) * S + c] = -(acc0 + acc1);
    }
    __syncthreads();
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

// The same inverse computed by a group of 128 threads (t = 0..127) that synchronizes on named
// barrier `bar_id`.  It needs no scratch beyond sT: the intermediate products X are kept,
// transposed, in the part of sT above the block diagonal, which is cleared at the end.
__device__ __forceinline__ void tril_inverse_64_g128(const float* __restrict__ sL,
                                                     float* __restrict__ sT, int t, int bar_id) {
    constexpr int S = kTrilStride, NT = 128;
    if (t < 64) {  // diagonal 16x16 blocks
        const int b = t >> 4, col = t & 15, o = 16 * b;
        float x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc = 0.f;
#pragma unroll
            for (int m = 0; m < r; ++m)
                if (m >= col) acc = fmaf(sL[(o + r) * S + o + m], x[m], acc);
            x[r] = r < col ? 0.f : (r == col ? 1.f : -acc);
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) sT[(o + r) * S + o + col] = x[r];
    }
    group_bar(bar_id, NT);
    // 16x16 level, (I, J) = (1, 0) and (3, 2): X = L_IJ T_JJ, stored transposed in block (J, I)
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int idx = t + NT * k;
        const int I = (idx >> 8) ? 3 : 1, J = I - 1, r = (idx >> 4) & 15, c = idx & 15;
        const float* lrow = sL + (16 * I + r) * S + 16 * J;
        const float* tcol = sT + (16 * J) * S + 16 * J + c;
        float acc = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m)
            if (m >= c) acc = fmaf(lrow[m], tcol[m * S], acc);
        sT[(16 * J + c) * S + 16 * I + r] = acc;
    }
    group_bar(bar_id, NT);
    //      T_IJ = -T_II X
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int idx = t + NT * k;
        const int I = (idx >> 8) ? 3 : 1, J = I - 1, r = (idx >> 4) & 15, c = idx & 15;
        const float* trow = sT + (16 * I + r) * S + 16 * I;
        const float* xrow = sT + (16 * J + c) * S + 16 * I;
        float acc = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m)
            if (m <= r) acc = fmaf(trow[m], xrow[m], acc);
        sT[(16 * I + r) * S + 16 * J + c] = -acc;
    }
    group_bar(bar_id, NT);
    // 32x32 level: X = L[32:64, 0:32] T[0:32, 0:32], stored transposed in rows 0..31, cols 32..63
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int idx = t + NT * k, r = idx >> 5, c = idx & 31;
        const float* lrow = sL + (32 + r) * S;
        const float* tcol = sT + c;
        float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
        for (int m = 0; m < 32; m += 2) {
            if (m >= c) acc0 = fmaf(lrow[m], tcol[m * S], acc0);
            if (m + 1 >= c) acc1 = fmaf(lrow[m + 1], tcol[(m + 1) * S], acc1);
        }
        sT[c * S + 32 + r] = acc0 + acc1;
    }
    group_bar(bar_id, NT);
    //      T[32:64, 0:32] = -T[32:64, 32:64] X
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int idx = t + NT * k, r = idx >> 5, c = idx & 31;
        const float* trow = sT + (32 + r) * S + 32;
        const float* xrow = sT + c * S + 32;
        float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
        for (int m = 0; m < 32; m += 2) {
            if (m <= r) acc0 = fmaf(trow[m], xrow[m], acc0);
            if (m + 1 <= r) acc1 = fmaf(trow[m + 1], xrow[m + 1], acc1);
        }
        sT[(32 + r) * S + c] = -(acc0 + acc1);
    }
    group_bar(bar_id, NT);
    for (int idx = t; idx < 64 * 64; idx += NT) {  // clear everything above the block diagonal
        const int r = idx >> 6, c = idx & 63;
        if ((c >> 4) > (r >> 4)) sT[r * S + c] = 0.f;
    }
    group_bar(bar_id, NT);
}

}  // namespace osdn
