// chunk_walk.cuh -- the order in which a persistent CTA visits the 64-token chunks of a batch.
#pragma once

#include "common.cuh"

namespace osdn {

constexpr int kChunk = 64;

// Walks the chunks of the whole batch for a persistent CTA.  Work item w = (64-row window of
// the token rows, head); a window holds the start of at most one chunk of each sequence that
// overlaps it (chunk starts are 64 rows apart), so items are near-uniform in size whatever the
// sequence lengths.  Items w = blockIdx.x, blockIdx.x + gridDim.x, ...
struct ChunkWalk {
    const int32_t* cu;
    int N, T, H;
    int64_t rows, W, w;
    int n;          // next sequence to examine in the current window
    bool fresh;     // the current window's first sequence is not located yet
    // output of next(): the chunk
    int64_t row0;
    int Lc, h;

    __device__ void init(const int32_t* cu_, int N_, int T_, int H_, int64_t rows_) {
        cu = cu_;
        N = N_;
        T = T_;
        H = H_;
        rows = rows_;
        W = ((rows + kChunk - 1) / kChunk) * H;
        w = blockIdx.x;
        fresh = true;
    }
    // Last sequence whose first row is <= row (sequences are contiguous and ordered).
    __device__ int seq_at(int64_t row) const {
        if (!cu) {
            const int64_t q = row / T;
            return q < N - 1 ? (int)q : N - 1;
        }
        int lo = 0, hi = N - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if ((int64_t)__ldg(cu + mid) <= row) lo = mid; else hi = mid - 1;
        }
        return lo;
    }
    // Advance to the next chunk; false when the CTA's items are exhausted.
    __device__ bool next() {
        while (w < W) {
            const int64_t lo = (w / H) * kChunk;
            const int64_t hi = lo + kChunk < rows ? lo + kChunk : rows;
            if (fresh) {
                n = seq_at(lo);
                fresh = false;
            }
            while (n < N) {
                int64_t first, count;
                if (!seq_range(cu, n, N, T, first, count)) return false;
                if (first >= hi) break;
                ++n;
                const int64_t end = first + count;
                const int64_t s = first >= lo ? first : first + ((lo - first + kChunk - 1) / kChunk) * kChunk;
                if (s < hi && s < end) {
                    row0 = s;
                    Lc = end - s < kChunk ? (int)(end - s) : kChunk;
                    h = (int)(w % H);
                    return true;
                }
            }
            w += gridDim.x;
            fresh = true;
        }
        return false;
    }
};

}  // namespace osdn
