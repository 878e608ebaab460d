// common.cuh -- helpers shared by the libosdn kernels (device status word, I/O conversion,
// sequence bounds).  Part of the single translation unit built from osdn_lib.cu.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "osdn.h"

namespace osdn {

// First error recorded by any kernel since the host last read it (osdn_get_device_status).
__device__ int g_device_status = 0;

__device__ __forceinline__ void record_status(int code) {
    atomicCAS(&g_device_status, 0, code);
}

// Debug-bounds builds (compiled with -DOSDN_DEBUG_BOUNDS; `build.py --debug-bounds` writes
// libosdn_debug.so): the kernels' computed global stores check their index against the extent
// of the buffer they write; a violation records OSDN_ERR_DEVICE_BOUNDS and skips the store
// instead of writing outside the buffer.  Release builds compile the checks out.
#ifdef OSDN_DEBUG_BOUNDS
__device__ __forceinline__ bool bounds_ok(int64_t i, int64_t n) {
    if (i >= 0 && i < n) return true;
    record_status(OSDN_ERR_DEVICE_BOUNDS);
    return false;
}
#define OSDN_IN_BOUNDS(idx, extent) (::osdn::bounds_ok((int64_t)(idx), (int64_t)(extent)))
#else
#define OSDN_IN_BOUNDS(idx, extent) true
#endif

// Token range of sequence n: fixed length (cu == nullptr) or packed (device offsets).
// Returns false, after recording OSDN_ERR_DEVICE_BOUNDS, when the offsets are unusable.
__device__ __forceinline__ bool seq_range(const int32_t* __restrict__ cu, int n, int N, int T,
                                          int64_t& first, int64_t& count) {
    if (cu == nullptr) {
        first = (int64_t)n * T;
        count = T;
        return true;
    }
    const int32_t a = __ldg(cu + n), b = __ldg(cu + n + 1);
    const bool ok = a >= 0 && b >= a && b <= T && (n != 0 || a == 0) && (n != N - 1 || b == T);
    if (!ok) {
        record_status(OSDN_ERR_DEVICE_BOUNDS);
        return false;
    }
    first = a;
    count = (int64_t)b - a;
    return true;
}

// ---- io dtype traits --------------------------------------------------------------------
template <typename IO> struct io_traits;

template <> struct io_traits<float> {
    static __device__ __forceinline__ float to_f32(float x) { return x; }
    static __device__ __forceinline__ float from_f32(float x) { return x; }
};

template <> struct io_traits<__nv_bfloat16> {
    static __device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
    static __device__ __forceinline__ __nv_bfloat16 from_f32(float x) {
        return __float2bfloat16_rn(x);
    }
};

// Load / store 4 consecutive io elements as float4 (8-byte or 16-byte accesses).
template <typename IO> __device__ __forceinline__ float4 load4(const IO* p);
template <> __device__ __forceinline__ float4 load4<float>(const float* p) {
    return __ldg(reinterpret_cast<const float4*>(p));
}
template <> __device__ __forceinline__ float4 load4<__nv_bfloat16>(const __nv_bfloat16* p) {
    const uint2 raw = __ldg(reinterpret_cast<const uint2*>(p));
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
    const float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
    return make_float4(a.x, a.y, b.x, b.y);
}
template <typename IO> __device__ __forceinline__ void store4(IO* p, float4 v);
template <> __device__ __forceinline__ void store4<float>(float* p, float4 v) {
    *reinterpret_cast<float4*>(p) = v;
}
template <> __device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* p, float4 v) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(v.z, v.w);
    uint2 raw;
    raw.x = *reinterpret_cast<const uint32_t*>(&lo);
    raw.y = *reinterpret_cast<const uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(p) = raw;
}

// Load / store 2 consecutive io elements as float2.
template <typename IO> __device__ __forceinline__ float2 load2(const IO* p);
template <> __device__ __forceinline__ float2 load2<float>(const float* p) {
    return __ldg(reinterpret_cast<const float2*>(p));
}
template <> __device__ __forceinline__ float2 load2<__nv_bfloat16>(const __nv_bfloat16* p) {
    const uint32_t raw = __ldg(reinterpret_cast<const unsigned int*>(p));
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw));
}
template <typename IO> __device__ __forceinline__ void store2(IO* p, float2 v);
template <> __device__ __forceinline__ void store2<float>(float* p, float2 v) {
    *reinterpret_cast<float2*>(p) = v;
}
template <> __device__ __forceinline__ void store2<__nv_bfloat16>(__nv_bfloat16* p, float2 v) {
    *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(v.x, v.y);
}

}  // namespace osdn
