// osdn_lib.cu -- libosdn: host side of the C ABI declared in include/osdn.h.
//
// One translation unit holds every kernel (so the device status word is a single symbol).
// The host code validates arguments, picks a kernel for the sizes and dtype, and enqueues it
// on the caller's stream.  It never allocates memory and never synchronizes, except in
// osdn_get_device_status, whose job is to synchronize.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "osdn.h"
#include "common.cuh"
#include "scan_warp.cuh"
#include "chunk_simt.cuh"
#include "watchdog.cuh"
#include "chunk_tc.cuh"
#include "chunk_prep.cuh"
#include "step.cuh"
#include "scan_tc.cuh"
#include "rho_geomean.cuh"
#include "bwd.cuh"

namespace osdn {
namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

inline size_t io_size(osdn_dtype_t io) { return io == OSDN_BF16 ? 2 : 4; }

struct Dims {
    int32_t B, T, H, Dk, Dv, N;
    int64_t rows() const { return (int64_t)B * T; }
};

osdn_status_t check_common(const int32_t* cu, int32_t num_seqs, int32_t B, int32_t T, int32_t H,
                           int32_t Dk, osdn_dtype_t io, Dims& d) {
    if (io != OSDN_BF16 && io != OSDN_F32) return OSDN_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || H < 1 || num_seqs < 0) return OSDN_ERR_INVALID_ARG;
    if (cu && B != 1) return OSDN_ERR_INVALID_ARG;
    if (cu && !aligned16(cu)) return OSDN_ERR_ALIGNMENT;
    if (Dk != 64 && Dk != 128) return OSDN_ERR_UNSUPPORTED;
    d.B = B;
    d.T = T;
    d.H = H;
    d.Dk = Dk;
    d.Dv = Dk;
    d.N = cu ? num_seqs : B;
    return OSDN_OK;
}

inline osdn_status_t launch_status() {
    return cudaGetLastError() == cudaSuccess ? OSDN_OK : OSDN_ERR_CUDA;
}

template <typename KernelT>
inline bool set_smem(KernelT kernel, size_t bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)bytes) == cudaSuccess;
}

// ---------------------------------------------------------------- phase 1 dispatch
template <typename IO>
osdn_status_t launch_scan_warp(const void* k, const float* beta, const float* r, float eta,
                               const float* d0, void* k_tilde, void* kt_lo, float* d_all,
                               float* dT, float* rho, const int32_t* cu, const Dims& d,
                               cudaStream_t stream) {
    const int units = d.N * d.H;
    if (units == 0) return OSDN_OK;
    const dim3 block(128), grid((units + 3) / 4);
    if (d.Dk == 128)
        precond_scan_warp_kernel<128, IO><<<grid, block, 0, stream>>>(
            static_cast<const IO*>(k), beta, r, eta, d0, static_cast<IO*>(k_tilde),
            static_cast<IO*>(kt_lo), d_all, dT, rho, cu, d.N, d.T, d.H);
    else
        precond_scan_warp_kernel<64, IO><<<grid, block, 0, stream>>>(
            static_cast<const IO*>(k), beta, r, eta, d0, static_cast<IO*>(k_tilde),
            static_cast<IO*>(kt_lo), d_all, dT, rho, cu, d.N, d.T, d.H);
    return launch_status();
}

// ---------------------------------------------------------------- phase 2 dispatch
template <int DK, int DV, int C, typename IO>
osdn_status_t launch_chunk_simt(const void* q, const void* k, const void* kt, const void* kt_lo,
                                const void* v, const float* beta, const float* alpha, int apc,
                                float scale, const float* S0, void* o, float* ST,
                                const int32_t* cu, const Dims& d, cudaStream_t stream) {
    constexpr int BV = 32;
    const int64_t ctas = (int64_t)d.N * d.H * (DV / BV);
    if (ctas == 0) return OSDN_OK;
    if (ctas > 0x7fffffff) return OSDN_ERR_UNSUPPORTED;
    auto kernel = chunk_fwd_simt_kernel<DK, DV, BV, C, IO>;
    const size_t smem = SimtSmem<DK, BV, C>::bytes;
    if (!set_smem(kernel, smem)) return OSDN_ERR_CUDA;
    kernel<<<dim3((unsigned)ctas), dim3(256), smem, stream>>>(
        static_cast<const IO*>(q), static_cast<const IO*>(k), static_cast<const IO*>(kt),
        static_cast<const IO*>(kt_lo), static_cast<const IO*>(v), beta, alpha, apc, scale, S0,
        static_cast<IO*>(o), ST, cu, d.N, d.T, d.H);
    return launch_status();
}

template <int DK, int DV, typename IO>
osdn_status_t launch_chunk_c(int chunk, const void* q, const void* k, const void* kt,
                             const void* kt_lo, const void* v, const float* beta,
                             const float* alpha, int apc, float scale, const float* S0, void* o,
                             float* ST, const int32_t* cu, const Dims& d, cudaStream_t stream) {
    switch (chunk) {
        case 16:
            return launch_chunk_simt<DK, DV, 16, IO>(q, k, kt, kt_lo, v, beta, alpha, apc, scale, S0,
                                                     o, ST, cu, d, stream);
        case 32:
            return launch_chunk_simt<DK, DV, 32, IO>(q, k, kt, kt_lo, v, beta, alpha, apc, scale, S0,
                                                     o, ST, cu, d, stream);
        case 64:
            return launch_chunk_simt<DK, DV, 64, IO>(q, k, kt, kt_lo, v, beta, alpha, apc, scale, S0,
                                                     o, ST, cu, d, stream);
        default:
            return OSDN_ERR_UNSUPPORTED;
    }
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime (the library
// does not link libcuda directly).
using EncodeTiledFn = PFN_cuTensorMapEncodeTiled_v12000;
EncodeTiledFn tensor_map_encoder() {
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// 3-D bf16 view [rows][H][D] of a [B, T, H, D] tensor; boxes of 64 channels x 1 head x 64
// tokens, 128-byte swizzle (the layout the MMA descriptors expect).
bool make_tile_map(CUtensorMap* m, const void* base, int D, int H, int64_t rows) {
    EncodeTiledFn enc = tensor_map_encoder();
    if (!enc || rows <= 0) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D fp32 view [rows][H][64] of a bf16 [B, T, H, 128] buffer (one 256-byte row per token and
// head); boxes of 64 values x 1 head x 64 tokens, no swizzle: the prep kernel's T_d tiles.
bool make_td_map(CUtensorMap* m, const void* base, int H, int64_t rows) {
    EncodeTiledFn enc = tensor_map_encoder();
    if (!enc || rows <= 0) return false;
    cuuint64_t dims[3] = {64, (cuuint64_t)H, (cuuint64_t)rows};
    cuuint64_t strides[2] = {256, (cuuint64_t)H * 256};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return 148;
    return n;
}

// Phase 1, bf16 with 128 key channels: T_d of every chunk (prep kernel, written into the k~
// buffer), then the chain across chunks (one CTA per (sequence, head)).
osdn_status_t launch_scan_tc(const void* k, const float* beta, const float* r, float eta,
                             const float* d0, void* k_tilde, void* kt_lo, float* d_all, float* dT,
                             float* rho, const int32_t* cu, const Dims& d, cudaStream_t stream) {
    const int64_t nh = (int64_t)d.N * d.H;
    if (nh == 0) return OSDN_OK;
    if (nh > 0x7fffffff) return OSDN_ERR_UNSUPPORTED;
    const int64_t rows = d.rows();  // > 0: token-free calls take the warp scan
    CUtensorMap mk, mtd, mkto, mktlo;
    if (!make_tile_map(&mk, k, 128, d.H, rows) || !make_td_map(&mtd, k_tilde, d.H, rows) ||
        !make_tile_map(&mkto, k_tilde, 128, d.H, rows) ||
        !make_tile_map(&mktlo, kt_lo ? kt_lo : k_tilde, 128, d.H, rows))
        return OSDN_ERR_CUDA;
    // persistent prep grid over (64-row window, head) items
    const int64_t items = ((rows + 63) / 64) * d.H;
    int64_t grid = (int64_t)SCAN_PREP_CTAS_PER_SM * sm_count();
    grid = grid < items ? grid : items;
    auto prep = precond_prep_kernel;
    if (!set_smem(prep, ScanPrepSmem::BYTES)) return OSDN_ERR_CUDA;
    prep<<<dim3((unsigned)grid), dim3(128), ScanPrepSmem::BYTES, stream>>>(
        mk, beta, r, eta, static_cast<float*>(k_tilde), cu, d.N, d.T, d.H, rows,
        (long long)kWaitLimitNs);
    const osdn_status_t st = launch_status();
    if (st != OSDN_OK) return st;
    auto chain = kt_lo ? (d_all ? precond_chain_kernel<true, true> : precond_chain_kernel<true, false>)
                       : (d_all ? precond_chain_kernel<false, true> : precond_chain_kernel<false, false>);
    if (!set_smem(chain, ScanChainSmem::BYTES)) return OSDN_ERR_CUDA;
    if (2 * nh > 0x7fffffff) return OSDN_ERR_UNSUPPORTED;
    // one 2-CTA cluster per (sequence, head): the chain and the k~ token pass on separate SMs
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * nh));
    cfg.blockDim = dim3(SCAN_CHAIN_THREADS);
    cfg.dynamicSmemBytes = ScanChainSmem::BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, chain, mk, mtd, mkto, mktlo, beta, r, eta, d0,
                           static_cast<__nv_bfloat16*>(k_tilde), static_cast<__nv_bfloat16*>(kt_lo),
                           d_all, dT, rho, cu, d.N, d.T, d.H, (long long)kWaitLimitNs) != cudaSuccess)
        return OSDN_ERR_CUDA;
    return launch_status();
}

// Phase 1: bf16 keys with 128 channels use the chunk-parallel kernel; fp32 I/O, 64 channels
// and token-free calls use the warp-per-(sequence, head) scan.  kt_lo (bf16 only; may be null):
// also write the residual bf16(k~ - k~_hi) of each key's rounding.
// d_all (may be null): also write d_t, the preconditioner of every token, as fp32 [B,T,H,Dk].
template <typename IO>
osdn_status_t launch_scan(const void* k, const float* beta, const float* r, float eta,
                          const float* d0, void* k_tilde, void* kt_lo, float* dT, float* rho,
                          const int32_t* cu, const Dims& d, cudaStream_t stream,
                          float* d_all = nullptr) {
    if constexpr (sizeof(IO) == 2) {
        if (d.Dk == 128 && d.rows() > 0 && d.rows() < (int64_t(1) << 31))
            return launch_scan_tc(k, beta, r, eta, d0, k_tilde, kt_lo, d_all, dT, rho, cu, d,
                                  stream);
    }
    return launch_scan_warp<IO>(k, beta, r, eta, d0, k_tilde, kt_lo, d_all, dT, rho, cu, d,
                                stream);
}

// 3-D fp32 view [rows][H][Dv / 2] of the bf16 output buffer; boxes of 32 values (one 128-byte
// slice of a row) x 1 head x 64 tokens: the WY factor's bf16 hi / lo operand tiles.
bool make_tp_map(CUtensorMap* m, const void* o, int Dv, int H, int64_t rows) {
    EncodeTiledFn enc = tensor_map_encoder();
    if (!enc || rows <= 0) return false;
    cuuint64_t dims[3] = {(cuuint64_t)Dv / 2, (cuuint64_t)H, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)Dv * 2, (cuuint64_t)H * Dv * 2};
    cuuint32_t box[3] = {32, 1, 64};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(o), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Phase 2, bf16 with d_k = d_v = 128: the WY factors of all chunks (persistent pre-kernel,
// written into o as bf16 hi / lo operand rows), then one CTA per (sequence, head, 64 value
// channels) for the state chain, the head's two CTAs as a cluster.
template <int DV>
osdn_status_t launch_chunk_tc(const void* q, const void* k, const void* kt, const void* kt_lo,
                              const void* v, const float* beta, float scale, const float* S0,
                              void* o, float* ST, const int32_t* cu, const Dims& d,
                              cudaStream_t stream) {
    const int64_t ctas = (int64_t)d.N * d.H * (DV / 64);
    if (ctas == 0) return OSDN_OK;
    if (ctas > 0x7fffffff) return OSDN_ERR_UNSUPPORTED;
    CUtensorMap mq, mk, mkt, mktlo, mv, mtp;
    const int64_t rows = d.rows();  // > 0 on this path
    const int has_lo = kt_lo != nullptr;
    if (!make_tile_map(&mq, q, 128, d.H, rows) || !make_tile_map(&mk, k, 128, d.H, rows) ||
        !make_tile_map(&mkt, kt, 128, d.H, rows) || !make_tile_map(&mv, v, DV, d.H, rows) ||
        !make_tp_map(&mtp, o, DV, d.H, rows) ||
        !make_tile_map(&mktlo, has_lo ? kt_lo : kt, 128, d.H, rows))
        return OSDN_ERR_CUDA;
    const int64_t items = ((rows + 63) / 64) * d.H;
    int64_t grid = (int64_t)WY_PREP_CTAS_PER_SM * sm_count();
    grid = grid < items ? grid : items;
    auto prep = wy_prep_kernel;
    if (!set_smem(prep, WyPrepSmem::BYTES)) return OSDN_ERR_CUDA;
    prep<<<dim3((unsigned)grid), dim3(128), WyPrepSmem::BYTES, stream>>>(
        mk, mkt, mktlo, has_lo, beta, static_cast<float*>(o), DV, cu, d.N, d.T, d.H, rows,
        (long long)kWaitLimitNs);
    const osdn_status_t st = launch_status();
    if (st != OSDN_OK) return st;
    auto kernel = chunk_fwd_tc_kernel<DV>;
    if (!set_smem(kernel, TcSmem::BYTES)) return OSDN_ERR_CUDA;
    // the head's two value-tile CTAs form a cluster (they share the WY hand-off in o)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)ctas);
    cfg.blockDim = dim3(TC_THREADS);
    cfg.dynamicSmemBytes = TcSmem::BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = DV / 64;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kernel, mq, mk, mkt, mv, mtp, mktlo, has_lo, beta, scale, S0,
                           static_cast<__nv_bfloat16*>(o), ST, cu, d.N, d.T, d.H,
                           (long long)kWaitLimitNs) != cudaSuccess)
        return OSDN_ERR_CUDA;
    return launch_status();
}

// kt_lo (may be null): the lo term of K~ handed over as bf16 hi + lo (k~ = kt + kt_lo).
// alpha (may be null): the decay of a gated backbone, per token (apc = 0) or per key channel.
template <typename IO>
osdn_status_t launch_chunk(int chunk, const void* q, const void* k, const void* kt,
                           const void* kt_lo, const void* v, const float* beta, const float* alpha,
                           int apc, float scale, const float* S0, void* o, float* ST,
                           const int32_t* cu, const Dims& d, cudaStream_t stream) {
    // bf16 I/O with 128 key and 128 value channels runs on the tensor cores; fp32 I/O, 64-channel
    // heads, gated backbones and token-free calls (states pass through) run the fp32 SIMT kernel.
    if constexpr (sizeof(IO) == 2) {
        if (!alpha && d.Dk == 128 && d.Dv == 128 && chunk == 64 && d.rows() > 0 &&
            d.rows() < (int64_t(1) << 31))
            return launch_chunk_tc<128>(q, k, kt, kt_lo, v, beta, scale, S0, o, ST, cu, d, stream);
    }
    if (d.Dk == 128 && d.Dv == 128)
        return launch_chunk_c<128, 128, IO>(chunk, q, k, kt, kt_lo, v, beta, alpha, apc, scale, S0,
                                            o, ST, cu, d, stream);
    if (d.Dk == 128 && d.Dv == 64)
        return launch_chunk_c<128, 64, IO>(chunk, q, k, kt, kt_lo, v, beta, alpha, apc, scale, S0, o,
                                           ST, cu, d, stream);
    if (d.Dk == 64 && d.Dv == 128)
        return launch_chunk_c<64, 128, IO>(chunk, q, k, kt, kt_lo, v, beta, alpha, apc, scale, S0, o,
                                           ST, cu, d, stream);
    return launch_chunk_c<64, 64, IO>(chunk, q, k, kt, kt_lo, v, beta, alpha, apc, scale, S0, o, ST,
                                      cu, d, stream);
}

// alpha: a device pointer of [B,T,H] (apc = 0) or [B,T,H,Dk] (apc = 1) float32, or null.
osdn_status_t validate_alpha(const float* alpha, int apc, const void* const* outs,
                             const size_t* out_bytes, int n_outs, const Dims& d) {
    if (apc != 0 && apc != 1) return OSDN_ERR_INVALID_ARG;
    if (!alpha) return OSDN_OK;
    if (!aligned16(alpha)) return OSDN_ERR_ALIGNMENT;
    const size_t ab = (size_t)d.rows() * d.H * (apc ? d.Dk : 1) * 4;
    for (int i = 0; i < n_outs; ++i)
        if (overlaps(alpha, ab, outs[i], out_bytes[i])) return OSDN_ERR_INVALID_ARG;
    return OSDN_OK;
}

osdn_status_t validate_scan(const void* k, const float* beta, const float* r, const float* d0,
                            const void* k_tilde, const float* dT, const float* rho, const Dims& d,
                            osdn_dtype_t io) {
    // token tensors may be NULL only when there are no tokens at all
    if (d.rows() * d.H > 0 && (!k || !beta || !k_tilde)) return OSDN_ERR_INVALID_ARG;
    const void* ptrs[] = {k, beta, r, d0, k_tilde, dT, rho};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return OSDN_ERR_ALIGNMENT;
    // the k~ buffer is written before the gates and states are read: no input may lie in it
    const size_t kbytes = (size_t)d.rows() * d.H * d.Dk * io_size(io);
    const size_t gbytes = (size_t)d.rows() * d.H * 4, sbytes = (size_t)d.N * d.H * d.Dk * 4;
    if (overlaps(k, kbytes, k_tilde, kbytes) || overlaps(beta, gbytes, k_tilde, kbytes) ||
        overlaps(r, gbytes, k_tilde, kbytes) || overlaps(d0, sbytes, k_tilde, kbytes) ||
        overlaps(dT, sbytes, k_tilde, kbytes) || overlaps(rho, gbytes, k_tilde, kbytes) ||
        overlaps(rho, gbytes, k, kbytes) || overlaps(rho, gbytes, beta, gbytes) ||
        overlaps(rho, gbytes, r, gbytes) || overlaps(rho, gbytes, d0, sbytes) ||
        overlaps(rho, gbytes, dT, sbytes))
        return OSDN_ERR_INVALID_ARG;
    return OSDN_OK;
}

osdn_status_t validate_chunk(const void* q, const void* k, const void* kt, const void* v,
                             const float* beta, const float* S0, const void* o, const float* ST,
                             const Dims& d, int chunk, osdn_dtype_t io) {
    if (d.rows() * d.H > 0 && (!q || !k || !kt || !v || !beta || !o)) return OSDN_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, kt, v, beta, S0, o, ST};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return OSDN_ERR_ALIGNMENT;
    if (d.Dv != 64 && d.Dv != 128) return OSDN_ERR_UNSUPPORTED;
    if (io == OSDN_BF16 ? chunk != 64 : (chunk != 16 && chunk != 32 && chunk != 64))
        return OSDN_ERR_UNSUPPORTED;
    const size_t es = io_size(io);
    const size_t kb = (size_t)d.rows() * d.H * d.Dk * es, vb = (size_t)d.rows() * d.H * d.Dv * es;
    // o is also scratch for per-chunk factors before it receives the outputs: nothing that is
    // read may lie in it
    const size_t gb = (size_t)d.rows() * d.H * 4, sb = (size_t)d.N * d.H * d.Dv * d.Dk * 4;
    if (overlaps(o, vb, q, kb) || overlaps(o, vb, k, kb) || overlaps(o, vb, kt, kb) ||
        overlaps(o, vb, v, vb) || overlaps(o, vb, beta, gb) || overlaps(o, vb, S0, sb) ||
        overlaps(o, vb, ST, sb))
        return OSDN_ERR_INVALID_ARG;
    return OSDN_OK;
}

}  // namespace
}  // namespace osdn

using namespace osdn;

namespace osdn {
namespace {
template <typename IO>
osdn_status_t launch_step_io(const void* q, const void* k, const void* v, const float* beta,
                             const float* r, const float* alpha, int apc, float eta, float scale,
                             float* S, float* d, void* o, void* kt, float* rho, int64_t nh, int Dk,
                             int Dv, cudaStream_t stream) {
    const IO *q_ = static_cast<const IO*>(q), *k_ = static_cast<const IO*>(k),
             *v_ = static_cast<const IO*>(v);
    IO *o_ = static_cast<IO*>(o), *kt_ = static_cast<IO*>(kt);
    const dim3 grid((unsigned)nh), block(step_threads(Dv));
    if (Dk == 128 && Dv == 128)
        osdn_step_kernel<128, 128, IO><<<grid, block, 0, stream>>>(q_, k_, v_, beta, r, eta, scale, S, d, o_, kt_, rho, alpha, apc, (int)nh);
    else if (Dk == 128 && Dv == 64)
        osdn_step_kernel<128, 64, IO><<<grid, block, 0, stream>>>(q_, k_, v_, beta, r, eta, scale, S, d, o_, kt_, rho, alpha, apc, (int)nh);
    else if (Dk == 64 && Dv == 128)
        osdn_step_kernel<64, 128, IO><<<grid, block, 0, stream>>>(q_, k_, v_, beta, r, eta, scale, S, d, o_, kt_, rho, alpha, apc, (int)nh);
    else
        osdn_step_kernel<64, 64, IO><<<grid, block, 0, stream>>>(q_, k_, v_, beta, r, eta, scale, S, d, o_, kt_, rho, alpha, apc, (int)nh);
    return launch_status();
}
}  // namespace
}  // namespace osdn


extern "C" {

int32_t osdn_abi_version(void) { return OSDN_ABI_VERSION; }

const char* osdn_status_string(osdn_status_t s) {
    switch (s) {
        case OSDN_OK: return "ok";
        case OSDN_ERR_INVALID_ARG: return "invalid argument";
        case OSDN_ERR_UNSUPPORTED: return "unsupported size or mode";
        case OSDN_ERR_ALIGNMENT: return "tensor pointer not 16-byte aligned";
        case OSDN_ERR_CUDA: return "CUDA runtime error";
        case OSDN_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
        case OSDN_ERR_DEVICE_BOUNDS: return "device-side cu_seqlens check failed";
    }
    return "unknown status";
}

osdn_status_t osdn_precond_scan(const void* k, const float* beta, const float* r, float eta,
                                const float* d0, void* k_tilde, float* dT, float* rho,
                                const int32_t* cu_seqlens, int32_t num_seqs, int32_t B,
                                int32_t T, int32_t H, int32_t Dk, osdn_dtype_t io,
                                void* stream) {
    Dims d;
    osdn_status_t st = check_common(cu_seqlens, num_seqs, B, T, H, Dk, io, d);
    if (st != OSDN_OK) return st;
    st = validate_scan(k, beta, r, d0, k_tilde, dT, rho, d, io);
    if (st != OSDN_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (io == OSDN_BF16)
        return launch_scan<__nv_bfloat16>(k, beta, r, eta, d0, k_tilde, nullptr, dT, rho, cu_seqlens,
                                          d, s);
    return launch_scan<float>(k, beta, r, eta, d0, k_tilde, nullptr, dT, rho, cu_seqlens, d, s);
}

osdn_status_t osdn_chunk_fwd(const void* q, const void* k, const void* k_tilde, const void* v,
                             const float* beta, const float* alpha, int32_t alpha_per_channel,
                             float scale, const float* S0, void* o, float* ST,
                             const int32_t* cu_seqlens, int32_t num_seqs, int32_t B, int32_t T,
                             int32_t H, int32_t Dk, int32_t Dv, int32_t chunk, osdn_dtype_t io,
                             void* stream) {
    Dims d;
    osdn_status_t st = check_common(cu_seqlens, num_seqs, B, T, H, Dk, io, d);
    if (st != OSDN_OK) return st;
    d.Dv = Dv;
    st = validate_chunk(q, k, k_tilde, v, beta, S0, o, ST, d, chunk, io);
    if (st != OSDN_OK) return st;
    {
        const void* outs[] = {o, ST};
        const size_t ob[] = {(size_t)d.rows() * d.H * d.Dv * io_size(io),
                             (size_t)d.N * d.H * d.Dv * d.Dk * 4};
        st = validate_alpha(alpha, alpha_per_channel, outs, ob, 2, d);
        if (st != OSDN_OK) return st;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (io == OSDN_BF16)
        return launch_chunk<__nv_bfloat16>(chunk, q, k, k_tilde, nullptr, v, beta, alpha,
                                           alpha_per_channel, scale, S0, o, ST, cu_seqlens, d, s);
    return launch_chunk<float>(chunk, q, k, k_tilde, nullptr, v, beta, alpha, alpha_per_channel,
                               scale, S0, o, ST, cu_seqlens, d, s);
}

// Workspace of osdn_fwd: k~ (used when the caller passes no k_tilde_out), then, for bf16, the
// residual of k~'s rounding to bf16, each part rounded up to 256 bytes.
static size_t kt_part_bytes(int32_t B, int32_t T, int32_t H, int32_t Dk, osdn_dtype_t io) {
    return (((size_t)B * T * H * Dk * io_size(io)) + 255) & ~(size_t)255;
}

size_t osdn_fwd_workspace_bytes(int32_t B, int32_t T, int32_t H, int32_t Dk, osdn_dtype_t io) {
    if (B < 0 || T < 0 || H < 1 || (Dk != 64 && Dk != 128) || (io != OSDN_BF16 && io != OSDN_F32))
        return 0;
    return kt_part_bytes(B, T, H, Dk, io) * (io == OSDN_BF16 ? 2 : 1);
}

osdn_status_t osdn_fwd(const void* q, const void* k, const void* v, const float* beta,
                       const float* r, const float* alpha, int32_t alpha_per_channel, float eta,
                       const float* d0, const float* S0, float scale, void* o, float* ST,
                       float* dT, float* rho, void* k_tilde_out, const int32_t* cu_seqlens,
                       int32_t num_seqs, int32_t B, int32_t T, int32_t H, int32_t Dk, int32_t Dv,
                       int32_t chunk, osdn_dtype_t io, void* workspace, size_t workspace_bytes,
                       void* stream) {
    Dims d;
    osdn_status_t st = check_common(cu_seqlens, num_seqs, B, T, H, Dk, io, d);
    if (st != OSDN_OK) return st;
    d.Dv = Dv;
    // where the preconditioned keys go: the caller's buffer, else the workspace's first part; for
    // bf16 the residual of their rounding goes to the workspace's second part, so phase 2 uses k~
    // to about 2^-17 of its size rather than to bf16's 2^-9
    const size_t need = osdn_fwd_workspace_bytes(B, T, H, Dk, io);
    void* kt = k_tilde_out;
    void* kt_lo = nullptr;
    if (need > 0) {
        if (!workspace || workspace_bytes < need) return OSDN_ERR_INVALID_ARG;
        if (reinterpret_cast<uintptr_t>(workspace) & 255u) return OSDN_ERR_ALIGNMENT;
        const size_t part = kt_part_bytes(B, T, H, Dk, io);
        if (!kt) kt = workspace;
        if (io == OSDN_BF16) kt_lo = static_cast<uint8_t*>(workspace) + part;
    }
    st = validate_scan(k, beta, r, d0, kt, dT, rho, d, io);
    if (st != OSDN_OK) return st;
    st = validate_chunk(q, k, kt, v, beta, S0, o, ST, d, chunk, io);
    if (st != OSDN_OK) return st;
    const size_t es = io_size(io);
    const size_t kb = (size_t)d.rows() * d.H * d.Dk * es, vb = (size_t)d.rows() * d.H * d.Dv * es;
    const size_t db = (size_t)d.N * d.H * d.Dk * 4;
    const size_t gb = (size_t)d.rows() * d.H * 4;
    // the lo part is written by phase 1 like k~ itself and read by phase 2 like k~
    if (kt_lo && (validate_scan(k, beta, r, d0, kt_lo, dT, rho, d, io) != OSDN_OK ||
                  validate_chunk(q, k, kt_lo, v, beta, S0, o, ST, d, chunk, io) != OSDN_OK ||
                  overlaps(kt_lo, kb, kt, kb) || overlaps(kt_lo, kb, q, kb) ||
                  overlaps(kt_lo, kb, v, vb)))
        return OSDN_ERR_INVALID_ARG;
    if (overlaps(kt, kb, q, kb) || overlaps(kt, kb, v, vb) || overlaps(o, vb, dT, db) ||
        overlaps(o, vb, rho, gb) || overlaps(rho, gb, q, kb) || overlaps(rho, gb, v, vb) ||
        overlaps(rho, gb, S0, (size_t)d.N * d.H * d.Dv * d.Dk * 4) ||
        overlaps(rho, gb, ST, (size_t)d.N * d.H * d.Dv * d.Dk * 4))
        return OSDN_ERR_INVALID_ARG;
    {
        const void* outs[] = {o, ST, dT, rho, kt, kt_lo};
        const size_t ob[] = {vb, (size_t)d.N * d.H * d.Dv * d.Dk * 4, db, gb, kb, kb};
        st = validate_alpha(alpha, alpha_per_channel, outs, ob, 6, d);
        if (st != OSDN_OK) return st;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (io == OSDN_BF16) {
        st = launch_scan<__nv_bfloat16>(k, beta, r, eta, d0, kt, kt_lo, dT, rho, cu_seqlens, d, s);
        if (st != OSDN_OK) return st;
        return launch_chunk<__nv_bfloat16>(chunk, q, k, kt, kt_lo, v, beta, alpha,
                                           alpha_per_channel, scale, S0, o, ST, cu_seqlens, d, s);
    }
    st = launch_scan<float>(k, beta, r, eta, d0, kt, nullptr, dT, rho, cu_seqlens, d, s);
    if (st != OSDN_OK) return st;
    return launch_chunk<float>(chunk, q, k, kt, nullptr, v, beta, alpha, alpha_per_channel, scale,
                               S0, o, ST, cu_seqlens, d, s);
}

osdn_status_t osdn_step(const void* q, const void* k, const void* v, const float* beta,
                        const float* r, const float* alpha, int32_t alpha_per_channel, float eta,
                        float scale, float* S, float* d, void* o, void* k_tilde, float* rho,
                        int32_t N, int32_t H, int32_t Dk, int32_t Dv, osdn_dtype_t io,
                        void* stream) {
    if (io != OSDN_BF16 && io != OSDN_F32) return OSDN_ERR_INVALID_ARG;
    if (alpha_per_channel != 0 && alpha_per_channel != 1) return OSDN_ERR_INVALID_ARG;
    if (N < 0 || H < 1) return OSDN_ERR_INVALID_ARG;
    if ((Dk != 64 && Dk != 128) || (Dv != 64 && Dv != 128)) return OSDN_ERR_UNSUPPORTED;
    const int64_t nh = (int64_t)N * H;
    if (nh == 0) return OSDN_OK;
    if (nh > 0x7fffffff) return OSDN_ERR_UNSUPPORTED;
    if (!q || !k || !v || !beta || !S || !d || !o) return OSDN_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, beta, r, alpha, S, d, o, k_tilde, rho};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return OSDN_ERR_ALIGNMENT;
    const size_t es = io_size(io);
    const size_t qb = nh * Dk * es, vb = nh * Dv * es, gb = nh * 4, sb = nh * Dv * Dk * 4,
                 db = nh * Dk * 4, ab = alpha_per_channel ? db : gb;
    // every written buffer (S, d, o, k_tilde, rho: slots 6..10) against every other buffer
    const void* all[] = {q, k, v, beta, r, alpha, S, d, o, k_tilde, rho};
    const size_t allb[] = {qb, qb, vb, gb, gb, ab, sb, db, vb, qb, gb};
    for (int a = 6; a < 11; ++a)
        for (int b = 0; b < 11; ++b)
            if (b != a && overlaps(all[a], allb[a], all[b], allb[b])) return OSDN_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (io == OSDN_BF16)
        return osdn::launch_step_io<__nv_bfloat16>(q, k, v, beta, r, alpha, alpha_per_channel, eta,
                                                   scale, S, d, o, k_tilde, rho, nh, Dk, Dv, s);
    return osdn::launch_step_io<float>(q, k, v, beta, r, alpha, alpha_per_channel, eta, scale, S, d,
                                       o, k_tilde, rho, nh, Dk, Dv, s);
}

osdn_status_t osdn_rho_geomean(const float* rho, const int32_t* cu_seqlens, int32_t num_seqs,
                               int32_t B, int32_t T, int32_t H, float* q_geo, void* stream) {
    if (B < 0 || T < 0 || H < 1 || num_seqs < 0) return OSDN_ERR_INVALID_ARG;
    if (cu_seqlens && B != 1) return OSDN_ERR_INVALID_ARG;
    const int64_t N = cu_seqlens ? num_seqs : B;
    const int64_t units = N * H;
    if (units == 0) return OSDN_OK;
    if (units > 0x7fffffff) return OSDN_ERR_UNSUPPORTED;
    if (!q_geo || ((int64_t)B * T > 0 && !rho)) return OSDN_ERR_INVALID_ARG;
    if ((rho && !aligned16(rho)) || !aligned16(q_geo) || (cu_seqlens && !aligned16(cu_seqlens)))
        return OSDN_ERR_ALIGNMENT;
    if (overlaps(rho, (size_t)B * T * H * 4, q_geo, (size_t)units * 4)) return OSDN_ERR_INVALID_ARG;
    rho_geomean_kernel<<<dim3((unsigned)units), dim3(GEOMEAN_THREADS), 0,
                         static_cast<cudaStream_t>(stream)>>>(rho, cu_seqlens, (int)N, T, H, q_geo);
    return launch_status();
}

}  // extern "C"

// ---------------------------------------------------------------- backward pass
namespace osdn {
namespace {

// Workspace of osdn_bwd, each part rounded up to 256 bytes: k~ (io dtype), d_t of every token,
// the state checkpoints (every BWD_C tokens), the per-value-tile shares of dq, dk, dk~ and dbeta,
// and deta per (sequence, head).
struct BwdWorkspace {
    size_t kt, dall, state, fw, dq, dk, dkt, dbeta, deta, total;
};

inline size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

BwdWorkspace bwd_workspace(int64_t rows, int64_t N, int32_t H, int32_t Dk, int32_t Dv,
                           osdn_dtype_t io) {
    BwdWorkspace w;
    const int64_t ntile = Dv / BWD_BV;
    const int64_t th = rows * H;
    size_t off = 0;
    w.kt = off;
    off += up256((size_t)th * Dk * io_size(io));
    w.dall = off;
    off += up256((size_t)th * Dk * 4);
    const size_t slots = (size_t)((rows + BWD_C - 1) / BWD_C + N + 1);
    w.state = off;
    off += up256(slots * H * Dv * Dk * 4);
    w.fw = off;
    off += up256(slots * H * ntile * BWD_FW * 4);
    w.dq = off;
    off += up256((size_t)ntile * th * Dk * 4);
    w.dk = off;
    off += up256((size_t)ntile * th * Dk * 4);
    w.dkt = off;
    off += up256((size_t)ntile * th * Dk * 4);
    w.dbeta = off;
    off += up256((size_t)ntile * th * 4);
    w.deta = off;
    off += up256((size_t)N * H * 4);
    w.total = off;
    return w;
}

template <int DK, typename IO>
osdn_status_t launch_bwd_kernels(const void* q, const void* k, const void* v, const float* beta,
                                 const float* r, float eta, const float* S0, float scale,
                                 const void* dO, const float* dST, const float* ddT, float* dq,
                                 float* dk, float* dv, float* dbeta, float* dr, float* deta,
                                 float* dS0, float* dd0, const int32_t* cu, const Dims& d,
                                 uint8_t* ws, const BwdWorkspace& w, cudaStream_t stream) {
    const int64_t rows = d.rows();
    const int ntile = d.Dv / BWD_BV;
    float* dall = reinterpret_cast<float*>(ws + w.dall);
    float* dq_part = reinterpret_cast<float*>(ws + w.dq);
    float* dk_part = reinterpret_cast<float*>(ws + w.dk);
    float* dkt_part = reinterpret_cast<float*>(ws + w.dkt);
    float* db_part = reinterpret_cast<float*>(ws + w.dbeta);
    float* deta_part = reinterpret_cast<float*>(ws + w.deta);
    const int64_t units = (int64_t)d.N * d.H;
    {
        auto kern = bwd_delta_kernel<DK, IO>;
        if (!set_smem(kern, BwdSmem<DK>::bytes)) return OSDN_ERR_CUDA;
        kern<<<dim3((unsigned)(units * ntile)), dim3(BWD_THREADS), BwdSmem<DK>::bytes, stream>>>(
            static_cast<const IO*>(q), static_cast<const IO*>(k), static_cast<const IO*>(v), beta,
            dall, S0, scale, static_cast<const IO*>(dO), dST, dv, dS0,
            reinterpret_cast<float*>(ws + w.state), reinterpret_cast<float*>(ws + w.fw), dq_part,
            dk_part, dkt_part, db_part, cu, d.N,
            d.T, d.H, d.Dv, rows);
        const osdn_status_t st = launch_status();
        if (st != OSDN_OK) return st;
    }
    if (rows > 0) {
        const int64_t n4 = rows * d.H * DK / 4, nb = rows * d.H;
        int64_t grid = (n4 + 255) / 256;
        const int64_t cap = 8LL * sm_count();
        grid = grid < cap ? grid : cap;
        bwd_reduce_kernel<<<dim3((unsigned)grid), dim3(256), 0, stream>>>(
            reinterpret_cast<const float4*>(dq_part), reinterpret_cast<float4*>(dk_part),
            reinterpret_cast<float4*>(dkt_part), db_part, ntile, n4, nb,
            reinterpret_cast<float4*>(dq));
        const osdn_status_t st = launch_status();
        if (st != OSDN_OK) return st;
    }
    {
        auto kern = bwd_precond_kernel<DK, IO>;
        if (!set_smem(kern, BwdPrecondSmem<DK, IO>::bytes)) return OSDN_ERR_CUDA;
        kern<<<dim3((unsigned)units), dim3(128), BwdPrecondSmem<DK, IO>::bytes, stream>>>(
            static_cast<const IO*>(k), beta, r, eta, dall, ddT, dk_part, dkt_part, db_part, dk, dbeta,
            dr, dd0, deta_part, cu, d.N, d.T, d.H);
        const osdn_status_t st = launch_status();
        if (st != OSDN_OK) return st;
    }
    if (deta) {
        bwd_sum_kernel<<<1, 256, 0, stream>>>(deta_part, units, deta);
        return launch_status();
    }
    return OSDN_OK;
}

}  // namespace
}  // namespace osdn

extern "C" {

size_t osdn_bwd_workspace_bytes(int32_t num_seqs, int32_t B, int32_t T, int32_t H, int32_t Dk,
                                int32_t Dv, osdn_dtype_t io) {
    if (B < 0 || T < 0 || H < 1 || num_seqs < 0 || (Dk != 64 && Dk != 128) ||
        (Dv != 64 && Dv != 128) || (io != OSDN_BF16 && io != OSDN_F32))
        return 0;
    const int64_t N = num_seqs > 0 ? num_seqs : B;
    return osdn::bwd_workspace((int64_t)B * T, N, H, Dk, Dv, io).total;
}

osdn_status_t osdn_bwd(const void* q, const void* k, const void* v, const float* beta,
                       const float* r, float eta, const float* d0, const float* S0, float scale,
                       const void* dO, const float* dST, const float* ddT, float* dq, float* dk,
                       float* dv, float* dbeta, float* dr, float* deta, float* dS0, float* dd0,
                       const int32_t* cu_seqlens, int32_t num_seqs, int32_t B, int32_t T,
                       int32_t H, int32_t Dk, int32_t Dv, osdn_dtype_t io, void* workspace,
                       size_t workspace_bytes, void* stream) {
    Dims d;
    osdn_status_t st = check_common(cu_seqlens, num_seqs, B, T, H, Dk, io, d);
    if (st != OSDN_OK) return st;
    if (Dv != 64 && Dv != 128) return OSDN_ERR_UNSUPPORTED;
    d.Dv = Dv;
    const int64_t th = d.rows() * d.H;
    const bool tokens = th > 0;
    if (tokens && (!q || !k || !v || !beta || !dO || !dq || !dk || !dv || !dbeta))
        return OSDN_ERR_INVALID_ARG;
    const void* ptrs[] = {q, k, v, beta, r, d0, S0, dO, dST, ddT, dq, dk, dv, dbeta, dr, deta,
                          dS0, dd0, cu_seqlens};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return OSDN_ERR_ALIGNMENT;
    const osdn::BwdWorkspace w = osdn::bwd_workspace(d.rows(), d.N, H, Dk, Dv, io);
    if (!workspace || workspace_bytes < w.total) return OSDN_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return OSDN_ERR_ALIGNMENT;
    // every output against every buffer (inputs, other outputs, the workspace)
    const size_t es = osdn::io_size(io);
    const size_t kb = (size_t)th * Dk * es, vb = (size_t)th * Dv * es, gb = (size_t)th * 4,
                 sb = (size_t)d.N * H * Dv * Dk * 4, db = (size_t)d.N * H * Dk * 4;
    const void* all[] = {q, k, v, beta, r, d0, S0, dO, dST, ddT, workspace,
                         dq, dk, dv, dbeta, dr, deta, dS0, dd0};
    const size_t allb[] = {kb, kb, vb, gb, gb, db, sb, vb, sb, db, w.total,
                           (size_t)th * Dk * 4, (size_t)th * Dk * 4, (size_t)th * Dv * 4, gb, gb, 4,
                           sb, db};
    for (int a = 11; a < 19; ++a)
        for (int b = 0; b < 19; ++b)
            if (b != a && osdn::overlaps(all[a], allb[a], all[b], allb[b])) return OSDN_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const int64_t units = (int64_t)d.N * H;
    if (units == 0) return OSDN_OK;
    if (units * (Dv / osdn::BWD_BV) > 0x7fffffff) return OSDN_ERR_UNSUPPORTED;
    // phase 1 forward: d_t of every token (k~ into the workspace, its own scratch)
    if (io == OSDN_BF16)
        st = osdn::launch_scan<__nv_bfloat16>(k, beta, r, eta, d0, ws + w.kt, nullptr, nullptr,
                                              nullptr, cu_seqlens, d, s,
                                              reinterpret_cast<float*>(ws + w.dall));
    else
        st = osdn::launch_scan<float>(k, beta, r, eta, d0, ws + w.kt, nullptr, nullptr, nullptr,
                                      cu_seqlens, d, s, reinterpret_cast<float*>(ws + w.dall));
    if (st != OSDN_OK) return st;
    if (io == OSDN_BF16) {
        if (Dk == 128)
            return osdn::launch_bwd_kernels<128, __nv_bfloat16>(q, k, v, beta, r, eta, S0, scale, dO,
                                                                dST, ddT, dq, dk, dv, dbeta, dr,
                                                                deta, dS0, dd0, cu_seqlens, d, ws,
                                                                w, s);
        return osdn::launch_bwd_kernels<64, __nv_bfloat16>(q, k, v, beta, r, eta, S0, scale, dO,
                                                           dST, ddT, dq, dk, dv, dbeta, dr, deta,
                                                           dS0, dd0, cu_seqlens, d, ws, w, s);
    }
    if (Dk == 128)
        return osdn::launch_bwd_kernels<128, float>(q, k, v, beta, r, eta, S0, scale, dO, dST, ddT,
                                                    dq, dk, dv, dbeta, dr, deta, dS0, dd0,
                                                    cu_seqlens, d, ws, w, s);
    return osdn::launch_bwd_kernels<64, float>(q, k, v, beta, r, eta, S0, scale, dO, dST, ddT, dq,
                                               dk, dv, dbeta, dr, deta, dS0, dd0, cu_seqlens, d,
                                               ws, w, s);
}

osdn_status_t osdn_get_device_status(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return OSDN_ERR_CUDA;
    int value = 0;
    const int zero = 0;
    if (cudaMemcpyFromSymbol(&value, g_device_status, sizeof(int)) != cudaSuccess)
        return OSDN_ERR_CUDA;
    if (value != 0 && cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess)
        return OSDN_ERR_CUDA;
    return static_cast<osdn_status_t>(value);
}

osdn_status_t osdn_debug_watchdog_selftest(int64_t spin_limit, void* stream) {
    if (spin_limit < 1 || spin_limit > (int64_t(1) << 30)) return OSDN_ERR_INVALID_ARG;
    watchdog_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(spin_limit);
    return launch_status();
}

}  // extern "C"

// ------------------------------------------------------------------------------------------
// osdn_fwd_noalloc: osdn_fwd for callers that cannot allocate device memory.
//
// The preconditioned keys that phase 1 hands to phase 2 normally live in a workspace the
// caller allocates.  Here they live in this file's fixed device array instead, so the caller
// passes only its inputs and outputs.  The array is part of the library image: every GPU that
// loads the library reserves it until the process exits.
// ------------------------------------------------------------------------------------------
#include <mutex>

namespace osdn {
namespace {

constexpr size_t kNoallocScratchBytes = OSDN_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};
void* g_noalloc_ctx[kMaxDevices] = {};  // the CUDA context the cached address belongs to

// cuCtxGetCurrent from the driver, looked up once through the runtime.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn ctx_get_current() {
    static CtxGetCurrentFn fn = []() -> CtxGetCurrentFn {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<CtxGetCurrentFn>(p);
    }();
    return fn;
}

// Device address of the array on the current device.  In host code the array's name is only a
// host-side stand-in, so the address is looked up with that device current and cached, together
// with the context it was found in; a new context (after cudaDeviceReset, say) looks it up anew
// instead of reusing an address that no longer exists.
osdn_status_t noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return OSDN_ERR_CUDA;
    CtxGetCurrentFn get_ctx = ctx_get_current();
    CUcontext ctx = nullptr;  // null until the runtime has made a context current on this thread
    if (!get_ctx || get_ctx(&ctx) != CUDA_SUCCESS) return OSDN_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (ctx == nullptr || g_noalloc_ptr[dev] == nullptr ||
        g_noalloc_ctx[dev] != static_cast<void*>(ctx)) {
        void* p = nullptr;  // the lookup also sets up the device's context when there is none yet
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
            return OSDN_ERR_CUDA;
        if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return OSDN_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
        g_noalloc_ctx[dev] = static_cast<void*>(ctx);
    }
    *out = g_noalloc_ptr[dev];
    return OSDN_OK;
}

}  // namespace
}  // namespace osdn

extern "C" osdn_status_t osdn_fwd_noalloc(const void* q, const void* k, const void* v,
                                          const float* beta, const float* r, const float* alpha,
                                          int32_t alpha_per_channel, float eta,
                                          const float* d0, const float* S0, float scale, void* o,
                                          float* ST, float* dT, float* rho,
                                          const int32_t* cu_seqlens,
                                          int32_t num_seqs, int32_t B, int32_t T, int32_t H,
                                          int32_t Dk, int32_t Dv, int32_t chunk,
                                          osdn_dtype_t io, void* stream) {
    if (B < 0 || T < 0 || H < 1 || (io != OSDN_BF16 && io != OSDN_F32))
        return OSDN_ERR_INVALID_ARG;
    if (Dk != 64 && Dk != 128) return OSDN_ERR_UNSUPPORTED;
    const size_t need = osdn_fwd_workspace_bytes(B, T, H, Dk, io);
    if (need > kNoallocScratchBytes) return OSDN_ERR_UNSUPPORTED;  // the hand-off does not fit
    void* scratch = nullptr;
    if (need > 0) {
        const osdn_status_t st = noalloc_scratch(&scratch);
        if (st != OSDN_OK) return st;
    }
    return osdn_fwd(q, k, v, beta, r, alpha, alpha_per_channel, eta, d0, S0, scale, o, ST, dT, rho,
                    nullptr, cu_seqlens, num_seqs, B, T, H, Dk, Dv, chunk, io, scratch,
                    need > 0 ? kNoallocScratchBytes : 0, stream);
}
