/*
 * osdn.h -- C ABI of libosdn, the B200 (sm_100a) forward pass of the Online Scaled DeltaNet
 * (OSDN) token mixer.
 *
 * The method is the one of "OSDN: Improving Delta Rule with Provable Online Preconditioning
 * in Linear Attention" (technical summary pages):
 *   - section 2.1: the right-preconditioned delta-rule step equals the delta rule with the
 *     write key k~_t = d_t (.) k_t, so the chunkwise WY pipeline of DeltaNet carries over
 *     with K~ in place of K in the chunk Gram matrix and the intra-chunk scores;
 *   - section 2.2: the preconditioner d follows online gradient descent on a surrogate whose
 *     closed form depends only on k_t, beta_t and d_t, which splits the forward pass into a
 *     light scan over the keys (phase 1) and the chunked DeltaNet pass (phase 2);
 *   - section 2.3: APF, a per-token, per-head retention gate r_{t,h} applied to d only.
 *
 * Per (sequence n, head h), tokens t = 0..T_n-1, with a_t = k_t (.) k_t:
 *   phase 1:  k~_t = d_t (.) k_t
 *             d_{t+1} = r_t d_t + eta * beta_t (1 - beta_t <d_t, a_t>) a_t / ||k_t||^2
 *             (descent on the surrogate; the step is 0 when ||k_t|| == 0; r == 1 without APF)
 *   phase 2:  S_t = S_{t-1} + beta_t (v_t - S_{t-1} k_t) k~_t^T,   o_t = scale * S_t q_t
 *
 * Conventions shared by every entry point
 *   - Pointers are DEVICE pointers to dense row-major tensors owned by the caller, unless a
 *     parameter says otherwise.  The library never allocates, frees or keeps a pointer.
 *   - Every tensor pointer must be 16-byte aligned (OSDN_ERR_ALIGNMENT otherwise).
 *   - Layouts:  q, k, k_tilde : [B, T, H, Dk]      v, o : [B, T, H, Dv]   (io dtype)
 *               beta, r       : [B, T, H]  float32 in every io mode
 *               S0, ST        : [N, H, Dv, Dk] float32 (row i of S is value channel i)
 *               d0, dT        : [N, H, Dk] float32
 *     Fixed length: cu_seqlens == NULL and N = B; sequence n is rows n*T .. n*T+T-1.
 *     Packed variable length: cu_seqlens != NULL (DEVICE int32 array of num_seqs+1 offsets,
 *     cu_seqlens[0] == 0, non-decreasing, cu_seqlens[num_seqs] == T), B == 1 and
 *     N = num_seqs; sequence n is rows cu_seqlens[n] .. cu_seqlens[n+1]-1.  Chunks restart
 *     at every sequence start and states are per sequence.  The offsets are checked on the
 *     device: a sequence whose offsets are out of order or out of range is skipped and the
 *     device status word records OSDN_ERR_DEVICE_BOUNDS (read it with
 *     osdn_get_device_status).
 *   - Supported sizes: Dk, Dv in {64, 128}; chunk 64 for OSDN_BF16, 16, 32 or 64 for
 *     OSDN_F32; T >= 0, B >= 0, H >= 1.  Anything else returns OSDN_ERR_UNSUPPORTED.
 *   - `stream` is a cudaStream_t (NULL: the legacy default stream).  Every call only
 *     enqueues work on it and returns; nothing synchronizes.  Calls on different streams
 *     may run concurrently as long as their output buffers do not overlap.
 *   - Argument errors are reported before anything is enqueued and leave outputs untouched.
 *     A failed kernel launch returns OSDN_ERR_CUDA.  No C++ exception crosses this ABI.
 *   - A debug-bounds build of this library (compiled with -DOSDN_DEBUG_BOUNDS; same symbols,
 *     same results) also checks every computed row or slot index of the kernels' global
 *     stores against its buffer's extent; an index outside it skips that store and records
 *     OSDN_ERR_DEVICE_BOUNDS.  The release build compiles these checks out.
 */
#ifndef OSDN_H_
#define OSDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define OSDN_ABI_VERSION 6

#if defined(__GNUC__)
#define OSDN_API __attribute__((visibility("default")))
#else
#define OSDN_API
#endif

typedef enum osdn_status {
    OSDN_OK = 0,
    OSDN_ERR_INVALID_ARG = 1,    /* NULL where a tensor is required, negative size, ...     */
    OSDN_ERR_UNSUPPORTED = 2,    /* a size or mode this build does not implement            */
    OSDN_ERR_ALIGNMENT = 3,      /* a tensor pointer that is not 16-byte aligned            */
    OSDN_ERR_CUDA = 4,           /* a CUDA runtime call or kernel launch failed             */
    OSDN_ERR_DEVICE_TIMEOUT = 5, /* a bounded device-side wait ran out (kernel returned)    */
    OSDN_ERR_DEVICE_BOUNDS = 6   /* device-side check of cu_seqlens failed; sequence skipped */
} osdn_status_t;

typedef enum osdn_dtype {
    OSDN_BF16 = 0, /* q, k, k_tilde, v, o in bfloat16; gates and states float32 */
    OSDN_F32 = 1   /* q, k, k_tilde, v, o in float32 (every product in fp32 FMA) */
} osdn_dtype_t;

/* Version of this ABI (OSDN_ABI_VERSION of the build). */
OSDN_API int32_t osdn_abi_version(void);

/* Short English text for a status code (static storage; never NULL). */
OSDN_API const char* osdn_status_string(osdn_status_t status);

/*
 * Phase 1: the preconditioner scan (section 2.2, first step of the two-phase split, with
 * the APF gate of section 2.3).
 *   k       [B,T,H,Dk] io dtype, read.
 *   beta    [B,T,H] float32, read.
 *   r       [B,T,H] float32 retention gate, or NULL for r == 1 (plain OSDN, no APF).
 *   eta     step size of the preconditioner's gradient descent (eta == 0 freezes d).
 *   d0      [N,H,Dk] initial preconditioner, or NULL for all ones.
 *   k_tilde [B,T,H,Dk] io dtype, written: k~_t = d_t (.) k_t.  Must not overlap k, beta, r,
 *           d0 or dT (OSDN_ERR_INVALID_ARG): for bf16 with Dk = 128 the call first uses this
 *           buffer as scratch for per-chunk factors, then overwrites it with k~.
 *   dT      [N,H,Dk] final preconditioner, written; NULL skips it.
 *   rho     [B,T,H] float32, written: the residual-contraction ratio of each write,
 *           rho_t = (1 - beta_t <d_t, k_t (.) k_t>)^2 (section 3: f_t(S_t) = rho_t f_t(S_{t-1}));
 *           NULL skips it.  Must not overlap any other buffer.
 */
OSDN_API osdn_status_t osdn_precond_scan(const void* k, const float* beta, const float* r, float eta,
                                const float* d0, void* k_tilde, float* dT, float* rho,
                                const int32_t* cu_seqlens, int32_t num_seqs, int32_t B,
                                int32_t T, int32_t H, int32_t Dk, osdn_dtype_t io,
                                void* stream);

/*
 * Phase 2: the chunkwise-parallel delta rule with write key K~ (section 2.1: K~ replaces K
 * in the chunk Gram matrix and in the intra-chunk scores).
 *   q, k    [B,T,H,Dk] io dtype, read (k is the erase/read key of the residual).
 *   k_tilde [B,T,H,Dk] io dtype, read (the write key).
 *   v       [B,T,H,Dv] io dtype, read.   beta [B,T,H] float32, read.
 *   alpha   decay of a gated backbone, or NULL for none: [B,T,H] float32 (Gated DeltaNet, one
 *           factor per token and head; alpha_per_channel = 0) or [B,T,H,Dk] float32 (Kimi Delta
 *           Attention, one per key channel; alpha_per_channel = 1).  The state's key channels
 *           decay before each write, S_t = S_{t-1} D_t + beta_t (v_t - S_{t-1} D_t k_t) k~_t^T
 *           with D_t = Diag(alpha_t) (the gated delta rule of the Gated DeltaNet-2 page,
 *           section 1, with OSDN's write key; phase 1 is unchanged).  Gated calls run phase 2 in
 *           fp32 FMA arithmetic (the SIMT kernel) in either io dtype.  alpha_per_channel must be
 *           0 or 1; alpha must not overlap an output.
 *   scale   multiplies o only (1.0 for unit-norm q).
 *   S0      [N,H,Dv,Dk] initial state, or NULL for zeros.
 *   o       [B,T,H,Dv] io dtype, written: o_t = scale * S_t q_t (state after token t).  Must
 *           not overlap q, k, k_tilde, v, beta, S0 or ST (OSDN_ERR_INVALID_ARG): for bf16 with
 *           Dk = 128 the call first uses it as scratch for per-chunk factors.
 *   ST      [N,H,Dv,Dk] final state, written; NULL skips it.
 *   chunk   tokens per chunk (64 for bf16; 16, 32 or 64 for f32).  The result does not
 *           depend on it beyond rounding.
 */
OSDN_API osdn_status_t osdn_chunk_fwd(const void* q, const void* k, const void* k_tilde, const void* v,
                             const float* beta, const float* alpha, int32_t alpha_per_channel,
                             float scale, const float* S0, void* o, float* ST,
                             const int32_t* cu_seqlens, int32_t num_seqs, int32_t B, int32_t T,
                             int32_t H, int32_t Dk, int32_t Dv, int32_t chunk, osdn_dtype_t io,
                             void* stream);

/* Bytes of device workspace osdn_fwd needs for these sizes: for bf16, two parts of
 * B*T*H*Dk*2 bytes each (k~ itself, used when k_tilde_out is NULL, and the residual of k~'s
 * rounding to bf16), each rounded up to 256 bytes; for fp32, one part of B*T*H*Dk*4 bytes
 * (rounded up likewise).  0 for unsupported sizes. */
OSDN_API size_t osdn_fwd_workspace_bytes(int32_t B, int32_t T, int32_t H, int32_t Dk, osdn_dtype_t io);

/*
 * Both phases (section 2.2's two-phase forward pass) on one stream.  Arguments are those of
 * osdn_precond_scan and osdn_chunk_fwd; in addition:
 *   k_tilde_out  [B,T,H,Dk] io dtype, or NULL.  When given, the preconditioned keys are
 *                written there (rounded to the io dtype) instead of to the workspace.
 *   workspace    device scratch of at least osdn_fwd_workspace_bytes(...) bytes, 256-byte
 *                aligned; NULL only if that size is 0.  In bf16 mode phase 1 hands k~ to
 *                phase 2 as two bf16 terms, k~ = hi + lo with hi = bf16(k~) and
 *                lo = bf16(k~ - hi) (about 2^-17 of |k~| left out), and every phase-2 product
 *                with K~ takes both terms, so phase 2 sees k~ essentially unrounded; the lo
 *                term lives in the workspace.  (The two-call path osdn_precond_scan ->
 *                osdn_chunk_fwd hands over hi only.)
 * The buffer rules of both phases apply; o must not overlap dT either.
 */
OSDN_API osdn_status_t osdn_fwd(const void* q, const void* k, const void* v, const float* beta,
                       const float* r, const float* alpha, int32_t alpha_per_channel, float eta,
                       const float* d0, const float* S0, float scale, void* o, float* ST,
                       float* dT, float* rho, void* k_tilde_out, const int32_t* cu_seqlens,
                       int32_t num_seqs, int32_t B, int32_t T, int32_t H, int32_t Dk, int32_t Dv,
                       int32_t chunk, osdn_dtype_t io, void* workspace, size_t workspace_bytes,
                       void* stream);

/*
 * osdn_fwd without any workspace, for callers that cannot allocate device memory: code that
 * runs inside a host application or plugin framework which owns every device allocation, or a
 * latency-critical service that forbids cudaMalloc after start-up (an allocation can
 * synchronize the device and fragments a fixed memory budget).  The original paper has no
 * counterpart: this is an interface convenience, not part of the method.
 *
 * Arguments are those of osdn_fwd minus k_tilde_out / workspace.  What osdn_fwd keeps in the
 * caller's workspace (the preconditioned keys phase 1 hands to phase 2, as bf16 hi and lo
 * terms in bf16 mode) goes to a fixed device array built into the library instead,
 * OSDN_NOALLOC_SCRATCH_BYTES (32 MiB) long, which every GPU that loads the library reserves
 * until the process exits.
 *   - Limit: osdn_fwd_workspace_bytes(B, T, H, Dk, io) must not exceed
 *     OSDN_NOALLOC_SCRATCH_BYTES (bf16: 2 * B * T * H * Dk * 2 bytes, each half rounded up to
 *     256 bytes); larger calls return OSDN_ERR_UNSUPPORTED before anything is enqueued.
 *   - The first call on each device (with that device current) looks up the array's device
 *     address in the device's current CUDA context and caches it; a later call looks it up
 *     again only if that context has changed (after cudaDeviceReset, for instance).  Make the
 *     first call on a device before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents.  Phase 1 rewrites
 *     every key before phase 2 reads it, so nothing needs clearing; but calls that overlap on
 *     the GPU (other streams, other host threads) race on it and must be serialized.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
#define OSDN_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
OSDN_API osdn_status_t osdn_fwd_noalloc(const void* q, const void* k, const void* v,
                                        const float* beta, const float* r, const float* alpha,
                                        int32_t alpha_per_channel, float eta,
                                        const float* d0, const float* S0, float scale, void* o,
                                        float* ST, float* dT, float* rho, const int32_t* cu_seqlens,
                                        int32_t num_seqs, int32_t B, int32_t T, int32_t H,
                                        int32_t Dk, int32_t Dv, int32_t chunk, osdn_dtype_t io,
                                        void* stream);

/*
 * Backward pass of osdn_fwd: the gradients of a loss L with respect to every input, given
 * dL/do, dL/dS_T and dL/dd_T.  The pages give no backward; this is the chain rule applied to the
 * forward recurrences (phase 1 and phase 2 as stated at the top of this header) in reverse order,
 * in fp32 FMA arithmetic (the path matches osdn_fwd's fp64 reference gradient, not a rounded one).
 *   q, k, v, beta, r, eta, d0, S0, scale   the forward pass's inputs (as for osdn_fwd).
 *   dO      [B,T,H,Dv] io dtype, read: dL/do.
 *   dST     [N,H,Dv,Dk] float32: dL/dS_T, or NULL for 0.   ddT [N,H,Dk] float32: dL/dd_T, or NULL.
 *   dq, dk  [B,T,H,Dk] float32, written.        dv [B,T,H,Dv] float32, written.
 *   dbeta   [B,T,H] float32, written.           dr [B,T,H] float32, written, or NULL to skip.
 *   deta    one float32, written (dL/deta), or NULL to skip.
 *   dS0     [N,H,Dv,Dk] float32, written, or NULL.   dd0 [N,H,Dk] float32, written, or NULL.
 *   workspace  device scratch of at least osdn_bwd_workspace_bytes(...) bytes, 256-byte aligned
 *           (about (4 + 3 Dv/64) x 4 B per key channel and token-head, plus, per 32 tokens and
 *           head, one Dv x Dk fp32 state and 24 KB per 64 value channels of chunk factors).
 * cu_seqlens, num_seqs, B, T, H as for the forward pass; Dk, Dv in {64, 128}.  Outputs must not
 * overlap one another, the inputs or the workspace (OSDN_ERR_INVALID_ARG).
 */
OSDN_API size_t osdn_bwd_workspace_bytes(int32_t num_seqs, int32_t B, int32_t T, int32_t H,
                                         int32_t Dk, int32_t Dv, osdn_dtype_t io);
OSDN_API osdn_status_t osdn_bwd(const void* q, const void* k, const void* v, const float* beta,
                                const float* r, float eta, const float* d0, const float* S0,
                                float scale, const void* dO, const float* dST, const float* ddT,
                                float* dq, float* dk, float* dv, float* dbeta, float* dr,
                                float* deta, float* dS0, float* dd0, const int32_t* cu_seqlens,
                                int32_t num_seqs, int32_t B, int32_t T, int32_t H, int32_t Dk,
                                int32_t Dv, osdn_dtype_t io, void* workspace,
                                size_t workspace_bytes, void* stream);

/*
 * q_geo, the residual-contraction diagnostic of section 3 (Theorem 5.2 bounds the product of
 * the token-local ratios rho_t = f_t(S_t) / f_t(S_{t-1}); the experiments of section 4.3
 * report their geometric mean): for every (sequence n, head h),
 *   q_geo[n][h] = exp( mean over the sequence's tokens of log rho[t][h] ).
 *   rho     [B,T,H] float32, read: the rho output of osdn_precond_scan or osdn_fwd (any
 *           non-negative ratios).  A ratio of 0 gives q_geo = 0.
 *   q_geo   [N,H] float32, written.  A sequence without tokens gets 1 (the empty product).
 * cu_seqlens, num_seqs, B and T as for the other calls.  Logs are taken in fp32 and summed in
 * fp64.  Pointers 16-byte aligned; q_geo must not overlap rho (OSDN_ERR_INVALID_ARG).
 */
OSDN_API osdn_status_t osdn_rho_geomean(const float* rho, const int32_t* cu_seqlens,
                                        int32_t num_seqs, int32_t B, int32_t T, int32_t H,
                                        float* q_geo, void* stream);

/*
 * One recurrent step per (sequence, head) -- the decode path (sections 2.1-2.3 applied to a
 * single token, the state carried in memory).  For each of the N*H (sequence, head) pairs, with
 * a = k (.) k, nk = ||k||^2 and s = <d, a>:
 *   k~ = d (.) k;  u = v - S k;  S <- S + beta u k~^T;  o = scale * S q;
 *   d <- r d + eta * beta * (1 - beta s) * a / nk   (0 when nk = 0).
 *   q, k     [N,H,Dk] io dtype, read.        v [N,H,Dv] io dtype, read.
 *   beta     [N,H] float32, read.            r [N,H] float32, or NULL for r == 1.
 *   S        [N,H,Dv,Dk] float32, read and written in place (row = value channel).
 *   d        [N,H,Dk] float32, read and written in place.
 *   o        [N,H,Dv] io dtype, written.     k_tilde [N,H,Dk] io dtype, written, or NULL.
 *   rho      [N,H] float32, written: (1 - beta s)^2, as for osdn_precond_scan; or NULL.
 *   alpha    decay of a gated backbone, or NULL for none: [N,H] float32 (Gated DeltaNet, one
 *            factor per token and head; alpha_per_channel = 0) or [N,H,Dk] float32 (Kimi Delta
 *            Attention, one per key channel; alpha_per_channel = 1).  The state's key channels
 *            decay first, S <- S Diag(alpha), then the step above runs on the decayed state (the
 *            gated delta rule of the Gated DeltaNet-2 page, section 1, with OSDN's write key; d
 *            is unchanged by the decay).  alpha_per_channel must be 0 or 1.
 * Dk, Dv in {64, 128}.  Pointers 16-byte aligned.  S, d, o and k_tilde must not overlap one
 * another or the inputs (OSDN_ERR_INVALID_ARG).  N == 0 is a no-op.  A sequence of steps
 * equals osdn_fwd over the same tokens (up to fp32 summation order).
 */
OSDN_API osdn_status_t osdn_step(const void* q, const void* k, const void* v, const float* beta,
                        const float* r, const float* alpha, int32_t alpha_per_channel, float eta,
                        float scale, float* S, float* d, void* o, void* k_tilde, float* rho,
                        int32_t N, int32_t H, int32_t Dk, int32_t Dv, osdn_dtype_t io,
                        void* stream);

/*
 * Synchronizes `stream`, then returns and clears the device status word of the current
 * device: OSDN_OK, OSDN_ERR_DEVICE_TIMEOUT or OSDN_ERR_DEVICE_BOUNDS (the first error any
 * kernel recorded since the last call; the word is shared by all streams of the device).
 * Returns OSDN_ERR_CUDA if the synchronization itself fails.
 */
OSDN_API osdn_status_t osdn_get_device_status(void* stream);

/*
 * Diagnostic: launches one block that waits on a shared-memory barrier nobody arrives at,
 * with at most `spin_limit` polls (1 .. 2^30), so the bounded wait runs out, records
 * OSDN_ERR_DEVICE_TIMEOUT in the device status word and returns.  Enqueue only.
 */
OSDN_API osdn_status_t osdn_debug_watchdog_selftest(int64_t spin_limit, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* OSDN_H_ */
