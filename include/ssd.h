/*
 * ssd.h — C ABI of the B200 (sm_100a) Mamba-2 SSD chunked-scan library (libssd.so).
 *
 * The operation is the State Space Duality (SSD) scan of Mamba-2, computed by the
 * five sub-modules named in "SSDi8: Accurate and Efficient 8-bit Quantization for
 * State Space Duality" (ICLR 2026 paper notes, section "overall framework"):
 * ChunkCumsum, ChunkState, StatePassing, ChunkBMM and ChunkScan (1 and 2).  It
 * produces the result of the recurrence, per batch row b and head h,
 *
 *     h_t = exp(dt_t * A_h) * h_{t-1} + dt_t * x_t B_{g(h),t}^T      (h_t is P x N)
 *     y_t = h_t C_{g(h),t} + D_h * x_t                                  (h_{-1} = 0)
 *
 * with g(h) = h / (H / G): B and C are stored per group and broadcast to blocks of
 * H/G consecutive heads.
 *
 * Two precision paths:
 *  - bf16 : bf16 inputs, fp32 accumulation, bf16 y, fp32 final state.
 *  - W8A8 : the persistent-INT8 scheme of the same notes: B and C quantised once per
 *           group (key design 3); ChunkState rebuilt as Q(LUT_state ⊙ X) x Q(B) with
 *           INT32 accumulation (key design 1, eq. 4 and the reconstruction); the
 *           state requantised to INT8 in registers with per-(H,P) scales, N left
 *           unquantised, and passed between chunks with a fixed-point decay and a
 *           shift by k = 7 (key design 2, eq. 6); ChunkBMM and ChunkScan1 on the
 *           INT8 B, C and state; ChunkScan2 in floating point with the CB
 *           dequantisation folded into LUT_Scan2.
 *
 * Conventions (all entry points):
 *  - Tensors are dense, row-major, in the layouts given per argument; every device
 *    pointer must be 16-byte aligned.  bf16 tensors are passed as uint16_t bit
 *    patterns.  The caller owns every buffer; the library allocates no memory.
 *  - Work is enqueued on `stream` and the call returns without synchronising.
 *    Argument and shape errors are detected on the host before anything is
 *    enqueued and are returned synchronously.  A failed launch returns SSD_ERR_CUDA.
 *  - Supported shapes: chunk in {64, 128, 256}; (headdim P, dstate N) in
 *    {(16,16), (64,128)}; nheads % ngroups == 0; any seqlen >= 0 (a final partial
 *    chunk behaves as if padded with dt = 0, x = B = C = 0 tokens).  Other shapes
 *    return SSD_ERR_UNSUPPORTED.
 *  - Preconditions not checked (the values are not scanned): dt >= 0 and finite,
 *    A <= 0, scales > 0 and finite.
 *  - The initial state is zero, except in the *_from_state entry points, which take
 *    one (the format of final_state).
 *  - No C++ exception crosses this interface.
 *
 * Beyond the scan, on the same conventions: the one-token decode step on the
 * persistent state (ssd_decode_step_bf16 / _i8), the SSD epilogue of the W8A8
 * pipeline (RMSNorm + INT8 output projection with the mean correction,
 * ssd_out_proj_i8) and a self-test of the device-side bounded wait.
 */
#ifndef SSD_B200_H
#define SSD_B200_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SSD_OK = 0,
    SSD_ERR_INVALID_ARG = 1,   /* null or misaligned pointer, negative size, bad parameter */
    SSD_ERR_UNSUPPORTED = 2,   /* shape outside the supported set */
    SSD_ERR_WORKSPACE = 3,     /* workspace missing or smaller than ssd_workspace_bytes() */
    SSD_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed */
    SSD_ERR_TIMEOUT = 5        /* a device-side bounded wait expired (read via ssd_workspace_status) */
} ssd_status;

typedef struct {
    int batch;     /* B  >= 0 */
    int seqlen;    /* L  >= 0 */
    int nheads;    /* H  >= 1 */
    int headdim;   /* P */
    int ngroups;   /* G  >= 1, divides H */
    int dstate;    /* N */
    int chunk;     /* Q, the chunk length l of the notes */
} ssd_shape;

/* Static symmetric INT8 scales (step sizes: real value = code * scale), device fp32.
 * Per-G for B and C, per-(H,P) for X_scaled and the state ("SSDi8" notes, key
 * designs 2 and 3). */
typedef struct {
    const float* s_B;      /* [G] */
    const float* s_C;      /* [G] */
    const float* s_x;      /* [H*P], scale of X_scaled = LUT_state ⊙ x */
    const float* s_s;      /* [H*P], scale of the INT8 state */
    int decay_shift;       /* k of eq. 6 (S = 2^k); 1..14, the notes use 7 */
    int storage;           /* 0: the library's layout (Acs fp32, CB kept on chip as INT32);
                            * otherwise flags of the notes' storage variant (overall
                            * framework; key design 2), for measurement and study:
                            * SSD_STORAGE_ACS_FP16 keeps Acs as IEEE half (every use reads
                            * the half value), SSD_STORAGE_CB_INT8 requantises each (b, c, g)
                            * CB tile to INT8 with one step amax|CB| / 127 (fp64; amax 0
                            * gives 1) and writes the codes to the workspace, from which
                            * ChunkScan2 reads them.  Flags need (P, N) = (64, 128) and
                            * chunk 256 (else SSD_ERR_UNSUPPORTED) and run the five-launch
                            * pipeline.  Zero-initialise the struct for the default. */
} ssd_i8_params;

#define SSD_STORAGE_ACS_FP16 1
#define SSD_STORAGE_CB_INT8 2

/* Human-readable name of a status code (static string). */
const char* ssd_status_string(ssd_status s);

/* The CUDA runtime's message for the error behind the calling thread's most recent
 * SSD_ERR_CUDA ("no error" if there was none); a static string. */
const char* ssd_last_cuda_error(void);

/* Bytes of device workspace that ssd_scan_fwd_bf16 (is_i8 = 0) or ssd_scan_fwd_i8
 * (is_i8 = 1) need for `shape`; 0 for an invalid or unsupported shape.  The
 * workspace holds the per-chunk cumulative decays, chunk states and passed states
 * plus a device status word (W8A8: also room for the single-launch scan's flags and
 * the storage variant's CB codes, so one size serves every W8A8 mode); its contents
 * are private to the library. */
size_t ssd_workspace_bytes(const ssd_shape* shape, int is_i8);

/* ChunkBMM/ChunkScan inputs quantised once along G ("SSDi8" notes, key design 3):
 *   Bq = clamp(rint(B * (1/s_B[g])), -127, 127), the same for C with s_C, in fp32 with
 *   round-to-nearest-even; 1/s is an IEEE division.
 * B, C : device bf16 [batch, seqlen, G, N].   s_B, s_C : device fp32 [G].
 * Bq, Cq : device int8 [batch, seqlen, G, N], written. */
ssd_status ssd_quantize_inputs(const ssd_shape* shape, const uint16_t* B, const uint16_t* C,
                               const float* s_B, const float* s_C,
                               int8_t* Bq, int8_t* Cq, cudaStream_t stream);

/* bf16 SSD forward.
 * x  : device bf16 [B, L, H, P]       dt : device fp32 [B, L, H] (after softplus, >= 0)
 * A  : device fp32 [H] (<= 0)         B, C : device bf16 [B, L, G, N]
 * D  : device fp32 [H]
 * y  : device bf16 [B, L, H, P], written
 * final_state : device fp32 [B, H, P, N], written (state after the last token)
 * workspace : device, at least ssd_workspace_bytes(shape, 0) bytes. */
ssd_status ssd_scan_fwd_bf16(const ssd_shape* shape, const uint16_t* x, const float* dt,
                             const float* A, const uint16_t* B, const uint16_t* C,
                             const float* D, uint16_t* y, float* final_state,
                             void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Size of the library's fixed device scratch used by ssd_scan_fwd_bf16_static. */
#define SSD_STATIC_SCRATCH_BYTES (32u << 20)

/* The bf16 SSD forward without a caller-provided workspace, for callers that cannot
 * allocate device memory (an allocator or arena that owns all device memory, a
 * plugin or embedded runtime that may not call cudaMalloc, a latency-critical thread
 * that must not take allocation locks).  The paper notes have no counterpart: this
 * is a packaging variant of ssd_scan_fwd_bf16, with the same arguments minus the
 * workspace and the same results.
 *  - Scratch lives in a fixed SSD_STATIC_SCRATCH_BYTES (32 MiB) array in the
 *    library's device memory, held by every GPU that loads the library until the
 *    process exits.  A shape whose ssd_workspace_bytes(shape, 0) exceeds it is
 *    rejected with SSD_ERR_WORKSPACE before anything is enqueued.
 *  - Nothing is allocated: no cudaMalloc/cudaFree or allocating library routine.
 *  - Every call looks up the array's device address with the calling device current
 *    (so a cudaDeviceReset or another context never sees a stale address).  Under lazy
 *    module loading (the CUDA default) the first call on a device loads the library's
 *    module, and the driver reserves the array's memory then: make that first call at
 *    start-up, before an arena takes the device's memory and before any stream capture.
 *  - All calls share the one array, which keeps the last call's contents (each call
 *    rewrites what it reads).  Calls whose GPU work overlaps (other streams, other
 *    host threads) race on it: serialise them.
 *  - A device-side error of the call (SSD_ERR_TIMEOUT from a bounded wait) is recorded
 *    in the array's status word: read it with ssd_static_scratch_status. */
ssd_status ssd_scan_fwd_bf16_static(const ssd_shape* shape, const uint16_t* x, const float* dt,
                                    const float* A, const uint16_t* B, const uint16_t* C,
                                    const float* D, uint16_t* y, float* final_state,
                                    cudaStream_t stream);

/* Status word of the fixed scratch used by ssd_scan_fwd_bf16_static (the counterpart of
 * ssd_workspace_status for callers that own no workspace): synchronises `stream`, returns
 * SSD_OK or the error a kernel of the last static call recorded (e.g. SSD_ERR_TIMEOUT),
 * and clears it.  Allocates nothing. */
ssd_status ssd_static_scratch_status(cudaStream_t stream);

/* ssd_scan_fwd_bf16 continuing from a given state: h_{-1} = initial_state (device fp32
 * [B, H, P, N], 16-byte aligned; null means zero, as in ssd_scan_fwd_bf16).  Feeding
 * a call's final_state to the next call over the following tokens reproduces one
 * call over both (bit for bit when the split falls on a chunk boundary).  With
 * seqlen 0, final_state receives a copy of initial_state.  The initial state enters
 * StatePassing as H_0 ("SSDi8" notes, eq. 6); everything else is unchanged. */
ssd_status ssd_scan_fwd_bf16_from_state(const ssd_shape* shape, const uint16_t* x, const float* dt,
                                        const float* A, const uint16_t* B, const uint16_t* C,
                                        const float* D, const float* initial_state, uint16_t* y,
                                        float* final_state, void* workspace, size_t workspace_bytes,
                                        cudaStream_t stream);

/* W8A8 SSD forward on the INT8 inputs of ssd_quantize_inputs.
 * x, dt, A, D, y : as in ssd_scan_fwd_bf16.   Bq, Cq : device int8 [B, L, G, N].
 * params : host pointer to the scales (device arrays) and the decay shift k.
 * final_state : device int8 [B, H, P, N], written; real value = code * s_s[h*P+p].
 * workspace : device, at least ssd_workspace_bytes(shape, 1) bytes.
 * Integer results (INT32 accumulators, INT8 states) are bit-exact with the
 * library's specification; see ssd_scan_fwd_i8_debug. */
ssd_status ssd_scan_fwd_i8(const ssd_shape* shape, const uint16_t* x, const float* dt,
                           const float* A, const int8_t* Bq, const int8_t* Cq, const float* D,
                           const ssd_i8_params* params, uint16_t* y, int8_t* final_state,
                           void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Optional device buffers that ssd_scan_fwd_i8_debug fills with the W8A8
 * intermediates (any may be NULL).  nc = ceil(L / Q); Lp = nc * Q.
 *   Acs       fp32  [B, H, nc, Q]     inclusive cumulative dt*A per chunk
 *   dq        int32 [B, H, nc]        decay codes rint(exp(Acs[Q-1]) * 2^k)
 *   Xq        int8  [B, Lp, H, P]     quantised X_scaled
 *   acc_state int32 [B, nc, H, P, N]  ChunkState accumulator Q(X_scaled)^T Q(B)
 *   S8        int8  [B, nc, H, P, N]  requantised chunk states
 *   H8        int8  [B, nc, H, P, N]  INT8 state entering each chunk
 *   cb        int32 [B, nc, G, Q, Q]  ChunkBMM accumulator Cq Bq^T (entries with i <= j;
 *                                     every entry with SSD_STORAGE_CB_INT8)
 *   acc_scan1 int32 [B, Lp, H, P]     ChunkScan1 accumulator Cq H8^T
 *   cb8       int8  [B, nc, G, Q, Q]  SSD_STORAGE_CB_INT8 only: the CB codes
 *   s_cb      fp64  [B, nc, G]        SSD_STORAGE_CB_INT8 only: their steps */
typedef struct {
    float* Acs;
    int32_t* dq;
    int8_t* Xq;
    int32_t* acc_state;
    int8_t* S8;
    int8_t* H8;
    int32_t* cb;
    int32_t* acc_scan1;
    int8_t* cb8;
    double* s_cb;
} ssd_i8_debug;

/* ssd_scan_fwd_i8 continuing from a given INT8 state: initial_state is device int8
 * [B, H, P, N] in the same codes as final_state (real value = code * s_s[h*P+p]),
 * 16-byte aligned; null means zero.  It is H_0 of the integer StatePassing (eq. 6),
 * so a call's final_state fed to the call over the following tokens reproduces
 * every integer of one call over both when the split falls on a chunk boundary. */
ssd_status ssd_scan_fwd_i8_from_state(const ssd_shape* shape, const uint16_t* x, const float* dt,
                                      const float* A, const int8_t* Bq, const int8_t* Cq, const float* D,
                                      const ssd_i8_params* params, const int8_t* initial_state, uint16_t* y,
                                      int8_t* final_state, void* workspace, size_t workspace_bytes,
                                      cudaStream_t stream);

/* ssd_scan_fwd_i8 that also writes the intermediates named in `dbg` (host pointer). */
ssd_status ssd_scan_fwd_i8_debug(const ssd_shape* shape, const uint16_t* x, const float* dt,
                                 const float* A, const int8_t* Bq, const int8_t* Cq,
                                 const float* D, const ssd_i8_params* params, uint16_t* y,
                                 int8_t* final_state, void* workspace, size_t workspace_bytes,
                                 const ssd_i8_debug* dbg, cudaStream_t stream);

/* Static calibration of the W8A8 scales over the first min(prefix, L) tokens of
 * every batch row (symmetric, step size = amax / 127, amax = 0 gives 1):
 *   s_B[g], s_C[g] : amax of |B|, |C| in group g
 *   s_x[h*P+p]     : amax of |X_scaled| = |dt_j exp(Acs_{Q-1} - Acs_j) x_j|
 *   s_s[h*P+p]     : amax over n of the chunk states S_c and the passed states
 *                    H_1..H_nc of the prefix (fp32 bf16-path arithmetic)
 * Inputs as in ssd_scan_fwd_bf16; outputs device fp32, written.  workspace: at
 * least ssd_calibrate_workspace_bytes(shape, prefix) bytes. */
size_t ssd_calibrate_workspace_bytes(const ssd_shape* shape, int prefix);
ssd_status ssd_calibrate_i8(const ssd_shape* shape, int prefix, const uint16_t* x,
                            const float* dt, const float* A, const uint16_t* B,
                            const uint16_t* C, float* s_B, float* s_C, float* s_x, float* s_s,
                            void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Device status word of a workspace used by a previous call: synchronises `stream`,
 * then returns SSD_OK or the error a kernel recorded (e.g. SSD_ERR_TIMEOUT), and
 * clears it. */
ssd_status ssd_workspace_status(void* workspace, cudaStream_t stream);

/* One token on the persistent state, in place (serving: the step after a scan, whose
 * final_state it continues; the recurrence the SSD factorises, one token at a time):
 *   h <- exp(dt*A) * h + dt * x B^T,      y = C . h + D * x
 * shape: batch, nheads, headdim, ngroups, dstate as in the scan; seqlen must be 1;
 *   chunk is not used.  Supported (P, N) as in the scan.
 * x  : device bf16 [B, H, P]          dt : device fp32 [B, H]
 * A, D : device fp32 [H]              B, C : device bf16 [B, G, N]
 * state : device fp32 [B, H, P, N], read and overwritten (the scan's final_state format)
 * y  : device bf16 [B, H, P], written.
 * All pointers 16-byte aligned.  Argument errors return before any launch. */
ssd_status ssd_decode_step_bf16(const ssd_shape* shape, const uint16_t* x, const float* dt, const float* A,
                                const uint16_t* B, const uint16_t* C, const float* D, float* state, uint16_t* y,
                                cudaStream_t stream);

/* W8A8 one-token step on the INT8 state of ssd_scan_fwd_i8 (codes, real value code *
 * s_s[h*P+p]), in place: the scan's integer steps with a chunk of one token ("SSDi8"
 * notes, key designs 1-3, eq. 6), so that the state codes equal those of
 * ssd_quantize_inputs + ssd_scan_fwd_i8_from_state over that token:
 *   Bq, Cq = the token's B, C quantised as ssd_quantize_inputs does (per group)
 *   a = dt*A;  Xq = clamp(rint(dt*x / s_x));  S8 = clamp(rint((Xq*Bq) * (s_x*s_B/s_s)))
 *   dq = rint(exp(a) * 2^k);  H <- sat127(S8 + ((dq*H + 2^(k-1)) >> k))
 *   y = (Cq.H_before)*s_C*s_s*exp(a) + (Cq.Bq)*s_C*s_B*dt*x + D*x     (bf16)
 * B, C : device bf16 [B, G, N] (one launch per token: no separate quantisation call).
 * params as in ssd_scan_fwd_i8.  state : device int8 [B, H, P, N], read and overwritten.
 * Other arguments as in ssd_decode_step_bf16. */
ssd_status ssd_decode_step_i8(const ssd_shape* shape, const uint16_t* x, const float* dt, const float* A,
                              const uint16_t* B, const uint16_t* C, const float* D, const ssd_i8_params* params,
                              int8_t* state, uint16_t* y, cudaStream_t stream);

/* SSD epilogue of the W8A8 pipeline ("SSDi8" notes, key design 4 and the training
 * strategy): RMSNorm of the scan output, static symmetric INT8 codes, the output
 * projection as an INT8 GEMM on the tensor cores, dequantisation and the mean
 * correction:
 *   u = y / sqrt(mean_k y^2 + 1e-5)             (per token, over k < d_inner)
 *   Aq = clamp(rint(u / s_a), +-127)             (codes kept in the workspace)
 *   out[t,d] = s_a * s_w[d] * sum_k Aq[t,k] Wq[d,k] + corr[d]     (bf16)
 * The RMSNorm weight is folded into Wq (gamma migration); corr = 0.15 c*, the mean
 * correction from calibration (null: none).
 * y : device bf16 [tokens, d_inner] (the scan's y seen as [B*L, H*P])
 * Wq : device int8 [d_model, d_inner]; s_w, corr : device fp32 [d_model]; s_a > 0
 * out : device bf16 [tokens, d_model], written
 * acc_debug : device int32 [tokens, d_model] or null: the INT32 accumulators
 * workspace : device, at least ssd_out_proj_workspace_bytes(tokens, d_inner) bytes
 * Supported: d_inner % 128 == 0, d_model % 256 == 0, tokens % 128 == 0 (else
 * SSD_ERR_UNSUPPORTED).  All pointers 16-byte aligned.  Asynchronous; a device-side
 * timeout is read back with ssd_out_proj_status. */
size_t ssd_out_proj_workspace_bytes(int tokens, int d_inner);
ssd_status ssd_out_proj_i8(int tokens, int d_inner, int d_model, const uint16_t* y, float s_a, const int8_t* Wq,
                           const float* s_w, const float* corr, uint16_t* out, int32_t* acc_debug, void* workspace,
                           size_t workspace_bytes, cudaStream_t stream);
/* Synchronises `stream` and returns the status word of an ssd_out_proj_i8 workspace. */
ssd_status ssd_out_proj_status(void* workspace, int tokens, int d_inner, cudaStream_t stream);

/* Self-test of the device-side bounded wait (the mechanism behind SSD_ERR_TIMEOUT):
 * launches, on `stream`, one CTA of two warps that wait on mbarriers nothing ever
 * completes.  Warp 0 gives up after `limit_cycles` SM clock cycles (0 < limit_cycles
 * <= about 4e9, i.e. two seconds), raises the CTA's abort flag and records
 * SSD_ERR_TIMEOUT in *status; warp 1, whose own limit is the kernels' full one,
 * must leave as soon as it sees the flag.  status: device int, cleared first, then
 * written by the kernel.  cycles: device array of 2 unsigned 64-bit counts, the
 * cycles each warp spent waiting.  Asynchronous: returns SSD_OK once launched,
 * SSD_ERR_INVALID_ARG for a null pointer or a limit out of range, SSD_ERR_CUDA if the
 * launch failed.  Neither warp faults, traps or waits past its limit. */
ssd_status ssd_selftest_bounded_wait(long long limit_cycles, int* status, unsigned long long* cycles,
                                     cudaStream_t stream);

/* Per-kernel timing (instrumentation, off by default).  While enabled, each kernel
 * the entry points enqueue is bracketed by two CUDA events on the caller's stream.
 * ssd_profile_read synchronises the recorded events and reports, for up to
 * `capacity` kernel names, the accumulated milliseconds and the number of launches
 * since the last reset; `count` receives the number of names known.  The name
 * strings are owned by the library and stay valid until it is unloaded. */
ssd_status ssd_profile_enable(int enable);
ssd_status ssd_profile_read(int capacity, const char** names, double* ms, long long* calls, int* count);
ssd_status ssd_profile_reset(void);
/* Restricts the per-kernel timing to the kernel named `name` (the names ssd_profile_read
 * reports; the string is copied), so that one kernel can be timed inside a loop with two
 * events per launch; NULL times every kernel again. */
ssd_status ssd_profile_filter(const char* name);

#ifdef __cplusplus
}
#endif

#endif /* SSD_B200_H */
