// kernels.h — launchers of the SSD scan kernels (internal to libssd.so).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ssd.h"
#include "common.cuh"

namespace ssd {

// Workspace layout of one scan call (offsets in bytes, 256-byte aligned regions).
struct WsLayout {
    size_t status, acs, lut, dtc, decay, states, passed, scales, cb8, total;
};
// `fp32_states`: chunk states kept in fp32 (calibration) instead of bf16 / int8.
WsLayout ws_layout(const Dims& d, bool i8, bool fp32_states = false);

// Optional W8A8 intermediates (device pointers, any may be null).
struct I8Debug {
    float* Acs;
    int32_t* dq;
    int8_t* Xq;
    int32_t* acc_state;
    int8_t* S8;
    int8_t* H8;
    int32_t* cb;
    int32_t* acc_scan1;
    int8_t* cb8;      // storage variant: CB codes [B,nc,G,Q,Q]
    double* s_cb;     // storage variant: their steps [B,nc,G]
};

struct I8Scales {
    const float* s_B;
    const float* s_C;
    const float* s_x;
    const float* s_s;
    int shift;
};

// a0: per-group INT8 quantisation of B and C.
cudaError_t launch_quantize_bc(const Dims& d, const uint16_t* B, const uint16_t* C,
                               const float* s_B, const float* s_C, int8_t* Bq, int8_t* Cq,
                               cudaStream_t st);

// a1: ChunkCumsum.  Writes Acs [B,H,nc,Q]; the bf16 path also the chunk decay
// exp(Acs[Q-1]) (fp32 [B,H,nc]); the W8A8 path the decay codes (int32 [B,H,nc]).
// Clears the workspace status word `status` (may be null) for the call.  `lut`
// (LUT_state) and `dtc` (dt) are optional [B,H,nc,Q] outputs.  W8A8 with `sc`: also
// inv_sx = 1/s_x and mq = s_x s_B / s_s per (h,p) ([H*P] each).  `acs_half`: Acs rounded
// to IEEE half as soon as it is formed, and stored as half (the storage variant).
cudaError_t launch_cumsum(const Dims& d, const float* dt, const float* A, float* Acs,
                          float* decay, int32_t* dq, int shift, int* status, float* lut, float* dtc,
                          cudaStream_t st, const I8Scales* sc = nullptr, float* inv_sx = nullptr,
                          float* mq = nullptr, bool acs_half = false);
// n IEEE half values to fp32 (debug copies).
cudaError_t launch_half_to_float(const void* src, float* dst, long long n, cudaStream_t st);

// a2: ChunkState.  bf16: fp32 states [B,nc,H,P,N]; W8A8: INT8 states.
// amax_xs / amax_s (calibration only): per-(h,p) running max of |X_scaled| and |S_c|.
cudaError_t launch_chunk_state_bf16(const Dims& d, const uint16_t* x, const float* dt,
                                    const float* Acs, const uint16_t* B, float* S,
                                    float* amax_xs, float* amax_s, cudaStream_t st);
cudaError_t launch_chunk_state_i8(const Dims& d, const uint16_t* x, const float* dt,
                                  const float* Acs, const int8_t* Bq, const I8Scales& sc,
                                  int8_t* S8, const I8Debug* dbg, cudaStream_t st);

// a3: StatePassing, sequential over chunks.
//   bf16: H_{c+1} = decay_c * H_c + S_c in fp32; writes the state entering each
//         chunk as bf16 (Hc) and/or fp32 (Hc32), the final state as fp32.
//   W8A8: H_{c+1} = sat127(S8_c + ((dq_c * H_c + 2^(k-1)) >> k)).
// One token on the persistent state (in place): bf16 path on an fp32 state, W8A8 on the
// INT8 state codes (B and C quantised inside).  x [B,H,P] bf16, dt [B,H], B/C bf16 [B,G,N], y [B,H,P] bf16.
cudaError_t launch_decode_bf16(const Dims& d, const uint16_t* x, const float* dt, const float* A, const uint16_t* B,
                               const uint16_t* C, const float* D, float* state, uint16_t* y, cudaStream_t st);
cudaError_t launch_decode_i8(const Dims& d, const uint16_t* x, const float* dt, const float* A, const uint16_t* B,
                             const uint16_t* C, const float* D, const I8Scales& sc, int8_t* state, uint16_t* y,
                             cudaStream_t st);

// SSD epilogue: RMSNorm codes of y [T,K] (bf16) into aq [T,K], then out [T,D] (bf16) =
// (aq Wq^T) * s_a * s_w[d] + corr[d] (corr may be null); acc_dbg [T,D] int32 optional.
cudaError_t launch_out_proj_norm(int T, int K, const uint16_t* y, float s_a, int8_t* aq, cudaStream_t st);
cudaError_t launch_out_proj_gemm(int T, int K, int D, const int8_t* aq, float s_a, const int8_t* Wq, const float* s_w,
                                 const float* corr, uint16_t* out, int32_t* acc_dbg, int* status, cudaStream_t st);

// init (fp32 [B,H,P,N]) / init8 (INT8 codes [B,H,P,N]): the state before the first chunk, or null for zero.
cudaError_t launch_state_passing_bf16(const Dims& d, const void* S, bool s_fp32, const float* decay,
                                      const float* init, uint16_t* Hc, float* final_state, float* amax_h,
                                      cudaStream_t st);
cudaError_t launch_state_passing_i8(const Dims& d, const int8_t* S8, const int32_t* dq, int shift,
                                    const int8_t* init8, int8_t* H8, int8_t* final_state, cudaStream_t st);

// a4-a7: ChunkBMM + ChunkScan2 (diagonal) + ChunkScan1 (off-diagonal) + D skip.
cudaError_t launch_chunk_scan_bf16(const Dims& d, const uint16_t* x, const float* dt,
                                   const float* Acs, const uint16_t* B, const uint16_t* C,
                                   const float* D, const uint16_t* Hc, uint16_t* y,
                                   cudaStream_t st);
cudaError_t launch_chunk_scan_i8(const Dims& d, const uint16_t* x, const float* dt,
                                 const float* Acs, const int8_t* Bq, const int8_t* Cq,
                                 const float* D, const I8Scales& sc, const int8_t* H8,
                                 uint16_t* y, const I8Debug* dbg, cudaStream_t st);

// 3D TMA tensor map over a [d2][d1][d0] tensor of bf16 (or int8 when is_i8) with the
// given byte strides of dims 1 and 2, a box of box1 x box0 elements, and a swizzle.
bool make_tmap_3d(CUtensorMap* m, bool is_i8, const void* base, unsigned long long d0, unsigned long long d1,
                  unsigned long long d2, unsigned long long stride1_bytes, unsigned long long stride2_bytes,
                  unsigned box0, unsigned box1, CUtensorMapSwizzle swizzle);

bool make_tmap_2d(CUtensorMap* m, bool is_i8, const void* base, unsigned long long d0, unsigned long long d1,
                  unsigned long long stride1_bytes, unsigned box0, unsigned box1, CUtensorMapSwizzle swizzle);

// Tensor-core ChunkBMM + ChunkScan2 + ChunkScan1 + D skip for P = 64, N = 128: one
// CTA per (chunk, batch row, block of up to `heads_per_cta` heads of one group).
// `Hc` is the state entering each chunk (bf16 or int8 [B,nc,H,P,N]); Acs and dtc
// are [B,H,nc,Q].
cudaError_t launch_chunk_scan_tc(const Dims& d, bool i8, const uint16_t* x, const void* Bmat,
                                 const void* Cmat, const float* Acs, const float* dtc, const float* D,
                                 const I8Scales& sc, const void* Hc, uint16_t* y, const I8Debug* dbg,
                                 int heads_per_cta, int* status, cudaStream_t st, const int8_t* cb8 = nullptr,
                                 const float* s_cb = nullptr, bool acs_half = false);

// ChunkBMM of the notes' storage variant (W8A8, chunk 256, N = 128): per (b, c, g) the
// INT32 CB tile, one fp64 step amax / 127, its INT8 codes to `cb8` [B,nc,G,Q,Q] and the
// step as fp32 to `s_cb` [B,nc,G].  chunk_bmm_i8_bytes: workspace bytes of both.
size_t chunk_bmm_i8_bytes(const Dims& d);
cudaError_t launch_chunk_bmm_i8(const Dims& d, const int8_t* Bq, const int8_t* Cq, int8_t* cb8, float* s_cb,
                                const I8Debug* dbg, int* status, cudaStream_t st);

// Tensor-core ChunkState for P = 64, N = 128: one CTA per (head, chunk, batch row)
// computes the chunk state transposed, S^T[n,p] = sum_j B[j,n] X_scaled[j,p], with
// tcgen05 (kind::f16, or kind::i8 on Xq and Bq).  `lut` is LUT_state [B,H,nc,Q].
// bf16 path: S written as bf16 (the passing accumulates in fp32).
// W8A8: `inv_sx` and `mq` are the per-(h,p) tables ChunkCumsum writes.
cudaError_t launch_chunk_state_tc(const Dims& d, bool i8, const uint16_t* x, const void* Bmat,
                                  const float* lut, const float* inv_sx, const float* mq, uint16_t* S, int8_t* S8,
                                  const I8Debug* dbg, int* status, cudaStream_t st);

// The whole W8A8 scan of one call (ChunkCumsum .. epilogue) as one persistent kernel
// for P = 64, N = 128 (fused_i8.cu).  Arguments of the kernel:
struct FusedI8Args {
    Dims d;
    int K;            // heads per work item
    int nhb_g;        // head blocks per group
    int nhb;          // head blocks per (batch row, chunk)
    int items;        // B * nc * nhb work items, chunk-major
    const float* dt;
    const float* A;
    const float* D;
    I8Scales sc;
    int* status;      // device status word (SSD_ERR_TIMEOUT on an expired wait)
    int* ticket;      // work-item counter, zero at launch
    int* hflag;       // [B, nc, H]: quarters of the state entering the chunk published (4 = ready)
    int8_t* Hpub;     // [B, nc, H, N, P] state entering each chunk (transposed)
    const float* inv_sx;  // [H*P] 1/s_x
    const float* mq;      // [H*P] s_x s_B / s_s (requantisation multiplier)
    const float* mulC;    // [H*P] s_C s_s (ChunkScan1 dequantisation)
    const int8_t* init8;
    int8_t* final8;
    I8Debug dbg;
};
// Workspace bytes of the fused W8A8 scan; *ctrl_bytes receives the size of the leading
// region (status word, ticket, flags) that is cleared before every launch.
size_t fused_i8_ws_bytes(const Dims& d, size_t* ctrl_bytes = nullptr);
int fused_heads_per_item(const Dims& d);
cudaError_t launch_fused_i8(const Dims& d, const uint16_t* x, const float* dt, const float* A, const int8_t* Bq,
                            const int8_t* Cq, const float* D, const I8Scales& sc, const int8_t* init8, uint16_t* y,
                            int8_t* final8, void* ws, const I8Debug* dbg, cudaStream_t st);

// Streaming multiprocessors of the current device (cached per device).
int device_sm_count();
// SSD_OK for cudaSuccess; otherwise SSD_ERR_CUDA, remembering `e` for ssd_last_cuda_error.
ssd_status from_cuda(cudaError_t e);

// Calibration helpers.
cudaError_t launch_amax_bc(const Dims& d, const uint16_t* B, const uint16_t* C, float* amax_B,
                           float* amax_C, cudaStream_t st);
cudaError_t launch_amax_to_scale(float* v, int n, cudaStream_t st);
cudaError_t launch_amax_pair_to_scale(const float* a1, const float* a2, float* out, int n,
                                      cudaStream_t st);

}  // namespace ssd
