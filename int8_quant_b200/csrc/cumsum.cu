// cumsum.cu — a1, ChunkCumsum: Acs[b,h,c,j] = sum_{i<=j} dt[b,cQ+i,h] * A[h] within each
// chunk, plus the chunk decay exp(Acs[Q-1]) (bf16 path) or its fixed-point code
// rint(exp(Acs[Q-1]) * 2^k) (W8A8 path, eq. 6 of the SSDi8 notes).  Optionally also
// LUT_state[b,h,c,j] = dt_j * exp(Acs[Q-1] - Acs[j]) (eq. 4; the W8A8 path uses the
// specified fp32 exp so that X_scaled's codes are reproducible) and dt in the same
// chunk-major layout, so that the tensor-core kernels read both contiguously.
// With `acs_half` (the notes' storage variant: dAcs kept in FP16) every Acs is rounded
// to IEEE half (nearest even) as soon as it is formed, LUT_state and the decay code are
// computed from the rounded values, and Acs is stored as half.
//
// One CTA per (chunk, block of 8 heads, batch row); warp k scans head h0 + k.  The
// dt rows of the chunk are staged in shared memory (32-byte row segments, 8 heads x
// fp32), transposed to one padded row per head.  In the scan, lane l owns the Q/32
// consecutive elements [l*m, (l+1)*m), sums them sequentially, combines the lane
// totals with a Kogge-Stone shuffle scan and adds the exclusive lane prefix.  Every
// add and multiply is an explicit round-to-nearest fp32 operation in this fixed
// order, so the result (and the W8A8 codes derived from it) is reproducible bit for
// bit.  The results go back through shared memory so that every global store of a
// warp covers 128 contiguous bytes.
#include <cuda_fp16.h>

#include "kernels.h"

namespace ssd {

namespace {

constexpr int kThreads = 256;
constexpr int kHeadsPerCta = kThreads / 32;

// padded position of element j in a per-head row: lane-strided (j = l*m + i) and
// contiguous (j = l + 32 i) accesses are both free of bank conflicts
__device__ __forceinline__ int pad(int j) { return j + (j >> 5); }

template <bool kI8>
__global__ void __launch_bounds__(kThreads)
cumsum_kernel(Dims d, const float* __restrict__ dt, const float* __restrict__ A,
              float* __restrict__ Acs, float* __restrict__ decay, int32_t* __restrict__ dq,
              int shift, int* __restrict__ status, float* __restrict__ lut, float* __restrict__ dtc,
              I8Scales sc, float* __restrict__ inv_sx, float* __restrict__ mq, int acs_half) {
    // this call's kernels record device-side errors in the workspace status word
    if (status && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0) *status = kStatusOk;
    // W8A8: per-(h,p) quantisation reciprocal 1/s_x and requantisation multiplier
    // s_x s_B / s_s of this block of heads, for ChunkState
    if (kI8 && inv_sx && blockIdx.x == 0 && blockIdx.z == 0) {
        for (int idx = threadIdx.x; idx < kHeadsPerCta * d.P; idx += kThreads) {
            const int h = blockIdx.y * kHeadsPerCta + idx / d.P;
            if (h < d.H) {
                const int o = h * d.P + idx % d.P;
                const float sx = __ldg(sc.s_x + o);
                inv_sx[o] = __frcp_rn(sx);
                mq[o] = __fdiv_rn(__fmul_rn(sx, __ldg(sc.s_B + h / d.hpg)), __ldg(sc.s_s + o));
            }
        }
    }
    extern __shared__ float smem[];
    const int Q = d.Q, ld = pad(Q);
    float* tile = smem;                             // [kHeadsPerCta][ld]  dt
    float* part = smem + kHeadsPerCta * ld;         // [kHeadsPerCta][ld]  Acs
    const int c = blockIdx.x, h0 = blockIdx.y * kHeadsPerCta, b = blockIdx.z;
    // all of this thread's loads first (Q * 8 / 256 <= 8), then the shared-memory stores
    constexpr int kLoads = 256 * kHeadsPerCta / kThreads;      // enough for Q = 256
    float vals[kLoads];
#pragma unroll
    for (int r = 0; r < kLoads; ++r) {
        const int idx = threadIdx.x + r * kThreads;
        const int j = idx / kHeadsPerCta, k = idx % kHeadsPerCta;
        const long long t = (long long)c * Q + j;
        const int h = h0 + k;
        vals[r] = (j < Q && t < d.L && h < d.H) ? __ldg(dt + ((long long)b * d.Ls + t) * d.H + h) : 0.f;
    }
#pragma unroll
    for (int r = 0; r < kLoads; ++r) {
        const int idx = threadIdx.x + r * kThreads;
        const int j = idx / kHeadsPerCta, k = idx % kHeadsPerCta;
        if (j < Q) tile[k * ld + pad(j)] = vals[r];
    }
    __syncthreads();
    const int k = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = h0 + k;
    if (h >= d.H) return;
    const float* dtk = tile + k * ld;
    float* acsk = part + k * ld;
    const int m = Q >> 5;                           // 2, 4 or 8
    const float ah = __ldg(A + h);
    float s[8];
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        if (i < m) {
            const float a = __fmul_rn(dtk[pad(lane * m + i)], ah);
            acc = (i == 0) ? a : __fadd_rn(acc, a);
            s[i] = acc;
        }
    }
    float v = acc;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v = __fadd_rn(u, v);
    }
    float e = __shfl_up_sync(0xffffffffu, v, 1);
    if (lane == 0) e = 0.f;
    float last = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        if (i < m) {
            last = __fadd_rn(e, s[i]);
            if (acs_half) last = __half2float(__float2half_rn(last));
            acsk[pad(lane * m + i)] = last;
        }
    }
    last = __shfl_sync(0xffffffffu, last, 31);          // Acs[Q-1]
    __syncwarp();
    const long long row = (((long long)b * d.H + h) * d.nc + c) * Q;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        if (i < m) {
            const int j = lane + 32 * i;
            const float a = acsk[pad(j)];
            if (acs_half) reinterpret_cast<__half*>(Acs)[row + j] = __float2half_rn(a);
            else Acs[row + j] = a;
            if (lut) {
                const float dtv = dtk[pad(j)];
                lut[row + j] = kI8 ? __fmul_rn(dtv, ssd_expf(__fsub_rn(last, a))) : dtv * expf(last - a);
                if (dtc) dtc[row + j] = dtv;
            }
        }
    }
    if (lane == 31) {
        const long long o = ((long long)b * d.H + h) * d.nc + c;
        if (kI8) {
            dq[o] = (int32_t)rintf(__fmul_rn(ssd_expf(last), (float)(1 << shift)));
        } else {
            decay[o] = expf(last);
        }
    }
}

// Half-precision values as fp32 (debug copies of a half Acs).
__global__ void half_to_float_kernel(const __half* __restrict__ src, float* __restrict__ dst, long long n) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        dst[i] = __half2float(src[i]);
}

}  // namespace

cudaError_t launch_half_to_float(const void* src, float* dst, long long n, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    const long long blocks = (n + 255) / 256;
    half_to_float_kernel<<<(unsigned)(blocks < 4096 ? blocks : 4096), 256, 0, st>>>(static_cast<const __half*>(src),
                                                                                   dst, n);
    return cudaGetLastError();
}

cudaError_t launch_cumsum(const Dims& d, const float* dt, const float* A, float* Acs,
                          float* decay, int32_t* dq, int shift, int* status, float* lut, float* dtc,
                          cudaStream_t st, const I8Scales* sc, float* inv_sx, float* mq, bool acs_half) {
    if (d.B == 0 || d.nc == 0) return cudaSuccess;
    dim3 grid(d.nc, (d.H + kHeadsPerCta - 1) / kHeadsPerCta, d.B);
    const size_t smem = (size_t)2 * kHeadsPerCta * (d.Q + d.Q / 32) * sizeof(float);
    if (dq) {
        cudaFuncSetAttribute(cumsum_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        cumsum_kernel<true><<<grid, kThreads, smem, st>>>(d, dt, A, Acs, decay, dq, shift, status, lut, dtc,
                                                          sc ? *sc : I8Scales{}, sc ? inv_sx : nullptr, mq,
                                                          acs_half ? 1 : 0);
    } else {
        cudaFuncSetAttribute(cumsum_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        cumsum_kernel<false><<<grid, kThreads, smem, st>>>(d, dt, A, Acs, decay, dq, shift, status, lut, dtc,
                                                           I8Scales{}, nullptr, nullptr, 0);
    }
    return cudaGetLastError();
}

}  // namespace ssd
