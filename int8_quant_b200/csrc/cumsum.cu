// cumsum.cu — a1, ChunkCumsum: Acs[b,h,c,j] = sum_{i<=j} dt[b,cQ+i,h] * A[h] within each
// chunk, plus the chunk decay exp(Acs[Q-1]) (bf16 path) or its fixed-point code
// rint(exp(Acs[Q-1]) * 2^k) (W8A8 path, eq. 6 of the SSDi8 notes).  Optionally also
// LUT_state[b,h,c,j] = dt_j * exp(Acs[Q-1] - Acs[j]) (eq. 4; the W8A8 path uses the
// specified fp32 exp so that X_scaled's codes are reproducible) and dt in the same
// chunk-major layout, so that the tensor-core kernels read both contiguously.
//
// One CTA per (chunk, block of 32 heads, batch row).  dt rows of the chunk are
// staged in shared memory with coalesced 128-byte row reads (32 heads x fp32),
// then each warp scans one head: lane l owns the Q/32 consecutive elements
// [l*m, (l+1)*m), sums them sequentially, combines the lane totals with a
// Kogge-Stone shuffle scan and adds the exclusive lane prefix.  Every add and
// multiply is an explicit round-to-nearest fp32 operation in this fixed order, so
// the result (and the W8A8 codes derived from it) is reproducible bit for bit.
#include "kernels.h"

namespace ssd {

namespace {

constexpr int kThreads = 256;
constexpr int kHeadsPerCta = 32;

template <bool kI8>
__global__ void __launch_bounds__(kThreads)
cumsum_kernel(Dims d, const float* __restrict__ dt, const float* __restrict__ A,
              float* __restrict__ Acs, float* __restrict__ decay, int32_t* __restrict__ dq,
              int shift, int* __restrict__ status, float* __restrict__ lut, float* __restrict__ dtc) {
    // this call's kernels record device-side errors in the workspace status word
    if (status && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0) *status = kStatusOk;
    extern __shared__ float tile[];                 // [Q][kHeadsPerCta + 1]
    const int c = blockIdx.x, h0 = blockIdx.y * kHeadsPerCta, b = blockIdx.z;
    const int Q = d.Q, ld = kHeadsPerCta + 1;
    for (int idx = threadIdx.x; idx < Q * kHeadsPerCta; idx += kThreads) {
        const int j = idx / kHeadsPerCta, k = idx % kHeadsPerCta;
        const long long t = (long long)c * Q + j;
        const int h = h0 + k;
        float v = 0.f;
        if (t < d.L && h < d.H) v = __ldg(dt + ((long long)b * d.Ls + t) * d.H + h);
        tile[j * ld + k] = v;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m = Q >> 5;                           // 2, 4 or 8
    for (int k = warp; k < kHeadsPerCta && h0 + k < d.H; k += kThreads / 32) {
        const int h = h0 + k;
        const float ah = __ldg(A + h);
        float s[8];
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (i < m) {
                const float a = __fmul_rn(tile[(lane * m + i) * ld + k], ah);
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
        const long long row = (((long long)b * d.H + h) * d.nc + c) * Q + lane * m;
        float* out = Acs + row;
        float acs[8];
        float last = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (i < m) {
                const float r = __fadd_rn(e, s[i]);
                out[i] = r;
                acs[i] = r;
                last = r;
            }
        }
        last = __shfl_sync(0xffffffffu, last, 31);          // Acs[Q-1]
        if (lut) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (i < m) {
                    const float dtv = tile[(lane * m + i) * ld + k];
                    lut[row + i] = kI8 ? __fmul_rn(dtv, ssd_expf(__fsub_rn(last, acs[i])))
                                       : dtv * expf(last - acs[i]);
                    if (dtc) dtc[row + i] = dtv;
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
}

}  // namespace

cudaError_t launch_cumsum(const Dims& d, const float* dt, const float* A, float* Acs,
                          float* decay, int32_t* dq, int shift, int* status, float* lut, float* dtc,
                          cudaStream_t st) {
    if (d.B == 0 || d.nc == 0) return cudaSuccess;
    dim3 grid(d.nc, (d.H + kHeadsPerCta - 1) / kHeadsPerCta, d.B);
    const size_t smem = (size_t)d.Q * (kHeadsPerCta + 1) * sizeof(float);
    if (dq) {
        cudaFuncSetAttribute(cumsum_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        cumsum_kernel<true><<<grid, kThreads, smem, st>>>(d, dt, A, Acs, decay, dq, shift, status, lut, dtc);
    } else {
        cudaFuncSetAttribute(cumsum_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        cumsum_kernel<false><<<grid, kThreads, smem, st>>>(d, dt, A, Acs, decay, dq, shift, status, lut, dtc);
    }
    return cudaGetLastError();
}

}  // namespace ssd
