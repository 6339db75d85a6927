// state_passing.cu — a3, StatePassing (SSDi8 notes, eq. 6), sequential over chunks.
//   bf16 : H_0 = 0, H_{c+1} = exp(Acs_c[Q-1]) * H_c + S_c  (fp32; S_c stored as bf16)
//   W8A8 : H_{c+1} = sat127(S8_c + ((dq_c * H_c + 2^(k-1)) >> k))       (int32, then INT8)
// Every (p,n) element of a (b,h) state is an independent scalar recurrence, so one
// thread owns one element and walks the chunks; consecutive threads own consecutive
// elements (coalesced loads and stores).  Loads of the next chunks' S are issued
// ahead of the dependent update.
#include "kernels.h"

namespace ssd {

namespace {

constexpr int kThreads = 256;
constexpr int kAhead = 4;

__device__ __forceinline__ float load_state(const float* p) { return __ldg(p); }
__device__ __forceinline__ float load_state(const uint16_t* p) { return bf16_bits_to_float(__ldg(p)); }

// TS: element type of the chunk states (bf16 bits from the scan, fp32 for calibration).
template <typename TS>
__global__ void __launch_bounds__(kThreads)
state_passing_bf16_kernel(Dims d, const TS* __restrict__ S, const float* __restrict__ decay,
                          uint16_t* __restrict__ Hc, float* __restrict__ final_state, float* amax_h) {
    const int PN = d.P * d.N;
    const int e = blockIdx.x * kThreads + threadIdx.x;
    const int h = blockIdx.y, b = blockIdx.z;
    if (e >= PN) return;
    const long long stride = (long long)d.H * PN;                 // between chunks
    const TS* s = S + ((long long)b * d.nc * d.H + h) * PN + e;
    uint16_t* hc = Hc ? Hc + ((long long)b * d.nc * d.H + h) * PN + e : nullptr;
    const float* dec = decay + ((long long)b * d.H + h) * d.nc;
    float hv = 0.f, amax = 0.f;
    for (int c0 = 0; c0 < d.nc; c0 += kAhead) {
        float sv[kAhead], dv[kAhead];
#pragma unroll
        for (int i = 0; i < kAhead; ++i) {
            const int c = c0 + i;
            sv[i] = c < d.nc ? load_state(s + c * stride) : 0.f;
            dv[i] = c < d.nc ? __ldg(dec + c) : 0.f;
        }
#pragma unroll
        for (int i = 0; i < kAhead; ++i) {
            const int c = c0 + i;
            if (c < d.nc) {
                if (hc) hc[c * stride] = float_to_bf16_bits(hv);
                hv = fmaf(dv[i], hv, sv[i]);
                amax = fmaxf(amax, fabsf(hv));
            }
        }
    }
    final_state[((long long)b * d.H + h) * PN + e] = hv;
    if (amax_h) atomic_max_nonneg(amax_h + h * d.P + e / d.N, amax);
}

__global__ void __launch_bounds__(kThreads)
state_passing_i8_kernel(Dims d, const int8_t* __restrict__ S8, const int32_t* __restrict__ dq,
                        int shift, int8_t* __restrict__ H8, int8_t* __restrict__ final_state) {
    const int PN = d.P * d.N;
    const int e = blockIdx.x * kThreads + threadIdx.x;
    const int h = blockIdx.y, b = blockIdx.z;
    if (e >= PN) return;
    const long long stride = (long long)d.H * PN;
    const int8_t* s = S8 + ((long long)b * d.nc * d.H + h) * PN + e;
    int8_t* hc = H8 + ((long long)b * d.nc * d.H + h) * PN + e;
    const int32_t* q = dq + ((long long)b * d.H + h) * d.nc;
    const int half = 1 << (shift - 1);
    int hv = 0;
    for (int c0 = 0; c0 < d.nc; c0 += kAhead) {
        int sv[kAhead], qv[kAhead];
#pragma unroll
        for (int i = 0; i < kAhead; ++i) {
            const int c = c0 + i;
            sv[i] = c < d.nc ? (int)s[c * stride] : 0;
            qv[i] = c < d.nc ? __ldg(q + c) : 0;
        }
#pragma unroll
        for (int i = 0; i < kAhead; ++i) {
            const int c = c0 + i;
            if (c < d.nc) {
                hc[c * stride] = (int8_t)hv;
                hv = sat127(sv[i] + ((qv[i] * hv + half) >> shift));
            }
        }
    }
    final_state[((long long)b * d.H + h) * PN + e] = (int8_t)hv;
}

}  // namespace

cudaError_t launch_state_passing_bf16(const Dims& d, const void* S, bool s_fp32, const float* decay,
                                      uint16_t* Hc, float* final_state, float* amax_h,
                                      cudaStream_t st) {
    if (d.B == 0) return cudaSuccess;
    dim3 grid((d.P * d.N + kThreads - 1) / kThreads, d.H, d.B);
    if (s_fp32)
        state_passing_bf16_kernel<float><<<grid, kThreads, 0, st>>>(d, static_cast<const float*>(S), decay, Hc,
                                                                     final_state, amax_h);
    else
        state_passing_bf16_kernel<uint16_t><<<grid, kThreads, 0, st>>>(d, static_cast<const uint16_t*>(S), decay,
                                                                        Hc, final_state, amax_h);
    return cudaGetLastError();
}

cudaError_t launch_state_passing_i8(const Dims& d, const int8_t* S8, const int32_t* dq, int shift,
                                    int8_t* H8, int8_t* final_state, cudaStream_t st) {
    if (d.B == 0) return cudaSuccess;
    dim3 grid((d.P * d.N + kThreads - 1) / kThreads, d.H, d.B);
    state_passing_i8_kernel<<<grid, kThreads, 0, st>>>(d, S8, dq, shift, H8, final_state);
    return cudaGetLastError();
}

}  // namespace ssd
