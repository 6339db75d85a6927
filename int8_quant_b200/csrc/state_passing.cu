// state_passing.cu — a3, StatePassing (SSDi8 notes, eq. 6), sequential over chunks.
//   bf16 : H_{c+1} = exp(Acs_c[Q-1]) * H_c + S_c  (fp32; S_c stored as bf16)
//   W8A8 : H_{c+1} = sat127(S8_c + ((dq_c * H_c + 2^(k-1)) >> k))       (int32, then INT8)
// H_0 is the caller's initial state (fp32, or INT8 codes in the s_s scales), or zero.
// Every (p,n) element of a (b,h) state is an independent scalar recurrence, so one
// thread owns 4 (bf16 path) or 16 (W8A8) consecutive elements and walks the chunks; consecutive threads own
// consecutive elements (coalesced vector loads and stores).  Loads of the next
// kAhead chunks' S are issued ahead of the dependent updates.
#include "kernels.h"

namespace ssd {

namespace {

constexpr int kThreads = 256;
constexpr int kVec = 4;                                  // elements per thread (P*N % 4 == 0)
constexpr int kAhead = 8;

struct F4 {
    float v[4];
};
__device__ __forceinline__ F4 load4(const float* p) {
    const float4 t = __ldg(reinterpret_cast<const float4*>(p));
    return F4{{t.x, t.y, t.z, t.w}};
}
__device__ __forceinline__ F4 load4(const uint16_t* p) {
    const uint2 t = __ldg(reinterpret_cast<const uint2*>(p));
    return F4{{__uint_as_float(t.x << 16), __uint_as_float(t.x & 0xffff0000u), __uint_as_float(t.y << 16),
               __uint_as_float(t.y & 0xffff0000u)}};
}

// TS: element type of the chunk states (bf16 bits from the scan, fp32 for calibration).
template <typename TS>
__global__ void __launch_bounds__(kThreads)
state_passing_bf16_kernel(Dims d, const TS* __restrict__ S, const float* __restrict__ decay,
                          const float* __restrict__ init, uint16_t* __restrict__ Hc, float* __restrict__ final_state,
                          float* amax_h) {
    const int PN = d.P * d.N;
    const int e = (blockIdx.x * kThreads + threadIdx.x) * kVec;
    const int h = blockIdx.y, b = blockIdx.z;
    if (e >= PN) return;
    const long long stride = (long long)d.H * PN;                 // between chunks
    const TS* s = S + ((long long)b * d.nc * d.H + h) * PN + e;
    uint16_t* hc = Hc ? Hc + ((long long)b * d.nc * d.H + h) * PN + e : nullptr;
    const float* dec = decay + ((long long)b * d.H + h) * d.nc;
    float hv[kVec] = {0.f, 0.f, 0.f, 0.f};
    if (init) {
        const F4 h0 = load4(init + ((long long)b * d.H + h) * PN + e);
#pragma unroll
        for (int v = 0; v < kVec; ++v) hv[v] = h0.v[v];
    }
    float amax = 0.f;
    for (int c0 = 0; c0 < d.nc; c0 += kAhead) {
        F4 sv[kAhead];
        float dv[kAhead];
#pragma unroll
        for (int i = 0; i < kAhead; ++i) {
            const int c = c0 + i;
            sv[i] = c < d.nc ? load4(s + c * stride) : F4{{0.f, 0.f, 0.f, 0.f}};
            dv[i] = c < d.nc ? __ldg(dec + c) : 0.f;
        }
#pragma unroll
        for (int i = 0; i < kAhead; ++i) {
            const int c = c0 + i;
            if (c < d.nc) {
                if (hc)
                    *reinterpret_cast<uint2*>(hc + c * stride) =
                        make_uint2((uint32_t)float_to_bf16_bits(hv[0]) | ((uint32_t)float_to_bf16_bits(hv[1]) << 16),
                                   (uint32_t)float_to_bf16_bits(hv[2]) | ((uint32_t)float_to_bf16_bits(hv[3]) << 16));
#pragma unroll
                for (int v = 0; v < kVec; ++v) {
                    hv[v] = fmaf(dv[i], hv[v], sv[i].v[v]);
                    amax = fmaxf(amax, fabsf(hv[v]));
                }
            }
        }
    }
    *reinterpret_cast<float4*>(final_state + ((long long)b * d.H + h) * PN + e) = make_float4(hv[0], hv[1], hv[2], hv[3]);
    if (amax_h) atomic_max_nonneg(amax_h + h * d.P + e / d.N, amax);  // the 4 elements share p
}

constexpr int kVecI8 = 16;                               // INT8 elements per thread: one 16-byte load

__global__ void __launch_bounds__(kThreads)
state_passing_i8_kernel(Dims d, const int8_t* __restrict__ S8, const int32_t* __restrict__ dq,
                        int shift, const int8_t* __restrict__ init8, int8_t* __restrict__ H8,
                        int8_t* __restrict__ final_state) {
    const int PN = d.P * d.N;
    const int e = (blockIdx.x * kThreads + threadIdx.x) * kVecI8;
    const int h = blockIdx.y, b = blockIdx.z;
    if (e >= PN) return;
    const long long stride = (long long)d.H * PN;
    const int8_t* s = S8 + ((long long)b * d.nc * d.H + h) * PN + e;
    int8_t* hc = H8 + ((long long)b * d.nc * d.H + h) * PN + e;
    const int32_t* q = dq + ((long long)b * d.H + h) * d.nc;
    // the state: 16 codes, four to a word (first code in the lowest byte)
    uint4 hw = init8 ? __ldg(reinterpret_cast<const uint4*>(init8 + ((long long)b * d.H + h) * PN + e))
                     : make_uint4(0, 0, 0, 0);
    const uint32_t lo = (129u << shift) * 0x10001u, hi = ((384u << shift) - 1u) * 0x10001u;
    constexpr int kAheadI8 = 4;
    for (int c0 = 0; c0 < d.nc; c0 += kAheadI8) {
        uint4 sv[kAheadI8];
        int qv[kAheadI8];
#pragma unroll
        for (int i = 0; i < kAheadI8; ++i) {
            const int c = c0 + i;
            sv[i] = c < d.nc ? __ldg(reinterpret_cast<const uint4*>(s + c * stride)) : make_uint4(0, 0, 0, 0);
            qv[i] = c < d.nc ? __ldg(q + c) : 0;
        }
#pragma unroll
        for (int i = 0; i < kAheadI8; ++i) {
            const int c = c0 + i;
            if (c < d.nc) {
                *reinterpret_cast<uint4*>(hc + c * stride) = hw;        // the state entering chunk c
                const uint32_t hv[4] = {hw.x, hw.y, hw.z, hw.w}, sw[4] = {sv[i].x, sv[i].y, sv[i].z, sv[i].w};
                uint32_t out[4];
                if (shift <= 7 && qv[i] <= (1 << shift)) {
                    // two codes per 16-bit field pair (decay codes are at most 2^k when A dt <= 0)
                    const uint32_t k0 = (uint32_t)((1 << (shift - 1)) + 128 * ((1 << shift) - qv[i])) * 0x10001u;
#pragma unroll
                    for (int j = 0; j < 4; ++j) out[j] = chain_word(hv[j], sw[j], (uint32_t)qv[i], k0, shift, lo, hi);
                } else {
                    const int half = 1 << (shift - 1);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        out[j] = 0u;
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            const int hs = (int)(int8_t)(hv[j] >> (8 * v)), sc = (int)(int8_t)(sw[j] >> (8 * v));
                            out[j] |= ((uint32_t)sat127(sc + ((qv[i] * hs + half) >> shift)) & 0xffu) << (8 * v);
                        }
                    }
                }
                hw = make_uint4(out[0], out[1], out[2], out[3]);
            }
        }
    }
    *reinterpret_cast<uint4*>(final_state + ((long long)b * d.H + h) * PN + e) = hw;
}

}  // namespace

cudaError_t launch_state_passing_bf16(const Dims& d, const void* S, bool s_fp32, const float* decay,
                                      const float* init, uint16_t* Hc, float* final_state, float* amax_h,
                                      cudaStream_t st) {
    if (d.B == 0) return cudaSuccess;
    if ((d.P * d.N) % kVec != 0 || d.N % kVec != 0) return cudaErrorInvalidValue;
    dim3 grid((d.P * d.N / kVec + kThreads - 1) / kThreads, d.H, d.B);
    if (s_fp32)
        state_passing_bf16_kernel<float><<<grid, kThreads, 0, st>>>(d, static_cast<const float*>(S), decay, init,
                                                                     Hc, final_state, amax_h);
    else
        state_passing_bf16_kernel<uint16_t><<<grid, kThreads, 0, st>>>(d, static_cast<const uint16_t*>(S), decay,
                                                                        init, Hc, final_state, amax_h);
    return cudaGetLastError();
}

cudaError_t launch_state_passing_i8(const Dims& d, const int8_t* S8, const int32_t* dq, int shift,
                                    const int8_t* init8, int8_t* H8, int8_t* final_state, cudaStream_t st) {
    if (d.B == 0) return cudaSuccess;
    if ((d.P * d.N) % kVecI8 != 0) return cudaErrorInvalidValue;
    dim3 grid((d.P * d.N / kVecI8 + kThreads - 1) / kThreads, d.H, d.B);
    state_passing_i8_kernel<<<grid, kThreads, 0, st>>>(d, S8, dq, shift, init8, H8, final_state);
    return cudaGetLastError();
}

}  // namespace ssd
