// quantize.cu — a0 (per-group INT8 quantisation of B and C) and the calibration
// reductions.  HBM-bound elementwise work: 16-byte loads of 8 bf16 values, 8-byte
// stores of 8 int8 codes, grid sized to a multiple of the SM count.
#include "kernels.h"

namespace ssd {

namespace {

constexpr int kThreads = 256;
constexpr int kMaxGroups = 64;                     // groups whose 1/s a CTA keeps in shared memory

__global__ void __launch_bounds__(kThreads)
quantize_bc_kernel(const uint4* __restrict__ B, const uint4* __restrict__ C,
                   const float* __restrict__ s_B, const float* __restrict__ s_C,
                   uint2* __restrict__ Bq, uint2* __restrict__ Cq, long long nvec, int G, int N) {
    const uint4* src = blockIdx.y == 0 ? B : C;
    uint2* dst = blockIdx.y == 0 ? Bq : Cq;
    const float* s = blockIdx.y == 0 ? s_B : s_C;
    // IEEE 1/s per group, once per CTA
    __shared__ float inv_s[kMaxGroups];
    for (int g = threadIdx.x; g < G && g < kMaxGroups; g += kThreads) inv_s[g] = __frcp_rn(__ldg(s + g));
    __syncthreads();
    const int vec_per_group = N / 8;
    const long long stride = (long long)gridDim.x * kThreads;
    constexpr int kUnroll = 4;                           // loads in flight per thread
    const float2 lo = make_float2(-127.0f, -127.0f), hi = make_float2(127.0f, 127.0f);
    const float2 rnd = make_float2(12582912.0f, 12582912.0f);   // 1.5 * 2^23
    for (long long i0 = blockIdx.x * (long long)kThreads + threadIdx.x; i0 < nvec; i0 += kUnroll * stride) {
        uint4 vv[kUnroll];
#pragma unroll
        for (int r = 0; r < kUnroll; ++r) {
            const long long i = i0 + r * stride;
            vv[r] = i < nvec ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int r = 0; r < kUnroll; ++r) {
            const long long i = i0 + r * stride;
            if (i >= nvec) break;
            const int g = (int)((i / vec_per_group) % G);
            const float inv = g < kMaxGroups ? inv_s[g] : __frcp_rn(__ldg(s + g));
            const float2 inv2 = make_float2(inv, inv);
            const uint4 v = vv[r];
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            uint32_t b[8];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                // clamp(rint(x / s), +-127): the product rounded in fp32, clamped (the same code:
                // +-127 are integers), rounded to nearest even by adding 1.5 * 2^23, whose low
                // byte is then the code's byte
                float2 q = __fmul2_rn(make_float2(__uint_as_float(w[k] << 16), __uint_as_float(w[k] & 0xffff0000u)),
                                      inv2);
                q.x = fminf(fmaxf(q.x, lo.x), hi.x);
                q.y = fminf(fmaxf(q.y, lo.y), hi.y);
                q = __fadd2_rn(q, rnd);
                b[2 * k] = __float_as_uint(q.x);
                b[2 * k + 1] = __float_as_uint(q.y);
            }
            dst[i] = make_uint2(__byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410),
                                __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410));
        }
    }
}

// Running amax of |B| and |C| per group over the first L tokens of each row.
__global__ void __launch_bounds__(kThreads)
amax_bc_kernel(const uint16_t* __restrict__ B, const uint16_t* __restrict__ C, float* amax_B,
               float* amax_C, Dims d) {
    const uint16_t* src = blockIdx.y == 0 ? B : C;
    float* out = blockIdx.y == 0 ? amax_B : amax_C;
    const long long per_row = (long long)d.L * d.G * d.N;
    const long long total = per_row * d.B;
    __shared__ float red[64];
    for (int g = threadIdx.x; g < 64; g += kThreads) red[g] = 0.f;
    __syncthreads();
    for (long long i = blockIdx.x * (long long)kThreads + threadIdx.x; i < total;
         i += (long long)gridDim.x * kThreads) {
        const long long b = i / per_row, r = i % per_row;
        const int g = (int)((r / d.N) % d.G);
        const float v = fabsf(bf16_bits_to_float(src[b * d.Ls * d.G * d.N + r]));
        atomic_max_nonneg(g < 64 ? &red[g] : out + g, v);
    }
    __syncthreads();
    for (int g = threadIdx.x; g < d.G && g < 64; g += kThreads) atomic_max_nonneg(out + g, red[g]);
}

__global__ void amax_to_scale_kernel(float* v, int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) {
        const float a = v[i];
        v[i] = a > 0.f ? __fdiv_rn(a, 127.0f) : 1.0f;
    }
}

__global__ void amax_pair_to_scale_kernel(const float* a1, const float* a2, float* out, int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) {
        const float a = fmaxf(a1[i], a2[i]);
        out[i] = a > 0.f ? __fdiv_rn(a, 127.0f) : 1.0f;
    }
}

int grid_for(long long work, int per_block) {
    int sms = 148;
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    long long blocks = (work + per_block - 1) / per_block;
    long long cap = (long long)sms * 8;
    if (blocks > cap) blocks = cap;
    return (int)(blocks < 1 ? 1 : blocks);
}

}  // namespace

cudaError_t launch_quantize_bc(const Dims& d, const uint16_t* B, const uint16_t* C,
                               const float* s_B, const float* s_C, int8_t* Bq, int8_t* Cq,
                               cudaStream_t st) {
    const long long nvec = (long long)d.B * d.L * d.G * d.N / 8;
    if (nvec == 0) return cudaSuccess;
    dim3 grid(grid_for(nvec, kThreads), 2);
    quantize_bc_kernel<<<grid, kThreads, 0, st>>>(reinterpret_cast<const uint4*>(B),
                                                  reinterpret_cast<const uint4*>(C), s_B, s_C,
                                                  reinterpret_cast<uint2*>(Bq),
                                                  reinterpret_cast<uint2*>(Cq), nvec, d.G, d.N);
    return cudaGetLastError();
}

cudaError_t launch_amax_bc(const Dims& d, const uint16_t* B, const uint16_t* C, float* amax_B,
                           float* amax_C, cudaStream_t st) {
    const long long total = (long long)d.B * d.L * d.G * d.N;
    if (total == 0) return cudaSuccess;
    dim3 grid(grid_for(total, kThreads), 2);
    amax_bc_kernel<<<grid, kThreads, 0, st>>>(B, C, amax_B, amax_C, d);
    return cudaGetLastError();
}

cudaError_t launch_amax_to_scale(float* v, int n, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    amax_to_scale_kernel<<<(n + 255) / 256, 256, 0, st>>>(v, n);
    return cudaGetLastError();
}

cudaError_t launch_amax_pair_to_scale(const float* a1, const float* a2, float* out, int n,
                                      cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    amax_pair_to_scale_kernel<<<(n + 255) / 256, 256, 0, st>>>(a1, a2, out, n);
    return cudaGetLastError();
}

}  // namespace ssd
