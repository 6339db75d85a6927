// common.cuh — shared device helpers of the SSD scan kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace ssd {

// Problem dimensions as the kernels see them.  `Ls` is the row stride of the
// token axis in elements of B*L-indexed tensors (equal to L except for the
// calibration prefix, which runs on the first L tokens of rows of length Ls).
struct Dims {
    int B, L, H, P, G, N, Q, nc, hpg;
    long long Ls;
    __host__ __device__ long long Lp() const { return (long long)nc * Q; }
};

// Device status word values (first int32 of the workspace).
enum : int { kStatusOk = 0, kStatusTimeout = 5 };

// ---------------------------------------------------------------- bf16 helpers
__device__ __forceinline__ float bf16_bits_to_float(uint16_t v) {
    return __uint_as_float(((uint32_t)v) << 16);
}
__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// ---------------------------------------------------------------- specified fp32 exp
// exp(x) with a fixed sequence of individually rounded fp32 operations, so that the
// W8A8 path's integer codes (X_scaled quantisation, decay codes) are reproducible
// on any IEEE-754 machine.  Method: Cody-Waite range reduction x = k ln2 + r with
// ln2 split into an 11-bit high part (k*ln2_hi exact for |k| < 2^13) and the rest,
// then the degree-7 Taylor polynomial of exp(r) by Horner's rule, then scaling by
// 2^k.  x < -87 gives 0; x is clamped to at most 88; exp(0) = 1 exactly.
// No contraction into FMA: every step is an explicit _rn intrinsic.
__device__ __forceinline__ float ssd_expf(float x) {
    if (x < -87.0f) return 0.0f;
    x = fminf(x, 88.0f);
    const float kLog2e = 1.4426950408889634f;
    const float kLn2Hi = 1420.0f / 2048.0f;
    const float kLn2Lo = (float)(0.6931471805599453 - 1420.0 / 2048.0);
    const float k = rintf(__fmul_rn(x, kLog2e));
    const float r = __fsub_rn(__fsub_rn(x, __fmul_rn(k, kLn2Hi)), __fmul_rn(k, kLn2Lo));
    float p = (float)(1.0 / 5040.0);
    p = __fadd_rn(__fmul_rn(p, r), (float)(1.0 / 720.0));
    p = __fadd_rn(__fmul_rn(p, r), (float)(1.0 / 120.0));
    p = __fadd_rn(__fmul_rn(p, r), (float)(1.0 / 24.0));
    p = __fadd_rn(__fmul_rn(p, r), (float)(1.0 / 6.0));
    p = __fadd_rn(__fmul_rn(p, r), 0.5f);
    p = __fadd_rn(__fmul_rn(p, r), 1.0f);
    p = __fadd_rn(__fmul_rn(p, r), 1.0f);
    int ki = (int)k;
    ki = ki < -126 ? -126 : (ki > 127 ? 127 : ki);
    const float two_k = __int_as_float((ki + 127) << 23);
    return __fmul_rn(p, two_k);
}

// Symmetric INT8 code: clamp(rint(v * inv_scale), -127, 127), fp32 round-to-nearest-even.
__device__ __forceinline__ int quant_i8(float v, float inv_scale) {
    float q = rintf(__fmul_rn(v, inv_scale));
    q = fminf(fmaxf(q, -127.0f), 127.0f);
    return (int)q;
}

__device__ __forceinline__ int sat127(int v) { return v < -127 ? -127 : (v > 127 ? 127 : v); }

// Lane-wise unsigned min / max of two 16-bit fields per word.
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
__device__ __forceinline__ uint32_t min_u16x2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("min.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// One link of the integer StatePassing (eq. 6) on four codes per word, for decay shifts
// k <= 7 and decay codes dq <= 2^k: H' = sat127(S8 + ((dq H + 2^(k-1)) >> k)).  With
// Hu = H + 128 and Su = S8 + 128 (the codes with the top bit flipped),
// V = dq Hu + 2^(k-1) + 128 (2^k - dq) + Su 2^k = dq H + 2^(k-1) + (S8 + 256) 2^k lies in
// [0, 2^16), so two codes share a 32-bit word as 16-bit fields; V >> k = H' + 256 before
// saturation, so clamping V to [129 2^k, 384 2^k - 1] (lo, hi: both fields) saturates, and
// the low byte of each field of V >> k is H' as an int8 code (bits shifted down from the
// upper field land at bit 16 - k >= 9, above it).  k0 = 2^(k-1) + 128 (2^k - dq) in both
// fields.
__device__ __forceinline__ uint32_t chain_word(uint32_t h4, uint32_t s4, uint32_t dq, uint32_t k0, int k,
                                               uint32_t lo, uint32_t hi) {
    const uint32_t hu = h4 ^ 0x80808080u, su = s4 ^ 0x80808080u;
    uint32_t v0 = __byte_perm(hu, 0, 0x4140) * dq + k0 + (__byte_perm(su, 0, 0x4140) << k);
    uint32_t v1 = __byte_perm(hu, 0, 0x4342) * dq + k0 + (__byte_perm(su, 0, 0x4342) << k);
    v0 = min_u16x2(max_u16x2(v0, lo), hi) >> k;
    v1 = min_u16x2(max_u16x2(v1, lo), hi) >> k;
    return __byte_perm(v0, v1, 0x6420);
}
// atomicMax on non-negative floats through their (monotone) bit patterns.
__device__ __forceinline__ void atomic_max_nonneg(float* addr, float v) {
    atomicMax(reinterpret_cast<unsigned int*>(addr), __float_as_uint(v));
}

}  // namespace ssd
