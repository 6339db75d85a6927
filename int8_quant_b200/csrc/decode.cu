// decode.cu — one token of the scan on the persistent state, the step on either side
// of the chunked scan when serving (the recurrence the SSD factorises, one token at a
// time):
//   h <- exp(dt*A) * h + dt * x B^T        y = C . h + D * x
// bf16 path: fp32 state.  W8A8 path: the INT8 state of the scan (real value code *
// s_s[h,p]) updated by the scan's own integer steps with a chunk of one token ("SSDi8"
// notes, key designs 1-2 and eq. 6): the chunk's cumulative sum is a = dt*A, the state
// LUT is dt * exp(a - a) = dt, X_scaled = dt * x is quantised per (h,p), the INT32
// product Xq * Bq is requantised to INT8 with s_x*s_B/s_s, and the state carried over
// the token is (dq * H + 2^(k-1)) >> k with dq = rint(exp(a) * 2^k); y is ChunkScan1
// (Cq . H on the state before the token, times s_C*s_s*exp(a)) plus ChunkScan2 (the
// single CB = Cq . Bq, times s_C*s_B*dt, as a bf16 factor of x) plus D*x.
//
// Both are one pass over the state (read and write once): one (b,h,p) row of N
// elements per N/4 lanes, four consecutive elements per lane (a 16-byte fp32 or
// 4-byte INT8 access), the row's C . h reduced by shuffles.
#include "kernels.h"

namespace ssd {

namespace {

constexpr int kThreads = 256;

struct RowIdx {
    long long r;   // (b*H + h)*P + p
    int b, h, p, g;
};

__device__ __forceinline__ RowIdx row_of(const Dims& d, long long row) {
    RowIdx i;
    i.r = row;
    i.p = (int)(row % d.P);
    const long long bh = row / d.P;
    i.h = (int)(bh % d.H);
    i.b = (int)(bh / d.H);
    i.g = i.h / d.hpg;
    return i;
}

template <int LPR, typename T>
__device__ __forceinline__ T row_sum(T v) {
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

template <int N>
__global__ void __launch_bounds__(kThreads)
decode_bf16_kernel(Dims d, const uint16_t* __restrict__ x, const float* __restrict__ dt, const float* __restrict__ A,
                   const uint16_t* __restrict__ Bm, const uint16_t* __restrict__ Cm, const float* __restrict__ D,
                   float* __restrict__ state, uint16_t* __restrict__ y) {
    constexpr int LPR = N / 4;                                   // lanes per state row
    const long long rows = (long long)d.B * d.H * d.P;
    const long long row = ((long long)blockIdx.x * kThreads + threadIdx.x) / LPR;
    const int sub = threadIdx.x % LPR, n0 = 4 * sub;
    const bool active = row < rows;                               // whole lane groups, shuffles stay full-warp
    const RowIdx i = row_of(d, active ? row : 0);
    float part = 0.f, xv = 0.f;
    if (active) {
        const long long bh = (long long)i.b * d.H + i.h;
        const float dtv = __ldg(dt + bh);
        const float dA = expf(dtv * __ldg(A + i.h));
        xv = bf16_bits_to_float(x[i.r]);
        const float u = dtv * xv;
        const uint2 bw = __ldg(reinterpret_cast<const uint2*>(Bm + ((long long)i.b * d.G + i.g) * N + n0));
        const uint2 cw = __ldg(reinterpret_cast<const uint2*>(Cm + ((long long)i.b * d.G + i.g) * N + n0));
        const float bv[4] = {__uint_as_float(bw.x << 16), __uint_as_float(bw.x & 0xffff0000u),
                             __uint_as_float(bw.y << 16), __uint_as_float(bw.y & 0xffff0000u)};
        const float cv[4] = {__uint_as_float(cw.x << 16), __uint_as_float(cw.x & 0xffff0000u),
                             __uint_as_float(cw.y << 16), __uint_as_float(cw.y & 0xffff0000u)};
        float4* sp = reinterpret_cast<float4*>(state + i.r * N + n0);
        const float4 h4 = *sp;
        float hv[4] = {h4.x, h4.y, h4.z, h4.w};
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            hv[v] = fmaf(dA, hv[v], u * bv[v]);
            part = fmaf(cv[v], hv[v], part);
        }
        *sp = make_float4(hv[0], hv[1], hv[2], hv[3]);
    }
    part = row_sum<LPR>(part);
    if (active && sub == 0) y[i.r] = float_to_bf16_bits(fmaf(__ldg(D + i.h), xv, part));
}

template <int N>
__global__ void __launch_bounds__(kThreads)
decode_i8_kernel(Dims d, const uint16_t* __restrict__ x, const float* __restrict__ dt, const float* __restrict__ A,
                 const int8_t* __restrict__ Bq, const int8_t* __restrict__ Cq, const float* __restrict__ D,
                 I8Scales sc, int8_t* __restrict__ state, uint16_t* __restrict__ y) {
    constexpr int LPR = N / 4;
    const long long rows = (long long)d.B * d.H * d.P;
    const long long row = ((long long)blockIdx.x * kThreads + threadIdx.x) / LPR;
    const int sub = threadIdx.x % LPR, n0 = 4 * sub;
    const bool active = row < rows;
    const RowIdx i = row_of(d, active ? row : 0);
    int acc1 = 0, cb = 0;
    float xv = 0.f, a = 0.f, dtv = 0.f;
    if (active) {
        const long long bh = (long long)i.b * d.H + i.h;
        const int hp = i.h * d.P + i.p;
        dtv = __ldg(dt + bh);
        a = __fmul_rn(dtv, __ldg(A + i.h));                        // ChunkCumsum of the one-token chunk
        xv = bf16_bits_to_float(x[i.r]);
        // ChunkState: X_scaled = LUT_state * x with LUT_state = dt * exp(a - a), its code
        const float lut = __fmul_rn(dtv, ssd_expf(__fsub_rn(a, a)));
        const float sx = __ldg(sc.s_x + hp);
        const int xq = quant_i8(__fmul_rn(lut, xv), __frcp_rn(sx));
        const float M = __fdiv_rn(__fmul_rn(sx, __ldg(sc.s_B + i.g)), __ldg(sc.s_s + hp));
        // StatePassing: the decay code and the rounding shift
        const int dq = (int)rintf(__fmul_rn(ssd_expf(a), (float)(1 << sc.shift)));
        const int half = 1 << (sc.shift - 1);
        const long long gn = ((long long)i.b * d.G + i.g) * N + n0;
        const uint32_t bw = __ldg(reinterpret_cast<const uint32_t*>(Bq + gn));
        const uint32_t cw = __ldg(reinterpret_cast<const uint32_t*>(Cq + gn));
        uint32_t* sp = reinterpret_cast<uint32_t*>(state + i.r * N + n0);
        const uint32_t hw = *sp;
        uint32_t out = 0;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int hs = (int)(int8_t)(hw >> (8 * v));
            const int bq = (int)(int8_t)(bw >> (8 * v));
            const int cq = (int)(int8_t)(cw >> (8 * v));
            const int s8 = quant_i8((float)(xq * bq), M);          // requantised INT32 state contribution
            const int hn = sat127(s8 + ((dq * hs + half) >> sc.shift));
            out |= ((uint32_t)hn & 0xffu) << (8 * v);
            acc1 += cq * hs;                                      // ChunkScan1 on the state before the token
            cb += cq * bq;                                        // ChunkBMM of the token with itself
        }
        *sp = out;
    }
    acc1 = row_sum<LPR>(acc1);
    cb = row_sum<LPR>(cb);
    if (active && sub == 0) {
        const int hp = i.h * d.P + i.p;
        const float sC = __ldg(sc.s_C + i.g);
        const float y_o = (float)acc1 * (sC * __ldg(sc.s_s + hp)) * expf(a);
        const float m = bf16_bits_to_float(float_to_bf16_bits((float)cb * (sC * __ldg(sc.s_B + i.g)) * dtv));
        y[i.r] = float_to_bf16_bits(fmaf(__ldg(D + i.h), xv, fmaf(m, xv, y_o)));
    }
}

}  // namespace

cudaError_t launch_decode_bf16(const Dims& d, const uint16_t* x, const float* dt, const float* A, const uint16_t* B,
                               const uint16_t* C, const float* D, float* state, uint16_t* y, cudaStream_t st) {
    const long long threads = (long long)d.B * d.H * d.P * (d.N / 4);
    if (threads == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((threads + kThreads - 1) / kThreads);
    if (d.N == 128) decode_bf16_kernel<128><<<grid, kThreads, 0, st>>>(d, x, dt, A, B, C, D, state, y);
    else if (d.N == 16) decode_bf16_kernel<16><<<grid, kThreads, 0, st>>>(d, x, dt, A, B, C, D, state, y);
    else return cudaErrorInvalidValue;
    return cudaGetLastError();
}

cudaError_t launch_decode_i8(const Dims& d, const uint16_t* x, const float* dt, const float* A, const int8_t* Bq,
                             const int8_t* Cq, const float* D, const I8Scales& sc, int8_t* state, uint16_t* y,
                             cudaStream_t st) {
    const long long threads = (long long)d.B * d.H * d.P * (d.N / 4);
    if (threads == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((threads + kThreads - 1) / kThreads);
    if (d.N == 128) decode_i8_kernel<128><<<grid, kThreads, 0, st>>>(d, x, dt, A, Bq, Cq, D, sc, state, y);
    else if (d.N == 16) decode_i8_kernel<16><<<grid, kThreads, 0, st>>>(d, x, dt, A, Bq, Cq, D, sc, state, y);
    else return cudaErrorInvalidValue;
    return cudaGetLastError();
}

}  // namespace ssd
