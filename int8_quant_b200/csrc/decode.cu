// decode.cu — one token of the scan on the persistent state, the step on either side
// of the chunked scan when serving (the recurrence the SSD factorises, one token at a
// time):
//   h <- exp(dt*A) * h + dt * x B^T        y = C . h + D * x
// bf16 path: fp32 state.  W8A8 path: the INT8 state of the scan (real value code *
// s_s[h,p]) updated by the scan's own integer steps with a chunk of one token ("SSDi8"
// notes, key designs 1-3 and eq. 6): the token's B and C are quantised per group as at
// the scan's entry, the chunk's cumulative sum is a = dt*A, the state
// LUT is dt * exp(a - a) = dt, X_scaled = dt * x is quantised per (h,p), the INT32
// product Xq * Bq is requantised to INT8 with s_x*s_B/s_s, and the state carried over
// the token is (dq * H + 2^(k-1)) >> k with dq = rint(exp(a) * 2^k); y is ChunkScan1
// (Cq . H on the state before the token, times s_C*s_s*exp(a)) plus ChunkScan2 (the
// single CB = Cq . Bq, times s_C*s_B*dt, as a bf16 factor of x) plus D*x.
//
// Both are one pass over the state (read and write once), one (b,h,p) row of N
// elements per group of lanes with a 16-byte access each (four fp32 elements, or
// sixteen INT8 codes, per lane), the state load issued before anything else; the
// row's C . h is reduced by shuffles.
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
    constexpr int VPL = N >= 64 ? 2 : 1;                          // float4s per lane (32 bytes in flight)
    constexpr int LPR = N / (4 * VPL);                            // lanes per state row
    const long long rows = (long long)d.B * d.H * d.P;
    const long long row = ((long long)blockIdx.x * kThreads + threadIdx.x) / LPR;
    const int sub = threadIdx.x % LPR;
    const bool active = row < rows;                               // whole lane groups, shuffles stay full-warp
    const RowIdx i = row_of(d, active ? row : 0);
    float part = 0.f, xv = 0.f;
    if (active) {
        // lane `sub` holds elements [4 (sub + LPR v), +4) for v < VPL: each access a coalesced row slice
        float4* sp = reinterpret_cast<float4*>(state + i.r * N);
        float4 h4[VPL];
#pragma unroll
        for (int v = 0; v < VPL; ++v) h4[v] = sp[sub + LPR * v];
        const long long bh = (long long)i.b * d.H + i.h;
        const float dtv = __ldg(dt + bh);
        const float dA = expf(dtv * __ldg(A + i.h));
        xv = bf16_bits_to_float(x[i.r]);
        const float u = dtv * xv;
        const uint2* bp = reinterpret_cast<const uint2*>(Bm + ((long long)i.b * d.G + i.g) * N);
        const uint2* cp = reinterpret_cast<const uint2*>(Cm + ((long long)i.b * d.G + i.g) * N);
#pragma unroll
        for (int v = 0; v < VPL; ++v) {
            const uint2 bw = __ldg(bp + sub + LPR * v), cw = __ldg(cp + sub + LPR * v);
            const float bv[4] = {__uint_as_float(bw.x << 16), __uint_as_float(bw.x & 0xffff0000u),
                                 __uint_as_float(bw.y << 16), __uint_as_float(bw.y & 0xffff0000u)};
            const float cv[4] = {__uint_as_float(cw.x << 16), __uint_as_float(cw.x & 0xffff0000u),
                                 __uint_as_float(cw.y << 16), __uint_as_float(cw.y & 0xffff0000u)};
            float hv[4] = {h4[v].x, h4[v].y, h4[v].z, h4[v].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                hv[e] = fmaf(dA, hv[e], u * bv[e]);
                part = fmaf(cv[e], hv[e], part);
            }
            sp[sub + LPR * v] = make_float4(hv[0], hv[1], hv[2], hv[3]);
        }
    }
    part = row_sum<LPR>(part);
    if (active && sub == 0) y[i.r] = float_to_bf16_bits(fmaf(__ldg(D + i.h), xv, part));
}

// Round-to-nearest-even of |v| < 2^22 to an int, and an int of magnitude < 2^22 to
// float, exactly and without conversion instructions: 1.5 * 2^23 + v is representable
// with the rounded value in its low mantissa bits (bit pattern 0x4B400000 + value).
__device__ __forceinline__ int rne_small(float v) { return __float_as_int(__fadd_rn(v, 12582912.0f)) - 0x4B400000; }
__device__ __forceinline__ float small_to_float(int a) { return __fsub_rn(__int_as_float(a + 0x4B400000), 12582912.0f); }
// clamp(rint(v * inv), +-127): the clamp first, then the rounding (the same result)
__device__ __forceinline__ int code_of(float v, float inv) {
    return rne_small(fminf(fmaxf(__fmul_rn(v, inv), -127.0f), 127.0f));
}

// RPT state rows of one (b, h) per lane group (rows p, p + RS, ...; RS lane groups per
// warp): the token's B, C codes and the head's decay are formed once for them, and
// RPT 16-byte state loads are in flight per lane.
template <int N, int RPT>
__global__ void __launch_bounds__(kThreads)
decode_i8_kernel(Dims d, const uint16_t* __restrict__ x, const float* __restrict__ dt, const float* __restrict__ A,
                 const uint16_t* __restrict__ Bm, const uint16_t* __restrict__ Cm, const float* __restrict__ D,
                 I8Scales sc, int8_t* __restrict__ state, uint16_t* __restrict__ y) {
    constexpr int LPR = N / 16;                                  // lanes per state row, 16 codes each
    constexpr int RS = 32 / LPR;                                 // lane groups per warp
    const long long rows = (long long)d.B * d.H * d.P;
    const long long grp = ((long long)blockIdx.x * kThreads + threadIdx.x) / LPR;
    const long long row0 = (grp / RS) * (RS * RPT) + grp % RS;  // this group's first row; the others + k RS
    const int sub = threadIdx.x % LPR, n0 = 16 * sub;
    const bool active = row0 < rows;                             // a group's rows share (b, h): P % (RS*RPT) == 0
    const RowIdx i = row_of(d, active ? row0 : 0);
    int acc1[RPT], cb = 0;
#pragma unroll
    for (int k = 0; k < RPT; ++k) acc1[k] = 0;
    float xv[RPT], a = 0.f, dtv = 0.f;
    if (active) {
        uint4* sp = reinterpret_cast<uint4*>(state + i.r * N + n0);
        uint4 hw4[RPT];
#pragma unroll
        for (int k = 0; k < RPT; ++k) hw4[k] = sp[(long long)k * RS * N / 16];
        const long long gn = ((long long)i.b * d.G + i.g) * N + n0;
        const uint4* bp = reinterpret_cast<const uint4*>(Bm + gn);          // 16 bf16 = two 16-byte loads
        const uint4* cp = reinterpret_cast<const uint4*>(Cm + gn);
        const uint4 braw[2] = {__ldg(bp), __ldg(bp + 1)};
        const uint4 craw[2] = {__ldg(cp), __ldg(cp + 1)};
        const long long bh = (long long)i.b * d.H + i.h;
        dtv = __ldg(dt + bh);
        const float Ah = __ldg(A + i.h), sB = __ldg(sc.s_B + i.g), sC = __ldg(sc.s_C + i.g);
        float sx[RPT], ss[RPT];
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            const int hp = i.h * d.P + i.p + k * RS;
            sx[k] = __ldg(sc.s_x + hp);
            ss[k] = __ldg(sc.s_s + hp);
            xv[k] = bf16_bits_to_float(x[i.r + k * RS]);
        }
        a = __fmul_rn(dtv, Ah);                                   // ChunkCumsum of the one-token chunk
        const float lut = __fmul_rn(dtv, ssd_expf(__fsub_rn(a, a)));   // LUT_state = dt * exp(a - a)
        const int dq = (int)rintf(__fmul_rn(ssd_expf(a), (float)(1 << sc.shift)));   // decay code
        const int half = 1 << (sc.shift - 1);
        // the token's B and C codes, as ssd_quantize_inputs forms them: clamp(rint(v * (1/s)), +-127)
        const float invB = __frcp_rn(sB), invC = __frcp_rn(sC);
        const uint32_t bb[8] = {braw[0].x, braw[0].y, braw[0].z, braw[0].w, braw[1].x, braw[1].y, braw[1].z, braw[1].w};
        const uint32_t cc[8] = {craw[0].x, craw[0].y, craw[0].z, craw[0].w, craw[1].x, craw[1].y, craw[1].z, craw[1].w};
        int bqv[16], cqv[16];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            bqv[2 * e] = code_of(__uint_as_float(bb[e] << 16), invB);
            bqv[2 * e + 1] = code_of(__uint_as_float(bb[e] & 0xffff0000u), invB);
            cqv[2 * e] = code_of(__uint_as_float(cc[e] << 16), invC);
            cqv[2 * e + 1] = code_of(__uint_as_float(cc[e] & 0xffff0000u), invC);
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) cb += cqv[e] * bqv[e];       // ChunkBMM of the token with itself
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            // ChunkState: X_scaled = LUT_state * x, its code; the requantisation factor
            const int xq = code_of(__fmul_rn(lut, xv[k]), __frcp_rn(sx[k]));
            const float M = __fdiv_rn(__fmul_rn(sx[k], sB), ss[k]);
            const uint32_t hw[4] = {hw4[k].x, hw4[k].y, hw4[k].z, hw4[k].w};
            uint32_t out[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                out[q] = 0;
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const int hs = (int)(int8_t)(hw[q] >> (8 * v));
                    const int s8 = code_of(small_to_float(xq * bqv[4 * q + v]), M);   // requantised contribution
                    const int hn = sat127(s8 + ((dq * hs + half) >> sc.shift));
                    out[q] |= ((uint32_t)hn & 0xffu) << (8 * v);
                    acc1[k] += cqv[4 * q + v] * hs;               // ChunkScan1 on the state before the token
                }
            }
            sp[(long long)k * RS * N / 16] = make_uint4(out[0], out[1], out[2], out[3]);
        }
    }
    cb = row_sum<LPR>(cb);
#pragma unroll
    for (int k = 0; k < RPT; ++k) acc1[k] = row_sum<LPR>(acc1[k]);
    if (active && sub == 0) {
        const float sC = __ldg(sc.s_C + i.g);
        const float m = bf16_bits_to_float(float_to_bf16_bits((float)cb * (sC * __ldg(sc.s_B + i.g)) * dtv));
        const float ea = expf(a), Dh = __ldg(D + i.h);
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            const float y_o = (float)acc1[k] * (sC * __ldg(sc.s_s + i.h * d.P + i.p + k * RS)) * ea;
            y[i.r + k * RS] = float_to_bf16_bits(fmaf(Dh, xv[k], fmaf(m, xv[k], y_o)));
        }
    }
}

// (P, N) = (64, 128): one (b, h) per CTA of 128 threads.  The token's B and C codes,
// the head's decay code and each row's X_scaled code and requantisation factor are
// formed once per CTA, into shared memory, while the state loads are in flight; then
// each lane carries 4 rows x 16 codes (rows rb, rb + 16, ...; 8 lanes per row): the
// requantised contribution on fp32 pairs, ChunkScan1 and ChunkBMM by dp4a, and for
// decay shifts k <= 7 (and dq <= 2^k) the eq. 6 carry on two codes per 32-bit word: with
// Hu = H + 128 and Su = S8 + 128, V = dq Hu + 2^(k-1) + 128 (2^k - dq) + Su 2^k
// = dq H + 2^(k-1) + (S8 + 256) 2^k < 2^16, V >> k = H' + 256 before saturation, so
// clamping V to [129 2^k, 384 2^k - 1] saturates and the low byte of V >> k is H'.
constexpr int kHeadThreads = 128;

__global__ void __launch_bounds__(kHeadThreads)
decode_i8_head_kernel(Dims d, const uint16_t* __restrict__ x, const float* __restrict__ dt,
                      const float* __restrict__ A, const uint16_t* __restrict__ Bm, const uint16_t* __restrict__ Cm,
                      const float* __restrict__ D, I8Scales sc, int8_t* __restrict__ state, uint16_t* __restrict__ y) {
    constexpr int P = 64, N = 128, RPT = 4;
    __shared__ __align__(16) float s_bqf[N];
    __shared__ __align__(16) int8_t s_bq[N];
    __shared__ __align__(16) int8_t s_cq[N];
    __shared__ float s_xqf[P], s_M[P], s_ys[P], s_xv[P];
    __shared__ int s_dq;
    __shared__ float s_ea;
    const int t = threadIdx.x, sub = t & 7, rb = t >> 3;
    const long long bh = blockIdx.x;
    const int b = (int)(bh / d.H), h = (int)(bh % d.H), g = h / d.hpg;
    uint4* sp = reinterpret_cast<uint4*>(state + bh * (P * N)) + sub;      // row p at sp[p * N / 16]
    uint4 hw4[RPT];
#pragma unroll
    for (int j = 0; j < RPT; ++j) hw4[j] = sp[(rb + 16 * j) * (N / 16)];
    const float dtv = __ldg(dt + bh);
    const float a = __fmul_rn(dtv, __ldg(A + h));                   // ChunkCumsum of the one-token chunk
    const float sB = __ldg(sc.s_B + g), sC = __ldg(sc.s_C + g);
    if (t < P) {
        // row p: X_scaled = LUT_state * x with LUT_state = dt * exp(a - a), its code; the
        // requantisation factor s_x s_B / s_s; y's factor s_C s_s
        const int p = t, hp = h * P + p;
        const float sx = __ldg(sc.s_x + hp), ss = __ldg(sc.s_s + hp);
        const float lut = __fmul_rn(dtv, ssd_expf(__fsub_rn(a, a)));
        const float xv = bf16_bits_to_float(x[bh * P + p]);
        s_xv[p] = xv;
        s_xqf[p] = (float)code_of(__fmul_rn(lut, xv), __frcp_rn(sx));
        s_M[p] = __fdiv_rn(__fmul_rn(sx, sB), ss);
        s_ys[p] = sC * ss;
    } else {
        // the token's B and C codes n and n + 64, as ssd_quantize_inputs forms them
        const int n = t - P;
        const long long gn = ((long long)b * d.G + g) * N;
        const float invB = __frcp_rn(sB), invC = __frcp_rn(sC);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int nn = n + 64 * e;
            const int bq = code_of(bf16_bits_to_float(Bm[gn + nn]), invB);
            s_bqf[nn] = (float)bq;
            s_bq[nn] = (int8_t)bq;
            s_cq[nn] = (int8_t)code_of(bf16_bits_to_float(Cm[gn + nn]), invC);
        }
        if (n == 0) s_dq = (int)rintf(__fmul_rn(ssd_expf(a), (float)(1 << sc.shift)));   // decay code
        if (n == 1) s_ea = expf(a);
    }
    __syncthreads();
    const uint4 bq4 = *reinterpret_cast<const uint4*>(s_bq + 16 * sub);
    const uint4 cq4 = *reinterpret_cast<const uint4*>(s_cq + 16 * sub);
    const int bw[4] = {(int)bq4.x, (int)bq4.y, (int)bq4.z, (int)bq4.w};
    const int cw[4] = {(int)cq4.x, (int)cq4.y, (int)cq4.z, (int)cq4.w};
    int cb = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) cb = __dp4a(cw[q], bw[q], cb);           // ChunkBMM of the token with itself
    cb = row_sum<8>(cb);
    float2 bqf[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 f = *reinterpret_cast<const float4*>(s_bqf + 16 * sub + 4 * q);
        bqf[2 * q] = make_float2(f.x, f.y);
        bqf[2 * q + 1] = make_float2(f.z, f.w);
    }
    const int k = sc.shift, dq = s_dq;
    const bool packed = k <= 7 && dq <= (1 << k);                          // dq <= 2^k when A dt <= 0
    const uint32_t k0 = (uint32_t)((1 << (k - 1)) + 128 * ((1 << k) - dq));
    const uint32_t k0x2 = k0 | (k0 << 16);
    const uint32_t lo = (129u << k) * 0x10001u, hi = ((384u << k) - 1u) * 0x10001u;
    const float2 lim_lo = make_float2(-127.0f, -127.0f), lim_hi = make_float2(127.0f, 127.0f);
    const float2 rnd = make_float2(12582912.0f + 128.0f, 12582912.0f + 128.0f);   // 1.5 2^23 + 128
    int acc1[RPT];
#pragma unroll
    for (int j = 0; j < RPT; ++j) {
        const int p = rb + 16 * j;
        const float xq = s_xqf[p], M = s_M[p];
        const float2 xq2 = make_float2(xq, xq), M2 = make_float2(M, M);
        const uint32_t hw[4] = {hw4[j].x, hw4[j].y, hw4[j].z, hw4[j].w};
        uint32_t out[4];
        int acc = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            acc = __dp4a((int)hw[q], cw[q], acc);                       // ChunkScan1 on the state before the token
            // S8 = clamp(rint(float(xq bq) * M), +-127) for codes 4q .. 4q+3: xq bq is exact in fp32
            uint32_t su[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float2 u = __fmul2_rn(__fmul2_rn(xq2, bqf[2 * q + e]), M2);
                u.x = fminf(fmaxf(u.x, lim_lo.x), lim_hi.x);
                u.y = fminf(fmaxf(u.y, lim_lo.y), lim_hi.y);
                u = __fadd2_rn(u, rnd);                                  // bits 0x4B400000 + 128 + rint(u)
                su[e] = __byte_perm(__float_as_uint(u.x), __float_as_uint(u.y), 0x5410);
            }
            if (packed) {
                const uint32_t hu = hw[q] ^ 0x80808080u;
                uint32_t v0 = __byte_perm(hu, 0, 0x4140) * (uint32_t)dq + k0x2 + (su[0] << k);
                uint32_t v1 = __byte_perm(hu, 0, 0x4342) * (uint32_t)dq + k0x2 + (su[1] << k);
                v0 = min_u16x2(max_u16x2(v0, lo), hi) >> k;
                v1 = min_u16x2(max_u16x2(v1, lo), hi) >> k;
                out[q] = __byte_perm(v0, v1, 0x6420);
            } else {
                out[q] = 0;
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const int hs = (int)(int8_t)(hw[q] >> (8 * v));
                    const int s8 = (int)((su[v >> 1] >> (16 * (v & 1))) & 0xffffu) - 128;
                    const int hn = sat127(s8 + ((dq * hs + (1 << (k - 1))) >> k));
                    out[q] |= ((uint32_t)hn & 0xffu) << (8 * v);
                }
            }
        }
        acc1[j] = acc;
        sp[p * (N / 16)] = make_uint4(out[0], out[1], out[2], out[3]);
    }
#pragma unroll
    for (int j = 0; j < RPT; ++j) acc1[j] = row_sum<8>(acc1[j]);
    if (sub == 0) {
        const float m = bf16_bits_to_float(float_to_bf16_bits((float)cb * (sC * sB) * dtv));
        const float ea = s_ea, Dh = __ldg(D + h);
#pragma unroll
        for (int j = 0; j < RPT; ++j) {
            const int p = rb + 16 * j;
            const float xv = s_xv[p];
            const float y_o = (float)acc1[j] * s_ys[p] * ea;
            y[bh * P + p] = float_to_bf16_bits(fmaf(Dh, xv, fmaf(m, xv, y_o)));
        }
    }
}

}  // namespace

cudaError_t launch_decode_bf16(const Dims& d, const uint16_t* x, const float* dt, const float* A, const uint16_t* B,
                               const uint16_t* C, const float* D, float* state, uint16_t* y, cudaStream_t st) {
    const long long threads = (long long)d.B * d.H * d.P * (d.N >= 64 ? d.N / 8 : d.N / 4);
    if (threads == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((threads + kThreads - 1) / kThreads);
    if (d.N == 128) decode_bf16_kernel<128><<<grid, kThreads, 0, st>>>(d, x, dt, A, B, C, D, state, y);
    else if (d.N == 16) decode_bf16_kernel<16><<<grid, kThreads, 0, st>>>(d, x, dt, A, B, C, D, state, y);
    else return cudaErrorInvalidValue;
    return cudaGetLastError();
}

cudaError_t launch_decode_i8(const Dims& d, const uint16_t* x, const float* dt, const float* A, const uint16_t* Bq,
                             const uint16_t* Cq, const float* D, const I8Scales& sc, int8_t* state, uint16_t* y,
                             cudaStream_t st) {
    const long long heads = (long long)d.B * d.H;
    if (d.N == 128 && d.P == 64) {
        if (heads == 0) return cudaSuccess;
        decode_i8_head_kernel<<<(unsigned)heads, kHeadThreads, 0, st>>>(d, x, dt, A, Bq, Cq, D, sc, state, y);
        return cudaGetLastError();
    }
    // other P with N = 128: 2 rows per lane group, 8 rows of one head per warp; N = 16: one row
    constexpr int kRpt128 = 2;
    if (d.N == 128 && d.P % (4 * kRpt128) != 0) return cudaErrorInvalidValue;
    const long long threads = (long long)d.B * d.H * d.P * (d.N / 16) / (d.N == 128 ? kRpt128 : 1);
    if (threads == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((threads + kThreads - 1) / kThreads);
    if (d.N == 128) decode_i8_kernel<128, kRpt128><<<grid, kThreads, 0, st>>>(d, x, dt, A, Bq, Cq, D, sc, state, y);
    else if (d.N == 16) decode_i8_kernel<16, 1><<<grid, kThreads, 0, st>>>(d, x, dt, A, Bq, Cq, D, sc, state, y);
    else return cudaErrorInvalidValue;
    return cudaGetLastError();
}

}  // namespace ssd
