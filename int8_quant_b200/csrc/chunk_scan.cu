// chunk_scan.cu — a4..a7: ChunkBMM, ChunkScan2 (intra-chunk, causal), ChunkScan1
// (contribution of the state entering the chunk) and the D skip (SSDi8 notes,
// "overall framework" and key design 2):
//   CB[j,i]  = C_j . B_i                                   (ChunkBMM)
//   y_d[j,p] = sum_{i<=j} CB[j,i] exp(Acs_j - Acs_i) dt_i x[i,p]   (ChunkScan2)
//   y_o[j,p] = exp(Acs_j) * sum_n C[j,n] H_c[p,n]          (ChunkScan1)
//   y        = y_d + y_o + D x
// W8A8: CB and the ChunkScan1 sum are int32 over the INT8 B, C and state;
// LUT_Scan2[j,i] = s_C s_B exp(Acs_j - Acs_i) dt_i folds CB's dequantisation in;
// y_o = float(acc1) * s_C * s_s[h,p] * exp(Acs_j).
//
// One CTA per (64-row tile of a chunk, head, batch row).
#include "kernels.h"

namespace ssd {

namespace {

constexpr int kThreads = 256;
constexpr int kT = 64;        // rows per tile (j) and columns per inner tile (i)

template <int P, int N, bool kI8>
__global__ void __launch_bounds__(kThreads)
chunk_scan_kernel(Dims d, const uint16_t* __restrict__ x, const float* __restrict__ dt,
                  const float* __restrict__ Acs, const uint16_t* __restrict__ B,
                  const uint16_t* __restrict__ C, const int8_t* __restrict__ Bq,
                  const int8_t* __restrict__ Cq, const float* __restrict__ D, I8Scales sc,
                  const uint16_t* __restrict__ Hc, const int8_t* __restrict__ H8,
                  uint16_t* __restrict__ y, I8Debug dbg) {
    constexpr int kYOut = kT * P / kThreads;        // outputs per thread (>= 1)
    constexpr int kMOut = kT * kT / kThreads;       // 16
    constexpr int NP = N + 1;
    extern __shared__ float smem[];
    float* acs = smem;                              // [Q]
    float* dts = acs + d.Q;                         // [Q]
    float* ct = dts + d.Q;                          // [kT][NP]
    float* hs = ct + kT * NP;                       // [P][NP]
    float* bt = hs + P * NP;                        // [kT][NP]
    float* xt = bt + kT * NP;                       // [kT][P]
    float* mt = xt + kT * P;                        // [kT][kT + 1]
    const int tiles = d.Q / kT;
    const int jt = blockIdx.x % tiles, c = blockIdx.x / tiles;
    const int h = blockIdx.y, b = blockIdx.z, g = h / d.hpg;
    const long long t0 = (long long)c * d.Q;
    const float* acs_g = Acs + (((long long)b * d.H + h) * d.nc + c) * d.Q;
    for (int j = threadIdx.x; j < d.Q; j += kThreads) {
        acs[j] = acs_g[j];
        const long long t = t0 + j;
        dts[j] = t < d.L ? __ldg(dt + ((long long)b * d.Ls + t) * d.H + h) : 0.f;
    }
    // C rows of this tile and the state entering the chunk
    for (int idx = threadIdx.x; idx < kT * N; idx += kThreads) {
        const int jj = idx / N, n = idx % N;
        const long long t = t0 + jt * kT + jj;
        float v = 0.f;
        if (t < d.L) {
            const long long o = (((long long)b * d.Ls + t) * d.G + g) * N + n;
            v = kI8 ? (float)Cq[o] : bf16_bits_to_float(C[o]);
        }
        ct[jj * NP + n] = v;
    }
    const long long sbase = (((long long)b * d.nc + c) * d.H + h) * (long long)(P * N);
    for (int idx = threadIdx.x; idx < P * N; idx += kThreads) {
        const int p = idx / N, n = idx % N;
        hs[p * NP + n] = kI8 ? (float)H8[sbase + idx] : bf16_bits_to_float(Hc[sbase + idx]);
    }
    __syncthreads();

    float yacc[kYOut];
    int yacc_i[kYOut];
    // ChunkScan1
#pragma unroll
    for (int r = 0; r < kYOut; ++r) {
        const int o = threadIdx.x + r * kThreads;
        const int jj = o / P, p = o % P;
        if (kI8) {
            int a = 0;
            for (int n = 0; n < N; ++n) a += (int)ct[jj * NP + n] * (int)hs[p * NP + n];
            yacc_i[r] = a;
            yacc[r] = 0.f;
        } else {
            float a = 0.f;
            for (int n = 0; n < N; ++n) a = fmaf(ct[jj * NP + n], hs[p * NP + n], a);
            yacc[r] = a;
            yacc_i[r] = 0;
        }
    }
    // finish ChunkScan1: scale rows by exp(Acs_j) (and the W8A8 dequantisation)
#pragma unroll
    for (int r = 0; r < kYOut; ++r) {
        const int o = threadIdx.x + r * kThreads;
        const int jj = o / P, p = o % P;
        const float e = expf(acs[jt * kT + jj]);
        if (kI8) {
            const long long t = t0 + jt * kT + jj;
            if (dbg.acc_scan1) dbg.acc_scan1[(((long long)b * d.Lp() + t) * d.H + h) * P + p] = yacc_i[r];
            yacc[r] = (float)yacc_i[r] * (__ldg(sc.s_C + g) * __ldg(sc.s_s + h * P + p)) * e;
        } else {
            yacc[r] *= e;
        }
    }
    const float sCB = kI8 ? __ldg(sc.s_C + g) * __ldg(sc.s_B + g) : 1.f;
    // ChunkBMM + ChunkScan2 over the causal column tiles
    for (int it = 0; it <= jt; ++it) {
        __syncthreads();
        for (int idx = threadIdx.x; idx < kT * N; idx += kThreads) {
            const int ii = idx / N, n = idx % N;
            const long long t = t0 + it * kT + ii;
            float v = 0.f;
            if (t < d.L) {
                const long long o = (((long long)b * d.Ls + t) * d.G + g) * N + n;
                v = kI8 ? (float)Bq[o] : bf16_bits_to_float(B[o]);
            }
            bt[ii * NP + n] = v;
        }
        for (int idx = threadIdx.x; idx < kT * P; idx += kThreads) {
            const int ii = idx / P, p = idx % P;
            const long long t = t0 + it * kT + ii;
            xt[ii * P + p] = t < d.L ? bf16_bits_to_float(x[(((long long)b * d.Ls + t) * d.H + h) * P + p]) : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int r = 0; r < kMOut; ++r) {
            const int o = threadIdx.x + r * kThreads;
            const int jj = o / kT, ii = o % kT;
            const int j = jt * kT + jj, i = it * kT + ii;
            float m = 0.f;
            if (kI8) {
                int a = 0;
                for (int n = 0; n < N; ++n) a += (int)ct[jj * NP + n] * (int)bt[ii * NP + n];
                if (dbg.cb && (h % d.hpg) == 0)
                    dbg.cb[((((long long)b * d.nc + c) * d.G + g) * d.Q + j) * d.Q + i] = a;
                if (i <= j) m = (float)a * (sCB * expf(acs[j] - acs[i]) * dts[i]);
            } else {
                float a = 0.f;
                for (int n = 0; n < N; ++n) a = fmaf(ct[jj * NP + n], bt[ii * NP + n], a);
                if (i <= j) m = a * expf(acs[j] - acs[i]) * dts[i];
            }
            mt[jj * (kT + 1) + ii] = m;
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < kYOut; ++r) {
            const int o = threadIdx.x + r * kThreads;
            const int jj = o / P, p = o % P;
            float a = 0.f;
            for (int ii = 0; ii < kT; ++ii) a = fmaf(mt[jj * (kT + 1) + ii], xt[ii * P + p], a);
            yacc[r] += a;
        }
    }
    // D skip and store
    const float Dh = __ldg(D + h);
#pragma unroll
    for (int r = 0; r < kYOut; ++r) {
        const int o = threadIdx.x + r * kThreads;
        const int jj = o / P, p = o % P;
        const long long t = t0 + jt * kT + jj;
        if (t < d.L) {
            const long long off = (((long long)b * d.Ls + t) * d.H + h) * P + p;
            const float xv = bf16_bits_to_float(x[off]);
            y[off] = float_to_bf16_bits(yacc[r] + Dh * xv);
        }
    }
}

template <int P, int N, bool kI8>
cudaError_t launch_t(const Dims& d, const uint16_t* x, const float* dt, const float* Acs,
                     const uint16_t* B, const uint16_t* C, const int8_t* Bq, const int8_t* Cq,
                     const float* D, const I8Scales& sc, const uint16_t* Hc, const int8_t* H8,
                     uint16_t* y, const I8Debug* dbg, cudaStream_t st) {
    if (d.Q % kT) return cudaErrorInvalidValue;
    dim3 grid(d.nc * (d.Q / kT), d.H, d.B);
    const size_t smem = (size_t)(2 * d.Q + kT * (N + 1) * 2 + P * (N + 1) + kT * P + kT * (kT + 1)) * sizeof(float);
    auto k = chunk_scan_kernel<P, N, kI8>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    I8Debug none{};
    k<<<grid, kThreads, smem, st>>>(d, x, dt, Acs, B, C, Bq, Cq, D, sc, Hc, H8, y, dbg ? *dbg : none);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_scan_bf16(const Dims& d, const uint16_t* x, const float* dt,
                                   const float* Acs, const uint16_t* B, const uint16_t* C,
                                   const float* D, const uint16_t* Hc, uint16_t* y,
                                   cudaStream_t st) {
    if (d.B == 0 || d.nc == 0) return cudaSuccess;
    I8Scales none{};
    if (d.P == 64 && d.N == 128)
        return launch_t<64, 128, false>(d, x, dt, Acs, B, C, nullptr, nullptr, D, none, Hc, nullptr, y, nullptr, st);
    return launch_t<16, 16, false>(d, x, dt, Acs, B, C, nullptr, nullptr, D, none, Hc, nullptr, y, nullptr, st);
}

cudaError_t launch_chunk_scan_i8(const Dims& d, const uint16_t* x, const float* dt,
                                 const float* Acs, const int8_t* Bq, const int8_t* Cq,
                                 const float* D, const I8Scales& sc, const int8_t* H8,
                                 uint16_t* y, const I8Debug* dbg, cudaStream_t st) {
    if (d.B == 0 || d.nc == 0) return cudaSuccess;
    if (d.P == 64 && d.N == 128)
        return launch_t<64, 128, true>(d, x, dt, Acs, nullptr, nullptr, Bq, Cq, D, sc, nullptr, H8, y, dbg, st);
    return launch_t<16, 16, true>(d, x, dt, Acs, nullptr, nullptr, Bq, Cq, D, sc, nullptr, H8, y, dbg, st);
}

}  // namespace ssd
