// chunk_state.cu — a2, ChunkState (SSDi8 notes, key design 1, eq. 4 and the
// sparsity-aware reconstruction):
//   S_c[p,n] = sum_j X_scaled[j,p] * B[j,n],  X_scaled[j,p] = LUT_state[j] * x[j,p],
//   LUT_state[j] = dt_j * exp(Acs[Q-1] - Acs[j])
// The decay is applied to x (not to B), which is what lets the W8A8 path quantise
// X_scaled once per (h,p) and run the contraction on INT8 codes:
//   Xq = clamp(rint(X_scaled / s_x)), acc = sum_j Xq * Bq (int32),
//   S8 = clamp(rint(float(acc) * (s_x * s_B / s_s)), +-127)   (key design 2).
//
// One CTA per (chunk, head, batch row); rows of the chunk are staged through shared
// memory 32 tokens at a time.
#include "kernels.h"

namespace ssd {

namespace {

constexpr int kThreads = 256;
constexpr int kRows = 32;

template <int P, int N, bool kI8>
__global__ void __launch_bounds__(kThreads)
chunk_state_kernel(Dims d, const uint16_t* __restrict__ x, const float* __restrict__ dt,
                   const float* __restrict__ Acs, const uint16_t* __restrict__ B,
                   const int8_t* __restrict__ Bq, I8Scales sc, float* __restrict__ S,
                   int8_t* __restrict__ S8, float* amax_xs, float* amax_s, I8Debug dbg) {
    constexpr int kOut = (P * N + kThreads - 1) / kThreads;
    extern __shared__ float smem[];
    float* lut = smem;                              // [Q]
    float* xs = lut + d.Q;                          // [kRows][P]
    float* bt = xs + kRows * P;                     // [kRows][N]
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int g = h / d.hpg;
    const float* acs = Acs + (((long long)b * d.H + h) * d.nc + c) * d.Q;
    const float last = acs[d.Q - 1];
    for (int j = threadIdx.x; j < d.Q; j += kThreads) {
        const long long t = (long long)c * d.Q + j;
        const float dtv = t < d.L ? __ldg(dt + ((long long)b * d.Ls + t) * d.H + h) : 0.f;
        lut[j] = kI8 ? __fmul_rn(dtv, ssd_expf(__fsub_rn(last, acs[j]))) : dtv * expf(last - acs[j]);
    }
    float accf[kOut];
    int acci[kOut];
#pragma unroll
    for (int r = 0; r < kOut; ++r) { accf[r] = 0.f; acci[r] = 0; }
    __syncthreads();
    for (int j0 = 0; j0 < d.Q; j0 += kRows) {
        for (int idx = threadIdx.x; idx < kRows * P; idx += kThreads) {
            const int jj = idx / P, p = idx % P;
            const long long t = (long long)c * d.Q + j0 + jj;
            float xv = 0.f;
            if (t < d.L) xv = bf16_bits_to_float(x[(((long long)b * d.Ls + t) * d.H + h) * P + p]);
            float v;
            if (kI8) {
                const float xsv = __fmul_rn(lut[j0 + jj], xv);
                const int q = quant_i8(xsv, __frcp_rn(__ldg(sc.s_x + h * P + p)));
                v = (float)q;
                if (dbg.Xq) dbg.Xq[(((long long)b * d.Lp() + t) * d.H + h) * P + p] = (int8_t)q;
            } else {
                v = lut[j0 + jj] * xv;
                if (amax_xs && t < d.L) atomic_max_nonneg(amax_xs + h * P + p, fabsf(v));
            }
            xs[jj * P + p] = v;
        }
        for (int idx = threadIdx.x; idx < kRows * N; idx += kThreads) {
            const int jj = idx / N, n = idx % N;
            const long long t = (long long)c * d.Q + j0 + jj;
            float bv = 0.f;
            if (t < d.L) {
                const long long o = (((long long)b * d.Ls + t) * d.G + g) * N + n;
                bv = kI8 ? (float)Bq[o] : bf16_bits_to_float(B[o]);
            }
            bt[jj * N + n] = bv;
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < kOut; ++r) {
            const int o = threadIdx.x + r * kThreads;
            if (o < P * N) {
                const int p = o / N, n = o % N;
                if (kI8) {
#pragma unroll 8
                    for (int jj = 0; jj < kRows; ++jj)
                        acci[r] += (int)xs[jj * P + p] * (int)bt[jj * N + n];
                } else {
#pragma unroll 8
                    for (int jj = 0; jj < kRows; ++jj) accf[r] = fmaf(xs[jj * P + p], bt[jj * N + n], accf[r]);
                }
            }
        }
        __syncthreads();
    }
    const long long base = (((long long)b * d.nc + c) * d.H + h) * (long long)(P * N);
#pragma unroll
    for (int r = 0; r < kOut; ++r) {
        const int o = threadIdx.x + r * kThreads;
        if (o >= P * N) continue;
        if (kI8) {
            const int p = o / N;
            const float M = __fdiv_rn(__fmul_rn(__ldg(sc.s_x + h * P + p), __ldg(sc.s_B + g)),
                                      __ldg(sc.s_s + h * P + p));
            float q = rintf(__fmul_rn((float)acci[r], M));
            q = fminf(fmaxf(q, -127.f), 127.f);
            S8[base + o] = (int8_t)(int)q;
            if (dbg.acc_state) dbg.acc_state[base + o] = acci[r];
            if (dbg.S8) dbg.S8[base + o] = (int8_t)(int)q;
        } else {
            S[base + o] = accf[r];
            if (amax_s) atomic_max_nonneg(amax_s + h * P + o / N, fabsf(accf[r]));
        }
    }
}

template <int P, int N, bool kI8>
cudaError_t launch_t(const Dims& d, const uint16_t* x, const float* dt, const float* Acs,
                     const uint16_t* B, const int8_t* Bq, const I8Scales& sc, float* S, int8_t* S8,
                     float* amax_xs, float* amax_s, const I8Debug* dbg, cudaStream_t st) {
    dim3 grid(d.nc, d.H, d.B);
    const size_t smem = (size_t)(d.Q + kRows * P + kRows * N) * sizeof(float);
    auto k = chunk_state_kernel<P, N, kI8>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    I8Debug none{};
    k<<<grid, kThreads, smem, st>>>(d, x, dt, Acs, B, Bq, sc, S, S8, amax_xs, amax_s, dbg ? *dbg : none);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_state_bf16(const Dims& d, const uint16_t* x, const float* dt,
                                    const float* Acs, const uint16_t* B, float* S,
                                    float* amax_xs, float* amax_s, cudaStream_t st) {
    if (d.B == 0 || d.nc == 0) return cudaSuccess;
    I8Scales none{};
    if (d.P == 64 && d.N == 128)
        return launch_t<64, 128, false>(d, x, dt, Acs, B, nullptr, none, S, nullptr, amax_xs, amax_s, nullptr, st);
    return launch_t<16, 16, false>(d, x, dt, Acs, B, nullptr, none, S, nullptr, amax_xs, amax_s, nullptr, st);
}

cudaError_t launch_chunk_state_i8(const Dims& d, const uint16_t* x, const float* dt,
                                  const float* Acs, const int8_t* Bq, const I8Scales& sc,
                                  int8_t* S8, const I8Debug* dbg, cudaStream_t st) {
    if (d.B == 0 || d.nc == 0) return cudaSuccess;
    if (d.P == 64 && d.N == 128)
        return launch_t<64, 128, true>(d, x, dt, Acs, nullptr, Bq, sc, nullptr, S8, nullptr, nullptr, dbg, st);
    return launch_t<16, 16, true>(d, x, dt, Acs, nullptr, Bq, sc, nullptr, S8, nullptr, nullptr, dbg, st);
}

}  // namespace ssd
