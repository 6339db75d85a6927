// out_proj.cu — the SSD epilogue in the W8A8 pipeline ("SSDi8" notes, key design 4 and
// the training strategy): RMSNorm of the scan output, static symmetric INT8 codes,
// the output projection as an INT8 GEMM with INT32 accumulation on the tensor cores,
// dequantisation by s_a * s_w[d] and the mean correction c[d] (0.15 c*, computed at
// calibration), bf16 out.  The RMSNorm weight is folded into the projection (gamma
// migration), so the codes are those of y / sqrt(mean(y^2) + eps).
//
//   rmsnorm_quant_kernel  one CTA per token: sum of squares over the K = H*P features,
//                         then the codes clamp(rint(u * (1/s_a)), +-127).
//   out_proj_gemm_kernel  persistent, one CTA per SM over the 128 x 256 output tiles
//                         (tokens x output channels): a 4-stage TMA ring of 128-byte K
//                         slices of the codes (128 rows) and the weights (256 rows,
//                         128-byte swizzle), tcgen05.mma kind::i8 (M = 128, N = 256,
//                         K = 32) issued by one elected lane into one of two 256-column
//                         INT32 TMEM accumulators, and four epilogue warps (one per TMEM
//                         lane quarter) that dequantise, add c and store bf16 rows while
//                         the next tile accumulates in the other.
// Every wait is bounded; an expired wait raises the CTA's abort flag and records
// SSD_ERR_TIMEOUT in the status word.
#include "kernels.h"
#include "tc.cuh"

namespace ssd {

namespace {

constexpr float kNormEps = 1e-5f;
constexpr int kNormThreads = 256;

__global__ void __launch_bounds__(kNormThreads)
rmsnorm_quant_kernel(int K, const uint16_t* __restrict__ y, float inv_sa, int8_t* __restrict__ aq) {
    const long long row = blockIdx.x;
    const uint16_t* yr = y + row * K;
    int8_t* qr = aq + row * K;
    __shared__ float part[kNormThreads / 32];
    float ss = 0.f;
    for (int i = threadIdx.x * 8; i < K; i += kNormThreads * 8) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(yr + i));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float lo = __uint_as_float(w[e] << 16), hi = __uint_as_float(w[e] & 0xffff0000u);
            ss = fmaf(lo, lo, ss);
            ss = fmaf(hi, hi, ss);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int i = 0; i < kNormThreads / 32; ++i) tot += part[i];
    const float r = rsqrtf(tot / (float)K + kNormEps);
    const float mul = r * inv_sa;
    for (int i = threadIdx.x * 8; i < K; i += kNormThreads * 8) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(yr + i));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t out[2] = {0u, 0u};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int q0 = quant_i8(__uint_as_float(w[e] << 16), mul);
            const int q1 = quant_i8(__uint_as_float(w[e] & 0xffff0000u), mul);
            out[e >> 1] |= (((uint32_t)q0 & 0xffu) | (((uint32_t)q1 & 0xffu) << 8)) << (16 * (e & 1));
        }
        *reinterpret_cast<uint2*>(qr + i) = make_uint2(out[0], out[1]);
    }
}

constexpr int kBM = 128, kBN = 256, kBK = 128, kStages = 4, kAcc = 2;
constexpr int kGemmWarps = 6;                        // 0 TMA, 1 MMA, 2-5 epilogue
constexpr int A_BYTES = kBM * kBK, W_BYTES = kBN * kBK;
constexpr int OFF_A = 0, OFF_W = kStages * A_BYTES, OFF_BAR = OFF_W + kStages * W_BYTES;
constexpr int B_FULL = 0, B_EMPTY = kStages, B_AFULL = 2 * kStages, B_AEMPTY = 2 * kStages + kAcc,
              NBAR = 2 * kStages + 2 * kAcc;
constexpr int OFF_FLAG = OFF_BAR + NBAR * 8, OFF_TMEM = OFF_FLAG + 8, GEMM_SMEM = OFF_TMEM + 8;

// Persistent: CTA i takes tiles i, i + grid, ... in the order (token tile, output-channel tile) with the
// channel tile fastest, so the CTAs working at one time share their token rows of codes through L2.  The
// stage ring runs on across tiles, and two TMEM accumulators let the epilogue of one tile overlap the
// MMAs of the next.
__global__ void __launch_bounds__(kGemmWarps * 32, 1)
out_proj_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_w, int K,
                     int D, int tiles_n, int tiles, float s_a, const float* __restrict__ s_w,
                     const float* __restrict__ corr, uint16_t* __restrict__ out, int32_t* __restrict__ acc_dbg,
                     int* __restrict__ status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_FLAG);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_TMEM);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = K / kBK;
    if (threadIdx.x == 0) {
        for (int i = 0; i < NBAR; ++i) tc::mbar_init(bar + i, i >= B_AEMPTY ? 4 : 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, kAcc * kBN);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            tc::prefetch_tmap(&tm_a);
            tc::prefetch_tmap(&tm_w);
            long long kc = 0;                                     // K slices issued so far (ring position)
            bool ok = true;
            for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
                const int m0 = (t / tiles_n) * kBM, n0 = (t % tiles_n) * kBN;
                for (int k = 0; k < nk; ++k, ++kc) {
                    const int s = (int)(kc % kStages);
                    if (!(ok = tc::wait_or_abort(bar + B_EMPTY + s, (((uint32_t)(kc / kStages)) & 1) ^ 1, abort_flag,
                                                 status, kStatusTimeout)))
                        break;
                    tc::mbar_arrive_expect_tx(bar + B_FULL + s, A_BYTES + W_BYTES);
                    tc::tma_load_2d(sm + OFF_A + s * A_BYTES, &tm_a, bar + B_FULL + s, k * kBK, m0);
                    tc::tma_load_2d(sm + OFF_W + s * W_BYTES, &tm_w, bar + B_FULL + s, k * kBK, n0);
                }
            }
        }
    } else if (warp == 1) {
        const uint32_t idesc = tc::idesc_s8_s32(kBM, kBN, tc::kMajorK, tc::kMajorK);
        long long kc = 0;
        int it = 0;                                               // tiles of this CTA so far
        bool ok = true;
        for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++it) {
            const int a = it & 1;
            // the epilogue has drained this accumulator (its use two tiles ago)
            ok = __all_sync(0xffffffffu, tc::wait_or_abort(bar + B_AEMPTY + a, (((uint32_t)(it >> 1)) & 1) ^ 1,
                                                          abort_flag, status, kStatusTimeout));
            if (!ok) break;
            const uint32_t dacc = tmem + (uint32_t)(a * kBN);
            for (int k = 0; k < nk; ++k, ++kc) {
                const int s = (int)(kc % kStages);
                ok = __all_sync(0xffffffffu, tc::wait_or_abort(bar + B_FULL + s, ((uint32_t)(kc / kStages)) & 1,
                                                              abort_flag, status, kStatusTimeout));
                if (!ok) break;
                tc::tc_fence_after();
                if (tc::elect_one()) {
                    const uint64_t da = tc::smem_desc(tc::smem_u32(sm + OFF_A + s * A_BYTES), 16, 1024, tc::kLayoutSw128);
                    const uint64_t dw = tc::smem_desc(tc::smem_u32(sm + OFF_W + s * W_BYTES), 16, 1024, tc::kLayoutSw128);
#pragma unroll
                    for (int kk = 0; kk < kBK / 32; ++kk)            // K = 32 codes = 32 bytes per MMA
                        tc::mma_i8_ss(dacc, da + (uint64_t)(kk * 2), dw + (uint64_t)(kk * 2), idesc, (k | kk) != 0);
                    tc::mma_commit(bar + B_EMPTY + s);
                    if (k == nk - 1) tc::mma_commit(bar + B_AFULL + a);
                }
                __syncwarp();
            }
        }
    } else {
        // epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31, i.e. output rows m0 + 32 (w % 4) + lane
        const int quarter = warp & 3;
        int it = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++it) {
            const int a = it & 1;
            const int m0 = (t / tiles_n) * kBM, n0 = (t % tiles_n) * kBN;
            const int row = m0 + quarter * 32 + lane;
            const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(a * kBN);
            const bool ok = tc::wait_or_abort(bar + B_AFULL + a, ((uint32_t)(it >> 1)) & 1, abort_flag, status,
                                              kStatusTimeout);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc::tc_fence_after();
            for (int c = 0; c < kBN / 32; ++c) {
                uint32_t v[32];
                tc::tmem_ld32(trow + c * 32, v);
                tc::tmem_wait_ld();
                if (c == kBN / 32 - 1) {
                    // the whole accumulator is in registers: hand it back to the MMA warp
                    tc::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(bar + B_AEMPTY + a);
                }
                const int col0 = n0 + c * 32;
                uint32_t o[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int ca = col0 + 2 * i;
                    float f0 = (float)(int)v[2 * i] * (s_a * __ldg(s_w + ca));
                    float f1 = (float)(int)v[2 * i + 1] * (s_a * __ldg(s_w + ca + 1));
                    if (corr) {
                        f0 += __ldg(corr + ca);
                        f1 += __ldg(corr + ca + 1);
                    }
                    o[i] = (uint32_t)float_to_bf16_bits(f0) | ((uint32_t)float_to_bf16_bits(f1) << 16);
                }
                uint4* dst = reinterpret_cast<uint4*>(out + (long long)row * D + col0);
#pragma unroll
                for (int q = 0; q < 4; ++q) dst[q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
                if (acc_dbg) {
                    int4* dd = reinterpret_cast<int4*>(acc_dbg + (long long)row * D + col0);
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        dd[q] = make_int4((int)v[4 * q], (int)v[4 * q + 1], (int)v[4 * q + 2], (int)v[4 * q + 3]);
                }
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(tmem, kAcc * kBN);
}

}  // namespace

cudaError_t launch_out_proj_norm(int T, int K, const uint16_t* y, float s_a, int8_t* aq, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    rmsnorm_quant_kernel<<<T, kNormThreads, 0, st>>>(K, y, 1.0f / s_a, aq);
    return cudaGetLastError();
}

cudaError_t launch_out_proj_gemm(int T, int K, int D, const int8_t* aq, float s_a, const int8_t* Wq, const float* s_w,
                                 const float* corr, uint16_t* out, int32_t* acc_dbg, int* status, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    cudaError_t e;
    CUtensorMap ma, mw;
    if (!make_tmap_2d(&ma, true, aq, (unsigned long long)K, (unsigned long long)T, (unsigned long long)K, kBK, kBM,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_2d(&mw, true, Wq, (unsigned long long)K, (unsigned long long)D, (unsigned long long)K, kBK, kBN,
                      CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const int smem = GEMM_SMEM + 1024;
    e = cudaFuncSetAttribute(out_proj_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int tiles_n = D / kBN, tiles = tiles_n * (T / kBM);
    const int grid = tiles < device_sm_count() ? tiles : device_sm_count();
    out_proj_gemm_kernel<<<grid, kGemmWarps * 32, smem, st>>>(ma, mw, K, D, tiles_n, tiles, s_a, s_w, corr, out,
                                                             acc_dbg, status);
    return cudaGetLastError();
}

}  // namespace ssd
