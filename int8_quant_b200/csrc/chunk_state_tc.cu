// chunk_state_tc.cu — a2, ChunkState on the tensor cores (P = 64, N = 128).
//
// SSDi8 notes, key design 1, eq. 4 and the reconstruction: the chunk state is
//   S_c = X_scaled^T B,  X_scaled[j,p] = LUT_state[j] * x[j,p],
// i.e. the decay is moved from B onto x so that, in the W8A8 path, X_scaled can be
// quantised once per (h,p) and the contraction run on INT8 codes with INT32
// accumulation; key design 2 then requantises the INT32 state to INT8 in registers:
//   S8 = clamp(rint(float(acc) * (s_x * s_B / s_s)), +-127).
//
// One CTA per (head, chunk, batch row); consecutive CTAs share (b, c) so the B tile
// is served from L2.  TMA brings the x tile [Q x 64] and the B tile [Q x 128] into
// 128-byte-swizzled shared memory; four warps scale x by LUT_state in place (bf16)
// or quantise it into a 64-byte-swizzled Xq tile (W8A8); one thread issues the
// tcgen05 MMAs for the transposed state S^T[n,p] = sum_j B[j,n] X[j,p]
// (M = n = 128, N = p = 64, K = j: both operands MN-major, as loaded), accumulating
// in TMEM; each warp then reads its 32 TMEM lanes (n) and writes S[p][n] rows with
// coalesced stores.
#include "kernels.h"
#include "tc.cuh"

namespace ssd {

namespace {

constexpr int kThreads = 128;
constexpr int kP = 64;
constexpr int kN = 128;

template <int Q, bool kI8>
struct StateSmem {
    static constexpr int kX = 0;                                  // x tile, bf16 [Q][64], SW128
    static constexpr int kB = kX + Q * 128;                       // B tile (bf16: 2 x [Q][64]; i8: [Q][128])
    static constexpr int kBBytes = kI8 ? Q * 128 : 2 * Q * 128;
    static constexpr int kXq = kB + kBBytes;                      // W8A8: Xq int8 [Q][64], SW64
    static constexpr int kXqBytes = kI8 ? Q * 64 : 0;
    static constexpr int kLut = kXq + kXqBytes;                   // float [Q]
    static constexpr int kScal = kLut + Q * 4;                    // float [64] M, float [64] 1/s_x
    static constexpr int kBar = kScal + 2 * 64 * 4;               // 2 x mbarrier
    static constexpr int kTmem = kBar + 16;
    static constexpr int kBytes = kTmem + 16;
    static constexpr int kTmaBytes = Q * 128 + kBBytes;
};

template <int Q, bool kI8>
__global__ void __launch_bounds__(kThreads, 1)
chunk_state_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                      Dims d, const float* __restrict__ lut_g, I8Scales sc, uint16_t* __restrict__ S,
                      int8_t* __restrict__ S8, I8Debug dbg, int* __restrict__ status) {
    using L = StateSmem<Q, kI8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    const int h = blockIdx.x, c = blockIdx.y, b = blockIdx.z;
    const int g = h / d.hpg;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + L::kBar);
    uint64_t* bar_mma = bar_tma + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::kTmem);
    float* lut = reinterpret_cast<float*>(sm + L::kLut);
    float* Mq = reinterpret_cast<float*>(sm + L::kScal);
    float* inv_sx = Mq + 64;

    if (tid == 0) {
        tc::mbar_init(bar_tma, 1);
        tc::mbar_init(bar_mma, 1);
        tc::fence_mbar_init();
        tc::prefetch_tmap(&tm_x);
        tc::prefetch_tmap(&tm_b);
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, 64);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (tid == 0) {
        tc::mbar_arrive_expect_tx(bar_tma, L::kTmaBytes);
        tc::tma_load_3d(sm + L::kX, &tm_x, bar_tma, h * kP, c * Q, b);
        tc::tma_load_3d(sm + L::kB, &tm_b, bar_tma, g * kN, c * Q, b);
        if (!kI8) tc::tma_load_3d(sm + L::kB + Q * 128, &tm_b, bar_tma, g * kN + 64, c * Q, b);
    }
    const float* lg = lut_g + (((long long)b * d.H + h) * d.nc + c) * Q;
    for (int j = tid; j < Q; j += kThreads) lut[j] = lg[j];
    if (kI8 && tid < kP) {
        const float sx = __ldg(sc.s_x + h * kP + tid);
        Mq[tid] = __fdiv_rn(__fmul_rn(sx, __ldg(sc.s_B + g)), __ldg(sc.s_s + h * kP + tid));
        inv_sx[tid] = __frcp_rn(sx);
    }
    __syncthreads();
    bool ok = tc::mbar_wait(bar_tma, 0, tc::kWaitLimit);

    if (ok) {
        // X_scaled = LUT_state[j] * x[j,p].  Each 16-byte chunk holds 8 consecutive p
        // of one row; the 128-byte swizzle only permutes chunks within a row.
        for (int k = tid; k < Q * 8; k += kThreads) {
            const int row = k >> 3;
            uint4* src = reinterpret_cast<uint4*>(sm + L::kX + k * 16);
            uint4 v = *src;
            uint32_t w[4] = {v.x, v.y, v.z, v.w};
            const float f = lut[row];
            if (!kI8) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float lo = bf16_bits_to_float((uint16_t)(w[i] & 0xffffu)) * f;
                    const float hi = bf16_bits_to_float((uint16_t)(w[i] >> 16)) * f;
                    w[i] = (uint32_t)float_to_bf16_bits(lo) | ((uint32_t)float_to_bf16_bits(hi) << 16);
                }
                *src = make_uint4(w[0], w[1], w[2], w[3]);
            } else {
                const int p0 = ((k & 7) ^ (row & 7)) * 8;          // logical first column of this chunk
                uint32_t q[2] = {0u, 0u};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint16_t bits = (uint16_t)(w[i >> 1] >> ((i & 1) * 16));
                    const float xs = __fmul_rn(f, bf16_bits_to_float(bits));
                    const int qi = quant_i8(xs, inv_sx[p0 + i]);
                    q[i >> 2] |= ((uint32_t)(qi & 0xff)) << ((i & 3) * 8);
                }
                // 64-byte swizzle: 16-byte chunk index (p / 16) XOR address bits 7..8
                const int off = row * 64 + ((((p0 >> 4) ^ ((row >> 1) & 3))) << 4) + (p0 & 15);
                *reinterpret_cast<uint2*>(sm + L::kXq + off) = make_uint2(q[0], q[1]);
                if (dbg.Xq) {
                    const long long t = (long long)c * Q + row;
                    *reinterpret_cast<uint2*>(dbg.Xq + (((long long)b * d.Lp() + t) * d.H + h) * kP + p0) =
                        make_uint2(q[0], q[1]);
                }
            }
        }
        tc::fence_proxy_async_smem();
    }
    __syncthreads();

    if (ok && tid == 0) {
        tc::tc_fence_after();
        if (!kI8) {
            const uint32_t idesc = tc::idesc_bf16_f32(128, kP, tc::kMajorMN, tc::kMajorMN);
            const uint32_t aB = tc::smem_u32(sm + L::kB), aX = tc::smem_u32(sm + L::kX);
#pragma unroll 4
            for (int s = 0; s < Q / 16; ++s) {
                const uint64_t da = tc::smem_desc(aB + s * 2048, Q * 128, 1024, tc::kLayoutSw128);
                const uint64_t db = tc::smem_desc(aX + s * 2048, Q * 128, 1024, tc::kLayoutSw128);
                tc::mma_f16_ss(tmem, da, db, idesc, s > 0 ? 1u : 0u);
            }
        } else {
            const uint32_t idesc = tc::idesc_s8_s32(128, kP, tc::kMajorMN, tc::kMajorMN);
            const uint32_t aB = tc::smem_u32(sm + L::kB), aX = tc::smem_u32(sm + L::kXq);
#pragma unroll 4
            for (int s = 0; s < Q / 32; ++s) {
                const uint64_t da = tc::smem_desc(aB + s * 4096, 0, 1024, tc::kLayoutSw128);
                const uint64_t db = tc::smem_desc(aX + s * 2048, 0, 512, tc::kLayoutSw64);
                tc::mma_i8_ss(tmem, da, db, idesc, s > 0 ? 1u : 0u);
            }
        }
        tc::mma_commit(bar_mma);
    }
    if (ok) ok = tc::mbar_wait(bar_mma, 0, tc::kWaitLimit);
    tc::tc_fence_after();

    if (ok) {
        uint32_t v0[32], v1[32];
        const uint32_t ta = tmem + ((uint32_t)(warp * 32) << 16);
        tc::tmem_ld32(ta, v0);
        tc::tmem_ld32(ta + 32, v1);
        tc::tmem_wait_ld();
        const int n = warp * 32 + lane;
        const long long base = (((long long)b * d.nc + c) * d.H + h) * (long long)(kP * kN) + n;
#pragma unroll
        for (int p = 0; p < kP; ++p) {
            const uint32_t raw = p < 32 ? v0[p] : v1[p - 32];
            if (!kI8) {
                S[base + p * kN] = float_to_bf16_bits(__uint_as_float(raw));
            } else {
                const int acc = (int)raw;
                float q = rintf(__fmul_rn(__int2float_rn(acc), Mq[p]));
                q = fminf(fmaxf(q, -127.f), 127.f);
                S8[base + p * kN] = (int8_t)(int)q;
                if (dbg.acc_state) dbg.acc_state[base + p * kN] = acc;
                if (dbg.S8) dbg.S8[base + p * kN] = (int8_t)(int)q;
            }
        }
    } else {
        // a wait expired: record it, give in-flight copies a bounded chance to land
        // before the shared memory is released, free TMEM and return
        if (tid == 0 && status) atomicExch(status, kStatusTimeout);
        tc::mbar_wait(bar_tma, 0, tc::kWaitLimit);
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 64);
}

template <int Q, bool kI8>
cudaError_t launch_q(const Dims& d, const CUtensorMap& tx, const CUtensorMap& tb, const float* lut,
                     const I8Scales& sc, uint16_t* S, int8_t* S8, const I8Debug* dbg, int* status, cudaStream_t st) {
    using L = StateSmem<Q, kI8>;
    auto k = chunk_state_tc_kernel<Q, kI8>;
    const int smem = L::kBytes + 1024;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    I8Debug none{};
    k<<<dim3(d.H, d.nc, d.B), kThreads, smem, st>>>(tx, tb, d, lut, sc, S, S8, dbg ? *dbg : none, status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_state_tc(const Dims& d, bool i8, const uint16_t* x, const void* Bmat,
                                  const float* lut, const I8Scales& sc, uint16_t* S, int8_t* S8,
                                  const I8Debug* dbg, int* status, cudaStream_t st) {
    if (d.B == 0 || d.nc == 0) return cudaSuccess;
    if (d.P != kP || d.N != kN) return cudaErrorInvalidValue;
    CUtensorMap tx, tb;
    const unsigned long long HP = (unsigned long long)d.H * kP, GN = (unsigned long long)d.G * kN;
    if (!make_tmap_3d(&tx, false, x, HP, d.L, d.B, HP * 2, d.Ls * HP * 2, 64, d.Q, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const bool ok_b = i8 ? make_tmap_3d(&tb, true, Bmat, GN, d.L, d.B, GN, d.Ls * GN, 128, d.Q,
                                        CU_TENSOR_MAP_SWIZZLE_128B)
                         : make_tmap_3d(&tb, false, Bmat, GN, d.L, d.B, GN * 2, d.Ls * GN * 2, 64, d.Q,
                                        CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok_b) return cudaErrorInvalidValue;
    switch (d.Q) {
        case 64: return i8 ? launch_q<64, true>(d, tx, tb, lut, sc, S, S8, dbg, status, st)
                           : launch_q<64, false>(d, tx, tb, lut, sc, S, S8, dbg, status, st);
        case 128: return i8 ? launch_q<128, true>(d, tx, tb, lut, sc, S, S8, dbg, status, st)
                            : launch_q<128, false>(d, tx, tb, lut, sc, S, S8, dbg, status, st);
        case 256: return i8 ? launch_q<256, true>(d, tx, tb, lut, sc, S, S8, dbg, status, st)
                            : launch_q<256, false>(d, tx, tb, lut, sc, S, S8, dbg, status, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace ssd
