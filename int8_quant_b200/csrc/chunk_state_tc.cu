// chunk_state_tc.cu — a2, ChunkState on the tensor cores (P = 64, N = 128).
//
// SSDi8 notes, key design 1, eq. 4 and the reconstruction: the chunk state is
//   S_c = X_scaled^T B,  X_scaled[j,p] = LUT_state[j] * x[j,p],
// i.e. the decay is moved from B onto x so that, in the W8A8 path, X_scaled can be
// quantised once per (h,p) and the contraction run on INT8 codes with INT32
// accumulation; key design 2 then requantises the INT32 state to INT8 in registers:
//   S8 = clamp(rint(float(acc) * (s_x * s_B / s_s)), +-127).
//
// Persistent kernel: one CTA per SM walks a contiguous range of (batch row, chunk,
// head) units, heads fastest, so the B tile of a (b, c, group) is loaded once and
// serves all of its heads.  The warp roles hand work to each other through
// mbarriers:
//   warp 0      TMA producer: the B tile whenever the group changes (W8A8: double
//               buffered); per head the x tile [Q x 64] and its LUT_state row into a
//               3-stage ring.
//   warp 1      TMEM allocation and the MMA-issuing thread: the transposed state
//               S^T[n,p] = sum_j B[j,n] X_scaled[j,p] (M = n = 128, N = p = 64,
//               K = j; both operands MN-major, as loaded) into one of four TMEM
//               accumulators.
//   warps 2-5   epilogue: each reads its 32 TMEM lanes (n) and writes S[p][n] rows
//               as bf16, or requantised to S8.
//   warps 6-13  prep: X_scaled = LUT_state * x in place (bf16), or quantised into a
//               64-byte-swizzled Xq tile (W8A8).
// Every wait is bounded; an expired wait raises a shared abort flag that ends all
// roles and records SSD_ERR_TIMEOUT in the status word; in-flight copies and MMAs
// are waited for (again bounded) before the CTA frees TMEM and exits.
#include "kernels.h"
#include "tc.cuh"

namespace ssd {

namespace {

constexpr int kP = 64;
constexpr int kN = 128;
constexpr int kWarps = 14;
constexpr int kThreads = kWarps * 32;
constexpr int kEpiWarp0 = 2;
constexpr int kPrepWarp0 = 6;
constexpr int kPrepThreads = (kWarps - kPrepWarp0) * 32;
constexpr int kAcc = 4;                                       // TMEM accumulators of 64 columns
static_assert(kPrepWarp0 - kEpiWarp0 == 4, "one epilogue warp per TMEM lane quarter");

template <int Q, bool kI8>
struct StateCfg {
    static_assert(Q * 127 * 127 < (1 << 22), "INT32 state accumulators must stay below 2^22");
    static constexpr int NB = kI8 ? 2 : 1;                    // B tile buffers
    static constexpr int NS = kI8 ? 3 : 4;                    // x ring stages (W8A8: also Xq slots)
    static constexpr int B_BYTES = kI8 ? Q * 128 : 2 * Q * 128;
    static constexpr int X_BYTES = Q * 128;                   // bf16 [Q][64], 128B swizzle
    static constexpr int XQ_BYTES = kI8 ? Q * 64 : 0;         // int8 [Q][64], 64B swizzle
    static constexpr int OFF_B = 0;
    static constexpr int OFF_X = OFF_B + NB * B_BYTES;
    static constexpr int OFF_XQ = OFF_X + NS * X_BYTES;
    static constexpr int OFF_LUT = OFF_XQ + NS * XQ_BYTES;
    static constexpr int OFF_SX = OFF_LUT + NS * Q * 4;      // W8A8: 1/s_x of the stage's head
    static constexpr int SX_BYTES = kI8 ? kP * 4 : 0;
    static constexpr int STAGE_TX = X_BYTES + Q * 4 + SX_BYTES;
    // FULL: x tile landed; EMPTY: x slot reusable (bf16: its MMA finished; W8A8: quantised);
    // QEMPTY (W8A8): Xq slot reusable (its MMA finished); PREP: operand ready for the MMA
    enum { FULL = 0, EMPTY = FULL + NS, QEMPTY = EMPTY + NS, PREP = QEMPTY + NS, BFULL = PREP + NS, BEMPTY = BFULL + 2,
           TFULL = BEMPTY + 2, TEMPTY = TFULL + kAcc, DONE = TEMPTY + kAcc, NBAR = DONE + 1 };
    static constexpr int OFF_BAR = OFF_SX + NS * SX_BYTES;
    static constexpr int OFF_FLAG = OFF_BAR + NBAR * 8;
    static constexpr int OFF_TMEM = OFF_FLAG + 8;
    // W8A8: each epilogue warp's copy of its unit's 64 requantisation factors (16-byte aligned)
    static constexpr int OFF_MQ = (OFF_TMEM + 8 + 15) & ~15;
    static constexpr int BYTES = OFF_MQ + (kI8 ? 4 * kP * 4 : 0);
};

// INT8 code of an already scaled value, clamp(rint(v), +-127), without a conversion
// instruction: clamping first gives the same code (+-127 are integers), and adding
// 1.5 * 2^23 rounds to the nearest integer (ties to even) into the low mantissa bits,
// so the float's bits are 0x4B400000 + code; the low byte is the code's byte.
constexpr float kRound = 12582912.0f;                        // 1.5 * 2^23
constexpr int kRoundBits = 0x4B400000;
__device__ __forceinline__ int code_bits(float v) {
    return __float_as_int(__fadd_rn(fminf(fmaxf(v, -127.f), 127.f), kRound));
}
// Two IEEE fp32 products (round to nearest even) in one packed instruction.
__device__ __forceinline__ void mul_f32x2(float& r0, float& r1, float a0, float a1, float b0, float b1) {
    asm("{\n\t.reg .b64 a, b, r;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
        "mul.rn.f32x2 r, a, b;\n\tmov.b64 {%0, %1}, r;\n\t}"
        : "=f"(r0), "=f"(r1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
// code_bits of two values, the rounding additions packed.
__device__ __forceinline__ void code_bits2(int& q0, int& q1, float v0, float v1) {
    const float c0 = fminf(fmaxf(v0, -127.f), 127.f), c1 = fminf(fmaxf(v1, -127.f), 127.f);
    float r0, r1;
    asm("{\n\t.reg .b64 a, b, r;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %4};\n\t"
        "add.rn.f32x2 r, a, b;\n\tmov.b64 {%0, %1}, r;\n\t}"
        : "=f"(r0), "=f"(r1)
        : "f"(c0), "f"(c1), "f"(kRound));
    q0 = __float_as_int(r0);
    q1 = __float_as_int(r1);
}
// float(a) for |a| < 2^22, exactly, by the same device.
__device__ __forceinline__ float small_int_to_float(int a) { return __fsub_rn(__int_as_float(a + kRoundBits), kRound); }

// Low bytes of four codes, first in the lowest byte.
__device__ __forceinline__ uint32_t pack_i8x4(int a, int b, int c, int d) {
    return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// Walks the units (b, c, h), heads fastest, without divisions after the start;
// `hh` is h's index within its group, so a unit needs a new B tile when hh == 0.
struct Cursor {
    int b, c, h, g, hh;
    __device__ __forceinline__ void init(const Dims& d, int u) {
        h = u % d.H;
        const int bc = u / d.H;
        c = bc % d.nc;
        b = bc / d.nc;
        g = h / d.hpg;
        hh = h - g * d.hpg;
    }
    __device__ __forceinline__ void next(const Dims& d) {
        if (++hh == d.hpg) {
            hh = 0;
            ++g;
        }
        if (++h == d.H) {
            h = g = hh = 0;
            if (++c == d.nc) {
                c = 0;
                ++b;
            }
        }
    }
};

template <int Q, bool kI8>
__global__ void __launch_bounds__(kThreads, 1)
chunk_state_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                      Dims d, const float* __restrict__ lut_g, const float* __restrict__ inv_sx_g,
                      const float* __restrict__ mq_g, uint16_t* __restrict__ S,
                      int8_t* __restrict__ S8, I8Debug dbg, int* __restrict__ status) {
    using K = StateCfg<Q, kI8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + K::OFF_BAR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + K::OFF_FLAG);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + K::OFF_TMEM);
    const int units = d.B * d.nc * d.H;
    const int u0 = (int)((long long)units * blockIdx.x / gridDim.x);
    const int u1 = (int)((long long)units * (blockIdx.x + 1) / gridDim.x);

    if (tid == 0) {
        for (int i = 0; i < K::NBAR; ++i) {
            uint32_t cnt = 1;
            if (i >= K::PREP && i < K::PREP + K::NS) cnt = kPrepThreads / 32;
            if (kI8 && i >= K::EMPTY && i < K::EMPTY + K::NS) cnt = kPrepThreads / 32;
            if (i >= K::TEMPTY && i < K::TEMPTY + kAcc) cnt = 4;
            tc::mbar_init(bar + i, cnt);
        }
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, kAcc * 64);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tc::prefetch_tmap(&tm_x);
            tc::prefetch_tmap(&tm_b);
            int k = 0, nbl = 0;
            Cursor un;
            un.init(d, u0);
            for (int u = u0; u < u1; ++u, ++k, un.next(d)) {
                if (u == u0 || un.hh == 0) {
                    const int bs = nbl % K::NB;
                    if (!tc::wait_or_abort(bar + K::BEMPTY + bs, ((uint32_t)(nbl / K::NB) & 1) ^ 1, abort_flag,
                                           status, kStatusTimeout))
                        break;
                    uint8_t* dst = sm + K::OFF_B + bs * K::B_BYTES;
                    tc::mbar_arrive_expect_tx(bar + K::BFULL + bs, K::B_BYTES);
                    tc::tma_load_3d(dst, &tm_b, bar + K::BFULL + bs, un.g * kN, un.c * Q, un.b);
                    if (!kI8) tc::tma_load_3d(dst + Q * 128, &tm_b, bar + K::BFULL + bs, un.g * kN + 64, un.c * Q, un.b);
                    ++nbl;
                }
                const int s = k % K::NS;
                if (!tc::wait_or_abort(bar + K::EMPTY + s, ((uint32_t)(k / K::NS) & 1) ^ 1, abort_flag, status,
                                       kStatusTimeout))
                    break;
                tc::mbar_arrive_expect_tx(bar + K::FULL + s, K::STAGE_TX);
                tc::tma_load_3d(sm + K::OFF_X + s * K::X_BYTES, &tm_x, bar + K::FULL + s, un.h * kP, un.c * Q, un.b);
                const float* lrow = lut_g + (((long long)un.b * d.H + un.h) * d.nc + un.c) * Q;
                tc::bulk_load(sm + K::OFF_LUT + s * Q * 4, lrow, Q * 4, bar + K::FULL + s);
                if (kI8) tc::bulk_load(sm + K::OFF_SX + s * K::SX_BYTES, inv_sx_g + un.h * kP, K::SX_BYTES, bar + K::FULL + s);
            }
            // copies still in flight after an abort must land before the CTA exits
            for (int s = 0; s < K::NS; ++s) {
                const int n = k > s ? (k - 1 - s) / K::NS + 1 : 0;
                if (n > 0) tc::mbar_wait(bar + K::FULL + s, (uint32_t)(n - 1) & 1, tc::kWaitLimit);
            }
            for (int bs = 0; bs < K::NB; ++bs) {
                const int n = nbl > bs ? (nbl - 1 - bs) / K::NB + 1 : 0;
                if (n > 0) tc::mbar_wait(bar + K::BFULL + bs, (uint32_t)(n - 1) & 1, tc::kWaitLimit);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs the schedule and waits; one elected lane issues.
        constexpr int kSteps = kI8 ? Q / 32 : Q / 16;
        const uint32_t idesc = kI8 ? tc::idesc_s8_s32(128, kP, tc::kMajorMN, tc::kMajorMN)
                                   : tc::idesc_bf16_f32(128, kP, tc::kMajorMN, tc::kMajorMN);
        // A = B tile (MN-major, two 64-column blocks Q*128 bytes apart in bf16);
        // B = X_scaled (bf16, 128B swizzle) or Xq (int8, 64B swizzle).  A K step
        // is 16 rows (bf16) or 32 rows (int8) further into both tiles.
        const uint64_t dA0 = kI8 ? tc::smem_desc(tc::smem_u32(sm + K::OFF_B), 0, 1024, tc::kLayoutSw128)
                                 : tc::smem_desc(tc::smem_u32(sm + K::OFF_B), Q * 128, 1024, tc::kLayoutSw128);
        const uint64_t dX0 = kI8 ? tc::smem_desc(tc::smem_u32(sm + K::OFF_XQ), 0, 512, tc::kLayoutSw64)
                                 : tc::smem_desc(tc::smem_u32(sm + K::OFF_X), Q * 128, 1024, tc::kLayoutSw128);
        constexpr uint32_t kStepA = kI8 ? 4096 : 2048, kStepX = 2048;
        constexpr uint32_t kStageX = kI8 ? K::XQ_BYTES : K::X_BYTES;
        int nbl = 0, bs = 0, s = 0, t = 0;
        uint32_t sph = 0, tph = 0;                                 // phase bits of the rings
        Cursor un;
        un.init(d, u0);
        for (int u = u0; u < u1; ++u, un.next(d)) {
            bool ok = true;
            if (u == u0 || un.hh == 0) {
                bs = nbl % K::NB;
                ok = tc::wait_or_abort(bar + K::BFULL + bs, (uint32_t)(nbl / K::NB) & 1, abort_flag, status,
                                       kStatusTimeout);
                ++nbl;
            }
            const bool last_of_b = (u + 1 == u1) || un.hh == d.hpg - 1;
            ok = ok && tc::wait_or_abort(bar + K::PREP + s, sph, abort_flag, status, kStatusTimeout);
            ok = ok && tc::wait_or_abort(bar + K::TEMPTY + t, tph ^ 1, abort_flag, status, kStatusTimeout);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc::tc_fence_after();
            if (tc::elect_one()) {
                const uint64_t dA = dA0 + (uint64_t)((bs * K::B_BYTES) >> 4);
                const uint64_t dX = dX0 + (uint64_t)((s * kStageX) >> 4);
                const uint32_t acc = tmem + (uint32_t)(t * 64);
#pragma unroll
                for (int st = 0; st < kSteps; ++st) {
                    const uint64_t a = dA + (uint64_t)((st * kStepA) >> 4);
                    const uint64_t x = dX + (uint64_t)((st * kStepX) >> 4);
                    if (kI8) tc::mma_i8_ss(acc, a, x, idesc, st > 0 ? 1u : 0u);
                    else tc::mma_f16_ss(acc, a, x, idesc, st > 0 ? 1u : 0u);
                }
                tc::mma_commit(bar + (kI8 ? K::QEMPTY : K::EMPTY) + s);
                tc::mma_commit(bar + K::TFULL + t);
                if (last_of_b) tc::mma_commit(bar + K::BEMPTY + bs);
            }
            __syncwarp();
            if (++s == K::NS) { s = 0; sph ^= 1; }
            if (++t == kAcc) { t = 0; tph ^= 1; }
        }
        // MMAs still running after an abort must finish before TMEM is freed
        if (tc::elect_one()) tc::mma_commit(bar + K::DONE);
        __syncwarp();
        tc::mbar_wait(bar + K::DONE, 0, tc::kWaitLimit);
    } else if (warp < kPrepWarp0) {
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;
        const int n = quarter * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
        // requantisation multipliers of columns p = lane and lane + 32, loaded one unit ahead
        Cursor un;
        un.init(d, u0);
        float m0 = 0.f, m1 = 0.f;
        if (kI8) {
            m0 = __ldg(mq_g + un.h * kP + lane);
            m1 = __ldg(mq_g + un.h * kP + lane + 32);
        }
        int k = 0;
        for (int u = u0; u < u1; ++u, ++k, un.next(d)) {
            const float c0 = m0, c1 = m1;
            if (kI8 && u + 1 < u1) {
                const int h = un.h + 1 < d.H ? un.h + 1 : 0;
                m0 = __ldg(mq_g + h * kP + lane);
                m1 = __ldg(mq_g + h * kP + lane + 32);
            }
            const int t = k % kAcc;
            // the unit's factors, broadcast to the warp through shared memory (16-byte reads)
            float* mqw = reinterpret_cast<float*>(sm + K::OFF_MQ) + quarter * kP;
            if (kI8) {
                __syncwarp();                                          // the previous unit's reads are done
                mqw[lane] = c0;
                mqw[lane + 32] = c1;
                __syncwarp();
            }
            const bool ok = tc::wait_or_abort(bar + K::TFULL + t, (uint32_t)(k / kAcc) & 1, abort_flag, status,
                                              kStatusTimeout);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc::tc_fence_after();
            uint32_t v0[32], v1[32];
            tc::tmem_ld32(trow + t * 64, v0);
            tc::tmem_ld32(trow + t * 64 + 32, v1);
            tc::tmem_wait_ld();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar + K::TEMPTY + t);
            const long long base = (((long long)un.b * d.nc + un.c) * d.H + un.h) * (long long)(kP * kN) + n;
            if (!kI8) {
#pragma unroll
                for (int p = 0; p < kP; ++p)
                    S[base + p * kN] = float_to_bf16_bits(__uint_as_float(p < 32 ? v0[p] : v1[p - 32]));
            } else {
                // |acc| <= Q * 127 * 127 < 2^22; the code's byte is the low byte of code_bits
#pragma unroll
                for (int p = 0; p < kP; p += 2) {
                    const uint32_t a0 = p < 32 ? v0[p] : v1[p - 32], a1 = p < 32 ? v0[p + 1] : v1[p - 31];
                    const float2 mq2 = reinterpret_cast<const float2*>(mqw)[p >> 1];
                    const float mq0 = mq2.x, mq1 = mq2.y;
                    float f0, f1, r0, r1;
                    // int-to-float conversions: they run on a pipe of their own, which is idle here
                    f0 = __int2float_rn((int)a0);
                    f1 = __int2float_rn((int)a1);
                    mul_f32x2(r0, r1, f0, f1, mq0, mq1);
                    int q0, q1;
                    code_bits2(q0, q1, r0, r1);
                    S8[base + p * kN] = (int8_t)q0;
                    S8[base + (p + 1) * kN] = (int8_t)q1;
                }
                if (dbg.acc_state || dbg.S8) {
#pragma unroll
                    for (int p = 0; p < kP; ++p) {
                        const int acc = (int)(p < 32 ? v0[p] : v1[p - 32]);
                        const float mq = __shfl_sync(0xffffffffu, p < 32 ? c0 : c1, p & 31);
                        const int q = code_bits(__fmul_rn(small_int_to_float(acc), mq)) - kRoundBits;
                        if (dbg.acc_state) dbg.acc_state[base + p * kN] = acc;
                        if (dbg.S8) dbg.S8[base + p * kN] = (int8_t)q;
                    }
                }
            }
        }
    } else {
        // ------------------------------------------------------------ prep
        const int pt = tid - kPrepWarp0 * 32;
        // 16-byte chunk pt + kPrepThreads * i holds 8 consecutive p of one row; with 8
        // chunks per 128-byte row and kPrepThreads a multiple of 64, a thread always
        // sees the same swizzle phase, hence the same logical columns p0 .. p0 + 7
        const int p0 = ((pt & 7) ^ ((pt >> 3) & 7)) * 8;
        constexpr int kPer = Q * 8 / kPrepThreads;            // chunks per thread: 2, 4 or 8
        int k = 0;
        Cursor un;
        un.init(d, u0);
        for (int u = u0; u < u1; ++u, ++k, un.next(d)) {
            const int s = k % K::NS;
            bool ok = tc::wait_or_abort(bar + K::FULL + s, (uint32_t)(k / K::NS) & 1, abort_flag, status,
                                        kStatusTimeout);
            // W8A8: the Xq slot must have been read by its previous MMA
            if (kI8) ok = ok && tc::wait_or_abort(bar + K::QEMPTY + s, ((uint32_t)(k / K::NS) & 1) ^ 1, abort_flag,
                                                  status, kStatusTimeout);
            if (!__all_sync(0xffffffffu, ok)) break;
            const float* lut = reinterpret_cast<const float*>(sm + K::OFF_LUT + s * Q * 4);
            uint8_t* xt = sm + K::OFF_X + s * K::X_BYTES;
            float inv_sx[8];
            if (kI8) {
                const float4* sx4 = reinterpret_cast<const float4*>(sm + K::OFF_SX + s * K::SX_BYTES + p0 * 4);
                const float4 a0 = sx4[0], a1 = sx4[1];
                inv_sx[0] = a0.x; inv_sx[1] = a0.y; inv_sx[2] = a0.z; inv_sx[3] = a0.w;
                inv_sx[4] = a1.x; inv_sx[5] = a1.y; inv_sx[6] = a1.z; inv_sx[7] = a1.w;
            }
            // all loads first: the chunks are independent, so their latencies overlap
            uint4 v[kPer];
            float f[kPer];
#pragma unroll
            for (int i = 0; i < kPer; ++i) {
                const int ck = pt + i * kPrepThreads;
                v[i] = *reinterpret_cast<const uint4*>(xt + ck * 16);
                f[i] = lut[ck >> 3];
            }
#pragma unroll
            for (int i = 0; i < kPer; ++i) {
                const int ck = pt + i * kPrepThreads, row = ck >> 3;
                const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
                if (!kI8) {
                    uint32_t o[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        o[e] = pack_bf16(__uint_as_float(w[e] << 16) * f[i], __uint_as_float(w[e] & 0xffff0000u) * f[i]);
                    *reinterpret_cast<uint4*>(xt + ck * 16) = make_uint4(o[0], o[1], o[2], o[3]);
                } else {
                    int q[8];
#pragma unroll
                    for (int e = 0; e < 8; e += 2) {
                        // X_scaled = LUT * x and X_scaled / s_x, both rounded fp32 products, two lanes at once
                        float xs0, xs1, v0, v1;
                        mul_f32x2(xs0, xs1, f[i], f[i], __uint_as_float(w[e >> 1] << 16),
                                  __uint_as_float(w[e >> 1] & 0xffff0000u));
                        mul_f32x2(v0, v1, xs0, xs1, inv_sx[e], inv_sx[e + 1]);
                        code_bits2(q[e], q[e + 1], v0, v1);
                    }
                    const uint2 qq = make_uint2(pack_i8x4(q[0], q[1], q[2], q[3]), pack_i8x4(q[4], q[5], q[6], q[7]));
                    // 64-byte swizzle: 16-byte chunk index (p / 16) XOR address bits 7..8
                    const int off = row * 64 + (((p0 >> 4) ^ ((row >> 1) & 3)) << 4) + (p0 & 15);
                    *reinterpret_cast<uint2*>(sm + K::OFF_XQ + s * K::XQ_BYTES + off) = qq;
                    if (dbg.Xq) {
                        const long long tok = (long long)un.c * Q + row;
                        *reinterpret_cast<uint2*>(dbg.Xq + (((long long)un.b * d.Lp() + tok) * d.H + un.h) * kP +
                                                  p0) = qq;
                    }
                }
            }
            tc::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                if (kI8) tc::mbar_arrive(bar + K::EMPTY + s);          // x tile read: the slot may refill
                tc::mbar_arrive(bar + K::PREP + s);
            }
        }
    }
    __syncwarp();
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(tmem, kAcc * 64);
}

template <int Q, bool kI8>
cudaError_t launch_q(const Dims& d, const CUtensorMap& tx, const CUtensorMap& tb, const float* lut,
                     const float* inv_sx, const float* mq, uint16_t* S, int8_t* S8, const I8Debug* dbg, int* status,
                     cudaStream_t st) {
    using K = StateCfg<Q, kI8>;
    auto k = chunk_state_tc_kernel<Q, kI8>;
    const int smem = K::BYTES + 1024;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const long long units = (long long)d.B * d.nc * d.H;
    const int sms = device_sm_count();
    const int grid = (int)(units < sms ? units : sms);
    I8Debug none{};
    k<<<grid, kThreads, smem, st>>>(tx, tb, d, lut, inv_sx, mq, S, S8, dbg ? *dbg : none, status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_state_tc(const Dims& d, bool i8, const uint16_t* x, const void* Bmat,
                                  const float* lut, const float* inv_sx, const float* mq, uint16_t* S,
                                  int8_t* S8, const I8Debug* dbg, int* status, cudaStream_t st) {
    if (d.B == 0 || d.nc == 0) return cudaSuccess;
    if (d.P != kP || d.N != kN) return cudaErrorInvalidValue;
    if ((long long)d.B * d.nc * d.H > 0x7fffffffLL) return cudaErrorInvalidValue;
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
        case 64: return i8 ? launch_q<64, true>(d, tx, tb, lut, inv_sx, mq, S, S8, dbg, status, st)
                           : launch_q<64, false>(d, tx, tb, lut, inv_sx, mq, S, S8, dbg, status, st);
        case 128: return i8 ? launch_q<128, true>(d, tx, tb, lut, inv_sx, mq, S, S8, dbg, status, st)
                            : launch_q<128, false>(d, tx, tb, lut, inv_sx, mq, S, S8, dbg, status, st);
        case 256: return i8 ? launch_q<256, true>(d, tx, tb, lut, inv_sx, mq, S, S8, dbg, status, st)
                            : launch_q<256, false>(d, tx, tb, lut, inv_sx, mq, S, S8, dbg, status, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace ssd
