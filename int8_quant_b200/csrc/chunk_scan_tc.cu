// chunk_scan_tc.cu — a4..a7 on the tensor cores (P = 64, N = 128): ChunkBMM,
// ChunkScan1, ChunkScan2 and the D skip (SSDi8 notes, "overall framework" and key
// design 2):
//   CB[j,i]  = C_j . B_i                                        (ChunkBMM)
//   y[j,p]   = exp(Acs_j) sum_n C[j,n] H_c[p,n]                   (ChunkScan1)
//            + sum_{i<=j} CB[j,i] exp(Acs_j - Acs_i) dt_i x[i,p]    (ChunkScan2)
//            + D x[j,p]
// W8A8: CB and the ChunkScan1 sum are int32 (kind::i8 on Cq, Bq, H8); ChunkScan1 is
// dequantised with s_C s_s[h,p]; LUT_Scan2 = s_C s_B exp(Acs_j - Acs_i) dt_i folds
// CB's dequantisation into the ChunkScan2 matrix, which runs in bf16 (kind::f16).
//
// One CTA per (chunk, batch row, block of heads of one group; the block size comes from
// the caller's wave-count model, 20 heads at the Mamba-2 2.7B shape); B and C are
// shared by the block, so CB is computed once and kept in TMEM, packed to bf16
// pairs, for all heads.  The work is split over warp roles that run concurrently
// and hand off through mbarriers:
//   warp 0      TMA producer: per head the decay rows (Acs, dt), the state tile and
//               the x tile (two stages in bf16, three in W8A8, whose shared memory
//               has room: two heads' loads in flight ahead of the MMAs), plus C and B
//               once.
//   warp 1      TMEM allocation and the single MMA-issuing thread: CB; per head
//               y = C H^T into one of two TMEM accumulator slots (issued as soon as
//               the slot is free, ahead of the previous head's remaining work, since
//               the tensor pipe executes in order), then y += M x over the pieces of
//               the masked matrix as they arrive.
//   warps 2-9   builders: M[j,i] = CB[j,i] exp(Acs_j - Acs_i) dt_i, 64 columns per
//               piece, into a 2-slot ring in TMEM (bf16 pairs), which the y += M x
//               MMAs read as their A operand: M never touches shared memory, whose
//               bandwidth (128 B/clk) the skinny N = 64 MMAs already saturate.  All
//               eight warps build each piece, one 32 x 32 block each.  Below the
//               32-row diagonal blocks the decay factorises through the end r of the
//               block's columns, exp(Acs_j - Acs_r) * exp(Acs_r - Acs_i), both <= 1, so
//               only the diagonal blocks take an exponential per element.
//   warps 10-13 scalers: ChunkScan1 rows times exp(Acs_j) in TMEM (W8A8: dequantise).
//   warps 14-17 storers: y + D x, rounded to bf16 over the x tile, stored by TMA
//               (a warp's rows are 10 KB apart in y, so stores from registers would
//               not coalesce).
// Every wait is bounded; an expired wait raises a shared abort flag that ends all
// roles, records SSD_ERR_TIMEOUT in the status word, and the CTA frees TMEM.
//
// The notes' storage variant (W8A8, chunk 256): with kCB8 the CTA loads the INT8 CB
// codes that chunk_bmm.cu wrote (one step per tile, folded into the decay vectors)
// into the B tile's space instead of forming CB, and the builders widen them to bf16;
// with acs_half the Acs rows arrive as IEEE half and are widened when the decay
// vectors are formed.
#include <cuda_fp16.h>

#include "kernels.h"
#include "tc.cuh"

namespace ssd {

namespace {

constexpr int kP = 64;
constexpr int kN = 128;
constexpr int kWarps = 18;
constexpr int kThreads = kWarps * 32;
constexpr int kBuilderWarp0 = 2;
constexpr int kBuilderThreads = 256;
constexpr int kScaleWarp0 = 10;
constexpr int kStoreWarp0 = 14;
constexpr int kEpiThreads = 128;
constexpr int kRing = 2;
constexpr float kLog2e = 1.4426950408889634f;
enum : uint32_t { kIdBuild = 1, kIdScale = 2, kIdStore = 3 };

// kCB8 (W8A8, Q = 256; the notes' storage variant): ChunkScan2 reads CB as the INT8
// codes ChunkBMM wrote to HBM (one step per tile) instead of forming CB on chip; the
// B tile's space holds those codes and no ChunkBMM runs here.
template <int Q, bool kI8, bool kCB8 = false>
struct Cfg {
    static constexpr int JT = Q >= 128 ? Q / 128 : 1;            // 128-row tiles of the chunk
    static constexpr int CROWS = Q >= 128 ? Q : 128;             // C rows loaded (Q = 64: ghost rows)
    static constexpr int NCB0 = Q >= 128 ? 128 : Q;              // CB columns of tile 0
    static constexpr int NPIECE = JT == 2 ? 6 : NCB0 / 64;       // 64-column pieces of M per head
    // TMEM columns: packed CB of tile 1 at [0, 128) and of tile 0 at [128, 192), the M
    // ring at [192, 256), y slots at 256 + 128 s.  Before packing, the fp32 CB
    // accumulators use [128, 256) (tile 0) and [256, 512) (tile 1); tile 0 is packed in
    // place, each 32-column step writing over columns it has already read.
    static constexpr uint32_t CBF = 128, CBP0 = 128, CBP1 = 0, RING = 192, YCOL = 256, TMEM_COLS = 512;
    static constexpr int EB = kI8 ? 1 : 2;
    static constexpr int C_BYTES = CROWS * kN * EB;
    static constexpr int B_BYTES = kCB8 ? Q * Q : Q * kN * EB;
    static constexpr int H_BYTES = kP * kN * EB;
    static constexpr int NHB = kI8 ? 2 : 1;                      // state tile buffers
    static constexpr int X_BYTES = Q * 128;
    // x stages (each also holds its head's y until the store has read it): three when
    // shared memory allows, so that two heads' loads can be in flight ahead of the MMAs
    static constexpr int NXS = kI8 ? 3 : 2;
    static constexpr int OFF_C = 0;
    static constexpr int OFF_B = C_BYTES;
    static constexpr int OFF_X = (OFF_B + B_BYTES + 1023) & ~1023;
    static constexpr int OFF_H = OFF_X + NXS * X_BYTES;
    static constexpr int OFF_VEC = OFF_H + NHB * H_BYTES;        // 2 slots x {acs, dtc, a2, vB, dtw}[Q]
    static constexpr int VEC_SLOT = (kI8 ? 6 : 5) * Q * 4;
    static constexpr int OFF_BAR = OFF_VEC + 2 * VEC_SLOT;
    // barriers
    static constexpr int B_LOAD = 0, B_CB = 1, B_PACKED = 2, B_XFULL = 3, B_XEMPTY = 3 + NXS,
                         B_HFULL = 3 + 2 * NXS, B_HEMPTY = B_HFULL + 2, B_VFULL = B_HEMPTY + 2,
                         B_VEMPTY = B_VFULL + 2, B_RFULL = B_VEMPTY + 2, B_REMPTY = B_RFULL + kRing,
                         B_YOFULL = B_RFULL + 2 * kRing, B_YSCALED = B_YOFULL + 2, B_YFULL = B_YOFULL + 4,
                         B_YEMPTY = B_YOFULL + 6, B_VPREP = B_YOFULL + 8, NBAR = B_YOFULL + 10;
    static constexpr int OFF_FLAG = OFF_BAR + NBAR * 8;
    static constexpr int OFF_TMEM = OFF_FLAG + 8;
    static constexpr int BYTES = OFF_TMEM + 8;
};

__device__ __forceinline__ void piece_of(int Q, int k, int& J, int& ib) {
    if (Q == 256) {
        J = k < 2 ? 0 : 1;
        ib = k < 2 ? k : k - 2;
    } else {
        J = 0;
        ib = k;
    }
}

// Bounded mbarrier wait that gives up early once another role has aborted.  With
// kBackoff a failed poll sleeps 20 ns before the next: in the W8A8 instantiation the
// polls of waiting roles slowed the others measurably (a few per cent of the kernel);
// in the bf16 one the sleep cost more than it saved.
template <bool kBackoff = false>
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status) {
    const long long t0 = clock64();
    while (!tc::mbar_try_wait(bar, parity)) {
        if (*abort_flag) return false;
        if (clock64() - t0 > tc::kWaitLimit) {
            *abort_flag = 1;
            if (status) atomicExch(status, kStatusTimeout);
            return false;
        }
        if (kBackoff) __nanosleep(20);
    }
    return true;
}

// 2^x with the MUFU instruction (relative error about 2^-22); x <= 0 here, so the
// result is in (0, 1] and never overflows.
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Two IEEE fp32 additions (round to nearest even) in one packed instruction.
__device__ __forceinline__ void add_f32x2(float& r0, float& r1, float a0, float a1, float b0, float b1) {
    asm("{\n\t.reg .b64 a, b, r;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
        "add.rn.f32x2 r, a, b;\n\tmov.b64 {%0, %1}, r;\n\t}"
        : "=f"(r0), "=f"(r1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void mul_f32x2(float& r0, float& r1, float a0, float a1, float b0, float b1) {
    asm("{\n\t.reg .b64 a, b, r;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
        "mul.rn.f32x2 r, a, b;\n\tmov.b64 {%0, %1}, r;\n\t}"
        : "=f"(r0), "=f"(r1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
// r = a * b + c on fp32 pairs, fused, round to nearest even
__device__ __forceinline__ void fma_f32x2(float& r0, float& r1, float a0, float a1, float b0, float b1, float c0,
                                          float c1) {
    asm("{\n\t.reg .b64 a, b, c, r;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
        "mov.b64 c, {%6, %7};\n\tfma.rn.f32x2 r, a, b, c;\n\tmov.b64 {%0, %1}, r;\n\t}"
        : "=f"(r0), "=f"(r1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ float lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// float(a) for |a| < 2^22, exactly, without a conversion instruction: 1.5 * 2^23 + a is
// representable, so its bit pattern is 0x4B400000 + a.  The int32 accumulators here are
// sums of at most 128 products of INT8 codes, |a| <= 128 * 127 * 127 < 2^22.
__device__ __forceinline__ float small_int_to_float(uint32_t a) {
    return __fsub_rn(__int_as_float((int)a + 0x4B400000), 12582912.0f);
}

// Two bf16 products (round to nearest even) in one packed instruction.
__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// Sixteen INT8 codes (one 16-byte word, first code in the lowest byte) as eight bf16
// pairs: each code is exact in fp32 and in bf16 (at most 8 significant bits), so the
// bf16 bits are the upper half of the fp32 bits.
__device__ __forceinline__ void i8x16_to_bf16x8(const uint4 q, uint32_t (&o)[8]) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const uint32_t word = w[e >> 1] >> (16 * (e & 1));
        const float lo = (float)(int)(int8_t)(word & 0xffu), hi = (float)(int)(int8_t)((word >> 8) & 0xffu);
        o[e] = __byte_perm(__float_as_uint(lo), __float_as_uint(hi), 0x7632);
    }
}

template <int Q, bool kI8, bool kCB8>
__global__ void __launch_bounds__(kThreads, 1)
chunk_scan_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_h,
                     const __grid_constant__ CUtensorMap tm_y, Dims d, int heads_per_cta, int ctas_per_group,
                     const float* __restrict__ Acs, const float* __restrict__ dtc, const float* __restrict__ Dv,
                     I8Scales sc, I8Debug dbg, int* __restrict__ status, const float* __restrict__ s_cb,
                     int acs_half) {
    using K = Cfg<Q, kI8, kCB8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c = blockIdx.y, b = blockIdx.z;
    const int g = blockIdx.x / ctas_per_group;
    const int h0 = g * d.hpg + (blockIdx.x % ctas_per_group) * heads_per_cta;
    const int nh = min(heads_per_cta, g * d.hpg + d.hpg - h0);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + K::OFF_BAR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + K::OFF_FLAG);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + K::OFF_TMEM);
    const long long vec_row0 = (((long long)b * d.H) * d.nc + c) * Q;   // + h * nc * Q
    const long long hc_row0 = ((long long)b * d.nc + c) * d.H;           // state rows (hc_row0 + h) * 64
    float sCB = kI8 ? __fmul_rn(__ldg(sc.s_C + g), __ldg(sc.s_B + g)) : 1.f;
    if (kCB8) sCB = __fmul_rn(sCB, __ldg(s_cb + ((long long)b * d.nc + c) * d.G + g));   // the CB codes' step

    if (tid == 0) {
        for (int i = 0; i < K::NBAR; ++i) {
            uint32_t cnt = 1;
            if (i == K::B_PACKED) cnt = 8;
            if (i >= K::B_VEMPTY && i < K::B_VEMPTY + 2) cnt = 12;
            if (i >= K::B_RFULL && i < K::B_RFULL + kRing) cnt = 8;
            if (i >= K::B_YSCALED && i < K::B_YSCALED + 2) cnt = 4;
            if (i >= K::B_YEMPTY && i < K::B_YEMPTY + 2) cnt = 4;
            if (i >= K::B_VPREP && i < K::B_VPREP + 2) cnt = 4;
            tc::mbar_init(bar + i, cnt);
        }
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, K::TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto vec = [&](int s, int which) -> float* {
        return reinterpret_cast<float*>(sm + K::OFF_VEC + s * K::VEC_SLOT + which * Q * 4);
    };
    enum { kAcs = 0, kDtc = 1, kA2 = 2, kVB = 3, kDtw = 4, kMul = 5 };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tc::prefetch_tmap(&tm_x);
            tc::prefetch_tmap(&tm_b);
            tc::prefetch_tmap(&tm_c);
            tc::prefetch_tmap(&tm_h);
            tc::prefetch_tmap(&tm_y);
            tc::mbar_arrive_expect_tx(bar + K::B_LOAD, K::C_BYTES + K::B_BYTES);
            if (!kI8) {
                tc::tma_load_3d(sm + K::OFF_C, &tm_c, bar + K::B_LOAD, g * kN, c * Q, b);
                tc::tma_load_3d(sm + K::OFF_C + K::CROWS * 128, &tm_c, bar + K::B_LOAD, g * kN + 64, c * Q, b);
                tc::tma_load_3d(sm + K::OFF_B, &tm_b, bar + K::B_LOAD, g * kN, c * Q, b);
                tc::tma_load_3d(sm + K::OFF_B + Q * 128, &tm_b, bar + K::B_LOAD, g * kN + 64, c * Q, b);
            } else if (!kCB8) {
                tc::tma_load_3d(sm + K::OFF_C, &tm_c, bar + K::B_LOAD, g * kN, c * Q, b);
                tc::tma_load_3d(sm + K::OFF_B, &tm_b, bar + K::B_LOAD, g * kN, c * Q, b);
            } else {
                // the (b, c, g) CB codes as two 128-column halves, 128-byte swizzle
                const int crow = (int)((((long long)b * d.nc + c) * d.G + g) * Q);
                tc::tma_load_3d(sm + K::OFF_C, &tm_c, bar + K::B_LOAD, g * kN, c * Q, b);
                tc::tma_load_2d(sm + K::OFF_B, &tm_b, bar + K::B_LOAD, 0, crow);
                tc::tma_load_2d(sm + K::OFF_B + Q * 128, &tm_b, bar + K::B_LOAD, 128, crow);
            }
            for (int it = 0; it < nh; ++it) {
                const int h = h0 + it, s = it & 1;
                const uint32_t u = (uint32_t)(it >> 1);
                if (!wait_bar<kI8>(bar + K::B_VEMPTY + s, (u & 1) ^ 1, abort_flag, status)) break;
                const int acs_bytes = acs_half ? Q * 2 : Q * 4;
                tc::mbar_arrive_expect_tx(bar + K::B_VFULL + s, acs_bytes + Q * 4);
                const long long vr = vec_row0 + (long long)h * d.nc * Q;
                tc::bulk_load(vec(s, kAcs), reinterpret_cast<const uint8_t*>(Acs) + vr * (acs_half ? 2 : 4), acs_bytes,
                              bar + K::B_VFULL + s);
                tc::bulk_load(vec(s, kDtc), dtc + vr, Q * 4, bar + K::B_VFULL + s);
                const int hb = kI8 ? s : 0;
                const uint32_t hpar = kI8 ? ((u & 1) ^ 1) : (((uint32_t)it & 1) ^ 1);
                if (!wait_bar<kI8>(bar + K::B_HEMPTY + hb, hpar, abort_flag, status)) break;
                tc::mbar_arrive_expect_tx(bar + K::B_HFULL + hb, K::H_BYTES);
                const int hrow = (int)((hc_row0 + h) * kP);
                uint8_t* hdst = sm + K::OFF_H + hb * K::H_BYTES;
                tc::tma_load_2d(hdst, &tm_h, bar + K::B_HFULL + hb, 0, hrow);
                if (!kI8) tc::tma_load_2d(hdst + kP * 128, &tm_h, bar + K::B_HFULL + hb, 64, hrow);
                const int xst = it % K::NXS;
                const uint32_t xu = (uint32_t)(it / K::NXS);
                if (!wait_bar<kI8>(bar + K::B_XEMPTY + xst, (xu & 1) ^ 1, abort_flag, status)) break;
                tc::mbar_arrive_expect_tx(bar + K::B_XFULL + xst, K::X_BYTES);
                tc::tma_load_3d(sm + K::OFF_X + xst * K::X_BYTES, &tm_x, bar + K::B_XFULL + xst, h * kP, c * Q, b);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs the schedule, so that its values stay warp-uniform, and
        // one elected lane issues; every readiness test is made uniform with a vote.
        // Descriptors are precomputed and advanced by constant adds.  (Adding off >> 4
        // to a descriptor moves its start address by `off` bytes; addresses stay
        // inside shared memory, so the 14-bit field never carries.)
        constexpr int kSteps = kI8 ? 4 : 8;                      // K = 128 (n)
        const uint64_t dC = tc::smem_desc(tc::smem_u32(sm + K::OFF_C), 16, 1024, tc::kLayoutSw128);
        const uint64_t dB = tc::smem_desc(tc::smem_u32(sm + K::OFF_B), 16, 1024, tc::kLayoutSw128);
        const uint64_t dH0 = tc::smem_desc(tc::smem_u32(sm + K::OFF_H), 16, 1024, tc::kLayoutSw128);
        const uint64_t dX0 = tc::smem_desc(tc::smem_u32(sm + K::OFF_X), 0, 1024, tc::kLayoutSw128);
        // byte offset of K step s inside a K-major tile whose 128-byte atoms hold `rows` rows
        auto koff = [](int s, int rows) -> uint32_t {
            return kI8 ? (uint32_t)(s * 32) : (uint32_t)((s >> 2) * rows * 128 + (s & 3) * 32);
        };
        auto wait_all = [&](int which, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, wait_bar<kI8>(bar + which, parity, abort_flag, status));
        };
        auto ready = [&](int which, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, tc::mbar_test(bar + which, parity));
        };
        bool ok = wait_all(K::B_LOAD, 0);
        if (ok && kCB8) {
            // the CB codes are in shared memory: no ChunkBMM here
            if (tc::elect_one()) tc::mbar_arrive(bar + K::B_CB);
            __syncwarp();
            ok = wait_all(K::B_PACKED, 0);
        } else if (ok) {
            tc::tc_fence_after();
            if (tc::elect_one()) {
                const uint32_t id0 = kI8 ? tc::idesc_s8_s32(128, K::NCB0, tc::kMajorK, tc::kMajorK)
                                         : tc::idesc_bf16_f32(128, K::NCB0, tc::kMajorK, tc::kMajorK);
#pragma unroll
                for (int st = 0; st < kSteps; ++st) {
                    const uint64_t a = dC + (koff(st, K::CROWS) >> 4), bb = dB + (koff(st, Q) >> 4);
                    if (kI8) tc::mma_i8_ss(tmem + K::CBF, a, bb, id0, st > 0);
                    else tc::mma_f16_ss(tmem + K::CBF, a, bb, id0, st > 0);
                }
                if (K::JT == 2) {
                    const uint32_t id1 = kI8 ? tc::idesc_s8_s32(128, 256, tc::kMajorK, tc::kMajorK)
                                             : tc::idesc_bf16_f32(128, 256, tc::kMajorK, tc::kMajorK);
#pragma unroll
                    for (int st = 0; st < kSteps; ++st) {
                        const uint64_t a = dC + ((128 * 128 + koff(st, K::CROWS)) >> 4), bb = dB + (koff(st, Q) >> 4);
                        if (kI8) tc::mma_i8_ss(tmem + K::CBF + 128, a, bb, id1, st > 0);
                        else tc::mma_f16_ss(tmem + K::CBF + 128, a, bb, id1, st > 0);
                    }
                }
                tc::mma_commit(bar + K::B_CB);
            }
            __syncwarp();
            ok = wait_all(K::B_PACKED, 0);
        }
        const uint32_t id_o = kI8 ? tc::idesc_s8_s32(128, kP, tc::kMajorK, tc::kMajorK)
                                  : tc::idesc_bf16_f32(128, kP, tc::kMajorK, tc::kMajorK);
        const uint32_t id_d = tc::idesc_bf16_f32(128, kP, tc::kMajorK, tc::kMajorMN);
        // ChunkScan1 of head `yo` into slot yo & 1, once that slot and the state tile
        // are ready; `block` waits for them, otherwise the call only checks.
        int yo = 0;
        auto issue_yo = [&](bool block) -> bool {
            const int s = yo & 1;
            const uint32_t u = (uint32_t)(yo >> 1);
            const int hb = kI8 ? s : 0;
            const uint32_t hpar = kI8 ? (u & 1) : ((uint32_t)yo & 1);
            if (block) {
                if (!wait_all(K::B_YEMPTY + s, (u & 1) ^ 1)) return false;
                if (!wait_all(K::B_HFULL + hb, hpar)) return false;
            } else if (!ready(K::B_YEMPTY + s, (u & 1) ^ 1) || !ready(K::B_HFULL + hb, hpar)) {
                return true;                                      // not yet: try again later
            }
            tc::tc_fence_after();
            if (tc::elect_one()) {
                const uint64_t dH = dH0 + (uint64_t)((hb * K::H_BYTES) >> 4);
                const uint32_t ycol = tmem + K::YCOL + 128 * s;
#pragma unroll
                for (int J = 0; J < K::JT; ++J)
#pragma unroll
                    for (int st = 0; st < kSteps; ++st) {
                        const uint64_t a = dC + ((J * 128 * 128 + koff(st, K::CROWS)) >> 4);
                        const uint64_t bb = dH + (koff(st, kP) >> 4);
                        if (kI8) tc::mma_i8_ss(ycol + 64 * J, a, bb, id_o, st > 0);
                        else tc::mma_f16_ss(ycol + 64 * J, a, bb, id_o, st > 0);
                    }
                tc::mma_commit(bar + K::B_YOFULL + s);
                tc::mma_commit(bar + K::B_HEMPTY + hb);
            }
            __syncwarp();
            ++yo;
            return true;
        };
        int p = 0;                                                // ring piece counter
        for (int it = 0; ok && it < nh; ++it) {
            const int s = it & 1;
            const uint32_t u = (uint32_t)(it >> 1);
            if (yo == it && !(ok = issue_yo(true))) break;
            // waiting for this head's scaling: meanwhile start the next head's ChunkScan1
            // one look at the next head's ChunkScan1, then a suspending wait (no spinning:
            // the builders share this warp's scheduler)
            if (yo == it + 1 && yo < nh && !(ok = issue_yo(false))) break;
            if (!(ok = wait_all(K::B_YSCALED + s, u & 1))) break;
            const int xst = it % K::NXS;
            if (!(ok = wait_all(K::B_XFULL + xst, (uint32_t)(it / K::NXS) & 1))) break;
            const uint64_t dX = dX0 + (uint64_t)((xst * K::X_BYTES) >> 4);
            const uint32_t ycol = tmem + K::YCOL + 128 * s;
            for (int k = 0; k < K::NPIECE; ++k, ++p) {
                int J, ib;
                piece_of(Q, k, J, ib);
                const int slot = p & (kRing - 1);
                const uint32_t rpar = (uint32_t)((p / kRing) & 1);
                // W8A8: the next head's (cheaper, int8) ChunkScan1 may go between the pieces
                if (kI8 && yo == it + 1 && yo < nh && !(ok = issue_yo(false))) break;
                if (!(ok = wait_all(K::B_RFULL + slot, rpar))) break;
                tc::tc_fence_after();
                if (tc::elect_one()) {
                    const uint32_t am = tmem + K::RING + slot * 32;      // 64 bf16 = 32 columns
                    const uint64_t db = dX + (uint64_t)(ib * 512);        // x rows ib*64: 64*128 B >> 4
                    const uint32_t dcol = ycol + 64 * J;
#pragma unroll
                    for (int st = 0; st < 4; ++st) tc::mma_f16_ts(dcol, am + st * 8, db + st * 128, id_d, 1u);
                    tc::mma_commit(bar + K::B_REMPTY + slot);
                }
                __syncwarp();
            }
            if (!ok) break;
            if (tc::elect_one()) tc::mma_commit(bar + K::B_YFULL + s);
            // bf16: the next head's ChunkScan1 goes behind this head's pieces in the tensor pipe
            if (!kI8 && yo == it + 1 && yo < nh && !(ok = issue_yo(false))) break;
            __syncwarp();
        }
    } else if (warp < kScaleWarp0) {
        // ------------------------------------------------------------ builders
        const int set = (warp - kBuilderWarp0) >> 2;
        const int quarter = warp & 3;
        const int rrow = quarter * 32 + lane;                 // row within a 128-row tile
        const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
        bool ok = tc::named_and(kIdBuild, kBuilderThreads, wait_bar<kI8>(bar + K::B_CB, 0, abort_flag, status));
        tc::tc_fence_after();
        if (ok && set == 0 && !kCB8) {
            if (kI8 && dbg.cb && (blockIdx.x % ctas_per_group) == 0) {
                for (int J = 0; J < K::JT; ++J) {
                    const int ncol = J == 0 ? K::NCB0 : 256;
                    const int j = J * 128 + rrow;
                    for (int g32 = 0; g32 < ncol / 32; ++g32) {
                        uint32_t v[32];
                        tc::tmem_ld32(trow + K::CBF + (J == 0 ? 0 : 128) + g32 * 32, v);
                        tc::tmem_wait_ld();
                        if (j < Q) {
                            int32_t* dst = dbg.cb + ((((long long)b * d.nc + c) * d.G + g) * Q + j) * Q + g32 * 32;
#pragma unroll
                            for (int i = 0; i < 32; ++i) dst[i] = (int32_t)v[i];
                        }
                    }
                }
            }
        }
        if (ok) {
            // pack CB to bf16 pairs: tile 0 by set 0, tile 1 by set 1 (both in parallel;
            // the destinations do not overlap the other set's source columns)
            const int J = set;
            if (J < K::JT && !kCB8) {
                const int ncol = J == 0 ? K::NCB0 : 256;
                for (int g32 = 0; g32 < ncol / 32; ++g32) {
                    uint32_t v[32], w[16];
                    tc::tmem_ld32(trow + K::CBF + (J == 0 ? 0 : 128) + g32 * 32, v);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float lo = kI8 ? small_int_to_float(v[2 * i]) : __uint_as_float(v[2 * i]);
                        const float hi = kI8 ? small_int_to_float(v[2 * i + 1]) : __uint_as_float(v[2 * i + 1]);
                        w[i] = pack_bf16(lo, hi);
                    }
                    tc::tmem_st16(trow + (J == 0 ? K::CBP0 : K::CBP1) + g32 * 16, w);
                }
            }
            tc::tmem_wait_st();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar + K::B_PACKED);
        }
        ok = tc::named_and(kIdBuild, kBuilderThreads, ok && wait_bar<kI8>(bar + K::B_PACKED, 0, abort_flag, status));
        tc::tc_fence_after();
        // Every piece is built by all eight warps.  Warp (set, quarter) owns the 32
        // rows of its TMEM lane quarter and, of the piece's four 16-column groups, the
        // groups set and set + 2, i.e. columns [16 set, 16 set + 16) of each of the
        // piece's two 32-column blocks (so that the diagonal blocks' work is shared by
        // both warps of a quarter).  Per 32 x 32 block of M: below the diagonal the decay
        // factorises through the end r of the block's columns,
        // exp(Acs_j - Acs_r) * exp(Acs_r - Acs_i) (both <= 1); on the diagonal it takes
        // one exponential per element; above it is zero.  The next piece's CB columns
        // are loaded from TMEM while the current piece is computed.
        const int c0 = 16 * set;                                  // first column within a block
        // diagonal blocks: which halves of this row's column pairs (c0 + 2k, c0 + 2k + 1)
        // lie on or below the diagonal (column <= row = lane)
        uint32_t dmask[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int c = c0 + 2 * k;
            dmask[k] = c + 1 <= lane ? 0xffffffffu : (c == lane ? 0x0000ffffu : 0u);
        }
        int p = 0;
        for (int it = 0; ok && it < nh; ++it) {
            const int s = it & 1;
            const uint32_t u = (uint32_t)(it >> 1);
            // the scalers have prepared the head's decay vectors
            ok = __all_sync(0xffffffffu, wait_bar<kI8>(bar + K::B_VPREP + s, u & 1, abort_flag, status));
            if (!ok) break;
            const float* a2 = vec(s, kA2);
            const float* v32 = vec(s, kVB);
            const float* dtw = vec(s, kDtw);
            auto cb_cols = [&](int k) -> uint32_t {
                int J, ib;
                piece_of(Q, k, J, ib);
                return trow + (J == 0 ? K::CBP0 : K::CBP1) + ib * 32 + c0 / 2;
            };
            // one 16-column group of block `cb` (columns i0 + c0 .. i0 + c0 + 15)
            auto build16 = [&](const uint32_t (&v)[8], int jb, int cb, float aj, uint32_t (&out)[8]) {
                const int i0 = 32 * cb + c0;
                if (jb > cb) {
                    // row factor and column factors as bf16 pairs: two bf16x2 products per pair
                    const float uj = ex2(fminf(aj - a2[32 * cb + 31], 0.f));
                    const uint32_t ub = pack_bf16(uj, uj);
                    const uint4* v4 = reinterpret_cast<const uint4*>(reinterpret_cast<const uint32_t*>(v32) + i0 / 2);
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const uint4 f = v4[q];
                        out[4 * q] = mul_bf16x2(v[4 * q], mul_bf16x2(ub, f.x));
                        out[4 * q + 1] = mul_bf16x2(v[4 * q + 1], mul_bf16x2(ub, f.y));
                        out[4 * q + 2] = mul_bf16x2(v[4 * q + 2], mul_bf16x2(ub, f.z));
                        out[4 * q + 3] = mul_bf16x2(v[4 * q + 3], mul_bf16x2(ub, f.w));
                    }
                } else if (jb == cb) {
                    // exp(Acs_j - Acs_i) dt_i = 2^(a_j + (log2(dt_i) - a_i)), the column term
                    // prepared per head; masked entries (column > row) may overflow to inf
                    // and are cleared bitwise by the row's pair masks
                    const float4* l4 = reinterpret_cast<const float4*>(dtw + i0);
#pragma unroll
                    for (int e4 = 0; e4 < 4; ++e4) {
                        const float4 lv = l4[e4];
                        float x0, x1, x2, x3;
                        add_f32x2(x0, x1, aj, aj, lv.x, lv.y);
                        add_f32x2(x2, x3, aj, aj, lv.z, lv.w);
                        out[2 * e4] = mul_bf16x2(v[2 * e4], pack_bf16(ex2(x0), ex2(x1))) & dmask[2 * e4];
                        out[2 * e4 + 1] = mul_bf16x2(v[2 * e4 + 1], pack_bf16(ex2(x2), ex2(x3))) & dmask[2 * e4 + 1];
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) out[e] = 0u;
                }
            };
            // kCB8: the piece's two 16-code groups of row J*128 + rrow from the swizzled tile
            auto cb8_load = [&](int k, uint32_t (&o0)[8], uint32_t (&o1)[8]) {
                int J, ib;
                piece_of(Q, k, J, ib);
                const int row = J * 128 + rrow;
#pragma unroll
                for (int blk = 0; blk < 2; ++blk) {
                    const int col = 32 * (2 * ib + blk) + c0;
                    const int phys = ((col & 127) >> 4) ^ (row & 7);
                    const uint4 q = *reinterpret_cast<const uint4*>(sm + K::OFF_B + (col >> 7) * (Q * 128) + row * 128 +
                                                                    phys * 16);
                    i8x16_to_bf16x8(q, blk == 0 ? o0 : o1);
                }
            };
            uint32_t cbv[2][2][8];                                // [buffer][block of the piece][packed cols]
            if constexpr (kCB8) {
                cb8_load(0, cbv[0][0], cbv[0][1]);
            } else {
                tc::tmem_ld8(cb_cols(0), cbv[0][0]);
                tc::tmem_ld8(cb_cols(0) + 16, cbv[0][1]);
                tc::tmem_wait_ld();
            }
#pragma unroll
            for (int k = 0; k < K::NPIECE; ++k) {
                int J, ib;
                piece_of(Q, k, J, ib);
                const bool pre = k + 1 < K::NPIECE;
                if (pre) {
                    if constexpr (kCB8) {
                        cb8_load(k + 1, cbv[(k + 1) & 1][0], cbv[(k + 1) & 1][1]);
                    } else {
                        tc::tmem_ld8(cb_cols(k + 1), cbv[(k + 1) & 1][0]);
                        tc::tmem_ld8(cb_cols(k + 1) + 16, cbv[(k + 1) & 1][1]);
                    }
                }
                const int pp = p + k, slot = pp % kRing;
                const int jrow = J * 128 + rrow;                  // row of M (ghost rows >= Q when Q = 64)
                const int jb = 4 * J + quarter;                   // its 32-row block
                const float aj = a2[jrow < Q ? jrow : Q - 1];
                uint32_t out0[8], out1[8];
                build16(cbv[k & 1][0], jb, 2 * ib, aj, out0);
                build16(cbv[k & 1][1], jb, 2 * ib + 1, aj, out1);
                if (!__all_sync(0xffffffffu, wait_bar<kI8>(bar + K::B_REMPTY + slot, (uint32_t)(((pp / kRing) & 1) ^ 1),
                                                      abort_flag, status))) {
                    ok = false;
                    break;
                }
                const uint32_t dst = trow + K::RING + slot * 32 + c0 / 2;
                tc::tmem_st8(dst, out0);
                tc::tmem_st8(dst + 16, out1);
                tc::tmem_wait_st();
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bar + K::B_RFULL + slot);
                if (pre) tc::tmem_wait_ld();
            }
            tc::tmem_wait_ld();                                   // no load left in flight on an early exit
            if (!ok) break;
            p += K::NPIECE;
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar + K::B_VEMPTY + s);
        }
    } else if (warp < kStoreWarp0) {
        // ------------------------------------------------------------ scalers
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
        bool ok = true;
        for (int it = 0; ok && it < nh; ++it) {
            const int h = h0 + it, s = it & 1;
            const uint32_t u = (uint32_t)(it >> 1);
            if (!(ok = tc::named_and(kIdScale, kEpiThreads, wait_bar<kI8>(bar + K::B_VFULL + s, u & 1, abort_flag, status))))
                break;
            {
                // the builders' decay vectors: log2-scaled Acs, dt with CB's
                // dequantisation, and the column factor exp(Acs_r - Acs_i) dt_i towards
                // the end r of i's 32-column block
                const float* acs = vec(s, kAcs);
                const float* dts = vec(s, kDtc);
                float* a2 = vec(s, kA2);
                float* v32 = vec(s, kVB);
                float* dtw = vec(s, kDtw);
                if (kI8 && tid - kScaleWarp0 * 32 < kP) {
                    // ChunkScan1's dequantisation s_C s_s[h,p] per column
                    const int p = tid - kScaleWarp0 * 32;
                    vec(s, kMul)[p] = __ldg(sc.s_C + g) * __ldg(sc.s_s + h * kP + p);
                }
                const __half* acs_h = reinterpret_cast<const __half*>(acs);   // Acs stored as half
                for (int i = tid - kScaleWarp0 * 32; i < Q; i += kEpiThreads) {
                    // explicitly rounded steps (no contraction), as in the single-launch scan
                    const float acs_i = acs_half ? __half2float(acs_h[i]) : acs[i];
                    const float acs_r = acs_half ? __half2float(acs_h[i | 31]) : acs[i | 31];
                    const float ai = __fmul_rn(acs_i, kLog2e);
                    const float ar = __fmul_rn(acs_r, kLog2e);
                    const float dw = __fmul_rn(dts[i], sCB);
                    a2[i] = ai;
                    dtw[i] = __fsub_rn(lg2(dw), ai);              // log2(dt_i) - a_i; -inf when dt_i = 0
                    // column factors as bf16 pairs (consecutive lanes hold consecutive i)
                    const float vi = __fmul_rn(ex2(fminf(__fsub_rn(ar, ai), 0.f)), dw);
                    const float vn = __shfl_down_sync(0xffffffffu, vi, 1);
                    if ((i & 1) == 0) reinterpret_cast<uint32_t*>(v32)[i / 2] = pack_bf16(vi, vn);
                }
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bar + K::B_VPREP + s);
            }
            if (!(ok = tc::named_and(kIdScale, kEpiThreads, wait_bar<kI8>(bar + K::B_YOFULL + s, u & 1, abort_flag, status))))
                break;
            tc::tc_fence_after();
            const float* a2v = vec(s, kA2);                        // log2e * Acs, formed above
            const uint32_t ybase = trow + K::YCOL + 128 * s;
            for (int J = 0; J < K::JT; ++J) {
                const int j = J * 128 + r;
                const float e = ex2(fminf(a2v[j < Q ? j : Q - 1], 0.f));
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    uint32_t v[32];
                    tc::tmem_ld32(ybase + 64 * J + 32 * hf, v);
                    tc::tmem_wait_ld();
                    if (kI8 && dbg.acc_scan1 && j < Q) {
                        int32_t* dst = dbg.acc_scan1 + (((long long)b * d.Lp() + (long long)c * Q + j) * d.H + h) * kP +
                                       32 * hf;
#pragma unroll
                        for (int i = 0; i < 32; ++i) dst[i] = (int32_t)v[i];
                    }
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        float f0, f1;
                        if (kI8) {
                            const float2 m = *reinterpret_cast<const float2*>(vec(s, kMul) + 32 * hf + i);
                            add_f32x2(f0, f1, __int_as_float((int)v[i] + 0x4B400000),
                                      __int_as_float((int)v[i + 1] + 0x4B400000), -12582912.0f, -12582912.0f);
                            mul_f32x2(f0, f1, f0, f1, m.x, m.y);
                        } else {
                            f0 = __uint_as_float(v[i]);
                            f1 = __uint_as_float(v[i + 1]);
                        }
                        mul_f32x2(f0, f1, f0, f1, e, e);
                        v[i] = __float_as_uint(f0);
                        v[i + 1] = __float_as_uint(f1);
                    }
                    tc::tmem_st32(ybase + 64 * J + 32 * hf, v);
                }
            }
            tc::tmem_wait_st();
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                tc::mbar_arrive(bar + K::B_YSCALED + s);
                tc::mbar_arrive(bar + K::B_VEMPTY + s);
            }
        }
    } else {
        // ------------------------------------------------------------ storers
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
        bool ok = true;
        for (int it = 0; ok && it < nh; ++it) {
            const int h = h0 + it, s = it & 1;
            const uint32_t u = (uint32_t)(it >> 1);
            const int xst = it % K::NXS;
            bool w = wait_bar<kI8>(bar + K::B_YFULL + s, u & 1, abort_flag, status);
            w = w && wait_bar<kI8>(bar + K::B_XFULL + xst, (uint32_t)(it / K::NXS) & 1, abort_flag, status);
            if (!(ok = tc::named_and(kIdStore, kEpiThreads, w))) break;
            tc::tc_fence_after();
            uint8_t* xs = sm + K::OFF_X + xst * K::X_BYTES;
            const uint32_t ybase = trow + K::YCOL + 128 * s;
            const float Dh = __ldg(Dv + h);
            for (int J = 0; J < K::JT; ++J) {
                const int j = J * 128 + r;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    uint32_t v[32];
                    tc::tmem_ld32(ybase + 64 * J + 32 * hf, v);
                    tc::tmem_wait_ld();
                    if (j < Q) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int chunk = hf * 4 + q;
                            uint4* px = reinterpret_cast<uint4*>(xs + j * 128 + ((chunk ^ (j & 7)) << 4));
                            const uint4 xv = *px;
                            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
                            uint32_t o[4];
#pragma unroll
                            for (int e2 = 0; e2 < 4; ++e2) {
                                float o0, o1;
                                fma_f32x2(o0, o1, Dh, Dh, bf16lo(xw[e2]), bf16hi(xw[e2]), __uint_as_float(v[q * 8 + 2 * e2]),
                                          __uint_as_float(v[q * 8 + 2 * e2 + 1]));
                                o[e2] = pack_bf16(o0, o1);
                            }
                            *px = make_uint4(o[0], o[1], o[2], o[3]);
                        }
                    }
                }
            }
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar + K::B_YEMPTY + s);
            tc::fence_proxy_async_smem();
            tc::named_sync(kIdStore, kEpiThreads);
            if (warp == kStoreWarp0 && lane == 0) {
                tc::tma_store_3d(&tm_y, xs, h * kP, c * Q, b);
                tc::tma_store_commit();
                tc::tma_store_wait_read0();
                tc::mbar_arrive(bar + K::B_XEMPTY + xst);
            }
        }
        if (warp == kStoreWarp0 && lane == 0) tc::tma_store_wait0();
    }
    __syncwarp();
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(tmem, K::TMEM_COLS);
}

template <int Q, bool kI8, bool kCB8 = false>
cudaError_t launch_q(const Dims& d, const CUtensorMap* maps, int hpc, int cpg, const float* Acs, const float* dtc,
                     const float* D, const I8Scales& sc, const I8Debug* dbg, int* status, cudaStream_t st,
                     const float* s_cb = nullptr, bool acs_half = false) {
    using K = Cfg<Q, kI8, kCB8>;
    static_assert(K::BYTES + 1024 <= 232448, "shared memory");
    auto k = chunk_scan_tc_kernel<Q, kI8, kCB8>;
    const int smem = K::BYTES + 1024;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    I8Debug none{};
    k<<<dim3(d.G * cpg, d.nc, d.B), kThreads, smem, st>>>(maps[0], maps[1], maps[2], maps[3], maps[4], d, hpc, cpg,
                                                            Acs, dtc, D, sc, dbg ? *dbg : none, status, s_cb,
                                                            acs_half ? 1 : 0);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_scan_tc(const Dims& d, bool i8, const uint16_t* x, const void* Bmat,
                                 const void* Cmat, const float* Acs, const float* dtc, const float* D,
                                 const I8Scales& sc, const void* Hc, uint16_t* y, const I8Debug* dbg,
                                 int heads_per_cta, int* status, cudaStream_t st, const int8_t* cb8,
                                 const float* s_cb, bool acs_half) {
    if (d.B == 0 || d.nc == 0) return cudaSuccess;
    if (d.P != kP || d.N != kN) return cudaErrorInvalidValue;
    if ((cb8 || acs_half) && (!i8 || d.Q != 256)) return cudaErrorInvalidValue;
    const int hpc = heads_per_cta < 1 ? 1 : (heads_per_cta > d.hpg ? d.hpg : heads_per_cta);
    const int cpg = (d.hpg + hpc - 1) / hpc;
    CUtensorMap maps[5];
    const unsigned long long HP = (unsigned long long)d.H * kP, GN = (unsigned long long)d.G * kN;
    const unsigned crows = d.Q >= 128 ? d.Q : 128;
    bool ok = make_tmap_3d(&maps[0], false, x, HP, d.L, d.B, HP * 2, d.Ls * HP * 2, 64, d.Q,
                           CU_TENSOR_MAP_SWIZZLE_128B);
    if (i8) {
        ok = ok && make_tmap_3d(&maps[1], true, Bmat, GN, d.L, d.B, GN, d.Ls * GN, 128, d.Q, CU_TENSOR_MAP_SWIZZLE_128B);
        ok = ok && make_tmap_3d(&maps[2], true, Cmat, GN, d.L, d.B, GN, d.Ls * GN, 128, crows, CU_TENSOR_MAP_SWIZZLE_128B);
        ok = ok && make_tmap_2d(&maps[3], true, Hc, kN, (unsigned long long)d.B * d.nc * d.H * kP, kN, 128, kP,
                                CU_TENSOR_MAP_SWIZZLE_128B);
    } else {
        ok = ok && make_tmap_3d(&maps[1], false, Bmat, GN, d.L, d.B, GN * 2, d.Ls * GN * 2, 64, d.Q,
                                CU_TENSOR_MAP_SWIZZLE_128B);
        ok = ok && make_tmap_3d(&maps[2], false, Cmat, GN, d.L, d.B, GN * 2, d.Ls * GN * 2, 64, crows,
                                CU_TENSOR_MAP_SWIZZLE_128B);
        ok = ok && make_tmap_2d(&maps[3], false, Hc, kN, (unsigned long long)d.B * d.nc * d.H * kP, kN * 2, 64, kP,
                                CU_TENSOR_MAP_SWIZZLE_128B);
    }
    ok = ok && make_tmap_3d(&maps[4], false, y, HP, d.L, d.B, HP * 2, d.Ls * HP * 2, 64, d.Q,
                            CU_TENSOR_MAP_SWIZZLE_128B);
    if (cb8)   // the CB codes, [B * nc * G * Q rows][Q] int8, in 128-column halves
        ok = ok && make_tmap_2d(&maps[1], true, cb8, d.Q, (unsigned long long)d.B * d.nc * d.G * d.Q, d.Q, 128, d.Q,
                                CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) return cudaErrorInvalidValue;
    if (cb8) return launch_q<256, true, true>(d, maps, hpc, cpg, Acs, dtc, D, sc, dbg, status, st, s_cb, acs_half);
    if (acs_half) return launch_q<256, true>(d, maps, hpc, cpg, Acs, dtc, D, sc, dbg, status, st, nullptr, true);
    switch (d.Q) {
        case 64: return i8 ? launch_q<64, true>(d, maps, hpc, cpg, Acs, dtc, D, sc, dbg, status, st)
                           : launch_q<64, false>(d, maps, hpc, cpg, Acs, dtc, D, sc, dbg, status, st);
        case 128: return i8 ? launch_q<128, true>(d, maps, hpc, cpg, Acs, dtc, D, sc, dbg, status, st)
                            : launch_q<128, false>(d, maps, hpc, cpg, Acs, dtc, D, sc, dbg, status, st);
        case 256: return i8 ? launch_q<256, true>(d, maps, hpc, cpg, Acs, dtc, D, sc, dbg, status, st)
                            : launch_q<256, false>(d, maps, hpc, cpg, Acs, dtc, D, sc, dbg, status, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace ssd
