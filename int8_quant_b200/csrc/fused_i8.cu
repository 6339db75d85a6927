// fused_i8.cu — the W8A8 SSD scan of one call (a1-a7) as a single persistent kernel
// (P = 64, N = 128), so that x is read from HBM once, y written once, and neither the
// chunk states nor the per-chunk vectors round-trip HBM.
//
// SSDi8 notes ("overall framework" and key designs 1-3): per chunk c of Q tokens,
//   ChunkCumsum  Acs_j = sum_{i<=j} dt_i A,  LUT_state_j = dt_j exp(Acs_{Q-1} - Acs_j),
//                dq = rint(exp(Acs_{Q-1}) 2^k)
//   ChunkState   S8 = clamp(rint(float(Q(LUT_state ⊙ x)^T Bq) s_x s_B / s_s))   (INT32 acc.)
//   StatePassing H_{c+1} = sat127(S8_c + ((dq_c H_c + 2^(k-1)) >> k))            (eq. 6)
//   ChunkBMM     CB = Cq Bq^T                                                    (INT32)
//   ChunkScan1   y_o = (Cq H8_c^T) s_C s_s exp(Acs_j)                            (INT32 acc.)
//   ChunkScan2   y_d = sum_{i<=j} CB_ji s_C s_B exp(Acs_j - Acs_i) dt_i x_i       (bf16 MMA)
//   y = y_d + y_o + D x.
//
// Work items are (chunk, batch row, block of heads of one group), claimed in
// chunk-major order from a global ticket counter by one CTA per SM.  StatePassing is
// carried by the items themselves: when an item has requantised a head's chunk state
// S8_c (still in registers), it reads H_c (published by the item of chunk c - 1 of the
// same heads, in L2) and publishes H_{c+1} with a release flag that the item of chunk
// c + 1 acquires before loading it for ChunkScan1; the last chunk writes the final
// state.  An item waits only for items of earlier chunks, which were claimed before it
// and are resident, so the schedule cannot deadlock.  States are stored transposed,
// [n][p] with p contiguous: one n per thread in the ChunkState epilogue writes whole
// rows, and ChunkScan1 reads H8^T as an MN-major operand.
//
// Warp roles (24 warps):
//   0      TMA producer: tickets, the Bq/Cq tiles of each item (3-slot ring), x per
//          head (3 stages).
//   1      TMEM allocation; MMA issue for the y-slot jobs in order: per item one
//          ChunkBMM job (six 128 x 64 CB units through a y slot), per head and 128-row
//          tile one ChunkScan1 job, each followed one job later by the ChunkScan2 pieces
//          of that tile (A = M from the TMEM ring, B = x).
//   2      vector warp: per head the cumulative sums (specified order), LUT_state, dq
//          and the ChunkScan2 decay vectors.
//   3      passed states: H_0 of this CTA's share of the chains, then per head of its
//          items the state entering the chunk, loaded once its flag is set.
//   4-7    state warps: Xq = Q(LUT_state ⊙ x) into shared memory; the ChunkState MMA
//          (S^T = Bq^T Xq, issued by one of them); the INT32 state requantised to INT8
//          and one StatePassing link.
//   8-15   builders: M = CB ⊙ exp(Acs_j - Acs_i) dt_i (bf16) in 64-column pieces.
//   16-19  scalers: CB units packed to bf16 in TMEM; ChunkScan1 dequantised in place.
//   20-23  storers: y + D x over the x tile, stored by TMA.
// The MMA issuers follow fixed schedules with suspending waits.  TMEM (512 columns):
// packed CB [0,192), M ring [192,256), three 64-column y slots [256,448), the
// ChunkState accumulator [448,512).  The per-(h,p) factors 1/s_x, s_x s_B / s_s and
// s_C s_s come precomputed from a small kernel launched before this one.
// Every wait is bounded; an expired wait raises the CTA's abort flag and records
// SSD_ERR_TIMEOUT; in-flight copies, MMAs and stores are waited for before exit.
#include "kernels.h"
#include "tc.cuh"

namespace ssd {

namespace {

constexpr int kP = 64;
constexpr int kN = 128;
enum : int {
    kWarpProd = 0,
    kWarpMma = 1,
    kWarpVec = 2,
    kWarpH = 3,
    kWarpState = 4,
    kWarpBuild = 8,
    kWarpScale = 16,
    kWarpStore = 20,
    kWarps = 24
};
constexpr int kThreads = kWarps * 32;
// item-ring consumers: MMA, vector, passed states, state (4), builders (8), scalers (4), storers (4)
constexpr int kItemConsumers = 1 + 1 + 1 + 4 + 8 + 4 + 4;
constexpr int kNI = 4, kNT = 3, kNX = 3, kNS = 2, kNC = 3, kNY = 3, kRing = 2;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kIdStore = 1, kIdState = 2;
constexpr float kRound = 12582912.0f;                         // 1.5 * 2^23
constexpr int kRoundBits = 0x4B400000;

template <int Q>
struct Cfg {
    static constexpr int JT = Q >= 128 ? Q / 128 : 1;           // 128-row tiles of a chunk
    static constexpr int CROWS = Q >= 128 ? Q : 128;            // C rows loaded (Q = 64: ghost rows)
    static constexpr int NCB0 = Q >= 128 ? 128 : Q;             // CB columns of row tile 0
    static constexpr int NPIECE = JT == 2 ? 6 : NCB0 / 64;      // 64-column pieces (= CB units) per head
    static constexpr int NP0 = JT == 2 ? 2 : NPIECE;            // pieces of row tile 0
    static constexpr uint32_t CBP1 = 0, CBP0 = JT == 2 ? 128 : 0, RING = 192, YCOL = 256, SCOL = 448;
    static constexpr int B_BYTES = Q * 128, C_BYTES = CROWS * 128, TILE = CROWS * 128;
    static constexpr int X_BYTES = Q * 128, XQ_BYTES = Q * 64, H_BYTES = kN * kP;
    // state vectors: LUT_state[Q], dq
    static constexpr int SV_LUT = 0, SV_DQ = Q * 4, SV_BYTES = SV_DQ + 16;
    // scan vectors: log2-scaled Acs[Q], log2(dt s_C s_B) - a2 [Q], column factors (bf16 pairs) [Q/2]
    static constexpr int CV_A2 = 0, CV_DTW = Q * 4, CV_VB = 2 * Q * 4, CV_BYTES = CV_VB + Q * 2;
    static constexpr int OFF_TILE = 0;
    static constexpr int OFF_X = OFF_TILE + kNT * TILE;
    static constexpr int OFF_XQ = OFF_X + kNX * X_BYTES;
    static constexpr int OFF_H = OFF_XQ + XQ_BYTES;
    static constexpr int OFF_SV = OFF_H + H_BYTES;
    static constexpr int OFF_CV = OFF_SV + kNS * SV_BYTES;
    static constexpr int OFF_BAR = (OFF_CV + kNC * CV_BYTES + 15) & ~15;
    enum {
        ITEM_FULL = 0,
        ITEM_EMPTY = ITEM_FULL + kNI,
        TILE_FULL = ITEM_EMPTY + kNI,
        TILE_EMPTY = TILE_FULL + kNT,
        X_FULL = TILE_EMPTY + kNT,
        X_EMPTY = X_FULL + kNX,
        XPREP = X_EMPTY + kNX,
        XQ_FULL = XPREP + kNX,
        XQ_EMPTY,
        S_FULL,
        S_EMPTY,
        H_FULL,
        H_EMPTY,
        SV_FULL,
        SV_EMPTY = SV_FULL + kNS,
        CV_FULL = SV_EMPTY + kNS,
        CV_EMPTY = CV_FULL + kNC,
        RFULL = CV_EMPTY + kNC,
        REMPTY = RFULL + kRing,
        YO_FULL = REMPTY + kRing,
        YSCALED = YO_FULL + kNY,
        YFULL = YSCALED + kNY,
        YEMPTY = YFULL + kNY,
        CBU_FULL = YEMPTY + kNY,
        CBU_EMPTY,
        CBU_FREE,
        CBU_PACKED = CBU_FREE + NPIECE,
        DONE_Y = CBU_PACKED + NPIECE,
        DONE_S,
        NBAR
    };
    static constexpr int OFF_ITEMS = OFF_BAR + NBAR * 8;
    static constexpr int OFF_FLAG = OFF_ITEMS + kNI * 4;
    static constexpr int OFF_TMEM = OFF_FLAG + 4;
    static constexpr int BYTES = OFF_TMEM + 4;
    // requested: BYTES + kSmemSlack; the kernel checks that the 1024-byte-aligned start of
    // its buffers leaves them inside the allocation
    static_assert(BYTES + 128 <= 232448, "shared memory budget of one CTA");
    static_assert(Q * 127 * 127 < (1 << 22), "INT32 accumulators stay below 2^22");
};

struct Item {
    int b, c, g, h0, nh;
};

__device__ __forceinline__ Item item_of(const FusedI8Args& a, int t) {
    Item it;
    const int hbk = t % a.nhb, bc = t / a.nhb;
    it.b = bc % a.d.B;
    it.c = bc / a.d.B;
    it.g = hbk / a.nhb_g;
    const int hb = hbk - it.g * a.nhb_g;
    it.h0 = it.g * a.d.hpg + hb * a.K;
    it.nh = min(a.K, a.d.hpg - hb * a.K);
    return it;
}

// 128-row tile J and 64-column block ib of piece (and CB unit) k.
template <int Q>
__device__ __forceinline__ void piece_of(int k, int& J, int& ib) {
    if (Q == 256) {
        J = k < 2 ? 0 : 1;
        ib = k < 2 ? k : k - 2;
    } else {
        J = 0;
        ib = k;
    }
}

// The i-th piece (and CB unit) in processing order.  With two row tiles, tile 1 goes
// first: its epilogue then writes y over x rows 128..255, which no later MMA reads,
// while tile 0's pieces (x rows 0..127) are still running; tile 0's epilogue follows
// the completion of every earlier MMA, tile 1's pieces included.
template <int Q>
__device__ __forceinline__ int piece_at(int i) {
    return Q == 256 ? (i < 4 ? i + 2 : i - 4) : i;
}

// ---------------------------------------------------------------- small device helpers
__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void red_release_add(int* p, int v) {
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ void mul_f32x2(float& r0, float& r1, float a0, float a1, float b0, float b1) {
    asm("{\n\t.reg .b64 a, b, r;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
        "mul.rn.f32x2 r, a, b;\n\tmov.b64 {%0, %1}, r;\n\t}"
        : "=f"(r0), "=f"(r1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void add_f32x2(float& r0, float& r1, float a0, float a1, float b0, float b1) {
    asm("{\n\t.reg .b64 a, b, r;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
        "add.rn.f32x2 r, a, b;\n\tmov.b64 {%0, %1}, r;\n\t}"
        : "=f"(r0), "=f"(r1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void fma_f32x2(float& r0, float& r1, float a0, float a1, float b0, float b1, float c0,
                                          float c1) {
    asm("{\n\t.reg .b64 a, b, c, r;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
        "mov.b64 c, {%6, %7};\n\tfma.rn.f32x2 r, a, b, c;\n\tmov.b64 {%0, %1}, r;\n\t}"
        : "=f"(r0), "=f"(r1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
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
// INT8 codes of two scaled values, clamp(rint(v), +-127): clamping first gives the same
// code, and adding 1.5 * 2^23 rounds to nearest (ties to even) into the low mantissa
// bits, so each result's low byte is the code's byte.
__device__ __forceinline__ void code_bits2(int& q0, int& q1, float v0, float v1) {
    const float c0 = fminf(fmaxf(v0, -127.f), 127.f), c1 = fminf(fmaxf(v1, -127.f), 127.f);
    float r0, r1;
    add_f32x2(r0, r1, c0, c1, kRound, kRound);
    q0 = __float_as_int(r0);
    q1 = __float_as_int(r1);
}
__device__ __forceinline__ uint32_t pack_i8x4(int a, int b, int c, int d) {
    return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// mbarrier wait (try_wait: the hardware may suspend the thread for a short, system-defined
// time before it returns false).
__device__ __forceinline__ bool try_wait_hw(uint64_t* bar, uint32_t parity) { return tc::mbar_try_wait(bar, parity); }
// Bounded wait: false once the CTA's abort flag is raised or, after
// tc::kWaitLimit cycles, with the flag raised and SSD_ERR_TIMEOUT recorded.
__device__ __noinline__ bool wait_sleep_slow(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status) {
    const long long t0 = clock64();
    for (;;) {
        if (try_wait_hw(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > tc::kWaitLimit) {
            *abort_flag = 1;
            if (status) atomicExch(status, kStatusTimeout);
            return false;
        }
    }
}
__device__ __forceinline__ bool wait_sleep(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status) {
    if (try_wait_hw(bar, parity)) return true;
    return wait_sleep_slow(bar, parity, abort_flag, status);
}

// Bounded wait by every lane of a warp; false (for all lanes) on abort or timeout.
__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status) {
    return __all_sync(0xffffffffu, wait_sleep(bar, parity, abort_flag, status));
}

// Single-thread bounded poll of a global flag until it is >= want (want > 0) or, with
// want == 0, nonzero; returns the value read, or 0 on abort or timeout.
__device__ __noinline__ int poll_flag(const int* f, int want, volatile int* abort_flag, int* status) {
    const long long t0 = clock64();
    for (;;) {
        const int v = ld_acquire(f);
        if (want > 0 ? v >= want : v != 0) return v;
        if (*abort_flag) return 0;
        if (clock64() - t0 > tc::kWaitLimit) {
            *abort_flag = 1;
            atomicExch(status, kStatusTimeout);
            return 0;
        }
        __nanosleep(64);
    }
}

// The same link, one code at a time (any k): w holds S8 (in) and H_{c+1} (out) for the
// 64 codes of row n; hrow is H_c's row (64 bytes).
__device__ __noinline__ void chain_row_generic(uint32_t* w, const uint32_t* hrow, int dq, int k) {
    for (int e = 0; e < 16; ++e) {
        uint32_t r = 0;
        for (int i = 0; i < 4; ++i) {
            const int h = (int)(int8_t)((hrow[e] >> (8 * i)) & 0xff);
            const int sv = (int)(int8_t)((w[e] >> (8 * i)) & 0xff);
            const int v = sv + ((dq * h + (1 << (k - 1))) >> k);
            r |= ((uint32_t)(v < -127 ? -127 : (v > 127 ? 127 : v)) & 0xffu) << (8 * i);
        }
        w[e] = r;
    }
}

// Out-of-line helpers for debug copies and rare paths, so that the hot loops stay small
// (the kernel's warps run many different roles; their code must share the SM's
// instruction caches) and keep their registers.
// 32 int32 accumulators to dst[i * stride].
__device__ __noinline__ void dump32(int32_t* dst, long long stride, const uint32_t* v) {
    for (int i = 0; i < 32; ++i) dst[i * stride] = (int32_t)v[i];
}
// 64 int8 codes (16 words, first code in the lowest byte) to dst[p * stride].
__device__ __noinline__ void dump_codes64(int8_t* dst, long long stride, const uint32_t* w) {
    for (int p = 0; p < 64; ++p) dst[p * stride] = (int8_t)(w[p >> 2] >> (8 * (p & 3)));
}
// The quantised X_scaled tile (int8 [Q][64], 64-byte swizzle) of one (b, c, h) into
// dbg [B, Lp, H, P]; `t` is a thread index among `nt` cooperating threads.
__device__ __noinline__ void dump_xq(const uint8_t* xq, int Q, int8_t* dst, long long row_stride, int t, int nt) {
    for (int i = t; i < Q * 4; i += nt) {
        const int row = i >> 2, c4 = i & 3;
        const uint4 v = *reinterpret_cast<const uint4*>(xq + row * 64 + ((c4 ^ ((row >> 1) & 3)) << 4));
        *reinterpret_cast<uint4*>(dst + row * row_stride + c4 * 16) = v;
    }
}

// The specified fp32 exp, called out of line by the vector warp (same operations).
__device__ __noinline__ float ssd_expf_call(float x) { return ssd_expf(x); }

template <int Q>
__global__ void __launch_bounds__(kThreads, 1)
ssd_fused_i8_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_y,
                    const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_c,
                    const __grid_constant__ CUtensorMap tm_h, const FusedI8Args a) {
    using K = Cfg<Q>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t pad = (1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u;
    if (pad > 128u) {
        // the buffers would not fit behind a 1024-byte boundary: report, touch nothing
        if (threadIdx.x == 0) atomicExch(a.status, 2);
        return;
    }
    uint8_t* sm = smem_raw + pad;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + K::OFF_BAR);
    volatile int* items = reinterpret_cast<volatile int*>(sm + K::OFF_ITEMS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + K::OFF_FLAG);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + K::OFF_TMEM);
    const Dims& d = a.d;
    int* status = a.status;

    if (tid == 0) {
        for (int i = 0; i < K::NBAR; ++i) {
            uint32_t cnt = 1;
            if (i >= K::ITEM_EMPTY && i < K::ITEM_EMPTY + kNI) cnt = kItemConsumers;
            if (i >= K::TILE_EMPTY && i < K::TILE_EMPTY + kNT) cnt = 2;          // both MMA warps
            if (i >= K::XPREP && i < K::XPREP + kNX) cnt = 4;
            if (i >= K::SV_EMPTY && i < K::SV_EMPTY + kNS) cnt = 4;
            if (i >= K::CV_EMPTY && i < K::CV_EMPTY + kNC) cnt = 12;           // builders + scalers
            if (i >= K::RFULL && i < K::RFULL + kRing) cnt = 8;
            if (i >= K::YSCALED && i < K::YSCALED + kNY) cnt = 4;
            if (i >= K::YEMPTY && i < K::YEMPTY + kNY) cnt = 4;
            if (i == K::CBU_EMPTY) cnt = 4;
            if (i >= K::CBU_FREE && i < K::CBU_FREE + K::NPIECE) cnt = 8;
            if (i >= K::CBU_PACKED && i < K::CBU_PACKED + K::NPIECE) cnt = 4;
            tc::mbar_init(bar + i, cnt);
        }
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == kWarpMma) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const long long nc = d.nc;

    // the item ring, as every consumer warp reads it
    auto item_get = [&](int n) -> int {
        if (!wait_all(bar + K::ITEM_FULL + n % kNI, (uint32_t)(n / kNI) & 1, abort_flag, status)) return -2;
        return items[n % kNI];
    };
    auto item_release = [&](int n) {
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(bar + K::ITEM_EMPTY + n % kNI);
    };
    auto sv = [&](int s) -> float* { return reinterpret_cast<float*>(sm + K::OFF_SV + s * K::SV_BYTES); };
    auto cv = [&](int s) -> float* { return reinterpret_cast<float*>(sm + K::OFF_CV + s * K::CV_BYTES); };

    if (warp == kWarpProd) {
        // ================================================================ TMA producer
        if (lane == 0) {
            tc::prefetch_tmap(&tm_x);
            tc::prefetch_tmap(&tm_y);
            tc::prefetch_tmap(&tm_b);
            tc::prefetch_tmap(&tm_c);
            tc::prefetch_tmap(&tm_h);
            int nt = 0, kx = 0;
            bool ok = true;
            for (int n = 0; ok; ++n) {
                int t = atomicAdd(a.ticket, 1);
                if (t >= a.items) t = -1;
                const int is = n % kNI;
                if (!wait_sleep(bar + K::ITEM_EMPTY + is, ((uint32_t)(n / kNI) & 1) ^ 1, abort_flag, status)) break;
                items[is] = t;
                tc::mbar_arrive(bar + K::ITEM_FULL + is);
                if (t < 0) break;
                const Item it = item_of(a, t);
                for (int w = 0; w < 2 && ok; ++w) {                  // Bq, then Cq
                    const int ts = nt % kNT;
                    if (!wait_sleep(bar + K::TILE_EMPTY + ts, ((uint32_t)(nt / kNT) & 1) ^ 1, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    tc::mbar_arrive_expect_tx(bar + K::TILE_FULL + ts, w == 0 ? K::B_BYTES : K::C_BYTES);
                    tc::tma_load_3d(sm + K::OFF_TILE + ts * K::TILE, w == 0 ? &tm_b : &tm_c, bar + K::TILE_FULL + ts,
                                    it.g * kN, it.c * Q, it.b);
                    ++nt;
                }
                for (int hh = 0; hh < it.nh && ok; ++hh) {
                    const int xs = kx % kNX;
                    if (!wait_sleep(bar + K::X_EMPTY + xs, ((uint32_t)(kx / kNX) & 1) ^ 1, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    tc::mbar_arrive_expect_tx(bar + K::X_FULL + xs, K::X_BYTES);
                    tc::tma_load_3d(sm + K::OFF_X + xs * K::X_BYTES, &tm_x, bar + K::X_FULL + xs, (it.h0 + hh) * kP,
                                    it.c * Q, it.b);
                    ++kx;
                }
            }
            // copies still in flight after an abort must land before the CTA exits
            for (int s = 0; s < kNT; ++s) {
                const int cnt = nt > s ? (nt - 1 - s) / kNT + 1 : 0;
                if (cnt > 0) tc::mbar_wait(bar + K::TILE_FULL + s, (uint32_t)(cnt - 1) & 1, tc::kWaitLimit);
            }
            for (int s = 0; s < kNX; ++s) {
                const int cnt = kx > s ? (kx - 1 - s) / kNX + 1 : 0;
                if (cnt > 0) tc::mbar_wait(bar + K::X_FULL + s, (uint32_t)(cnt - 1) & 1, tc::kWaitLimit);
            }
        }
    } else if (warp == kWarpMma) {
        // ================================================================ MMA: y-slot jobs
        // Jobs in order, one slot each (slot = job % 3): per item a ChunkBMM job (its CB
        // units), then per head and row tile (tile 1 first) a ChunkScan1 job.  The pieces
        // of a ChunkScan1 job are issued after the next job's ChunkScan1, so that the
        // next job's scaling overlaps them.  The whole warp runs the schedule and waits;
        // one elected lane issues.
        const uint32_t idCB = tc::idesc_s8_s32(128, 64, tc::kMajorK, tc::kMajorK);
        const uint32_t idO = tc::idesc_s8_s32(128, kP, tc::kMajorK, tc::kMajorMN);
        const uint32_t idD = tc::idesc_bf16_f32(128, kP, tc::kMajorK, tc::kMajorMN);
        const uint64_t dTileK = tc::smem_desc(tc::smem_u32(sm + K::OFF_TILE), 16, 1024, tc::kLayoutSw128);
        const uint64_t dH = tc::smem_desc(tc::smem_u32(sm + K::OFF_H), 0, 512, tc::kLayoutSw64);
        const uint64_t dX0 = tc::smem_desc(tc::smem_u32(sm + K::OFF_X), 0, 1024, tc::kLayoutSw128);
        int jk = 0, hk = 0, cbu = 0, pr = 0;
        uint32_t ru_par = 0;                                         // per-slot parity bits of ChunkScan1 jobs
        bool pend = false;                                           // a ChunkScan1 job awaits its pieces
        int pslot = 0, pJ = 0, pxs = 0;
        uint32_t ppar = 0;
        bool ok = true;
        auto pieces = [&]() -> bool {
            if (!wait_all(bar + K::YSCALED + pslot, ppar, abort_flag, status)) return false;
            const int kfirst = pJ == 0 ? 0 : K::NP0, klast = pJ == 0 ? K::NP0 : K::NPIECE;
            for (int kk = kfirst; kk < klast; ++kk, ++pr) {
                const int rs = pr % kRing;
                if (!wait_all(bar + K::RFULL + rs, (uint32_t)(pr / kRing) & 1, abort_flag, status)) return false;
                tc::tc_fence_after();
                int Jp, ib;
                piece_of<Q>(kk, Jp, ib);
                if (tc::elect_one()) {
                    const uint32_t am = tmem + K::RING + rs * 32;
                    const uint64_t db = dX0 + (uint64_t)((pxs * K::X_BYTES) >> 4) + (uint64_t)(ib * 512);
                    const uint32_t dcol = tmem + K::YCOL + 64 * pslot;
#pragma unroll
                    for (int st = 0; st < 4; ++st) tc::mma_f16_ts(dcol, am + st * 8, db + st * 128, idD, 1u);
                    tc::mma_commit(bar + K::REMPTY + rs);
                    if (kk + 1 == klast) tc::mma_commit(bar + K::YFULL + pslot);
                }
                __syncwarp();
            }
            pend = false;
            return true;
        };
        for (int n = 0; ok; ++n) {
            const int t = item_get(n);
            if (t < 0) break;
            const Item it = item_of(a, t);
            const int tb = 2 * n, tcq = 2 * n + 1;                   // the item's Bq and Cq tiles
            // ChunkBMM job: the previous item's last pieces first (the builders must finish
            // with its CB before the units are packed over it)
            if (pend && !(ok = pieces())) break;
            {
                const int slot = jk % kNY;
                ok = wait_all(bar + K::YEMPTY + slot, ((uint32_t)(jk / kNY) & 1) ^ 1, abort_flag, status) &&
                     wait_all(bar + K::TILE_FULL + tb % kNT, (uint32_t)(tb / kNT) & 1, abort_flag, status) &&
                     wait_all(bar + K::TILE_FULL + tcq % kNT, (uint32_t)(tcq / kNT) & 1, abort_flag, status);
                for (int ui = 0; ok && ui < K::NPIECE; ++ui, ++cbu) {
                    if (cbu > 0 && !(ok = wait_all(bar + K::CBU_EMPTY, (uint32_t)(cbu - 1) & 1, abort_flag, status)))
                        break;
                    tc::tc_fence_after();
                    int J, ib;
                    piece_of<Q>(piece_at<Q>(ui), J, ib);
                    if (tc::elect_one()) {
                        const uint64_t dA = dTileK + (uint64_t)(((tcq % kNT) * K::TILE) >> 4) +
                                            (uint64_t)((J * 128 * 128) >> 4);
                        const uint64_t dB = dTileK + (uint64_t)(((tb % kNT) * K::TILE) >> 4) +
                                            (uint64_t)((ib * 64 * 128) >> 4);
#pragma unroll
                        for (int st = 0; st < 4; ++st)
                            tc::mma_i8_ss(tmem + K::YCOL + 64 * slot, dA + (uint64_t)(st * 2), dB + (uint64_t)(st * 2),
                                          idCB, st > 0 ? 1u : 0u);
                        tc::mma_commit(bar + K::CBU_FULL);
                        if (ui + 1 == K::NPIECE) tc::mma_commit(bar + K::TILE_EMPTY + tb % kNT);
                    }
                    __syncwarp();
                }
                if (!ok) break;
                ++jk;
            }
            // ChunkScan1 jobs
            for (int hh = 0; ok && hh < it.nh; ++hh) {
                for (int jj = 0; jj < K::JT; ++jj) {
                    const int J = K::JT - 1 - jj, slot = jk % kNY;
                    ok = wait_all(bar + K::YEMPTY + slot, ((uint32_t)(jk / kNY) & 1) ^ 1, abort_flag, status);
                    if (ok && jj == 0) ok = wait_all(bar + K::H_FULL, (uint32_t)hk & 1, abort_flag, status);
                    if (!ok) break;
                    tc::tc_fence_after();
                    const bool last_j = jj == K::JT - 1;
                    if (tc::elect_one()) {
                        const uint64_t dA = dTileK + (uint64_t)(((tcq % kNT) * K::TILE) >> 4) +
                                            (uint64_t)((J * 128 * 128) >> 4);
#pragma unroll
                        for (int st = 0; st < 4; ++st)
                            tc::mma_i8_ss(tmem + K::YCOL + 64 * slot, dA + (uint64_t)(st * 2), dH + (uint64_t)(st * 128),
                                          idO, st > 0 ? 1u : 0u);
                        tc::mma_commit(bar + K::YO_FULL + slot);
                        if (last_j) tc::mma_commit(bar + K::H_EMPTY);
                        if (last_j && hh == it.nh - 1) tc::mma_commit(bar + K::TILE_EMPTY + tcq % kNT);
                    }
                    __syncwarp();
                    const uint32_t par = (ru_par >> slot) & 1;
                    ru_par ^= 1u << slot;
                    if (pend && !(ok = pieces())) break;
                    pend = true;
                    pslot = slot;
                    pJ = J;
                    pxs = hk % kNX;
                    ppar = par;
                    ++jk;
                    if (last_j) ++hk;
                }
            }
            if (!ok) break;
            item_release(n);
        }
        if (ok && pend) pieces();
        // MMAs still running (after an abort too) must finish before TMEM is freed
        if (tc::elect_one()) tc::mma_commit(bar + K::DONE_Y);
        __syncwarp();
        tc::mbar_wait(bar + K::DONE_Y, 0, tc::kWaitLimit);
    } else if (warp == kWarpVec) {
        // ================================================================ vector warp
        constexpr int m = Q / 32;                                   // elements per lane, consecutive
        int hk = 0;
        for (int n = 0;; ++n) {
            const int t = item_get(n);
            if (t < 0) break;
            const Item it = item_of(a, t);
            const float sCB = __fmul_rn(__ldg(a.sc.s_C + it.g), __ldg(a.sc.s_B + it.g));
            bool ok = true;
            for (int hh = 0; hh < it.nh; ++hh, ++hk) {
                const int h = it.h0 + hh, ss = hk % kNS, cs = hk % kNC;
                float dtv[m], acs[m];
#pragma unroll
                for (int i = 0; i < m; ++i) {
                    const long long tok = (long long)it.c * Q + lane * m + i;
                    dtv[i] = tok < d.L ? __ldg(a.dt + ((long long)it.b * d.Ls + tok) * d.H + h) : 0.f;
                }
                if (!wait_all(bar + K::SV_EMPTY + ss, ((uint32_t)(hk / kNS) & 1) ^ 1, abort_flag, status) ||
                    !wait_all(bar + K::CV_EMPTY + cs, ((uint32_t)(hk / kNC) & 1) ^ 1, abort_flag, status)) {
                    ok = false;
                    break;
                }
                const float ah = __ldg(a.A + h);
                // ChunkCumsum in the specified order: sequential in the lane, Kogge-Stone
                // over lane totals, exclusive lane prefix added
                float acc = 0.f;
#pragma unroll
                for (int i = 0; i < m; ++i) {
                    const float v = __fmul_rn(dtv[i], ah);
                    acc = i == 0 ? v : __fadd_rn(acc, v);
                    acs[i] = acc;
                }
                float v = acc;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float u = __shfl_up_sync(0xffffffffu, v, off);
                    if (lane >= off) v = __fadd_rn(u, v);
                }
                float e = __shfl_up_sync(0xffffffffu, v, 1);
                if (lane == 0) e = 0.f;
#pragma unroll
                for (int i = 0; i < m; ++i) acs[i] = __fadd_rn(e, acs[i]);
                const float last = __shfl_sync(0xffffffffu, acs[m - 1], 31);
                float* svp = sv(ss);
                float* cvp = cv(cs);
                // Acs and dt go to the scan vectors' slot first; the per-element exponentials
                // then run as a rolled loop (small code) that reads them back
#pragma unroll
                for (int i = 0; i < m; ++i) {
                    cvp[K::CV_A2 / 4 + lane * m + i] = acs[i];
                    cvp[K::CV_DTW / 4 + lane * m + i] = dtv[i];
                }
                if (a.dbg.Acs) {
                    float* dst = a.dbg.Acs + (((long long)it.b * d.H + h) * nc + it.c) * Q + lane * m;
#pragma unroll
                    for (int i = 0; i < m; ++i) dst[i] = acs[i];
                }
                // a2 at the end of the 32-element block of this lane's elements
                const float ar = __shfl_sync(0xffffffffu, __fmul_rn(acs[m - 1], kLog2e), lane | (32 / m - 1));
                __syncwarp();
#pragma unroll 1
                for (int i = 0; i < m; i += 2) {
                    const int j = lane * m + i;
                    const float c0v = cvp[K::CV_A2 / 4 + j], c1v = cvp[K::CV_A2 / 4 + j + 1];
                    const float t0 = cvp[K::CV_DTW / 4 + j], t1 = cvp[K::CV_DTW / 4 + j + 1];
                    svp[K::SV_LUT / 4 + j] = __fmul_rn(t0, ssd_expf_call(__fsub_rn(last, c0v)));
                    svp[K::SV_LUT / 4 + j + 1] = __fmul_rn(t1, ssd_expf_call(__fsub_rn(last, c1v)));
                    // explicitly rounded steps (no contraction), as in the five-launch ChunkScan
                    const float a0v = __fmul_rn(c0v, kLog2e), a1v = __fmul_rn(c1v, kLog2e);
                    const float dw0 = __fmul_rn(t0, sCB), dw1 = __fmul_rn(t1, sCB);
                    cvp[K::CV_A2 / 4 + j] = a0v;
                    cvp[K::CV_A2 / 4 + j + 1] = a1v;
                    cvp[K::CV_DTW / 4 + j] = __fsub_rn(lg2(dw0), a0v);
                    cvp[K::CV_DTW / 4 + j + 1] = __fsub_rn(lg2(dw1), a1v);
                    const float v0 = __fmul_rn(ex2(fminf(__fsub_rn(ar, a0v), 0.f)), dw0);
                    const float v1 = __fmul_rn(ex2(fminf(__fsub_rn(ar, a1v), 0.f)), dw1);
                    reinterpret_cast<uint32_t*>(cvp + K::CV_VB / 4)[j / 2] = pack_bf16(v0, v1);
                }
                if (lane == 31) {
                    const int dq = (int)rintf(__fmul_rn(ssd_expf_call(last), (float)(1 << a.sc.shift)));
                    reinterpret_cast<int*>(svp)[K::SV_DQ / 4] = dq;
                    if (a.dbg.dq) a.dbg.dq[((long long)it.b * d.H + h) * nc + it.c] = dq;
                }
                __syncwarp();
                if (lane == 0) {
                    tc::mbar_arrive(bar + K::SV_FULL + ss);
                    tc::mbar_arrive(bar + K::CV_FULL + cs);
                }
            }
            if (!ok) break;
            item_release(n);
        }
    } else if (warp == kWarpH) {
        // ================================================================ passed states
        // H_0 (the initial state or zero) of this CTA's share of the (batch row, head)
        // chains, published for the items of chunk 0; lane l writes rows n = l + 32 i of
        // the transposed [n][p] tile.
        for (int bh = blockIdx.x; bh < d.B * d.H; bh += gridDim.x) {
            const int h = bh % d.H, b = bh / d.H;
            const long long row0 = ((long long)b * nc) * d.H + h;
#pragma unroll 1
            for (int i = 0; i < 4; ++i) {
                const int n = lane + 32 * i;
                const int8_t* src = a.init8 ? a.init8 + (long long)bh * (kP * kN) + n : nullptr;
                uint4* pub = reinterpret_cast<uint4*>(a.Hpub + row0 * 8192 + n * 64);
#pragma unroll 1
                for (int c4 = 0; c4 < 4; ++c4) {
                    uint32_t w[4] = {0u, 0u, 0u, 0u};
                    if (src) {
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            w[e >> 2] |= ((uint32_t)(uint8_t)src[(16 * c4 + e) * kN]) << (8 * (e & 3));
                    }
                    pub[c4] = make_uint4(w[0], w[1], w[2], w[3]);
                    if (a.dbg.H8) {
                        int8_t* dst = a.dbg.H8 + row0 * (kP * kN) + n;
#pragma unroll
                        for (int e = 0; e < 16; ++e) dst[(16 * c4 + e) * kN] = (int8_t)(w[e >> 2] >> (8 * (e & 3)));
                    }
                }
            }
            __syncwarp();
            if (lane == 0) red_release_add(a.hflag + row0, 4);
        }
        // Then the state entering the chunk of every head of this CTA's items, into the
        // single H tile, in head order: poll the head's flag (while the tile may still be
        // in use), wait for the tile to be free (ChunkScan1 of the previous head), load it.
        int kh = 0;
        bool ok = true;
        for (int n = 0; ok; ++n) {
            const int t = item_get(n);
            if (t < 0) break;
            const Item it = item_of(a, t);
            if (lane == 0) {
                for (int hh = 0; hh < it.nh; ++hh, ++kh) {
                    const long long row = ((long long)it.b * nc + it.c) * d.H + it.h0 + hh;
                    if (poll_flag(a.hflag + row, 4, abort_flag, status) == 0 ||
                        !wait_sleep(bar + K::H_EMPTY, ((uint32_t)kh & 1) ^ 1, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    fence_proxy_async_global();
                    tc::mbar_arrive_expect_tx(bar + K::H_FULL, K::H_BYTES);
                    tc::tma_load_2d(sm + K::OFF_H, &tm_h, bar + K::H_FULL, 0, (int)(row * kN));
                }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            kh = __shfl_sync(0xffffffffu, kh, 0);
            if (ok) item_release(n);
        }
        // a copy still in flight after an abort must land before the CTA exits
        if (lane == 0 && kh > 0) tc::mbar_wait(bar + K::H_FULL, (uint32_t)(kh - 1) & 1, tc::kWaitLimit);
    } else if (warp < kWarpBuild) {
        // ================================================================ state warps
        const int quarter = warp & 3;
        const int pt = tid - kWarpState * 32;                       // 0..127
        const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
        // 16-byte chunk pt + 128 i of the x tile holds 8 consecutive p of row (pt >> 3) + 16 i;
        // every such chunk of this thread has the same swizzle phase, so the same p0
        const int p0 = ((pt & 7) ^ ((pt >> 3) & 7)) * 8;
        constexpr int kChunks = Q * 8 / 128;                       // 16-byte chunks per thread
        constexpr int kBatch = kChunks < 8 ? kChunks : 8;
        const int ksh = a.sc.shift;
        const bool packed = ksh <= 7;
        const uint32_t clo = (uint32_t)(129u << ksh) * 0x00010001u;
        const uint32_t chi = (uint32_t)((384u << ksh) - 1u) * 0x00010001u;
        const uint32_t idS = tc::idesc_s8_s32(128, kP, tc::kMajorMN, tc::kMajorMN);
        const uint64_t dTileMN = tc::smem_desc(tc::smem_u32(sm + K::OFF_TILE), 0, 1024, tc::kLayoutSw128);
        const uint64_t dXq = tc::smem_desc(tc::smem_u32(sm + K::OFF_XQ), 0, 512, tc::kLayoutSw64);
        const bool issuer = warp == kWarpState;                     // one elected lane issues the MMA
        int hk = 0;
        int pb = 0, pc = 0, ph = 0;                                  // head awaiting requantisation
        bool pending = false;
        // Head kk's INT32 chunk state S^T[n][p] (this warp's 32 rows n) requantised to INT8
        // codes (key design 2) into wq; afterwards the accumulator may be overwritten.
        auto requant_codes = [&](int kk, uint32_t (&wq)[16]) -> bool {
            if (!wait_all(bar + K::S_FULL, (uint32_t)kk & 1, abort_flag, status)) {
#pragma unroll
                for (int e = 0; e < 16; ++e) wq[e] = 0u;
                return false;
            }
            tc::tc_fence_after();
            const float* mq = a.mq + ph * kP;
            const int n = quarter * 32 + lane;
            const long long row = ((long long)pb * nc + pc) * d.H + ph;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                uint32_t v[32];
                tc::tmem_ld32(trow + K::SCOL + 32 * hf, v);
                tc::tmem_wait_ld();
#pragma unroll
                for (int p = 0; p < 32; p += 4) {
                    const float4 m4 = __ldg(reinterpret_cast<const float4*>(mq + 32 * hf + p));
                    float r0, r1, r2, r3;
                    mul_f32x2(r0, r1, __int2float_rn((int)v[p]), __int2float_rn((int)v[p + 1]), m4.x, m4.y);
                    mul_f32x2(r2, r3, __int2float_rn((int)v[p + 2]), __int2float_rn((int)v[p + 3]), m4.z, m4.w);
                    int q0, q1, q2, q3;
                    code_bits2(q0, q1, r0, r1);
                    code_bits2(q2, q3, r2, r3);
                    wq[8 * hf + p / 4] = pack_i8x4(q0, q1, q2, q3);
                }
                if (a.dbg.acc_state) dump32(a.dbg.acc_state + row * (kP * kN) + n + (long long)(32 * hf) * kN, kN, v);
            }
            tc::tc_fence_before();
            if (a.dbg.S8) dump_codes64(a.dbg.S8 + row * (kP * kN) + n, kN, wq);
            return true;
        };
        // One link of StatePassing (eq. 6) for this warp's rows: H_{c+1} = sat127(S8_c +
        // ((dq_c H_c + 2^(k-1)) >> k)), with H_c read from the published buffer (acquired
        // through its flag); H_{c+1} is published for the item of chunk c + 1, or is the
        // final state.
        auto link = [&](int kk, uint32_t (&wq)[16]) -> bool {
            const int s = kk % kNS;
            const int dq = reinterpret_cast<const int*>(sv(s))[K::SV_DQ / 4];
            const int n = quarter * 32 + lane;
            const long long row = ((long long)pb * nc + pc) * d.H + ph;
            int fv = 0;
            if (lane == 0) fv = poll_flag(a.hflag + row, 4, abort_flag, status);
            if (__shfl_sync(0xffffffffu, fv, 0) == 0) return false;
            const uint4* hsrc = reinterpret_cast<const uint4*>(a.Hpub + row * 8192 + n * 64);
            if (packed) {
                const uint32_t k0 = (uint32_t)((1 << (ksh - 1)) + 128 * ((1 << ksh) - dq)) * 0x00010001u;
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const uint4 hv = hsrc[c4];
                    wq[4 * c4] = chain_word(hv.x, wq[4 * c4], (uint32_t)dq, k0, ksh, clo, chi);
                    wq[4 * c4 + 1] = chain_word(hv.y, wq[4 * c4 + 1], (uint32_t)dq, k0, ksh, clo, chi);
                    wq[4 * c4 + 2] = chain_word(hv.z, wq[4 * c4 + 2], (uint32_t)dq, k0, ksh, clo, chi);
                    wq[4 * c4 + 3] = chain_word(hv.w, wq[4 * c4 + 3], (uint32_t)dq, k0, ksh, clo, chi);
                }
            } else {
                chain_row_generic(wq, reinterpret_cast<const uint32_t*>(hsrc), dq, ksh);
            }
            if (pc + 1 < d.nc) {
                const long long nrow = row + d.H;                     // chunk c + 1
                uint4* pub = reinterpret_cast<uint4*>(a.Hpub + nrow * 8192 + n * 64);
#pragma unroll
                for (int e = 0; e < 4; ++e) pub[e] = make_uint4(wq[4 * e], wq[4 * e + 1], wq[4 * e + 2], wq[4 * e + 3]);
                if (a.dbg.H8) dump_codes64(a.dbg.H8 + nrow * (kP * kN) + n, kN, wq);
                __syncwarp();
                if (lane == 0) red_release_add(a.hflag + nrow, 1);
            } else {
                dump_codes64(a.final8 + ((long long)pb * d.H + ph) * (kP * kN) + n, kN, wq);
            }
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar + K::SV_EMPTY + s);
            return true;
        };
        // One flat loop over this CTA's heads.  Iteration hk: the codes and the link of head
        // hk - 1 (its MMA was issued at the end of the previous iteration; the link comes
        // first so that H_{c+1} reaches the next chunk's item as early as possible), then the
        // prep of head hk and its ChunkState MMA.  An item is released once its last head's
        // link is done; its tiles (this issuer's arrival) after its last MMA.
        // Every exit from this loop is decided collectively: the four warps meet at named
        // barriers that also AND their success flags, so that none is left waiting at a
        // barrier after another has left on a failed (bounded) wait.
        bool ok = true;
        int n = -1, hh = 0, nh = 0, rel = -1;
        Item it{};
        for (;;) {
            bool lok = true;
            if (pending) {
                uint32_t wq[16];
                lok = requant_codes(hk - 1, wq);
                if (lok) lok = link(hk - 1, wq);
            }
            bool more = true;
            if (lok && hh == nh) {
                // this issuer is done with the previous item's tiles; the item itself is done
                // once its last link is (just above)
                if (n >= 0 && issuer) {
                    if (tc::elect_one()) {
                        tc::mma_commit(bar + K::TILE_EMPTY + (2 * n) % kNT);
                        tc::mma_commit(bar + K::TILE_EMPTY + (2 * n + 1) % kNT);
                    }
                    __syncwarp();
                }
                if (rel >= 0) {
                    item_release(rel);
                    rel = -1;
                }
                const int t = item_get(++n);
                if (t == -2) {
                    lok = false;
                } else if (t < 0) {
                    more = false;
                } else {
                    it = item_of(a, t);
                    hh = 0;
                    nh = it.nh;
                    rel = n;
                }
            }
            const int xs = hk % kNX, s = hk % kNS;
            if (lok && more) {
                bool w = wait_sleep(bar + K::X_FULL + xs, (uint32_t)(hk / kNX) & 1, abort_flag, status);
                w = w && wait_sleep(bar + K::SV_FULL + s, (uint32_t)(hk / kNS) & 1, abort_flag, status);
                w = w && wait_sleep(bar + K::XQ_EMPTY, ((uint32_t)hk & 1) ^ 1, abort_flag, status);
                lok = __all_sync(0xffffffffu, w);
            }
            if (!tc::named_and(kIdState, 128, lok)) {
                ok = false;
                break;
            }
            if (!more) break;
            {
                const int h = it.h0 + hh;
                const float* lut = sv(s) + K::SV_LUT / 4;
                float inv_sx[8];
                {
                    const float4* sx4 = reinterpret_cast<const float4*>(a.inv_sx + h * kP + p0);
                    const float4 a0 = __ldg(sx4), a1 = __ldg(sx4 + 1);
                    inv_sx[0] = a0.x; inv_sx[1] = a0.y; inv_sx[2] = a0.z; inv_sx[3] = a0.w;
                    inv_sx[4] = a1.x; inv_sx[5] = a1.y; inv_sx[6] = a1.z; inv_sx[7] = a1.w;
                }
                const uint8_t* xt = sm + K::OFF_X + xs * K::X_BYTES;
                uint8_t* xq = sm + K::OFF_XQ;
#pragma unroll 1
                for (int half = 0; half < kChunks; half += kBatch) {
                    uint4 v[kBatch];
                    float f[kBatch];
#pragma unroll
                    for (int i = 0; i < kBatch; ++i) {
                        const int ck = pt + (half + i) * 128;
                        v[i] = *reinterpret_cast<const uint4*>(xt + ck * 16);
                        f[i] = lut[ck >> 3];
                    }
#pragma unroll
                    for (int i = 0; i < kBatch; ++i) {
                        const int row = (pt >> 3) + (half + i) * 16;
                        const uint32_t wv[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
                        int q[8];
#pragma unroll
                        for (int e = 0; e < 8; e += 2) {
                            float xs0, xs1, u0, u1;
                            mul_f32x2(xs0, xs1, f[i], f[i], bf16lo(wv[e >> 1]), bf16hi(wv[e >> 1]));
                            mul_f32x2(u0, u1, xs0, xs1, inv_sx[e], inv_sx[e + 1]);
                            code_bits2(q[e], q[e + 1], u0, u1);
                        }
                        const uint2 qq = make_uint2(pack_i8x4(q[0], q[1], q[2], q[3]), pack_i8x4(q[4], q[5], q[6], q[7]));
                        // 64-byte swizzle: 16-byte chunk index (p / 16) XOR address bits 7..8
                        const int off = row * 64 + (((p0 >> 4) ^ ((row >> 1) & 3)) << 4) + (p0 & 15);
                        *reinterpret_cast<uint2*>(xq + off) = qq;
                    }
                }
                tc::fence_proxy_async_smem();
                if (a.dbg.Xq) {
                    tc::named_sync(kIdState, 128);                   // the whole tile is written
                    dump_xq(xq, Q, a.dbg.Xq + (((long long)it.b * d.Lp() + (long long)it.c * Q) * d.H + h) * kP,
                            (long long)d.H * kP, pt, 128);
                }
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bar + K::XPREP + xs);      // x no longer needed here
            }
            // Xq written by all four warps (and the accumulator drained at the top): the MMA
            if (!tc::named_and(kIdState, 128, true)) {
                ok = false;
                break;
            }
            if (issuer) {
                const int tb = 2 * n;
                if (hh == 0 && !wait_all(bar + K::TILE_FULL + tb % kNT, (uint32_t)(tb / kNT) & 1, abort_flag, status)) {
                    // the others see the missing MMA as an expired wait on its barrier
                } else {
                    tc::tc_fence_after();
                    if (tc::elect_one()) {
                        const uint64_t dA = dTileMN + (uint64_t)(((tb % kNT) * K::TILE) >> 4);
#pragma unroll
                        for (int st = 0; st < Q / 32; ++st)
                            tc::mma_i8_ss(tmem + K::SCOL, dA + (uint64_t)(st * 256), dXq + (uint64_t)(st * 128), idS,
                                          st > 0 ? 1u : 0u);
                        tc::mma_commit(bar + K::XQ_EMPTY);
                        tc::mma_commit(bar + K::S_FULL);
                    }
                    __syncwarp();
                }
            }
            pending = true;
            pb = it.b;
            pc = it.c;
            ph = it.h0 + hh;
            ++hh;
            ++hk;
        }
        if (rel >= 0 && ok) item_release(rel);
        // the MMAs this warp issued must finish before TMEM is freed
        if (issuer) {
            if (tc::elect_one()) tc::mma_commit(bar + K::DONE_S);
            __syncwarp();
            tc::mbar_wait(bar + K::DONE_S, 0, tc::kWaitLimit);
        }
    } else if (warp < kWarpScale) {
        // ================================================================ builders
        const int set = (warp - kWarpBuild) >> 2;
        const int quarter = warp & 3;
        const int rrow = quarter * 32 + lane;                       // row within a 128-row tile
        const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
        const int c0 = 16 * set;                                    // first column within a 32-column block
        uint32_t dmask[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int cc = c0 + 2 * k;
            dmask[k] = cc + 1 <= lane ? 0xffffffffu : (cc == lane ? 0x0000ffffu : 0u);
        }
        int hk = 0, p = 0;
        bool ok = true;
        for (int n = 0; ok; ++n) {
            const int t = item_get(n);
            if (t < 0) break;
            const Item it = item_of(a, t);
            for (int hh = 0; hh < it.nh; ++hh, ++hk) {
                const int s = hk % kNC;
                const bool first = hh == 0, last = hh == it.nh - 1;
                if (!wait_all(bar + K::CV_FULL + s, (uint32_t)(hk / kNC) & 1, abort_flag, status)) {
                    ok = false;
                    break;
                }
                const float* a2 = cv(s) + K::CV_A2 / 4;
                const float* dtw = cv(s) + K::CV_DTW / 4;
                const uint32_t* v32 = reinterpret_cast<const uint32_t*>(cv(s) + K::CV_VB / 4);
                auto cb_cols = [&](int k) -> uint32_t {
                    int J, ib;
                    piece_of<Q>(k, J, ib);
                    return trow + (J == 0 ? K::CBP0 : K::CBP1) + ib * 32 + c0 / 2;
                };
                // One 16-column group of 32 x 32 block `cb` of M for rows of block `jb`.
                // Below the diagonal the decay factorises through the end r of the block's
                // columns, exp(Acs_j - Acs_r) * exp(Acs_r - Acs_i) (both <= 1); on the
                // diagonal it takes one exponential per element; above it is zero.
                auto build16 = [&](const uint32_t (&v)[8], int jb, int cb, float aj, uint32_t (&out)[8]) {
                    const int i0 = 32 * cb + c0;
                    if (jb > cb) {
                        const float uj = ex2(fminf(aj - a2[32 * cb + 31], 0.f));
                        const uint32_t ub = pack_bf16(uj, uj);
                        const uint4* v4 = reinterpret_cast<const uint4*>(v32 + i0 / 2);
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            const uint4 f = v4[q];
                            out[4 * q] = mul_bf16x2(v[4 * q], mul_bf16x2(ub, f.x));
                            out[4 * q + 1] = mul_bf16x2(v[4 * q + 1], mul_bf16x2(ub, f.y));
                            out[4 * q + 2] = mul_bf16x2(v[4 * q + 2], mul_bf16x2(ub, f.z));
                            out[4 * q + 3] = mul_bf16x2(v[4 * q + 3], mul_bf16x2(ub, f.w));
                        }
                    } else if (jb == cb) {
                        // exp(Acs_j - Acs_i) dt_i = 2^(a_j + (log2(dt_i) - a_i)); entries above the
                        // diagonal may overflow and are cleared by the row's pair masks
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
                uint32_t cur0[8], cur1[8], nx0[8], nx1[8];
                const int k0 = piece_at<Q>(0);
                if (first && !wait_all(bar + K::CBU_PACKED + k0, (uint32_t)n & 1, abort_flag, status)) {
                    ok = false;
                    break;
                }
                tc::tc_fence_after();
                tc::tmem_ld8(cb_cols(k0), cur0);
                tc::tmem_ld8(cb_cols(k0) + 16, cur1);
                tc::tmem_wait_ld();
                if (last) {
                    tc::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(bar + K::CBU_FREE + k0);
                }
#pragma unroll 1
                for (int i = 0; i < K::NPIECE; ++i) {
                    const int k = piece_at<Q>(i);
                    int J, ib;
                    piece_of<Q>(k, J, ib);
                    const bool pre = i + 1 < K::NPIECE;
                    const int kn = pre ? piece_at<Q>(i + 1) : 0;
                    if (pre) {
                        if (first && !wait_all(bar + K::CBU_PACKED + kn, (uint32_t)n & 1, abort_flag, status)) {
                            ok = false;
                            break;
                        }
                        tc::tc_fence_after();
                        tc::tmem_ld8(cb_cols(kn), nx0);
                        tc::tmem_ld8(cb_cols(kn) + 16, nx1);
                    }
                    const int slot = p % kRing;
                    const int jrow = J * 128 + rrow;
                    const int jb = 4 * J + quarter;
                    const float aj = a2[jrow < Q ? jrow : Q - 1];
                    uint32_t out0[8], out1[8];
                    build16(cur0, jb, 2 * ib, aj, out0);
                    build16(cur1, jb, 2 * ib + 1, aj, out1);
                    if (!wait_all(bar + K::REMPTY + slot, ((uint32_t)(p / kRing) & 1) ^ 1, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    const uint32_t dst = trow + K::RING + slot * 32 + c0 / 2;
                    tc::tmem_st8(dst, out0);
                    tc::tmem_st8(dst + 16, out1);
                    tc::tmem_wait_st();
                    tc::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(bar + K::RFULL + slot);
                    ++p;
                    if (pre) {
                        tc::tmem_wait_ld();
                        if (last) {
                            tc::tc_fence_before();
                            __syncwarp();
                            if (lane == 0) tc::mbar_arrive(bar + K::CBU_FREE + kn);
                        }
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            cur0[e] = nx0[e];
                            cur1[e] = nx1[e];
                        }
                    }
                }
                tc::tmem_wait_ld();
                if (!ok) break;
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bar + K::CV_EMPTY + s);
            }
            if (!ok) break;
            item_release(n);
        }
    } else if (warp < kWarpStore) {
        // ================================================================ scalers
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
        int yk = 0, hk = 0, cbu = 0;
        uint32_t ru_par = 0;
        bool ok = true;
        for (int n = 0; ok; ++n) {
            const int t = item_get(n);
            if (t < 0) break;
            const Item it = item_of(a, t);
            // ChunkBMM job: the CB units, packed to bf16 pairs in TMEM
            {
                const int slot = yk % kNY;
                for (int ui = 0; ui < K::NPIECE; ++ui, ++cbu) {
                    const int u = piece_at<Q>(ui);
                    if (n > 0 && !wait_all(bar + K::CBU_FREE + u, (uint32_t)(n - 1) & 1, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    if (!wait_all(bar + K::CBU_FULL, (uint32_t)cbu & 1, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
                    int J, ib;
                    piece_of<Q>(u, J, ib);
                    const int j = J * 128 + r;
                    const bool dump = a.dbg.cb && j < Q && it.h0 == it.g * d.hpg;   // one item per group
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        uint32_t v[32], w[16];
                        tc::tmem_ld32(trow + K::YCOL + 64 * slot + 32 * hf, v);
                        tc::tmem_wait_ld();
                        if (hf == 1) {
                            // the staging columns have been read: the next unit may go there
                            tc::tc_fence_before();
                            __syncwarp();
                            if (lane == 0) tc::mbar_arrive(bar + K::CBU_EMPTY);
                        }
                        if (dump)
                            dump32(a.dbg.cb + ((((long long)it.b * nc + it.c) * d.G + it.g) * Q + j) * Q + ib * 64 +
                                       32 * hf,
                                   1, v);
#pragma unroll
                        for (int i = 0; i < 16; ++i) w[i] = pack_bf16((float)(int)v[2 * i], (float)(int)v[2 * i + 1]);
                        tc::tmem_st16(trow + (J == 0 ? K::CBP0 : K::CBP1) + ib * 32 + 16 * hf, w);
                    }
                    tc::tmem_wait_st();
                    tc::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(bar + K::CBU_PACKED + u);
                }
                if (!ok) break;
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bar + K::YEMPTY + slot);
                ++yk;
            }
            // ChunkScan1 jobs: dequantise in place, rows times exp(Acs_j)
            for (int hh = 0; hh < it.nh && ok; ++hh, ++hk) {
                const int s = hk % kNC;
                const int h = it.h0 + hh;
                if (!wait_all(bar + K::CV_FULL + s, (uint32_t)(hk / kNC) & 1, abort_flag, status)) {
                    ok = false;
                    break;
                }
                const float* a2 = cv(s) + K::CV_A2 / 4;
                const float* mul = a.mulC + h * kP;
                for (int jj = 0; jj < K::JT; ++jj) {
                    const int J = K::JT - 1 - jj;
                    const int slot = yk % kNY;
                    const uint32_t par = (ru_par >> slot) & 1;
                    ru_par ^= 1u << slot;
                    if (!wait_all(bar + K::YO_FULL + slot, par, abort_flag, status)) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
                    const int j = J * 128 + r;
                    const float e = ex2(fminf(a2[j < Q ? j : Q - 1], 0.f));
                    const uint32_t ybase = trow + K::YCOL + 64 * slot;
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        uint32_t v[32];
                        tc::tmem_ld32(ybase + 32 * hf, v);
                        tc::tmem_wait_ld();
                        if (a.dbg.acc_scan1 && j < Q)
                            dump32(a.dbg.acc_scan1 +
                                       (((long long)it.b * d.Lp() + (long long)it.c * Q + j) * d.H + h) * kP + 32 * hf,
                                   1, v);
#pragma unroll
                        for (int i = 0; i < 32; i += 2) {
                            const float2 mm = __ldg(reinterpret_cast<const float2*>(mul + 32 * hf + i));
                            float f0, f1;
                            add_f32x2(f0, f1, __int_as_float((int)v[i] + kRoundBits),
                                      __int_as_float((int)v[i + 1] + kRoundBits), -kRound, -kRound);
                            mul_f32x2(f0, f1, f0, f1, mm.x, mm.y);
                            mul_f32x2(f0, f1, f0, f1, e, e);
                            v[i] = __float_as_uint(f0);
                            v[i + 1] = __float_as_uint(f1);
                        }
                        tc::tmem_st32(ybase + 32 * hf, v);
                    }
                    tc::tmem_wait_st();
                    tc::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(bar + K::YSCALED + slot);
                    ++yk;
                }
                if (!ok) break;
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bar + K::CV_EMPTY + s);
            }
            if (!ok) break;
            item_release(n);
        }
    } else {
        // ================================================================ storers
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
        const bool issuer = warp == kWarpStore && lane == 0;
        int yk = 0, hk = 0;
        uint32_t ru_par = 0;
        bool ok = true;
        for (int n = 0; ok; ++n) {
            const int t = item_get(n);
            if (t < 0) break;
            const Item it = item_of(a, t);
            ++yk;                                                   // the item's ChunkBMM job
            for (int hh = 0; hh < it.nh && ok; ++hh, ++hk) {
                const int xs = hk % kNX, h = it.h0 + hh;
                uint8_t* xt = sm + K::OFF_X + xs * K::X_BYTES;
                const float Dh = __ldg(a.D + h);
                for (int jj = 0; jj < K::JT; ++jj) {
                    const int J = K::JT - 1 - jj;
                    const int slot = yk % kNY;
                    const uint32_t par = (ru_par >> slot) & 1;
                    ru_par ^= 1u << slot;
                    bool w = wait_sleep(bar + K::YFULL + slot, par, abort_flag, status);
                    if (jj == 0)
                        w = w && wait_sleep(bar + K::XPREP + xs, (uint32_t)(hk / kNX) & 1, abort_flag, status);
                    if (!tc::named_and(kIdStore, 128, w)) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
                    const uint32_t ybase = trow + K::YCOL + 64 * slot;
                    const int j = J * 128 + r;
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        uint32_t v[32];
                        tc::tmem_ld32(ybase + 32 * hf, v);
                        tc::tmem_wait_ld();
                        if (hf == 1) {
                            tc::tc_fence_before();
                            __syncwarp();
                            if (lane == 0) tc::mbar_arrive(bar + K::YEMPTY + slot);
                        }
                        if (j < Q) {
#pragma unroll
                            for (int q = 4 * hf; q < 4 * hf + 4; ++q) {
                                uint4* px = reinterpret_cast<uint4*>(xt + j * 128 + ((q ^ (j & 7)) << 4));
                                const uint4 xv = *px;
                                const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
                                uint32_t o[4];
#pragma unroll
                                for (int e2 = 0; e2 < 4; ++e2) {
                                    const int col = (q - 4 * hf) * 8 + 2 * e2;
                                    float o0, o1;
                                    fma_f32x2(o0, o1, Dh, Dh, bf16lo(xw[e2]), bf16hi(xw[e2]), __uint_as_float(v[col]),
                                              __uint_as_float(v[col + 1]));
                                    o[e2] = pack_bf16(o0, o1);
                                }
                                *px = make_uint4(o[0], o[1], o[2], o[3]);
                            }
                        }
                    }
                    tc::fence_proxy_async_smem();
                    tc::named_sync(kIdStore, 128);
                    if (issuer) {
                        tc::tma_store_3d(&tm_y, xt + J * 128 * 128, h * kP, it.c * Q + J * 128, it.b);
                        tc::tma_store_commit();
                        if (jj == K::JT - 1) {
                            // the head's stores have read the tile: the x stage may refill
                            tc::tma_store_wait_read0();
                            tc::mbar_arrive(bar + K::X_EMPTY + xs);
                        }
                    }
                    ++yk;
                }
            }
            if (!ok) break;
            item_release(n);
        }
        if (issuer) tc::tma_store_wait0();
    }
    __syncwarp();
    tc::tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) tc::tmem_dealloc(tmem, 512);
}

// The per-(h,p) factors of the W8A8 scan, in the fp32 operation order of the
// specification: 1/s_x (IEEE division), s_x s_B / s_s, and s_C s_s.
__global__ void fused_i8_tables_kernel(int HP, int P, int hpg, I8Scales sc, float* inv_sx, float* mq, float* mulC) {
    const int o = blockIdx.x * blockDim.x + threadIdx.x;
    if (o >= HP) return;
    const int g = o / P / hpg;
    const float sx = __ldg(sc.s_x + o), ss = __ldg(sc.s_s + o);
    inv_sx[o] = __frcp_rn(sx);
    mq[o] = __fdiv_rn(__fmul_rn(sx, __ldg(sc.s_B + g)), ss);
    mulC[o] = __ldg(sc.s_C + g) * ss;
}

template <int Q>
cudaError_t launch_q(const FusedI8Args& a, const CUtensorMap* maps, cudaStream_t st) {
    using K = Cfg<Q>;
    auto k = ssd_fused_i8_kernel<Q>;
    const int smem = K::BYTES + 128;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int sms = device_sm_count();
    const int grid = a.items < sms ? a.items : sms;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;          // every CTA resident
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, maps[0], maps[1], maps[2], maps[3], maps[4], a);
}

}  // namespace

size_t fused_i8_ws_bytes(const Dims& d, size_t* ctrl_bytes) {
    const size_t bch = (size_t)d.B * d.nc * d.H;
    const size_t ctrl = ((256 + bch * sizeof(int)) + 255) & ~(size_t)255;    // status, ticket, flags
    if (ctrl_bytes) *ctrl_bytes = ctrl;
    const size_t tables = ((size_t)3 * d.H * kP * sizeof(float) + 255) & ~(size_t)255;
    return ctrl + tables + ((bch * kP * kN + 255) & ~(size_t)255);
}

int fused_heads_per_item(const Dims& d) {
    // Few heads per item pay the item's ChunkBMM job and pipeline turn-over often; many
    // leave a longer ragged end.  Cost in head-times per SM: (heads + 1.5 per item) / SMs
    // plus half an item for the end.
    const int sms = device_sm_count();
    int best = d.hpg;
    double best_cost = -1.0;
    for (int K : {4, 5, 6, 8, 10, 12, 16, 20}) {
        const int k = K < d.hpg ? K : d.hpg;
        const double items = (double)d.G * ((d.hpg + k - 1) / k) * d.nc * d.B;
        const double cost = ((double)d.B * d.nc * d.H + 1.5 * items) / sms + 0.5 * (k + 1.5);
        if (best_cost < 0 || cost < best_cost - 1e-9) {
            best_cost = cost;
            best = k;
        }
    }
    const char* env = getenv("SSD_FUSED_HEADS");
    if (env) {
        const int v = atoi(env);
        if (v >= 1) best = v < d.hpg ? v : d.hpg;
    }
    return best;
}

cudaError_t launch_fused_i8(const Dims& d, const uint16_t* x, const float* dt, const float* A, const int8_t* Bq,
                            const int8_t* Cq, const float* D, const I8Scales& sc, const int8_t* init8, uint16_t* y,
                            int8_t* final8, void* ws, const I8Debug* dbg, cudaStream_t st) {
    if (d.B == 0 || d.nc == 0) return cudaSuccess;
    if (d.P != kP || d.N != kN) return cudaErrorInvalidValue;
    size_t ctrl = 0;
    fused_i8_ws_bytes(d, &ctrl);
    const size_t bch = (size_t)d.B * d.nc * d.H;
    char* w = static_cast<char*>(ws);
    FusedI8Args a{};
    a.d = d;
    a.K = fused_heads_per_item(d);
    a.nhb_g = (d.hpg + a.K - 1) / a.K;
    a.nhb = d.G * a.nhb_g;
    const long long items = (long long)d.B * d.nc * a.nhb;
    if (items > 0x7fffffffLL || bch * kN > 0x7fffffffULL) return cudaErrorInvalidValue;
    a.items = (int)items;
    a.dt = dt;
    a.A = A;
    a.D = D;
    a.sc = sc;
    a.status = reinterpret_cast<int*>(w);
    a.ticket = reinterpret_cast<int*>(w) + 1;
    a.hflag = reinterpret_cast<int*>(w + 256);
    const int HP = d.H * kP;
    float* tables = reinterpret_cast<float*>(w + ctrl);
    a.inv_sx = tables;
    a.mq = tables + HP;
    a.mulC = tables + 2 * HP;
    a.Hpub = reinterpret_cast<int8_t*>(w + ctrl + ((((size_t)3 * HP * sizeof(float)) + 255) & ~(size_t)255));
    a.init8 = init8;
    a.final8 = final8;
    if (dbg) a.dbg = *dbg;
    cudaError_t e = cudaMemsetAsync(w, 0, ctrl, st);
    if (e != cudaSuccess) return e;
    fused_i8_tables_kernel<<<(HP + 255) / 256, 256, 0, st>>>(HP, kP, d.hpg, sc, tables, tables + HP, tables + 2 * HP);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    CUtensorMap maps[5];
    const unsigned long long HPu = (unsigned long long)HP, GN = (unsigned long long)d.G * kN;
    const unsigned crows = d.Q >= 128 ? d.Q : 128, yrows = d.Q >= 128 ? 128 : d.Q;
    bool ok = make_tmap_3d(&maps[0], false, x, HPu, d.L, d.B, HPu * 2, d.Ls * HPu * 2, 64, d.Q,
                           CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_tmap_3d(&maps[1], false, y, HPu, d.L, d.B, HPu * 2, d.Ls * HPu * 2, 64, yrows,
                            CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_tmap_3d(&maps[2], true, Bq, GN, d.L, d.B, GN, d.Ls * GN, 128, d.Q, CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_tmap_3d(&maps[3], true, Cq, GN, d.L, d.B, GN, d.Ls * GN, 128, crows, CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_tmap_2d(&maps[4], true, a.Hpub, kP, (unsigned long long)bch * kN, kP, 64, kN,
                            CU_TENSOR_MAP_SWIZZLE_64B);
    if (!ok) return cudaErrorInvalidValue;
    switch (d.Q) {
        case 64: return launch_q<64>(a, maps, st);
        case 128: return launch_q<128>(a, maps, st);
        case 256: return launch_q<256>(a, maps, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace ssd
