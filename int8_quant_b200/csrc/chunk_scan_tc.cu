// chunk_scan_tc.cu — a4..a7 on the tensor cores (P = 64, N = 128): ChunkBMM,
// ChunkScan1, ChunkScan2 and the D skip (SSDi8 notes, "overall framework" and key
// design 2):
//   CB[j,i]  = C_j . B_i                                      (ChunkBMM)
//   y[j,p]   = exp(Acs_j) sum_n C[j,n] H_c[p,n]                 (ChunkScan1)
//            + sum_{i<=j} CB[j,i] exp(Acs_j - Acs_i) dt_i x[i,p]  (ChunkScan2)
//            + D x[j,p]
// W8A8: CB and the ChunkScan1 sum are int32 (kind::i8 on Cq, Bq, H8); the ChunkScan1
// result is dequantised with s_C s_s[h,p]; LUT_Scan2 = s_C s_B exp(Acs_j - Acs_i) dt_i
// folds CB's dequantisation into the ChunkScan2 matrix, which runs in bf16 (kind::f16).
//
// One CTA per (chunk, batch row, block of heads of one group).  B and C are shared
// by the block, so CB = C B^T is computed once (rows j in tiles of 128, causal
// columns only) and kept in TMEM for all heads.  Per head:
//  1. MMA: y = C H^T into the head's TMEM accumulator (one [128 x 64] tile per
//     128 rows of the chunk);
//  2. eight warps scale each accumulator row by exp(Acs_j) (W8A8: convert the
//     int32 sums and apply s_C s_s[p]) in place, and turn CB rows into the masked
//     matrix M[j,i] = CB[j,i] exp(Acs_j - Acs_i) dt_i (bf16, K-major, 128-byte
//     swizzle) in shared memory — for the block below the 128-row diagonal the
//     decay factorises as exp(Acs_j - Acs_127) * exp(Acs_127 - Acs_i), both <= 1,
//     so only diagonal blocks take one exponential per element;
//  3. MMA: y += M x, with x as TMA loaded it (MN-major) — M pieces of 128 columns
//     stream through two 32 KB buffers so building and multiplying overlap;
//  4. eight warps add D x, round to bf16 in place of the x tile, and one thread
//     stores the tile with TMA.
// TMA brings the next head's x (double-buffered) and state while this head runs.
#include "kernels.h"
#include "tc.cuh"

namespace ssd {

namespace {

constexpr int kThreads = 256;
constexpr int kP = 64;
constexpr int kN = 128;
constexpr float kLog2e = 1.4426950408889634f;

template <int Q, bool kI8>
struct ScanCfg {
    static constexpr int JT = Q >= 128 ? Q / 128 : 1;            // 128-row tiles of the chunk
    static constexpr int CROWS = Q >= 128 ? Q : 128;             // C rows loaded (Q = 64: 64 ghost rows)
    static constexpr int NCB0 = Q >= 128 ? 128 : Q;              // CB columns of tile 0
    static constexpr int CB1_COL = NCB0;                         // CB tile 1 (JT = 2): 256 columns
    static constexpr int Y_COL = JT == 2 ? 384 : NCB0;           // y accumulators, 64 columns per tile
    static constexpr int TMEM_COLS = JT == 2 ? 512 : (Q == 128 ? 256 : 128);
    static constexpr int EB = kI8 ? 1 : 2;                       // bytes per B/C/state element
    static constexpr int ATOM_ROWS_C = CROWS;                    // rows of one 128-byte K atom of C
    static constexpr int C_BYTES = CROWS * kN * EB;
    static constexpr int B_BYTES = Q * kN * EB;
    static constexpr int H_BYTES = kP * kN * EB;
    static constexpr int X_BYTES = Q * 128;                      // x tile bf16 [Q][64]
    static constexpr int MPIECE = 128 * 128 * 2;                 // [128 rows][128 i] bf16
    static constexpr int M_BYTES = (JT == 2 ? 2 : 1) * MPIECE;
    static constexpr int OFF_C = 0;
    static constexpr int OFF_B = OFF_C + C_BYTES;
    // bf16: the M pieces reuse the B tile once CB is computed (B is then dead)
    static constexpr int OFF_M = kI8 ? OFF_B + B_BYTES : OFF_B;
    static constexpr int BM_END = kI8 ? OFF_M + M_BYTES : OFF_B + (B_BYTES > M_BYTES ? B_BYTES : M_BYTES);
    static constexpr int OFF_X = (BM_END + 1023) & ~1023;
    static constexpr int OFF_H = OFF_X + 2 * X_BYTES;
    static constexpr int OFF_A2 = OFF_H + H_BYTES;               // float [Q]  Acs * log2(e)
    static constexpr int OFF_DTW = OFF_A2 + Q * 4;               // float [Q]  dt (* s_C s_B)
    static constexpr int OFF_VL = OFF_DTW + Q * 4;               // float [128] exp(Acs_127 - Acs_i) dtw_i
    static constexpr int OFF_SCS = OFF_VL + 128 * 4;             // float [64] s_C s_s[h,p] (W8A8)
    static constexpr int OFF_BAR = OFF_SCS + 64 * 4;             // mbarriers
    static constexpr int NBAR = 10;
    static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_TMEM + 16;
};

// K-major 128B-swizzled tile: element (row, k) of a tile whose 128-byte K atoms hold
// `rows` rows each, at byte offset (within the tile) of its 16-byte chunk.
__device__ __forceinline__ int kmajor_chunk_off(int row, int katom, int chunk, int rows) {
    return katom * rows * 128 + row * 128 + ((chunk ^ (row & 7)) << 4);
}

// Bounded wait whose outcome every thread of the block agrees on (the block then
// leaves the head loop together when a wait expires).
__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity) {
    const bool ok = tc::mbar_wait(bar, parity, tc::kWaitLimit);
    return __syncthreads_and(ok ? 1 : 0) != 0;
}

template <int Q, bool kI8>
__global__ void __launch_bounds__(kThreads, 1)
chunk_scan_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_h,
                     const __grid_constant__ CUtensorMap tm_y, Dims d, int heads_per_cta, int ctas_per_group,
                     const float* __restrict__ Acs, const float* __restrict__ dtc, const float* __restrict__ Dv,
                     I8Scales sc, I8Debug dbg, int* __restrict__ status) {
    using K = ScanCfg<Q, kI8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, half = warp >> 2;
    const int c = blockIdx.y, b = blockIdx.z;
    const int g = blockIdx.x / ctas_per_group;
    const int h0 = g * d.hpg + (blockIdx.x % ctas_per_group) * heads_per_cta;
    const int nh = min(heads_per_cta, g * d.hpg + d.hpg - h0);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + K::OFF_BAR);
    uint64_t* bar_load = bar + 0;       // C and B tiles
    uint64_t* bar_x = bar + 1;          // [2] x tiles
    uint64_t* bar_h = bar + 3;          // state tile
    uint64_t* bar_cb = bar + 4;         // CB MMAs
    uint64_t* bar_yo = bar + 5;         // ChunkScan1 MMAs
    uint64_t* bar_y0 = bar + 6;         // ChunkScan2, tile 0
    uint64_t* bar_y1a = bar + 7;        // ChunkScan2, tile 1, columns 0..127
    uint64_t* bar_y1b = bar + 8;        // ChunkScan2, tile 1, columns 128..255
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + K::OFF_TMEM);
    float* a2 = reinterpret_cast<float*>(sm + K::OFF_A2);
    float* dtw = reinterpret_cast<float*>(sm + K::OFF_DTW);
    float* vL = reinterpret_cast<float*>(sm + K::OFF_VL);
    float* sCs = reinterpret_cast<float*>(sm + K::OFF_SCS);

    if (tid == 0) {
        for (int i = 0; i < K::NBAR; ++i) tc::mbar_init(bar + i, 1);
        tc::fence_mbar_init();
        tc::prefetch_tmap(&tm_x);
        tc::prefetch_tmap(&tm_b);
        tc::prefetch_tmap(&tm_c);
        tc::prefetch_tmap(&tm_h);
        tc::prefetch_tmap(&tm_y);
    }
    if (warp == 0) {
        tc::tmem_alloc(tmem_slot, K::TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const long long hc_row0 = ((long long)b * d.nc + c) * d.H;      // state rows: (hc_row0 + h) * 64

    if (tid == 0) {
        // C (and its ghost rows for Q = 64), B, the first x tiles and the first state
        tc::mbar_arrive_expect_tx(bar_load, K::C_BYTES + K::B_BYTES);
        if (!kI8) {
            tc::tma_load_3d(sm + K::OFF_C, &tm_c, bar_load, g * kN, c * Q, b);
            tc::tma_load_3d(sm + K::OFF_C + K::CROWS * 128, &tm_c, bar_load, g * kN + 64, c * Q, b);
            tc::tma_load_3d(sm + K::OFF_B, &tm_b, bar_load, g * kN, c * Q, b);
            tc::tma_load_3d(sm + K::OFF_B + Q * 128, &tm_b, bar_load, g * kN + 64, c * Q, b);
        } else {
            tc::tma_load_3d(sm + K::OFF_C, &tm_c, bar_load, g * kN, c * Q, b);
            tc::tma_load_3d(sm + K::OFF_B, &tm_b, bar_load, g * kN, c * Q, b);
        }
        for (int i = 0; i < 2 && i < nh; ++i) {
            tc::mbar_arrive_expect_tx(bar_x + i, K::X_BYTES);
            tc::tma_load_3d(sm + K::OFF_X + i * K::X_BYTES, &tm_x, bar_x + i, (h0 + i) * kP, c * Q, b);
        }
        tc::mbar_arrive_expect_tx(bar_h, K::H_BYTES);
        if (!kI8) {
            tc::tma_load_2d(sm + K::OFF_H, &tm_h, bar_h, 0, (int)((hc_row0 + h0) * kP));
            tc::tma_load_2d(sm + K::OFF_H + kP * 128, &tm_h, bar_h, 64, (int)((hc_row0 + h0) * kP));
        } else {
            tc::tma_load_2d(sm + K::OFF_H, &tm_h, bar_h, 0, (int)((hc_row0 + h0) * kP));
        }
    }
    bool ok = wait_all(bar_load, 0);

    const uint32_t aC = tc::smem_u32(sm + K::OFF_C);
    const uint32_t aB = tc::smem_u32(sm + K::OFF_B);
    const uint32_t aH = tc::smem_u32(sm + K::OFF_H);
    const uint32_t aM = tc::smem_u32(sm + K::OFF_M);
    // A operand (C rows from r0), K step s: bf16 K atoms of 64 n, 4 steps of 16 per atom;
    // int8 one atom of 128 n, 4 steps of 32.
    auto descC = [&](int r0, int s) -> uint64_t {
        const uint32_t off = kI8 ? (uint32_t)(s * 32) : (uint32_t)((s >> 2) * K::CROWS * 128 + (s & 3) * 32);
        return tc::smem_desc(aC + r0 * 128 + off, 16, 1024, tc::kLayoutSw128);
    };
    auto descB = [&](int s) -> uint64_t {
        const uint32_t off = kI8 ? (uint32_t)(s * 32) : (uint32_t)((s >> 2) * Q * 128 + (s & 3) * 32);
        return tc::smem_desc(aB + off, 16, 1024, tc::kLayoutSw128);
    };
    auto descH = [&](int s) -> uint64_t {
        const uint32_t off = kI8 ? (uint32_t)(s * 32) : (uint32_t)((s >> 2) * kP * 128 + (s & 3) * 32);
        return tc::smem_desc(aH + off, 16, 1024, tc::kLayoutSw128);
    };
    constexpr int kSteps = kI8 ? 4 : 8;          // K = 128 (n) in MMA steps

    // ---- ChunkBMM: CB = C B^T, causal column range of each 128-row tile
    if (ok && tid == 0) {
        tc::tc_fence_after();
        if (!kI8) {
            const uint32_t id0 = tc::idesc_bf16_f32(128, K::NCB0, tc::kMajorK, tc::kMajorK);
            for (int s = 0; s < kSteps; ++s) tc::mma_f16_ss(tmem, descC(0, s), descB(s), id0, s > 0);
            if (K::JT == 2) {
                const uint32_t id1 = tc::idesc_bf16_f32(128, 256, tc::kMajorK, tc::kMajorK);
                for (int s = 0; s < kSteps; ++s)
                    tc::mma_f16_ss(tmem + K::CB1_COL, descC(128, s), descB(s), id1, s > 0);
            }
        } else {
            const uint32_t id0 = tc::idesc_s8_s32(128, K::NCB0, tc::kMajorK, tc::kMajorK);
            for (int s = 0; s < kSteps; ++s) tc::mma_i8_ss(tmem, descC(0, s), descB(s), id0, s > 0);
            if (K::JT == 2) {
                const uint32_t id1 = tc::idesc_s8_s32(128, 256, tc::kMajorK, tc::kMajorK);
                for (int s = 0; s < kSteps; ++s)
                    tc::mma_i8_ss(tmem + K::CB1_COL, descC(128, s), descB(s), id1, s > 0);
            }
        }
        tc::mma_commit(bar_cb);
    }
    if (ok) ok = wait_all(bar_cb, 0);
    tc::tc_fence_after();
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);  // this warp's TMEM lanes

    // W8A8 debug: the ChunkBMM accumulator, written once per (b, c, g)
    if (kI8 && ok && dbg.cb && (blockIdx.x % ctas_per_group) == 0) {
        for (int J = 0; J < K::JT; ++J) {
            const int ncol = J == 0 ? K::NCB0 : 256;
            const int j = J * 128 + quarter * 32 + lane;
            for (int g32 = half; g32 < ncol / 32; g32 += 2) {
                uint32_t v[32];
                tc::tmem_ld32(trow + (J == 0 ? 0 : K::CB1_COL) + g32 * 32, v);
                tc::tmem_wait_ld();
                if (j < Q) {
                    int32_t* dst = dbg.cb + ((((long long)b * d.nc + c) * d.G + g) * Q + j) * Q + g32 * 32;
#pragma unroll
                    for (int i = 0; i < 32; ++i) dst[i] = (int32_t)v[i];
                }
            }
        }
    }

    const float sCB = kI8 ? __ldg(sc.s_C + g) * __ldg(sc.s_B + g) : 1.f;
    for (int it = 0; it < nh && ok; ++it) {
        const int h = h0 + it;
        const int xb = it & 1;
        const uint32_t par = (uint32_t)(it & 1);
        const uint32_t xpar = (uint32_t)((it >> 1) & 1);
        uint8_t* xs = sm + K::OFF_X + xb * K::X_BYTES;
        const uint32_t aX = tc::smem_u32(xs);

        // per-head rows: Acs * log2(e), dt (with the W8A8 CB scale), decay factors
        {
            const long long r = (((long long)b * d.H + h) * d.nc + c) * Q;
            if (tid < Q) {
                a2[tid] = Acs[r + tid] * kLog2e;
                dtw[tid] = dtc[r + tid] * sCB;
            }
            if (K::JT == 2 && tid < 128) {
                const float a127 = Acs[r + 127] * kLog2e;
                vL[tid] = exp2f(a127 - Acs[r + tid] * kLog2e) * (dtc[r + tid] * sCB);
            }
            if (kI8 && tid < kP) sCs[tid] = __ldg(sc.s_C + g) * __ldg(sc.s_s + h * kP + tid);
        }
        __syncthreads();

        // 1. ChunkScan1 MMA into the head's accumulators
        ok = wait_all(bar_h, par);
        if (!ok) break;
        if (tid == 0) {
            tc::tc_fence_after();
            for (int J = 0; J < K::JT; ++J) {
                const uint32_t dcol = tmem + K::Y_COL + J * 64;
                if (!kI8) {
                    const uint32_t id = tc::idesc_bf16_f32(128, kP, tc::kMajorK, tc::kMajorK);
                    for (int s = 0; s < kSteps; ++s) tc::mma_f16_ss(dcol, descC(J * 128, s), descH(s), id, s > 0);
                } else {
                    const uint32_t id = tc::idesc_s8_s32(128, kP, tc::kMajorK, tc::kMajorK);
                    for (int s = 0; s < kSteps; ++s) tc::mma_i8_ss(dcol, descC(J * 128, s), descH(s), id, s > 0);
                }
            }
            tc::mma_commit(bar_yo);
        }
        ok = wait_all(bar_yo, par);
        if (!ok) break;
        tc::tc_fence_after();
        if (tid == 0 && it + 1 < nh) {          // the state tile is free: fetch the next head's
            tc::mbar_arrive_expect_tx(bar_h, K::H_BYTES);
            const int row = (int)((hc_row0 + h + 1) * kP);
            tc::tma_load_2d(sm + K::OFF_H, &tm_h, bar_h, 0, row);
            if (!kI8) tc::tma_load_2d(sm + K::OFF_H + kP * 128, &tm_h, bar_h, 64, row);
        }
        ok = wait_all(bar_x + xb, xpar);
        if (!ok) break;

        // 2a. scale the ChunkScan1 rows by exp(Acs_j) (W8A8: dequantise) in place
        for (int J = 0; J < K::JT; ++J) {
            const int j = J * 128 + quarter * 32 + lane;
            const uint32_t ta = trow + K::Y_COL + J * 64 + half * 32;
            uint32_t v[32];
            tc::tmem_ld32(ta, v);
            tc::tmem_wait_ld();
            const float e = exp2f(a2[j < Q ? j : Q - 1]);
            if (kI8 && dbg.acc_scan1 && j < Q) {
                int32_t* dst = dbg.acc_scan1 + (((long long)b * d.Lp() + (long long)c * Q + j) * d.H + h) * kP +
                               half * 32;
#pragma unroll
                for (int i = 0; i < 32; ++i) dst[i] = (int32_t)v[i];
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float f = kI8 ? (float)(int32_t)v[i] * sCs[half * 32 + i] : __uint_as_float(v[i]);
                v[i] = __float_as_uint(f * e);
            }
            tc::tmem_st32(ta, v);
        }
        tc::tmem_wait_st();

        // Builds 32 columns [col0, col0 + 32) of M for row j of tile J into a piece.
        // diag: columns are in the diagonal 128-block (per-element exponential);
        // otherwise below it (factorised decay u_j * vL_i).
        auto build32 = [&](int J, uint32_t cb_col, int col0, int piece_off, int piece_col0, bool diag) {
            const int j = J * 128 + quarter * 32 + lane;
            const int r = quarter * 32 + lane;                   // row within the piece
            uint32_t v[32];
            tc::tmem_ld32(trow + cb_col + col0, v);
            tc::tmem_wait_ld();
            const float aj = a2[j < Q ? j : Q - 1];
            const float u = diag ? 0.f : exp2f(aj - a2[127]);
            uint32_t packed[16];
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
                float m2[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int ii = col0 + i + e;
                    const float cbv = kI8 ? (float)(int32_t)v[i + e] : __uint_as_float(v[i + e]);
                    float m;
                    if (diag) m = (ii <= j) ? cbv * exp2f(aj - a2[ii]) * dtw[ii] : 0.f;
                    else m = cbv * u * vL[ii];
                    m2[e] = m;
                }
                packed[i >> 1] = (uint32_t)float_to_bf16_bits(m2[0]) | ((uint32_t)float_to_bf16_bits(m2[1]) << 16);
            }
            const int pc = col0 - piece_col0;                    // column within the piece
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int col = pc + q * 8;
                const int off = piece_off + kmajor_chunk_off(r, col >> 6, (col & 63) >> 3, 128);
                *reinterpret_cast<uint4*>(sm + K::OFF_M + off) =
                    make_uint4(packed[q * 4], packed[q * 4 + 1], packed[q * 4 + 2], packed[q * 4 + 3]);
            }
        };
        auto mma_yd = [&](int J, uint32_t piece_addr, int k0, int nk, bool acc_first, uint64_t* done) {
            tc::tc_fence_after();
            const uint32_t id = tc::idesc_bf16_f32(128, kP, tc::kMajorK, tc::kMajorMN);
            const uint32_t dcol = tmem + K::Y_COL + J * 64;
            for (int s = 0; s < nk / 16; ++s) {
                const uint32_t am = piece_addr + (uint32_t)((s >> 2) * 128 * 128 + (s & 3) * 32);
                const uint64_t da = tc::smem_desc(am, 16, 1024, tc::kLayoutSw128);
                const uint64_t db = tc::smem_desc(aX + (uint32_t)((k0 + s * 16) * 128), 0, 1024, tc::kLayoutSw128);
                tc::mma_f16_ss(dcol, da, db, id, (acc_first || s > 0) ? 1u : 0u);
            }
            tc::mma_commit(done);
        };

        // 2b/3. tile 0 (diagonal block): M into piece 0, then y0 += M x[0:NCB0]
        for (int g32 = half; g32 < K::NCB0 / 32; g32 += 2) build32(0, 0, g32 * 32, 0, 0, true);
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        if (tid == 0) mma_yd(0, aM, 0, K::NCB0, true, bar_y0);
        if (K::JT == 2) {
            // tile 1, columns 0..127 (below the diagonal block): piece 1
            for (int g32 = half; g32 < 4; g32 += 2) build32(1, K::CB1_COL, g32 * 32, K::MPIECE, 0, false);
            tc::fence_proxy_async_smem();
            tc::tc_fence_before();
            __syncthreads();
            if (tid == 0) mma_yd(1, aM + K::MPIECE, 0, 128, true, bar_y1a);
            // tile 1, columns 128..255 (diagonal block): piece 0 once tile 0's MMAs are done
            ok = wait_all(bar_y0, par);
            if (!ok) break;
            for (int g32 = 4 + half; g32 < 8; g32 += 2) build32(1, K::CB1_COL, g32 * 32, 0, 128, true);
            tc::fence_proxy_async_smem();
            tc::tc_fence_before();
            __syncthreads();
            if (tid == 0) mma_yd(1, aM, 128, 128, true, bar_y1b);
            ok = wait_all(bar_y1b, par);
        } else {
            ok = wait_all(bar_y0, par);
        }
        if (!ok) break;
        tc::tc_fence_after();

        // 4. y = acc + D x, bf16, written over the x tile, then stored by TMA
        const float Dh = __ldg(Dv + h);
        for (int J = 0; J < K::JT; ++J) {
            const int j = J * 128 + quarter * 32 + lane;
            uint32_t v[32];
            tc::tmem_ld32(trow + K::Y_COL + J * 64 + half * 32, v);
            tc::tmem_wait_ld();
            if (j < Q) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int chunk = half * 4 + q;                 // 8 columns p = chunk*8 ..
                    uint4* px = reinterpret_cast<uint4*>(xs + j * 128 + ((chunk ^ (j & 7)) << 4));
                    const uint4 xv = *px;
                    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
                    uint32_t o[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float lo = __uint_as_float(v[q * 8 + 2 * e]) +
                                         Dh * bf16_bits_to_float((uint16_t)(xw[e] & 0xffffu));
                        const float hi = __uint_as_float(v[q * 8 + 2 * e + 1]) +
                                         Dh * bf16_bits_to_float((uint16_t)(xw[e] >> 16));
                        o[e] = (uint32_t)float_to_bf16_bits(lo) | ((uint32_t)float_to_bf16_bits(hi) << 16);
                    }
                    *px = make_uint4(o[0], o[1], o[2], o[3]);
                }
            }
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc::tma_store_3d(&tm_y, xs, h * kP, c * Q, b);
            tc::tma_store_commit();
            if (it + 2 < nh) {                  // this x buffer is next needed for head it + 2
                tc::tma_store_wait_read0();
                tc::mbar_arrive_expect_tx(bar_x + xb, K::X_BYTES);
                tc::tma_load_3d(xs, &tm_x, bar_x + xb, (h + 2) * kP, c * Q, b);
            }
        }
    }
    if (!ok && tid == 0 && status) atomicExch(status, kStatusTimeout);
    if (tid == 0) tc::tma_store_wait0();
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, K::TMEM_COLS);
}

template <int Q, bool kI8>
cudaError_t launch_q(const Dims& d, const CUtensorMap* maps, int hpc, int cpg, const float* Acs, const float* dtc,
                     const float* D, const I8Scales& sc, const I8Debug* dbg, int* status, cudaStream_t st) {
    using K = ScanCfg<Q, kI8>;
    auto k = chunk_scan_tc_kernel<Q, kI8>;
    const int smem = K::BYTES + 1024;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    I8Debug none{};
    k<<<dim3(d.G * cpg, d.nc, d.B), kThreads, smem, st>>>(maps[0], maps[1], maps[2], maps[3], maps[4], d, hpc, cpg,
                                                            Acs, dtc, D, sc, dbg ? *dbg : none, status);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_scan_tc(const Dims& d, bool i8, const uint16_t* x, const void* Bmat,
                                 const void* Cmat, const float* Acs, const float* dtc, const float* D,
                                 const I8Scales& sc, const void* Hc, uint16_t* y, const I8Debug* dbg,
                                 int heads_per_cta, int* status, cudaStream_t st) {
    if (d.B == 0 || d.nc == 0) return cudaSuccess;
    if (d.P != kP || d.N != kN) return cudaErrorInvalidValue;
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
    if (!ok) return cudaErrorInvalidValue;
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
