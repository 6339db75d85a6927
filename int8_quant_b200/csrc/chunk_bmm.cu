// chunk_bmm.cu — ChunkBMM of the notes' storage variant ("SSDi8" notes, key design 2:
// CB is requantised to INT8 because it is larger than X; overall framework).  Per
// (b, c, g) tile of chunk 256: the INT32 product CB = Cq Bq^T over every entry (two
// 128 x 256 tcgen05 kind::i8 MMAs into all 512 TMEM columns), one step
// s = amax|CB| / 127 in fp64 (amax 0 gives 1), and the codes clamp(rint(CB / s), +-127)
// (fp64 division, round half to even), written to HBM as int8 [B, nc, G, Q, Q] with s
// as fp32 [B, nc, G] for ChunkScan2's dequantisation.  The library's own layout keeps
// CB on chip instead (ChunkScan forms it from the INT8 B and C it loads anyway).
//
// Warps: 0 TMA (Cq and Bq tiles, 128-byte swizzle), 1 TMEM allocation and MMA issue,
// 2..5 epilogue (one TMEM lane quarter each): amax over the tile (warp shuffles, then
// the four warps through shared memory), then the codes.  Waits are bounded: an
// expired wait raises the CTA's abort flag and records SSD_ERR_TIMEOUT; copies and
// MMAs in flight are waited for before TMEM is freed.
#include "kernels.h"
#include "tc.cuh"

namespace ssd {

namespace {

constexpr int kQ = 256;
constexpr int kN = 128;
constexpr int kThreads = 6 * 32;
constexpr int kEpiWarp0 = 2;
constexpr int OFF_C = 0;                          // Cq tile [256][128], 32 KB, 1024-aligned
constexpr int OFF_B = kQ * kN;                    // Bq tile [256][128]
constexpr int OFF_BAR = 2 * kQ * kN;
constexpr int BAR_LOAD = 0, BAR_MMA = 1, NBAR = 2;
constexpr int OFF_FLAG = OFF_BAR + NBAR * 8;
constexpr int OFF_TMEM = OFF_FLAG + 8;
constexpr int OFF_RED = OFF_TMEM + 8;
constexpr int BYTES = OFF_RED + 4 * 4;
constexpr uint32_t kIdEpi = 1;                    // named barrier of the epilogue warps

__global__ void __launch_bounds__(kThreads, 1)
chunk_bmm_i8_kernel(const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_c, Dims d,
                    int8_t* __restrict__ cb8, float* __restrict__ s_cb, int* __restrict__ status,
                    int32_t* __restrict__ dbg_cb, int8_t* __restrict__ dbg_cb8, double* __restrict__ dbg_s_cb) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = blockIdx.x, c = blockIdx.y, b = blockIdx.z;
    const long long tile = ((long long)b * d.nc + c) * d.G + g;
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_FLAG);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_TMEM);
    int* red = reinterpret_cast<int*>(sm + OFF_RED);

    if (tid == 0) {
        tc::mbar_init(bar + BAR_LOAD, 1);
        tc::mbar_init(bar + BAR_MMA, 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            tc::prefetch_tmap(&tm_b);
            tc::prefetch_tmap(&tm_c);
            tc::mbar_arrive_expect_tx(bar + BAR_LOAD, 2 * kQ * kN);
            tc::tma_load_3d(sm + OFF_C, &tm_c, bar + BAR_LOAD, g * kN, c * kQ, b);
            tc::tma_load_3d(sm + OFF_B, &tm_b, bar + BAR_LOAD, g * kN, c * kQ, b);
            // the copies must land before the CTA may exit
            tc::mbar_wait(bar + BAR_LOAD, 0, tc::kWaitLimit);
        }
    } else if (warp == 1) {
        const bool ok = __all_sync(0xffffffffu, tc::wait_or_abort(bar + BAR_LOAD, 0, abort_flag, status,
                                                                   kStatusTimeout));
        if (ok) {
            tc::tc_fence_after();
            if (tc::elect_one()) {
                // A = Cq rows (K-major), B = Bq rows (K-major, N = 256); K = 128 in four steps of 32
                const uint64_t dC = tc::smem_desc(tc::smem_u32(sm + OFF_C), 16, 1024, tc::kLayoutSw128);
                const uint64_t dB = tc::smem_desc(tc::smem_u32(sm + OFF_B), 16, 1024, tc::kLayoutSw128);
                const uint32_t id = tc::idesc_s8_s32(128, 256, tc::kMajorK, tc::kMajorK);
#pragma unroll
                for (int J = 0; J < 2; ++J)
#pragma unroll
                    for (int st = 0; st < 4; ++st)
                        tc::mma_i8_ss(tmem + 256 * J, dC + (uint64_t)((J * 128 * 128 + st * 32) >> 4),
                                      dB + (uint64_t)((st * 32) >> 4), id, st > 0 ? 1u : 0u);
                tc::mma_commit(bar + BAR_MMA);
            }
            __syncwarp();
            // the MMAs must complete before TMEM is freed
            tc::mbar_wait(bar + BAR_MMA, 0, tc::kWaitLimit);
        }
    } else {
        const int quarter = warp & 3;                             // TMEM lanes of this warp
        const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
        bool ok = __all_sync(0xffffffffu, tc::wait_or_abort(bar + BAR_MMA, 0, abort_flag, status, kStatusTimeout));
        tc::tc_fence_after();
        int amax = 0;
        if (ok) {
            for (int J = 0; J < 2; ++J) {
                const int row = J * 128 + quarter * 32 + lane;
                for (int g32 = 0; g32 < 8; ++g32) {
                    uint32_t v[32];
                    tc::tmem_ld32(trow + 256 * J + 32 * g32, v);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) amax = max(amax, abs((int)v[i]));
                    if (dbg_cb) {
                        int32_t* dst = dbg_cb + (tile * kQ + row) * kQ + 32 * g32;
#pragma unroll
                        for (int i = 0; i < 32; ++i) dst[i] = (int32_t)v[i];
                    }
                }
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        if (lane == 0) red[quarter] = amax;
        ok = tc::named_and(kIdEpi, 128, ok);
        amax = max(max(red[0], red[1]), max(red[2], red[3]));
        const double s = amax > 0 ? (double)amax / 127.0 : 1.0;
        if (tid == kEpiWarp0 * 32) {
            s_cb[tile] = (float)s;
            if (dbg_s_cb) dbg_s_cb[tile] = s;
        }
        if (ok) {
            for (int J = 0; J < 2; ++J) {
                const int row = J * 128 + quarter * 32 + lane;
                for (int g32 = 0; g32 < 8; ++g32) {
                    uint32_t v[32];
                    tc::tmem_ld32(trow + 256 * J + 32 * g32, v);
                    tc::tmem_wait_ld();
                    uint32_t w[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) w[i] = 0u;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        double q = rint(__ddiv_rn((double)(int)v[i], s));
                        q = fmin(fmax(q, -127.0), 127.0);
                        w[i >> 2] |= ((uint32_t)(int)q & 0xffu) << (8 * (i & 3));
                    }
                    const long long o = (tile * kQ + row) * kQ + 32 * g32;
                    uint4* dst = reinterpret_cast<uint4*>(cb8 + o);
                    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
                    if (dbg_cb8) {
                        uint4* dd = reinterpret_cast<uint4*>(dbg_cb8 + o);
                        dd[0] = make_uint4(w[0], w[1], w[2], w[3]);
                        dd[1] = make_uint4(w[4], w[5], w[6], w[7]);
                    }
                }
            }
        }
    }
    __syncwarp();
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

}  // namespace

size_t chunk_bmm_i8_bytes(const Dims& d) {
    const size_t tiles = (size_t)d.B * d.nc * d.G;
    return tiles * kQ * kQ + ((tiles * sizeof(float) + 255) & ~(size_t)255) + 256;
}

cudaError_t launch_chunk_bmm_i8(const Dims& d, const int8_t* Bq, const int8_t* Cq, int8_t* cb8, float* s_cb,
                                const I8Debug* dbg, int* status, cudaStream_t st) {
    if (d.B == 0 || d.nc == 0) return cudaSuccess;
    if (d.Q != kQ || d.N != kN) return cudaErrorInvalidValue;
    const unsigned long long GN = (unsigned long long)d.G * kN;
    CUtensorMap mb, mc;
    bool ok = make_tmap_3d(&mb, true, Bq, GN, d.L, d.B, GN, d.Ls * GN, 128, kQ, CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_tmap_3d(&mc, true, Cq, GN, d.L, d.B, GN, d.Ls * GN, 128, kQ, CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) return cudaErrorInvalidValue;
    // more than half of the SM's shared memory: one CTA per SM, so that no second CTA waits
    // in its TMEM allocation for the first one's 512 columns
    const int smem = BYTES + 1024 > 120 * 1024 ? BYTES + 1024 : 120 * 1024;
    cudaError_t e = cudaFuncSetAttribute(chunk_bmm_i8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    chunk_bmm_i8_kernel<<<dim3(d.G, d.nc, d.B), kThreads, smem, st>>>(
        mb, mc, d, cb8, s_cb, status, dbg ? dbg->cb : nullptr, dbg ? dbg->cb8 : nullptr, dbg ? dbg->s_cb : nullptr);
    return cudaGetLastError();
}

}  // namespace ssd
