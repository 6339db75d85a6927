// api.cu — the C ABI of libssd.so: argument validation, workspace layout and the
// launch sequence of each entry point on the caller's stream.
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/ssd.h"
#include "kernels.h"

namespace ssd {

namespace {

inline size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// Validates a shape; fills `d`.  Returns SSD_OK, SSD_ERR_INVALID_ARG or SSD_ERR_UNSUPPORTED.
ssd_status make_dims(const ssd_shape* s, Dims* d) {
    if (!s) return SSD_ERR_INVALID_ARG;
    if (s->batch < 0 || s->seqlen < 0 || s->nheads < 1 || s->ngroups < 1 || s->headdim < 1 ||
        s->dstate < 1 || s->chunk < 1)
        return SSD_ERR_INVALID_ARG;
    if (s->nheads % s->ngroups != 0) return SSD_ERR_INVALID_ARG;
    if (s->chunk != 64 && s->chunk != 128 && s->chunk != 256) return SSD_ERR_UNSUPPORTED;
    const bool pn_ok = (s->headdim == 64 && s->dstate == 128) || (s->headdim == 16 && s->dstate == 16);
    if (!pn_ok) return SSD_ERR_UNSUPPORTED;
    d->B = s->batch;
    d->L = s->seqlen;
    d->H = s->nheads;
    d->P = s->headdim;
    d->G = s->ngroups;
    d->N = s->dstate;
    d->Q = s->chunk;
    d->nc = (s->seqlen + s->chunk - 1) / s->chunk;
    d->hpg = s->nheads / s->ngroups;
    d->Ls = s->seqlen;
    return SSD_OK;
}

// Shapes served by the tensor-core kernels; the (16,16) test shape uses the
// CUDA-core kernels.
bool tensor_core_shape(const Dims& d) { return d.P == 64 && d.N == 128; }

// The W8A8 scan of the tensor-core shapes runs as the five-launch sequence (quantize,
// ChunkCumsum, ChunkState, StatePassing, ChunkScan), the faster of the two designs on
// B200; SSD_I8_FUSED=1 in the environment selects the single persistent kernel
// (fused_i8.cu), which gives the same integers bit for bit.
bool i8_fused(const Dims& d) {
    const char* e = getenv("SSD_I8_FUSED");
    return tensor_core_shape(d) && e && e[0] == '1';
}

}  // namespace

int device_sm_count() {
    static int n[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    if (n[dev] == 0) {
        int v = 0;
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        n[dev] = v > 0 ? v : 1;
    }
    return n[dev];
}

namespace {

// Heads that share one ChunkBMM result in a tensor-core ChunkScan CTA.  One CTA runs per
// SM, so the grid runs in waves; a CTA costs about one head's time for its prologue (C and
// B tiles, ChunkBMM, packing) plus one per head.  Among a few block sizes, take the one
// whose waves x (1 + heads) is smallest: fewer prologues against a full last wave.
int scan_heads_per_cta(const Dims& d) {
    const int sms = device_sm_count();
    int best = 8;
    long long best_cost = -1;
    for (int hpc : {8, 10, 12, 16, 20}) {
        const int per = hpc < d.hpg ? hpc : d.hpg;
        const long long ctas = (long long)d.G * ((d.hpg + per - 1) / per) * d.nc * d.B;
        const long long cost = ((ctas + sms - 1) / sms) * (1 + per);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = per;
        }
    }
    return best;
}

}  // namespace

// The CUDA error behind this thread's last SSD_ERR_CUDA (cudaSuccess if none).
thread_local cudaError_t g_last_cuda_error = cudaSuccess;

ssd_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return SSD_OK;
    g_last_cuda_error = e;
    return SSD_ERR_CUDA;
}

namespace {

#define SSD_TRY(expr)                                  \
    do {                                               \
        cudaError_t _e = (expr);                       \
        if (_e != cudaSuccess) return from_cuda(_e);   \
    } while (0)

template <typename T>
T* at(void* base, size_t off) { return reinterpret_cast<T*>(reinterpret_cast<char*>(base) + off); }

}  // namespace

WsLayout ws_layout(const Dims& d, bool i8, bool fp32_states) {
    WsLayout w{};
    const size_t chains = (size_t)d.B * d.H;
    const size_t states = (size_t)d.B * d.nc * d.H * d.P * d.N;
    size_t off = 0;
    w.status = off;  off += 256;
    w.acs = off;     off += align256(chains * d.nc * d.Q * sizeof(float));
    w.lut = off;     off += align256(chains * d.nc * d.Q * sizeof(float));   // LUT_state
    w.dtc = off;     off += align256(chains * d.nc * d.Q * sizeof(float));   // dt, chunk-major
    w.decay = off;   off += align256(chains * d.nc * sizeof(float));   // fp32 decay or int32 code
    // chunk states: int8 (W8A8), bf16 (tensor-core bf16 path), fp32 (CUDA-core path, calibration)
    const size_t s_elem = i8 ? 1 : (fp32_states || !tensor_core_shape(d)) ? sizeof(float) : sizeof(uint16_t);
    w.states = off;  off += align256(states * s_elem);
    w.passed = off;  off += align256(states * (i8 ? 1 : sizeof(uint16_t)));
    w.scales = off;  off += align256(i8 ? (size_t)2 * d.H * d.P * sizeof(float) : 0);   // 1/s_x, s_x s_B / s_s
    // the storage variant's CB codes and steps (W8A8, tensor-core shape, chunk 256)
    w.cb8 = off;     off += (i8 && tensor_core_shape(d) && d.Q == 256) ? align256(chunk_bmm_i8_bytes(d)) : 0;
    w.total = off;
    return w;
}

size_t ws_bytes(const Dims& d, bool i8) {
    const size_t staged = ws_layout(d, i8).total;
    if (!i8 || !tensor_core_shape(d)) return staged;
    const size_t fused = fused_i8_ws_bytes(d);
    return fused > staged ? fused : staged;
}

// ---------------------------------------------------------------- per-kernel timing
// While enabled, every kernel the entry points enqueue is bracketed by two CUDA
// events on the call's stream; ssd_profile_read() turns them into milliseconds per
// kernel name.  Events come from a pool owned by the library.
namespace prof {

struct Pending { int kernel; cudaEvent_t a, b; };
std::mutex mu;
bool enabled = false;
std::vector<std::string> names;
std::vector<double> ms;
std::vector<long long> calls;
std::vector<Pending> pending;
std::vector<cudaEvent_t> pool;
std::string filter;                     // empty: every kernel

cudaEvent_t get_event() {
    if (!pool.empty()) { cudaEvent_t e = pool.back(); pool.pop_back(); return e; }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

int kernel_id(const char* name) {
    for (size_t i = 0; i < names.size(); ++i) if (names[i] == name) return (int)i;
    names.emplace_back(name);
    ms.push_back(0.0);
    calls.push_back(0);
    return (int)names.size() - 1;
}

struct Scope {
    cudaStream_t st;
    int k = -1;
    cudaEvent_t b = nullptr;
    Scope(const char* name, cudaStream_t s) : st(s) {
        std::lock_guard<std::mutex> g(mu);
        if (!enabled || (!filter.empty() && filter != name)) return;
        k = kernel_id(name);
        cudaEvent_t a = get_event();
        b = get_event();
        cudaEventRecord(a, st);
        pending.push_back({k, a, b});
    }
    ~Scope() {
        if (k >= 0) cudaEventRecord(b, st);
    }
};

}  // namespace prof

#define SSD_STAGE(name, expr)                                      \
    do {                                                           \
        prof::Scope _scope(name, stream);                          \
        cudaError_t _e = (expr);                                   \
        if (_e != cudaSuccess) return from_cuda(_e);               \
    } while (0)

}  // namespace ssd

using namespace ssd;

extern "C" {

const char* ssd_status_string(ssd_status s) {
    switch (s) {
        case SSD_OK: return "SSD_OK";
        case SSD_ERR_INVALID_ARG: return "SSD_ERR_INVALID_ARG: null or misaligned pointer, or invalid parameter";
        case SSD_ERR_UNSUPPORTED: return "SSD_ERR_UNSUPPORTED: shape outside the supported set";
        case SSD_ERR_WORKSPACE: return "SSD_ERR_WORKSPACE: workspace missing or too small";
        case SSD_ERR_CUDA: return "SSD_ERR_CUDA: a CUDA call or kernel launch failed";
        case SSD_ERR_TIMEOUT: return "SSD_ERR_TIMEOUT: a device-side bounded wait expired";
    }
    return "unknown ssd_status";
}

const char* ssd_last_cuda_error(void) { return cudaGetErrorString(g_last_cuda_error); }

size_t ssd_workspace_bytes(const ssd_shape* shape, int is_i8) {
    Dims d;
    if (make_dims(shape, &d) != SSD_OK) return 0;
    return ws_bytes(d, is_i8 != 0);
}

ssd_status ssd_quantize_inputs(const ssd_shape* shape, const uint16_t* B, const uint16_t* C,
                               const float* s_B, const float* s_C, int8_t* Bq, int8_t* Cq,
                               cudaStream_t stream) {
    Dims d;
    ssd_status st = make_dims(shape, &d);
    if (st != SSD_OK) return st;
    const long long n = (long long)d.B * d.L;
    if (n == 0) return SSD_OK;
    if (!B || !C || !s_B || !s_C || !Bq || !Cq) return SSD_ERR_INVALID_ARG;
    if (!aligned16(B) || !aligned16(C) || !aligned16(Bq) || !aligned16(Cq)) return SSD_ERR_INVALID_ARG;
    SSD_STAGE("quantize_inputs", launch_quantize_bc(d, B, C, s_B, s_C, Bq, Cq, stream));
    return SSD_OK;
}

static ssd_status check_common(const Dims& d, const void* x, const float* dt, const float* A,
                               const void* B, const void* C, const float* D, const void* y,
                               const void* final_state, void* ws, size_t ws_size, bool i8) {
    if (!final_state || !A || !D) return SSD_ERR_INVALID_ARG;
    if (!aligned16(final_state)) return SSD_ERR_INVALID_ARG;
    if ((long long)d.B * d.L > 0) {
        if (!x || !dt || !B || !C || !y) return SSD_ERR_INVALID_ARG;
        if (!aligned16(x) || !aligned16(dt) || !aligned16(B) || !aligned16(C) || !aligned16(y))
            return SSD_ERR_INVALID_ARG;
    }
    if (!ws || !aligned16(ws)) return SSD_ERR_WORKSPACE;
    if (ws_size < ws_bytes(d, i8)) return SSD_ERR_WORKSPACE;
    return SSD_OK;
}

static ssd_status scan_bf16(const ssd_shape* shape, const uint16_t* x, const float* dt, const float* A,
                            const uint16_t* B, const uint16_t* C, const float* D, const float* initial_state,
                            uint16_t* y, float* final_state, void* workspace, size_t workspace_bytes,
                            cudaStream_t stream) {
    Dims d;
    ssd_status st = make_dims(shape, &d);
    if (st != SSD_OK) return st;
    if (d.B == 0) return SSD_OK;
    st = check_common(d, x, dt, A, B, C, D, y, final_state, workspace, workspace_bytes, false);
    if (st != SSD_OK) return st;
    if (initial_state && !aligned16(initial_state)) return SSD_ERR_INVALID_ARG;
    const size_t fs_bytes = (size_t)d.B * d.H * d.P * d.N * sizeof(float);
    const WsLayout w = ws_layout(d, false);
    if (d.L == 0) {
        SSD_TRY(cudaMemsetAsync(at<int>(workspace, w.status), 0, sizeof(int), stream));
        if (initial_state)
            return from_cuda(cudaMemcpyAsync(final_state, initial_state, fs_bytes, cudaMemcpyDeviceToDevice, stream));
        return from_cuda(cudaMemsetAsync(final_state, 0, fs_bytes, stream));
    }
    float* Acs = at<float>(workspace, w.acs);
    float* decay = at<float>(workspace, w.decay);
    uint16_t* Hc = at<uint16_t>(workspace, w.passed);
    float* lut = at<float>(workspace, w.lut);
    float* dtc = at<float>(workspace, w.dtc);
    int* status = at<int>(workspace, w.status);
    SSD_STAGE("chunk_cumsum", launch_cumsum(d, dt, A, Acs, decay, nullptr, 0, status, lut, dtc, stream));
    // bf16 chunk states on the tensor-core path, fp32 on the CUDA-core (small-shape) path
    const bool tcs = tensor_core_shape(d);
    void* S = at<void>(workspace, w.states);
    if (tcs)
        SSD_STAGE("chunk_state", launch_chunk_state_tc(d, false, x, B, lut, nullptr, nullptr, static_cast<uint16_t*>(S),
                                                       nullptr, nullptr, status, stream));
    else
        SSD_STAGE("chunk_state", launch_chunk_state_bf16(d, x, dt, Acs, B, static_cast<float*>(S), nullptr, nullptr,
                                                         stream));
    SSD_STAGE("state_passing",
              launch_state_passing_bf16(d, S, !tcs, decay, initial_state, Hc, final_state, nullptr, stream));
    if (tensor_core_shape(d))
        SSD_STAGE("chunk_scan", launch_chunk_scan_tc(d, false, x, B, C, Acs, dtc, D, I8Scales{}, Hc, y, nullptr,
                                                     scan_heads_per_cta(d), status, stream));
    else
        SSD_STAGE("chunk_scan", launch_chunk_scan_bf16(d, x, dt, Acs, B, C, D, Hc, y, stream));
    return SSD_OK;
}

ssd_status ssd_scan_fwd_bf16(const ssd_shape* shape, const uint16_t* x, const float* dt,
                             const float* A, const uint16_t* B, const uint16_t* C,
                             const float* D, uint16_t* y, float* final_state, void* workspace,
                             size_t workspace_bytes, cudaStream_t stream) {
    return scan_bf16(shape, x, dt, A, B, C, D, nullptr, y, final_state, workspace, workspace_bytes, stream);
}

ssd_status ssd_scan_fwd_bf16_from_state(const ssd_shape* shape, const uint16_t* x, const float* dt,
                                        const float* A, const uint16_t* B, const uint16_t* C,
                                        const float* D, const float* initial_state, uint16_t* y,
                                        float* final_state, void* workspace, size_t workspace_bytes,
                                        cudaStream_t stream) {
    return scan_bf16(shape, x, dt, A, B, C, D, initial_state, y, final_state, workspace, workspace_bytes, stream);
}

static ssd_status scan_i8(const ssd_shape* shape, const uint16_t* x, const float* dt, const float* A,
                          const int8_t* Bq, const int8_t* Cq, const float* D, const ssd_i8_params* params,
                          const int8_t* initial_state, uint16_t* y, int8_t* final_state, void* workspace,
                          size_t workspace_bytes, const ssd_i8_debug* dbg, cudaStream_t stream) {
    Dims d;
    ssd_status st = make_dims(shape, &d);
    if (st != SSD_OK) return st;
    if (!params || !params->s_B || !params->s_C || !params->s_x || !params->s_s) return SSD_ERR_INVALID_ARG;
    if (params->decay_shift < 1 || params->decay_shift > 14) return SSD_ERR_INVALID_ARG;
    const int storage = params->storage;
    if (storage & ~(SSD_STORAGE_ACS_FP16 | SSD_STORAGE_CB_INT8)) return SSD_ERR_INVALID_ARG;
    if (storage && (!tensor_core_shape(d) || d.Q != 256)) return SSD_ERR_UNSUPPORTED;
    const bool acs_half = (storage & SSD_STORAGE_ACS_FP16) != 0, cb_int8 = (storage & SSD_STORAGE_CB_INT8) != 0;
    if (d.B == 0) return SSD_OK;
    st = check_common(d, x, dt, A, Bq, Cq, D, y, final_state, workspace, workspace_bytes, true);
    if (st != SSD_OK) return st;
    if (initial_state && !aligned16(initial_state)) return SSD_ERR_INVALID_ARG;
    const size_t fs_bytes = (size_t)d.B * d.H * d.P * d.N;
    const WsLayout w = ws_layout(d, true);
    if (d.L == 0) {
        SSD_TRY(cudaMemsetAsync(at<int>(workspace, w.status), 0, sizeof(int), stream));
        if (initial_state)
            return from_cuda(cudaMemcpyAsync(final_state, initial_state, fs_bytes, cudaMemcpyDeviceToDevice, stream));
        return from_cuda(cudaMemsetAsync(final_state, 0, fs_bytes, stream));
    }
    I8Scales sc{params->s_B, params->s_C, params->s_x, params->s_s, params->decay_shift};
    I8Debug dd{};
    if (dbg)
        dd = I8Debug{dbg->Acs, dbg->dq, dbg->Xq, dbg->acc_state, dbg->S8, dbg->H8, dbg->cb, dbg->acc_scan1,
                     dbg->cb8, dbg->s_cb};
    if (i8_fused(d) && !storage) {
        SSD_STAGE("ssd_fused_i8", launch_fused_i8(d, x, dt, A, Bq, Cq, D, sc, initial_state, y, final_state, workspace,
                                                  dbg ? &dd : nullptr, stream));
        return SSD_OK;
    }
    float* Acs = at<float>(workspace, w.acs);
    int32_t* dq = at<int32_t>(workspace, w.decay);
    int8_t* S8 = at<int8_t>(workspace, w.states);
    int8_t* H8 = at<int8_t>(workspace, w.passed);
    float* lut = at<float>(workspace, w.lut);
    float* dtc = at<float>(workspace, w.dtc);
    int* status = at<int>(workspace, w.status);
    float* inv_sx = at<float>(workspace, w.scales);
    float* mq = inv_sx + d.H * d.P;
    SSD_STAGE("chunk_cumsum", launch_cumsum(d, dt, A, Acs, nullptr, dq, sc.shift, status, lut, dtc, stream, &sc, inv_sx, mq,
                                            acs_half));
    if (tensor_core_shape(d))
        SSD_STAGE("chunk_state", launch_chunk_state_tc(d, true, x, Bq, lut, inv_sx, mq, nullptr, S8, dbg ? &dd : nullptr,
                                                       status, stream));
    else
        SSD_STAGE("chunk_state", launch_chunk_state_i8(d, x, dt, Acs, Bq, sc, S8, dbg ? &dd : nullptr, stream));
    SSD_STAGE("state_passing", launch_state_passing_i8(d, S8, dq, sc.shift, initial_state, H8, final_state, stream));
    int8_t* cb8 = at<int8_t>(workspace, w.cb8);
    float* s_cb = at<float>(workspace, w.cb8 + (size_t)d.B * d.nc * d.G * d.Q * d.Q);
    if (cb_int8) SSD_STAGE("chunk_bmm", launch_chunk_bmm_i8(d, Bq, Cq, cb8, s_cb, dbg ? &dd : nullptr, status, stream));
    if (tensor_core_shape(d))
        SSD_STAGE("chunk_scan", launch_chunk_scan_tc(d, true, x, Bq, Cq, Acs, dtc, D, sc, H8, y, dbg ? &dd : nullptr,
                                                     scan_heads_per_cta(d), status, stream, cb_int8 ? cb8 : nullptr,
                                                     s_cb, acs_half));
    else
        SSD_STAGE("chunk_scan", launch_chunk_scan_i8(d, x, dt, Acs, Bq, Cq, D, sc, H8, y, dbg ? &dd : nullptr, stream));
    if (dbg) {
        const size_t chains = (size_t)d.B * d.H;
        const size_t states = (size_t)d.B * d.nc * d.H * d.P * d.N;
        if (dbg->Acs && acs_half) SSD_TRY(launch_half_to_float(Acs, dbg->Acs, (long long)(chains * d.nc * d.Q), stream));
        else if (dbg->Acs)
            SSD_TRY(cudaMemcpyAsync(dbg->Acs, Acs, chains * d.nc * d.Q * 4, cudaMemcpyDeviceToDevice, stream));
        if (dbg->dq) SSD_TRY(cudaMemcpyAsync(dbg->dq, dq, chains * d.nc * 4, cudaMemcpyDeviceToDevice, stream));
        if (dbg->H8) SSD_TRY(cudaMemcpyAsync(dbg->H8, H8, states, cudaMemcpyDeviceToDevice, stream));
    }
    return SSD_OK;
}

ssd_status ssd_scan_fwd_i8_debug(const ssd_shape* shape, const uint16_t* x, const float* dt,
                                 const float* A, const int8_t* Bq, const int8_t* Cq,
                                 const float* D, const ssd_i8_params* params, uint16_t* y,
                                 int8_t* final_state, void* workspace, size_t workspace_bytes,
                                 const ssd_i8_debug* dbg, cudaStream_t stream) {
    return scan_i8(shape, x, dt, A, Bq, Cq, D, params, nullptr, y, final_state, workspace, workspace_bytes, dbg,
                   stream);
}

ssd_status ssd_scan_fwd_i8(const ssd_shape* shape, const uint16_t* x, const float* dt,
                           const float* A, const int8_t* Bq, const int8_t* Cq, const float* D,
                           const ssd_i8_params* params, uint16_t* y, int8_t* final_state,
                           void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    return scan_i8(shape, x, dt, A, Bq, Cq, D, params, nullptr, y, final_state, workspace, workspace_bytes, nullptr,
                   stream);
}

ssd_status ssd_scan_fwd_i8_from_state(const ssd_shape* shape, const uint16_t* x, const float* dt,
                                      const float* A, const int8_t* Bq, const int8_t* Cq, const float* D,
                                      const ssd_i8_params* params, const int8_t* initial_state, uint16_t* y,
                                      int8_t* final_state, void* workspace, size_t workspace_bytes,
                                      cudaStream_t stream) {
    return scan_i8(shape, x, dt, A, Bq, Cq, D, params, initial_state, y, final_state, workspace, workspace_bytes,
                   nullptr, stream);
}

size_t ssd_out_proj_workspace_bytes(int tokens, int d_inner) {
    if (tokens < 0 || d_inner < 1) return 0;
    return align256((size_t)tokens * d_inner) + 256;
}

ssd_status ssd_out_proj_i8(int tokens, int d_inner, int d_model, const uint16_t* y, float s_a, const int8_t* Wq,
                           const float* s_w, const float* corr, uint16_t* out, int32_t* acc_debug, void* workspace,
                           size_t workspace_bytes, cudaStream_t stream) {
    if (tokens < 0 || d_inner < 1 || d_model < 1 || !(s_a > 0.f)) return SSD_ERR_INVALID_ARG;
    if (d_inner % 128 != 0 || d_model % 256 != 0 || tokens % 128 != 0) return SSD_ERR_UNSUPPORTED;
    if (!Wq || !s_w || !aligned16(Wq) || (corr && !aligned16(corr))) return SSD_ERR_INVALID_ARG;
    if (!workspace || !aligned16(workspace) || workspace_bytes < ssd_out_proj_workspace_bytes(tokens, d_inner))
        return SSD_ERR_WORKSPACE;
    int* status = at<int>(workspace, align256((size_t)tokens * d_inner));
    SSD_TRY(cudaMemsetAsync(status, 0, sizeof(int), stream));
    if (tokens == 0) return SSD_OK;
    if (!y || !out || !aligned16(y) || !aligned16(out) || (acc_debug && !aligned16(acc_debug)))
        return SSD_ERR_INVALID_ARG;
    int8_t* aq = static_cast<int8_t*>(workspace);
    SSD_STAGE("out_proj_norm", launch_out_proj_norm(tokens, d_inner, y, s_a, aq, stream));
    SSD_STAGE("out_proj_gemm", launch_out_proj_gemm(tokens, d_inner, d_model, aq, s_a, Wq, s_w, corr, out, acc_debug,
                                                    status, stream));
    return SSD_OK;
}

ssd_status ssd_out_proj_status(void* workspace, int tokens, int d_inner, cudaStream_t stream) {
    if (!workspace || tokens < 0 || d_inner < 1) return SSD_ERR_INVALID_ARG;
    int v = 0;
    SSD_TRY(cudaMemcpyAsync(&v, at<int>(workspace, align256((size_t)tokens * d_inner)), sizeof(int),
                            cudaMemcpyDeviceToHost, stream));
    SSD_TRY(cudaStreamSynchronize(stream));
    return v == 0 ? SSD_OK : (ssd_status)v;
}

// Shape of a one-token step: seqlen must be 1; chunk is not used.
static ssd_status decode_dims(const ssd_shape* s, Dims* d) {
    if (!s) return SSD_ERR_INVALID_ARG;
    if (s->batch < 0 || s->seqlen != 1 || s->nheads < 1 || s->ngroups < 1 || s->headdim < 1 || s->dstate < 1)
        return SSD_ERR_INVALID_ARG;
    if (s->nheads % s->ngroups != 0) return SSD_ERR_INVALID_ARG;
    const bool pn_ok = (s->headdim == 64 && s->dstate == 128) || (s->headdim == 16 && s->dstate == 16);
    if (!pn_ok) return SSD_ERR_UNSUPPORTED;
    *d = Dims{s->batch, 1, s->nheads, s->headdim, s->ngroups, s->dstate, 1, 1, s->nheads / s->ngroups, 1};
    return SSD_OK;
}

ssd_status ssd_decode_step_bf16(const ssd_shape* shape, const uint16_t* x, const float* dt, const float* A,
                                const uint16_t* B, const uint16_t* C, const float* D, float* state, uint16_t* y,
                                cudaStream_t stream) {
    Dims d;
    const ssd_status st = decode_dims(shape, &d);
    if (st != SSD_OK) return st;
    if (!A || !D) return SSD_ERR_INVALID_ARG;
    if (d.B == 0) return SSD_OK;
    if (!x || !dt || !B || !C || !state || !y) return SSD_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(dt) || !aligned16(B) || !aligned16(C) || !aligned16(state) || !aligned16(y))
        return SSD_ERR_INVALID_ARG;
    SSD_STAGE("decode_step", launch_decode_bf16(d, x, dt, A, B, C, D, state, y, stream));
    return SSD_OK;
}

ssd_status ssd_decode_step_i8(const ssd_shape* shape, const uint16_t* x, const float* dt, const float* A,
                              const uint16_t* B, const uint16_t* C, const float* D, const ssd_i8_params* params,
                              int8_t* state, uint16_t* y, cudaStream_t stream) {
    Dims d;
    const ssd_status st = decode_dims(shape, &d);
    if (st != SSD_OK) return st;
    if (!A || !D) return SSD_ERR_INVALID_ARG;
    if (!params || !params->s_B || !params->s_C || !params->s_x || !params->s_s) return SSD_ERR_INVALID_ARG;
    if (params->decay_shift < 1 || params->decay_shift > 14) return SSD_ERR_INVALID_ARG;
    if (d.B == 0) return SSD_OK;
    if (!x || !dt || !B || !C || !state || !y) return SSD_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(dt) || !aligned16(B) || !aligned16(C) || !aligned16(state) || !aligned16(y))
        return SSD_ERR_INVALID_ARG;
    const I8Scales sc{params->s_B, params->s_C, params->s_x, params->s_s, params->decay_shift};
    SSD_STAGE("decode_step", launch_decode_i8(d, x, dt, A, B, C, D, sc, state, y, stream));
    return SSD_OK;
}

static WsLayout calib_layout(const Dims& p, size_t* fin_off, size_t* amax_off) {
    WsLayout w = ws_layout(p, false, true);
    *fin_off = w.total;
    *amax_off = *fin_off + align256((size_t)p.B * p.H * p.P * p.N * sizeof(float));
    w.total = *amax_off + align256((size_t)(2 * p.G + 3 * p.H * p.P) * sizeof(float));
    return w;
}

static Dims prefix_dims(const Dims& d, int prefix) {
    Dims p = d;                 // the first T tokens of rows of length L
    p.L = prefix < d.L ? prefix : d.L;
    p.nc = (p.L + d.Q - 1) / d.Q;
    return p;
}

size_t ssd_calibrate_workspace_bytes(const ssd_shape* shape, int prefix) {
    Dims d;
    if (make_dims(shape, &d) != SSD_OK || prefix < 0) return 0;
    size_t fo, ao;
    return calib_layout(prefix_dims(d, prefix), &fo, &ao).total;
}

ssd_status ssd_calibrate_i8(const ssd_shape* shape, int prefix, const uint16_t* x,
                            const float* dt, const float* A, const uint16_t* B,
                            const uint16_t* C, float* s_B, float* s_C, float* s_x, float* s_s,
                            void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    Dims d;
    ssd_status st = make_dims(shape, &d);
    if (st != SSD_OK) return st;
    if (prefix < 0 || !A || !s_B || !s_C || !s_x || !s_s) return SSD_ERR_INVALID_ARG;
    const Dims p = prefix_dims(d, prefix);
    size_t fin_off, amax_off;
    const WsLayout w = calib_layout(p, &fin_off, &amax_off);
    if (!workspace || !aligned16(workspace)) return SSD_ERR_WORKSPACE;
    if (workspace_bytes < w.total) return SSD_ERR_WORKSPACE;
    const bool work = (long long)p.B * p.L > 0;
    if (work) {
        if (!x || !dt || !B || !C) return SSD_ERR_INVALID_ARG;
        if (!aligned16(x) || !aligned16(dt) || !aligned16(B) || !aligned16(C)) return SSD_ERR_INVALID_ARG;
    }
    float* aB = at<float>(workspace, amax_off);
    float* aC = aB + d.G;
    float* ax = aC + d.G;
    float* as = ax + d.H * d.P;
    float* ah = as + d.H * d.P;
    SSD_TRY(cudaMemsetAsync(aB, 0, (size_t)(2 * d.G + 3 * d.H * d.P) * sizeof(float), stream));
    if (work) {
        float* Acs = at<float>(workspace, w.acs);
        float* decay = at<float>(workspace, w.decay);
        float* S = at<float>(workspace, w.states);
        float* fin = at<float>(workspace, fin_off);
        SSD_TRY(launch_amax_bc(p, B, C, aB, aC, stream));
        SSD_TRY(launch_cumsum(p, dt, A, Acs, decay, nullptr, 0, nullptr, nullptr, nullptr, stream));
        SSD_TRY(launch_chunk_state_bf16(p, x, dt, Acs, B, S, ax, as, stream));
        SSD_TRY(launch_state_passing_bf16(p, S, true, decay, nullptr, nullptr, fin, ah, stream));
    }
    SSD_TRY(launch_amax_to_scale(aB, 2 * d.G + d.H * d.P, stream));       // s_B, s_C, s_x
    SSD_TRY(launch_amax_pair_to_scale(as, ah, s_s, d.H * d.P, stream));    // s_s over S and H
    SSD_TRY(cudaMemcpyAsync(s_B, aB, d.G * sizeof(float), cudaMemcpyDeviceToDevice, stream));
    SSD_TRY(cudaMemcpyAsync(s_C, aC, d.G * sizeof(float), cudaMemcpyDeviceToDevice, stream));
    SSD_TRY(cudaMemcpyAsync(s_x, ax, (size_t)d.H * d.P * sizeof(float), cudaMemcpyDeviceToDevice, stream));
    return SSD_OK;
}

ssd_status ssd_profile_enable(int enable) {
    std::lock_guard<std::mutex> g(prof::mu);
    prof::enabled = enable != 0;
    return SSD_OK;
}

ssd_status ssd_profile_read(int capacity, const char** names, double* ms, long long* calls, int* count) {
    std::lock_guard<std::mutex> g(prof::mu);
    for (const auto& p : prof::pending) {
        if (cudaEventSynchronize(p.b) != cudaSuccess) return SSD_ERR_CUDA;
        float t = 0.f;
        if (cudaEventElapsedTime(&t, p.a, p.b) != cudaSuccess) return SSD_ERR_CUDA;
        prof::ms[p.kernel] += t;
        prof::calls[p.kernel] += 1;
        prof::pool.push_back(p.a);
        prof::pool.push_back(p.b);
    }
    prof::pending.clear();
    const int n = (int)prof::names.size();
    if (count) *count = n;
    for (int i = 0; i < n && i < capacity; ++i) {
        if (names) names[i] = prof::names[i].c_str();
        if (ms) ms[i] = prof::ms[i];
        if (calls) calls[i] = prof::calls[i];
    }
    return SSD_OK;
}

ssd_status ssd_profile_filter(const char* name) {
    std::lock_guard<std::mutex> g(prof::mu);
    prof::filter = name ? std::string(name) : std::string();
    return SSD_OK;
}

ssd_status ssd_profile_reset(void) {
    std::lock_guard<std::mutex> g(prof::mu);
    for (const auto& p : prof::pending) {
        cudaEventSynchronize(p.b);
        prof::pool.push_back(p.a);
        prof::pool.push_back(p.b);
    }
    prof::pending.clear();
    for (auto& v : prof::ms) v = 0.0;
    for (auto& c : prof::calls) c = 0;
    return SSD_OK;
}

ssd_status ssd_workspace_status(void* workspace, cudaStream_t stream) {
    if (!workspace) return SSD_ERR_INVALID_ARG;
    int v = 0;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return SSD_ERR_CUDA;
    if (cudaMemcpy(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SSD_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpy(workspace, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return SSD_ERR_CUDA;
    }
    return v == 0 ? SSD_OK : (ssd_status)v;
}

}  // extern "C"
