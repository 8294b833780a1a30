// mtla_api.cu -- the C ABI of libmtla.so: argument checks, scratch layout,
// device status word and dispatch to the kernels. See include/mtla.h.
#include <mutex>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>

#include "../../include/mtla.h"
#include "mtla_internal.h"

namespace mtla {

// Device status word, one per device that loads the library: the first error
// a kernel finds (a position beyond the cache, a bounded wait that ran out).
__device__ int g_device_status;

static std::atomic<uint64_t> g_launches{0};

static thread_local char g_error_detail[256] = "";

cudaError_t note_error(const char* where, cudaError_t e) {
    if (e != cudaSuccess)
        snprintf(g_error_detail, sizeof(g_error_detail), "%s: %s (%s)", where, cudaGetErrorName(e),
                 cudaGetErrorString(e));
    return e;
}

static void* const* g_prof_events = nullptr;
static int32_t g_prof_pairs = 0;
static int32_t g_prof_next = 0;
static bool g_prof_open = false;

// Record a profile event: a plain record, or an event node while `st` is
// being captured into a graph.
static cudaError_t record_profile_event(void* ev, cudaStream_t st) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return cudaGetLastError();
    if (cs == cudaStreamCaptureStatusActive)
        return cudaEventRecordWithFlags((cudaEvent_t)ev, st, cudaEventRecordExternal);
    return cudaEventRecord((cudaEvent_t)ev, st);
}

void profile_begin(cudaStream_t st) {
    g_prof_open = false;
    if (g_prof_events && g_prof_next < g_prof_pairs) {
        if (record_profile_event(g_prof_events[2 * g_prof_next], st) == cudaSuccess) {
            g_prof_open = true;
        } else {
            cudaGetLastError();            // a bad handle turns the hook off, not the call
            g_prof_events = nullptr;
        }
    }
}

void profile_end(cudaStream_t st) {
    if (g_prof_open) {
        if (record_profile_event(g_prof_events[2 * g_prof_next + 1], st) == cudaSuccess) {
            ++g_prof_next;
        } else {
            cudaGetLastError();
            g_prof_events = nullptr;
        }
        g_prof_open = false;
    }
}

// Address of g_device_status on the current device (looked up once per device).
static cudaError_t status_ptr(int** out) {
    static std::mutex mu;
    static int* cached[64] = {nullptr};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!cached[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_device_status);
        if (e != cudaSuccess) return e;
        cached[dev] = (int*)p;
    }
    *out = cached[dev];
    return cudaSuccess;
}

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// Validate a config; fill the resolved shape.
static mtla_status check_config(const mtla_config* cfg, Shape* sh) {
    if (!cfg) return MTLA_ERR_INVALID_ARG;
    if (cfg->batch <= 0 || cfg->heads <= 0 || cfg->d_h <= 0 || cfg->d_c <= 0 || cfg->d_r <= 0 ||
        cfg->stride <= 0 || cfg->max_slots <= 0)
        return MTLA_ERR_INVALID_ARG;
    if (cfg->dtype != MTLA_BF16 && cfg->dtype != MTLA_FP32 && cfg->dtype != MTLA_FP16) return MTLA_ERR_INVALID_ARG;
    if (cfg->gate_mode < MTLA_GATE_COMPUTED || cfg->gate_mode > MTLA_GATE_CHANNEL_SUPPLIED)
        return MTLA_ERR_INVALID_ARG;
    if (!(cfg->softmax_scale >= 0.f) || !std::isfinite(cfg->softmax_scale)) return MTLA_ERR_INVALID_ARG;
    if (!(cfg->rope_base >= 0.f) || !std::isfinite(cfg->rope_base) ||
        (cfg->rope_base != 0.f && cfg->rope_base <= 1.f))
        return MTLA_ERR_INVALID_ARG;
    if (cfg->d_h % 16 || cfg->d_c % 16 || cfg->d_r % 16) return MTLA_ERR_UNSUPPORTED;
    if (cfg->d_c + cfg->d_r > 576 || cfg->d_c > 512 || cfg->heads > 128 || cfg->d_h > 256 ||
        cfg->stride > 8)
        return MTLA_ERR_UNSUPPORTED;
    if ((int64_t)cfg->max_slots * cfg->stride > INT32_MAX) return MTLA_ERR_UNSUPPORTED;
    // per-channel gates: the scan keeps a lane's RoPE pairs in registers (d_r <= 128)
    if (cfg->gate_mode >= MTLA_GATE_CHANNEL_COMPUTED && cfg->d_r > 128) return MTLA_ERR_UNSUPPORTED;
    sh->B = cfg->batch;
    sh->H = cfg->heads;
    sh->d_h = cfg->d_h;
    sh->d_c = cfg->d_c;
    sh->d_r = cfg->d_r;
    sh->s = cfg->stride;
    sh->D = cfg->d_c + cfg->d_r;
    sh->gate_mode = cfg->gate_mode;
    sh->dtype = cfg->dtype;
    sh->max_slots = cfg->max_slots;
    sh->scale = cfg->softmax_scale != 0.f ? cfg->softmax_scale
                                          : (float)(1.0 / std::sqrt((double)(cfg->d_h + cfg->d_r)));
    sh->log2_rope_base = std::log2(cfg->rope_base != 0.f ? (double)cfg->rope_base : 10000.0);
    sh->log2_pe_base = std::log2(10000.0);
    return MTLA_OK;
}

// bf16 and fp16 decode run on the tensor cores where the shape fits the
// kernel (heads <= 32, d_c a multiple of 128, slot width <= 384), and with
// 32 < heads <= 128 on the cluster kernel; fp32 and the other shapes on the
// CUDA-core kernels.
static bool use_tc_decode(const mtla_config* cfg, const Shape& sh) {
    return (cfg->dtype == MTLA_BF16 || cfg->dtype == MTLA_FP16) && tc_decode_supported(sh);
}
// bf16 or fp16 with 32 < heads <= 128: the cluster kernel with all heads as M = 128.
static bool use_tc_decode_lh(const mtla_config* cfg, const Shape& sh) {
    return (cfg->dtype == MTLA_BF16 || cfg->dtype == MTLA_FP16) && !tc_decode_supported(sh) &&
           tc_decode_lh_supported(sh);
}

static size_t decode_ws(const mtla_config* cfg, const Shape& sh) {
    if (use_tc_decode(cfg, sh)) return tc_decode_workspace(sh);
    if (use_tc_decode_lh(cfg, sh)) return tc_decode_lh_workspace(sh);
    return simt_decode_workspace(sh);
}
// bf16 and fp16 prefill run on the tensor cores where the shape fits the
// kernel (d_h = 64, d_R = 32, d_c 128 or 256); the rest on the CUDA cores.
static bool use_tc_prefill(const mtla_config* cfg, const Shape& sh) {
    return (cfg->dtype == MTLA_BF16 || cfg->dtype == MTLA_FP16) && tc_prefill_supported(sh);
}

static size_t prefill_ws(const mtla_config* cfg, const Shape& sh, int T) {
    return use_tc_prefill(cfg, sh) ? tc_prefill_workspace(sh, T) : simt_prefill_workspace(sh, T);
}

static mtla_status check_gate_ptrs(const mtla_config* cfg, const float* gate_w, const float* gate_b,
                                   const float* gate_in) {
    if (cfg->gate_mode == MTLA_GATE_COMPUTED || cfg->gate_mode == MTLA_GATE_CHANNEL_COMPUTED) {
        if (!gate_w || !gate_b || !aligned16(gate_w) || !aligned16(gate_b)) return MTLA_ERR_INVALID_ARG;
    }
    if (cfg->gate_mode == MTLA_GATE_SUPPLIED || cfg->gate_mode == MTLA_GATE_CHANNEL_SUPPLIED) {
        if (!gate_in || !aligned16(gate_in)) return MTLA_ERR_INVALID_ARG;
    }
    return MTLA_OK;
}

size_t prefill_seed_bytes(const Shape& sh) { return align256((size_t)sh.B * sh.D * sizeof(float)); }

cudaError_t prefill_seed(PrefillArgs& a, void* seed_ws, cudaStream_t st) {
    if (!a.open_slot_in) return cudaSuccess;
    cudaError_t e = cudaMemcpyAsync(seed_ws, a.open_slot_in, (size_t)a.sh.B * a.sh.D * sizeof(float),
                                    cudaMemcpyDeviceToDevice, st);
    a.open_slot_in = (const float*)seed_ws;
    return note_error("prefill open-slot copy", e);
}

}  // namespace mtla

using namespace mtla;

extern "C" {

mtla_status mtla_workspace_size(const mtla_config* cfg, int32_t max_tokens, size_t* bytes) {
    Shape sh;
    if (!bytes || max_tokens < 0) return MTLA_ERR_INVALID_ARG;
    mtla_status st = check_config(cfg, &sh);
    if (st != MTLA_OK) return st;
    size_t d = decode_ws(cfg, sh);
    size_t p = max_tokens > 0 ? prefill_ws(cfg, sh, max_tokens) : 0;
    *bytes = d > p ? d : p;
    return MTLA_OK;
}

mtla_status mtla_decode_step(const mtla_config* cfg, const void* c_new, const void* kr_new,
                             const void* q_c, const void* q_r, const void* w_uk, const void* w_uv,
                             const float* gate_w, const float* gate_b, const float* gate_in,
                             const int32_t* pos, void* cache, float* open_slot, void* out,
                             void* workspace, size_t workspace_bytes, void* stream) {
    Shape sh;
    mtla_status st = check_config(cfg, &sh);
    if (st != MTLA_OK) return st;
    const void* req[] = {c_new, kr_new, q_c, q_r, w_uk, w_uv, pos, cache, open_slot, out, workspace};
    for (const void* p : req)
        if (!p || !aligned16(p)) return MTLA_ERR_INVALID_ARG;
    st = check_gate_ptrs(cfg, gate_w, gate_b, gate_in);
    if (st != MTLA_OK) return st;
    if (workspace_bytes < decode_ws(cfg, sh)) return MTLA_ERR_WORKSPACE;
    DecodeArgs a;
    a.sh = sh;
    a.c_new = c_new;
    a.kr_new = kr_new;
    a.q_c = q_c;
    a.q_r = q_r;
    a.w_uk = w_uk;
    a.w_uv = w_uv;
    a.gate_w = gate_w;
    a.gate_b = gate_b;
    a.gate_in = gate_in;
    a.pos = pos;
    a.cache = cache;
    a.open_slot = open_slot;
    a.out = out;
    a.workspace = workspace;
    a.workspace_bytes = workspace_bytes;
    g_error_detail[0] = 0;
    if (note_error("device status word", status_ptr(&a.status)) != cudaSuccess) return MTLA_ERR_CUDA;
    uint64_t n = 0;
    cudaError_t e = use_tc_decode(cfg, sh)      ? tc_decode(a, (cudaStream_t)stream, &n)
                    : use_tc_decode_lh(cfg, sh) ? tc_decode_lh(a, (cudaStream_t)stream, &n)
                                                : simt_decode(a, cfg->dtype, (cudaStream_t)stream, &n);
    g_launches += n;
    if (e != cudaSuccess && !g_error_detail[0]) note_error("decode launch", e);
    return e == cudaSuccess ? MTLA_OK : MTLA_ERR_CUDA;
}

static mtla_status prefill_common(const mtla_config* cfg, int32_t t0, int32_t T, const void* c, const void* kr,
                                  const void* q_c, const void* q_r, const void* w_uk, const void* w_uv,
                                  const float* gate_w, const float* gate_b, const float* gate_in, void* out,
                                  void* cache, const float* open_in, float* open_out, void* workspace,
                                  size_t workspace_bytes, void* stream) {
    Shape sh;
    mtla_status st = check_config(cfg, &sh);
    if (st != MTLA_OK) return st;
    if (T <= 0 || t0 < 0) return MTLA_ERR_INVALID_ARG;
    const void* req[] = {c, kr, q_c, q_r, w_uk, w_uv, out, cache, workspace};
    for (const void* p : req)
        if (!p || !aligned16(p)) return MTLA_ERR_INVALID_ARG;
    if (open_out && !aligned16(open_out)) return MTLA_ERR_INVALID_ARG;
    if (t0 % sh.s != 0 && (!open_in || !aligned16(open_in))) return MTLA_ERR_INVALID_ARG;
    st = check_gate_ptrs(cfg, gate_w, gate_b, gate_in);
    if (st != MTLA_OK) return st;
    if (((int64_t)t0 + T + sh.s - 1) / sh.s > sh.max_slots) return MTLA_ERR_CAPACITY;
    if (workspace_bytes < prefill_ws(cfg, sh, T)) return MTLA_ERR_WORKSPACE;
    PrefillArgs a;
    a.sh = sh;
    a.T = T;
    a.t0 = t0;
    a.open_slot_in = t0 % sh.s != 0 ? open_in : nullptr;
    a.c = c;
    a.kr = kr;
    a.q_c = q_c;
    a.q_r = q_r;
    a.w_uk = w_uk;
    a.w_uv = w_uv;
    a.gate_w = gate_w;
    a.gate_b = gate_b;
    a.gate_in = gate_in;
    a.out = out;
    a.cache_out = cache;
    a.open_slot_out = open_out;
    a.workspace = workspace;
    a.workspace_bytes = workspace_bytes;
    g_error_detail[0] = 0;
    if (note_error("device status word", status_ptr(&a.status)) != cudaSuccess) return MTLA_ERR_CUDA;
    uint64_t n = 0;
    cudaError_t e = use_tc_prefill(cfg, sh) ? tc_prefill(a, (cudaStream_t)stream, &n)
                                            : simt_prefill(a, cfg->dtype, (cudaStream_t)stream, &n);
    g_launches += n;
    if (e != cudaSuccess && !g_error_detail[0]) note_error("prefill launch", e);
    return e == cudaSuccess ? MTLA_OK : MTLA_ERR_CUDA;
}

mtla_status mtla_prefill(const mtla_config* cfg, int32_t T, const void* c, const void* kr,
                         const void* q_c, const void* q_r, const void* w_uk, const void* w_uv,
                         const float* gate_w, const float* gate_b, const float* gate_in, void* out,
                         void* cache_out, float* open_slot_out, void* workspace,
                         size_t workspace_bytes, void* stream) {
    return prefill_common(cfg, 0, T, c, kr, q_c, q_r, w_uk, w_uv, gate_w, gate_b, gate_in, out, cache_out,
                          nullptr, open_slot_out, workspace, workspace_bytes, stream);
}

mtla_status mtla_prefill_from(const mtla_config* cfg, int32_t t0, int32_t T, const void* c, const void* kr,
                              const void* q_c, const void* q_r, const void* w_uk, const void* w_uv,
                              const float* gate_w, const float* gate_b, const float* gate_in, void* out,
                              void* cache, float* open_slot, void* workspace, size_t workspace_bytes,
                              void* stream) {
    if (!open_slot) return MTLA_ERR_INVALID_ARG;
    return prefill_common(cfg, t0, T, c, kr, q_c, q_r, w_uk, w_uv, gate_w, gate_b, gate_in, out, cache,
                          open_slot, open_slot, workspace, workspace_bytes, stream);
}

static mtla_status backward_check(const mtla_config* cfg, int32_t T, Shape* sh) {
    mtla_status st = check_config(cfg, sh);
    if (st != MTLA_OK) return st;
    if (T <= 0) return MTLA_ERR_INVALID_ARG;
    if (cfg->gate_mode > MTLA_GATE_UNIT || cfg->batch > 65535 || (int64_t)cfg->batch * T > INT32_MAX)
        return MTLA_ERR_UNSUPPORTED;
    return MTLA_OK;
}

mtla_status mtla_prefill_backward_workspace_size(const mtla_config* cfg, int32_t T, size_t* bytes) {
    Shape sh;
    if (!bytes) return MTLA_ERR_INVALID_ARG;
    mtla_status st = backward_check(cfg, T, &sh);
    if (st != MTLA_OK) return st;
    *bytes = prefill_backward_workspace(sh, T, cfg->dtype);
    return MTLA_OK;
}

mtla_status mtla_prefill_backward(const mtla_config* cfg, int32_t T, const void* c, const void* kr,
                                  const void* q_c, const void* q_r, const void* w_uk, const void* w_uv,
                                  const float* gate_w, const float* gate_b, const float* gate_in,
                                  const void* dout, float* dc, float* dkr, float* dq_c, float* dq_r,
                                  float* dw_uk, float* dw_uv, float* dgate_w, float* dgate_b, float* dgate_in,
                                  void* workspace, size_t workspace_bytes, void* stream) {
    Shape sh;
    mtla_status st = backward_check(cfg, T, &sh);
    if (st != MTLA_OK) return st;
    const void* req[] = {c, kr, q_c, q_r, w_uk, w_uv, dout, dc, dkr, dq_c, dq_r, dw_uk, dw_uv, workspace};
    for (const void* p : req)
        if (!p || !aligned16(p)) return MTLA_ERR_INVALID_ARG;
    st = check_gate_ptrs(cfg, gate_w, gate_b, gate_in);
    if (st != MTLA_OK) return st;
    if (cfg->gate_mode == MTLA_GATE_COMPUTED &&
        (!dgate_w || !dgate_b || !aligned16(dgate_w) || !aligned16(dgate_b)))
        return MTLA_ERR_INVALID_ARG;
    if (cfg->gate_mode == MTLA_GATE_SUPPLIED && (!dgate_in || !aligned16(dgate_in))) return MTLA_ERR_INVALID_ARG;
    if (workspace_bytes < prefill_backward_workspace(sh, T, cfg->dtype))
        return MTLA_ERR_WORKSPACE;
    PrefillArgs a = {};
    a.sh = sh;
    a.T = T;
    a.c = c;
    a.kr = kr;
    a.q_c = q_c;
    a.q_r = q_r;
    a.w_uk = w_uk;
    a.w_uv = w_uv;
    a.gate_w = gate_w;
    a.gate_b = gate_b;
    a.gate_in = gate_in;
    a.workspace = workspace;
    a.workspace_bytes = workspace_bytes;
    BackwardGrads g = {dout, dc, dkr, dq_c, dq_r, dw_uk, dw_uv, dgate_w, dgate_b, dgate_in};
    g_error_detail[0] = 0;
    if (note_error("device status word", status_ptr(&a.status)) != cudaSuccess) return MTLA_ERR_CUDA;
    uint64_t n = 0;
    cudaError_t e = prefill_backward(a, g, cfg->dtype, (cudaStream_t)stream, &n);
    g_launches += n;
    if (e != cudaSuccess && !g_error_detail[0]) note_error("backward launch", e);
    return e == cudaSuccess ? MTLA_OK : MTLA_ERR_CUDA;
}

static mtla_status train_check(const mtla_config* cfg, int32_t T, Shape* sh) {
    mtla_status st = backward_check(cfg, T, sh);
    if (st != MTLA_OK) return st;
    return prefill_train_supported(*sh) ? MTLA_OK : MTLA_ERR_UNSUPPORTED;
}

mtla_status mtla_prefill_train_saved_size(const mtla_config* cfg, int32_t T, size_t* bytes) {
    Shape sh;
    if (!bytes) return MTLA_ERR_INVALID_ARG;
    mtla_status st = train_check(cfg, T, &sh);
    if (st != MTLA_OK) return st;
    *bytes = prefill_train_saved_bytes(sh, T);
    return MTLA_OK;
}

mtla_status mtla_prefill_backward_saved_workspace_size(const mtla_config* cfg, int32_t T, size_t* bytes) {
    Shape sh;
    if (!bytes) return MTLA_ERR_INVALID_ARG;
    mtla_status st = train_check(cfg, T, &sh);
    if (st != MTLA_OK) return st;
    *bytes = prefill_backward_saved_workspace(sh, T);
    return MTLA_OK;
}

static PrefillArgs train_args(const Shape& sh, int32_t T, const void* c, const void* kr, const void* q_c,
                              const void* q_r, const void* w_uk, const void* w_uv, const float* gate_w,
                              const float* gate_b, const float* gate_in) {
    PrefillArgs a = {};
    a.sh = sh;
    a.T = T;
    a.c = c;
    a.kr = kr;
    a.q_c = q_c;
    a.q_r = q_r;
    a.w_uk = w_uk;
    a.w_uv = w_uv;
    a.gate_w = gate_w;
    a.gate_b = gate_b;
    a.gate_in = gate_in;
    return a;
}

mtla_status mtla_prefill_train(const mtla_config* cfg, int32_t T, const void* c, const void* kr, const void* q_c,
                               const void* q_r, const void* w_uk, const void* w_uv, const float* gate_w,
                               const float* gate_b, const float* gate_in, void* out, void* saved, size_t saved_bytes,
                               void* stream) {
    Shape sh;
    mtla_status st = train_check(cfg, T, &sh);
    if (st != MTLA_OK) return st;
    const void* req[] = {c, kr, q_c, q_r, w_uk, w_uv, out, saved};
    for (const void* p : req)
        if (!p || !aligned16(p)) return MTLA_ERR_INVALID_ARG;
    st = check_gate_ptrs(cfg, gate_w, gate_b, gate_in);
    if (st != MTLA_OK) return st;
    if (saved_bytes < prefill_train_saved_bytes(sh, T)) return MTLA_ERR_WORKSPACE;
    PrefillArgs a = train_args(sh, T, c, kr, q_c, q_r, w_uk, w_uv, gate_w, gate_b, gate_in);
    a.out = out;
    g_error_detail[0] = 0;
    if (note_error("device status word", status_ptr(&a.status)) != cudaSuccess) return MTLA_ERR_CUDA;
    uint64_t n = 0;
    cudaError_t e = prefill_train(a, saved, (cudaStream_t)stream, &n);
    g_launches += n;
    if (e != cudaSuccess && !g_error_detail[0]) note_error("training forward launch", e);
    return e == cudaSuccess ? MTLA_OK : MTLA_ERR_CUDA;
}

mtla_status mtla_prefill_backward_saved(const mtla_config* cfg, int32_t T, const void* c, const void* kr,
                                        const void* q_c, const void* q_r, const void* w_uk, const void* w_uv,
                                        const float* gate_w, const float* gate_b, const float* gate_in,
                                        const void* saved, const void* dout, float* dc, float* dkr, float* dq_c,
                                        float* dq_r, float* dw_uk, float* dw_uv, float* dgate_w, float* dgate_b,
                                        float* dgate_in, void* workspace, size_t workspace_bytes, void* stream) {
    Shape sh;
    mtla_status st = train_check(cfg, T, &sh);
    if (st != MTLA_OK) return st;
    const void* req[] = {c, kr, q_c, q_r, w_uk, w_uv, saved, dout, dc, dkr, dq_c, dq_r, dw_uk, dw_uv, workspace};
    for (const void* p : req)
        if (!p || !aligned16(p)) return MTLA_ERR_INVALID_ARG;
    st = check_gate_ptrs(cfg, gate_w, gate_b, gate_in);
    if (st != MTLA_OK) return st;
    if (cfg->gate_mode == MTLA_GATE_COMPUTED &&
        (!dgate_w || !dgate_b || !aligned16(dgate_w) || !aligned16(dgate_b)))
        return MTLA_ERR_INVALID_ARG;
    if (cfg->gate_mode == MTLA_GATE_SUPPLIED && (!dgate_in || !aligned16(dgate_in))) return MTLA_ERR_INVALID_ARG;
    if (workspace_bytes < prefill_backward_saved_workspace(sh, T)) return MTLA_ERR_WORKSPACE;
    PrefillArgs a = train_args(sh, T, c, kr, q_c, q_r, w_uk, w_uv, gate_w, gate_b, gate_in);
    a.workspace = workspace;
    a.workspace_bytes = workspace_bytes;
    BackwardGrads g = {dout, dc, dkr, dq_c, dq_r, dw_uk, dw_uv, dgate_w, dgate_b, dgate_in};
    g_error_detail[0] = 0;
    if (note_error("device status word", status_ptr(&a.status)) != cudaSuccess) return MTLA_ERR_CUDA;
    uint64_t n = 0;
    cudaError_t e = prefill_backward_saved(a, g, saved, (cudaStream_t)stream, &n);
    g_launches += n;
    if (e != cudaSuccess && !g_error_detail[0]) note_error("backward launch", e);
    return e == cudaSuccess ? MTLA_OK : MTLA_ERR_CUDA;
}

mtla_status mtla_linear(const void* x, const void* w, void* y, int32_t M, int32_t N, int32_t K, void* stream) {
    if (M <= 0 || N <= 0 || K <= 0 || K % 8 != 0) return MTLA_ERR_INVALID_ARG;
    if (!x || !w || !y || !aligned16(x) || !aligned16(w) || !aligned16(y)) return MTLA_ERR_INVALID_ARG;
    g_error_detail[0] = 0;
    int* status = nullptr;
    if (note_error("device status word", status_ptr(&status)) != cudaSuccess) return MTLA_ERR_CUDA;
    uint64_t n = 0;
    cudaError_t e = gemm_bf16(x, K, w, K, y, N, M, N, K, status, (cudaStream_t)stream, &n);
    g_launches += n;
    return e == cudaSuccess ? MTLA_OK : MTLA_ERR_CUDA;
}

// The layer around the path: activations of M = B*T tokens in the workspace
// (c, k, qC, qR, o; bf16, 256-byte aligned regions), then the path's scratch.
struct LayerWs {
    size_t c, kr, qc, qr, o, path, total;
};
static LayerWs layer_ws_layout(const Shape& sh, int64_t M, size_t path_bytes) {
    LayerWs l;
    l.c = 0;
    l.kr = l.c + align256((size_t)M * sh.d_c * 2);
    l.qc = l.kr + align256((size_t)M * sh.d_r * 2);
    l.qr = l.qc + align256((size_t)M * sh.H * sh.d_h * 2);
    l.o = l.qr + align256((size_t)M * sh.H * sh.d_r * 2);
    l.path = l.o + align256((size_t)M * sh.H * sh.d_h * 2);
    l.total = l.path + path_bytes;
    return l;
}

static mtla_status layer_check(const mtla_config* cfg, int32_t d_model, Shape* sh) {
    mtla_status st = check_config(cfg, sh);
    if (st != MTLA_OK) return st;
    if (d_model <= 0 || d_model % 8 != 0) return MTLA_ERR_INVALID_ARG;
    if (cfg->dtype != MTLA_BF16) return MTLA_ERR_UNSUPPORTED;
    return MTLA_OK;
}

static mtla_status layer_weights_ok(const mtla_layer_weights* w) {
    if (!w) return MTLA_ERR_INVALID_ARG;
    const void* p[] = {w->w_dkv, w->w_kr, w->w_q, w->w_qr, w->w_uk, w->w_uv, w->w_o};
    for (const void* q : p)
        if (!q || !aligned16(q)) return MTLA_ERR_INVALID_ARG;
    return MTLA_OK;
}

// The four projections of M tokens of h into the workspace activations.
static cudaError_t layer_project(const Shape& sh, int d_model, int64_t M, const void* h,
                                 const mtla_layer_weights* w, char* ws, const LayerWs& l, int* status,
                                 cudaStream_t st, uint64_t* n) {
    const int m = (int)M;
    cudaError_t e = gemm_bf16(h, d_model, w->w_dkv, d_model, ws + l.c, sh.d_c, m, sh.d_c, d_model, status, st, n);
    if (e == cudaSuccess) e = gemm_bf16(h, d_model, w->w_kr, d_model, ws + l.kr, sh.d_r, m, sh.d_r, d_model, status, st, n);
    if (e == cudaSuccess)
        e = gemm_bf16(h, d_model, w->w_q, d_model, ws + l.qc, sh.H * sh.d_h, m, sh.H * sh.d_h, d_model, status, st, n);
    if (e == cudaSuccess)
        e = gemm_bf16(h, d_model, w->w_qr, d_model, ws + l.qr, sh.H * sh.d_r, m, sh.H * sh.d_r, d_model, status, st, n);
    return e;
}

mtla_status mtla_layer_workspace_size(const mtla_config* cfg, int32_t d_model, int32_t max_tokens, size_t* bytes) {
    Shape sh;
    if (!bytes || max_tokens < 0) return MTLA_ERR_INVALID_ARG;
    mtla_status st = layer_check(cfg, d_model, &sh);
    if (st != MTLA_OK) return st;
    const size_t dec = layer_ws_layout(sh, sh.B, decode_ws(cfg, sh)).total;
    const size_t pre = max_tokens > 0 ? layer_ws_layout(sh, (int64_t)sh.B * max_tokens, prefill_ws(cfg, sh, max_tokens)).total : 0;
    *bytes = dec > pre ? dec : pre;
    return MTLA_OK;
}

mtla_status mtla_layer_forward(const mtla_config* cfg, int32_t d_model, int32_t t0, int32_t T, const void* h,
                               const mtla_layer_weights* w, const float* gate_w, const float* gate_b,
                               const float* gate_in, void* y, void* cache, float* open_slot, void* workspace,
                               size_t workspace_bytes, void* stream) {
    Shape sh;
    mtla_status st = layer_check(cfg, d_model, &sh);
    if (st != MTLA_OK) return st;
    if (T <= 0 || t0 < 0) return MTLA_ERR_INVALID_ARG;
    if ((st = layer_weights_ok(w)) != MTLA_OK) return st;
    const void* req[] = {h, y, cache, open_slot, workspace};
    for (const void* p : req)
        if (!p || !aligned16(p)) return MTLA_ERR_INVALID_ARG;
    st = check_gate_ptrs(cfg, gate_w, gate_b, gate_in);
    if (st != MTLA_OK) return st;
    if (((int64_t)t0 + T + sh.s - 1) / sh.s > sh.max_slots) return MTLA_ERR_CAPACITY;
    const int64_t M = (int64_t)sh.B * T;
    const LayerWs l = layer_ws_layout(sh, M, prefill_ws(cfg, sh, T));
    if (workspace_bytes < l.total) return MTLA_ERR_WORKSPACE;
    char* ws = (char*)workspace;
    g_error_detail[0] = 0;
    int* status = nullptr;
    if (note_error("device status word", status_ptr(&status)) != cudaSuccess) return MTLA_ERR_CUDA;
    uint64_t n = 0;
    cudaStream_t s_ = (cudaStream_t)stream;
    cudaError_t e = layer_project(sh, d_model, M, h, w, ws, l, status, s_, &n);
    g_launches += n;
    if (e != cudaSuccess) return MTLA_ERR_CUDA;
    st = prefill_common(cfg, t0, T, ws + l.c, ws + l.kr, ws + l.qc, ws + l.qr, w->w_uk, w->w_uv, gate_w, gate_b,
                        gate_in, ws + l.o, cache, open_slot, open_slot, ws + l.path, workspace_bytes - l.path, stream);
    if (st != MTLA_OK) return st;
    n = 0;
    e = gemm_bf16(ws + l.o, sh.H * sh.d_h, w->w_o, sh.H * sh.d_h, y, d_model, (int)M, d_model, sh.H * sh.d_h,
                  status, s_, &n);
    g_launches += n;
    return e == cudaSuccess ? MTLA_OK : MTLA_ERR_CUDA;
}

mtla_status mtla_layer_decode_step(const mtla_config* cfg, int32_t d_model, const void* h,
                                   const mtla_layer_weights* w, const float* gate_w, const float* gate_b,
                                   const float* gate_in, const int32_t* pos, void* cache, float* open_slot,
                                   void* y, void* workspace, size_t workspace_bytes, void* stream) {
    Shape sh;
    mtla_status st = layer_check(cfg, d_model, &sh);
    if (st != MTLA_OK) return st;
    if ((st = layer_weights_ok(w)) != MTLA_OK) return st;
    const void* req[] = {h, y, pos, cache, open_slot, workspace};
    for (const void* p : req)
        if (!p || !aligned16(p)) return MTLA_ERR_INVALID_ARG;
    st = check_gate_ptrs(cfg, gate_w, gate_b, gate_in);
    if (st != MTLA_OK) return st;
    const LayerWs l = layer_ws_layout(sh, sh.B, decode_ws(cfg, sh));
    if (workspace_bytes < l.total) return MTLA_ERR_WORKSPACE;
    char* ws = (char*)workspace;
    g_error_detail[0] = 0;
    int* status = nullptr;
    if (note_error("device status word", status_ptr(&status)) != cudaSuccess) return MTLA_ERR_CUDA;
    uint64_t n = 0;
    cudaStream_t s_ = (cudaStream_t)stream;
    cudaError_t e = layer_project(sh, d_model, sh.B, h, w, ws, l, status, s_, &n);
    g_launches += n;
    if (e != cudaSuccess) return MTLA_ERR_CUDA;
    st = mtla_decode_step(cfg, ws + l.c, ws + l.kr, ws + l.qc, ws + l.qr, w->w_uk, w->w_uv, gate_w, gate_b, gate_in,
                          pos, cache, open_slot, ws + l.o, ws + l.path, workspace_bytes - l.path, stream);
    if (st != MTLA_OK) return st;
    n = 0;
    e = gemm_bf16(ws + l.o, sh.H * sh.d_h, w->w_o, sh.H * sh.d_h, y, d_model, sh.B, d_model, sh.H * sh.d_h, status,
                  s_, &n);
    g_launches += n;
    return e == cudaSuccess ? MTLA_OK : MTLA_ERR_CUDA;
}

mtla_status mtla_test_wait_timeout(uint64_t limit_ns, void* scratch, void* stream) {
    if (!scratch || !aligned16(scratch) || limit_ns == 0 || limit_ns > 1000000000ull) return MTLA_ERR_INVALID_ARG;
    g_error_detail[0] = 0;
    int* status = nullptr;
    if (note_error("device status word", status_ptr(&status)) != cudaSuccess) return MTLA_ERR_CUDA;
    uint64_t n = 0;
    cudaError_t e = wait_probe(limit_ns, scratch, status, (cudaStream_t)stream, &n);
    g_launches += n;
    return e == cudaSuccess ? MTLA_OK : MTLA_ERR_CUDA;
}

mtla_status mtla_get_device_status(void* stream) {
    int* p = nullptr;
    if (status_ptr(&p) != cudaSuccess) return MTLA_ERR_CUDA;
    cudaStream_t s = (cudaStream_t)stream;
    int v = 0;
    if (cudaMemcpyAsync(&v, p, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return MTLA_ERR_CUDA;
    if (cudaMemsetAsync(p, 0, sizeof(int), s) != cudaSuccess) return MTLA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MTLA_ERR_CUDA;
    return (mtla_status)v;
}

const char* mtla_status_string(mtla_status s) {
    switch (s) {
        case MTLA_OK: return "ok";
        case MTLA_ERR_INVALID_ARG: return "invalid argument";
        case MTLA_ERR_UNSUPPORTED: return "unsupported shape or option";
        case MTLA_ERR_CAPACITY: return "position beyond the cache capacity";
        case MTLA_ERR_CUDA: return "CUDA runtime error";
        case MTLA_ERR_TIMEOUT: return "device wait timed out";
        case MTLA_ERR_WORKSPACE: return "workspace too small";
    }
    return "unknown status";
}

mtla_status mtla_reorder_cache(const mtla_config* cfg, const int32_t* src, const int32_t* n_tokens,
                               const void* cache_in, const float* open_in, void* cache_out,
                               float* open_out, void* stream) {
    Shape sh;
    mtla_status st = check_config(cfg, &sh);
    if (st != MTLA_OK) return st;
    const void* req[] = {src, n_tokens, cache_in, open_in, cache_out, open_out};
    for (const void* p : req)
        if (!p || !aligned16(p)) return MTLA_ERR_INVALID_ARG;
    const size_t esize = cfg->dtype == MTLA_FP32 ? 4 : 2;
    const size_t cache_bytes = (size_t)sh.B * sh.max_slots * sh.D * esize;
    const size_t open_bytes = (size_t)sh.B * sh.D * sizeof(float);
    auto overlap = [](const void* a, size_t na, const void* b, size_t nb) {
        const uintptr_t x = (uintptr_t)a, y = (uintptr_t)b;
        return x < y + nb && y < x + na;
    };
    if (overlap(cache_in, cache_bytes, cache_out, cache_bytes) || overlap(open_in, open_bytes, open_out, open_bytes))
        return MTLA_ERR_INVALID_ARG;
    g_error_detail[0] = 0;
    int* status = nullptr;
    if (note_error("device status word", status_ptr(&status)) != cudaSuccess) return MTLA_ERR_CUDA;
    uint64_t n = 0;
    cudaError_t e = reorder_cache(sh, esize, src, n_tokens, cache_in, open_in, cache_out, open_out, status,
                                  (cudaStream_t)stream, &n);
    g_launches += n;
    return e == cudaSuccess ? MTLA_OK : MTLA_ERR_CUDA;
}

uint64_t mtla_kernel_launches(void) { return g_launches.load(); }

const char* mtla_last_error_detail(void) { return g_error_detail; }

void mtla_set_profile_events(void* const* events, int32_t n_pairs) {
    g_prof_events = (events && n_pairs > 0) ? events : nullptr;
    g_prof_pairs = g_prof_events ? n_pairs : 0;
    g_prof_next = 0;
    g_prof_open = false;
}

int32_t mtla_profile_events_recorded(void) { return g_prof_next; }

}  // extern "C"
