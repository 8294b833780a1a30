// mtla_static.cu -- a decode-step entry point that allocates nothing.
//
// Some callers cannot hand the library a workspace: they run inside a host
// framework whose pool allocator owns all device memory and forbids raw
// cudaMalloc (so that its own accounting stays right), or in a serving loop
// where a cudaMalloc/cudaFree could synchronise the device in the middle of a
// latency budget, or in a plug-in host that passes only input and output
// buffers. For them, mtla_decode_step_noalloc() takes the decode step's scratch
// from one fixed array in device memory that this file declares. Every GPU
// that loads libmtla.so holds that array until the process exits.
#include <mutex>

#include "../../include/mtla.h"

namespace {

// The scratch every call of mtla_decode_step_noalloc shares, on each device.
__device__ __align__(256) unsigned char g_noalloc_scratch[MTLA_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch, looked up once per device. In host code
// the array's name only stands in for the symbol; a kernel must be given the
// address that cudaGetSymbolAddress returns on the current device.
cudaError_t noalloc_scratch_address(void** out) {
    static std::mutex mu;
    static void* addr[64] = {nullptr};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = p;
    }
    *out = addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" mtla_status mtla_decode_step_noalloc(
    const mtla_config* cfg, const void* c_new, const void* kr_new, const void* q_c,
    const void* q_r, const void* w_uk, const void* w_uv, const float* gate_w,
    const float* gate_b, const float* gate_in, const int32_t* pos, void* cache, float* open_slot,
    void* out, void* stream) {
    // Size check first, on the host: a config whose decode scratch does not fit
    // in the built-in array is refused before anything touches the device.
    size_t need = 0;
    mtla_status st = mtla_workspace_size(cfg, 0, &need);
    if (st != MTLA_OK) return st;
    if (need > (size_t)MTLA_NOALLOC_SCRATCH_BYTES) return MTLA_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (noalloc_scratch_address(&scratch) != cudaSuccess) return MTLA_ERR_CUDA;
    // The decode kernels write every scratch byte before they read it, so the
    // previous call's leftovers need no clearing.
    return mtla_decode_step(cfg, c_new, kr_new, q_c, q_r, w_uk, w_uv, gate_w, gate_b, gate_in,
                            pos, cache, open_slot, out, scratch, (size_t)MTLA_NOALLOC_SCRATCH_BYTES,
                            stream);
}
