// common.cuh -- device helpers shared by the MTLA kernels (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mtla {

// Device-side status codes (same values as mtla_status).
enum : int { kStatusOk = 0, kStatusCapacity = 3, kStatusTimeout = 5 };

// Record the first device-side error; later ones keep the first.
__device__ __forceinline__ void latch_status(int* status, int code) {
    atomicCAS(status, 0, code);
}

typedef __nv_bfloat16 bf16;
typedef __half f16;

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<bf16>(bf16 x) { return __bfloat162float(x); }
template <> __device__ __forceinline__ float to_f<f16>(f16 x) { return __half2float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float x) { return __float2bfloat16_rn(x); }
template <> __device__ __forceinline__ f16 from_f<f16>(float x) { return __float2half_rn(x); }

// Storage rounding: what a value becomes once written to the cache.
template <typename T> __device__ __forceinline__ float round_to(float x) { return to_f<T>(from_f<T>(x)); }

// Angle t * base^(-2k/d) of rotation pair k, reduced to [-pi, pi] in double
// (positions reach 2^16 and beyond, where a float angle would lose ~1e-2 rad),
// then sine and cosine in float. Used for the sinusoidal PE (base 10000 over
// the latent width) and for RoPE (rope_base over d_r).
__device__ __forceinline__ void pair_sincos(int64_t t, int k, int d, double log2_base,
                                            float* sn, float* cs) {
    const double inv_freq = exp2(-(2.0 * k / (double)d) * log2_base);
    double a = (double)t * inv_freq;
    a = fma(-6.283185307179586476925, rint(a * 0.15915494309189533577), a);
    sincosf((float)a, sn, cs);
}

// Same angle with the frequency given (precomputed per block).
__device__ __forceinline__ void pair_sincos_f(int64_t t, double inv_freq, float* sn, float* cs) {
    double a = (double)t * inv_freq;
    a = fma(-6.283185307179586476925, rint(a * 0.15915494309189533577), a);
    sincosf((float)a, sn, cs);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Block-wide sum; every thread gets the result. `red` holds >= 32 floats.
__device__ __forceinline__ float block_sum(float v, float* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nw = (blockDim.x + 31) >> 5;
    v = warp_sum(v);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float r = (lane < nw) ? red[lane] : 0.f;
    r = warp_sum(r);
    return r;
}

// Two floats as one 32-bit word of two 16-bit values of type E (round to
// nearest even), `lo` at the lower address; and the two halves back.
template <typename E> __device__ __forceinline__ uint32_t pack2(float lo, float hi);
template <> __device__ __forceinline__ uint32_t pack2<f16>(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}
template <typename E> __device__ __forceinline__ float lo_of(uint32_t w);
template <typename E> __device__ __forceinline__ float hi_of(uint32_t w);
template <> __device__ __forceinline__ float lo_of<bf16>(uint32_t w) { return __uint_as_float(w << 16); }
template <> __device__ __forceinline__ float hi_of<bf16>(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
template <> __device__ __forceinline__ float lo_of<f16>(uint32_t w) {
    return __half2float(__ushort_as_half((unsigned short)(w & 0xffffu)));
}
template <> __device__ __forceinline__ float hi_of<f16>(uint32_t w) {
    return __half2float(__ushort_as_half((unsigned short)(w >> 16)));
}
// Two floats as bf16 (round to nearest even), `lo` at the lower address.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}
template <> __device__ __forceinline__ uint32_t pack2<bf16>(float lo, float hi) { return pack_bf16x2(lo, hi); }

__device__ __forceinline__ float sigmoidf_(float z) { return 1.f / (1.f + expf(-z)); }

// Programmatic dependent launch: let the next kernel in the stream start its
// prologue; wait until the previous kernel's results are visible (both are
// no-ops when the launch was an ordinary one).
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

}  // namespace mtla
