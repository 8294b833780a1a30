// prep.cuh -- per-token work in front of the attention: the merging gate
// ("Multi-head Temporal Latent Attention", Sec. 4.1, Eq. 13), the RoPE of the
// decoupled key (Sec. 4.3), the in-place update of the slot being filled
// (Method (1)), and the query absorption [W_UK^T qC ; RoPE(qR)] (absorption
// kept from MLA). Device functions shared by the CUDA-core and tensor-core
// decode paths and by the prefill.
#pragma once
#include "common.cuh"
#include "mtla_internal.h"

namespace mtla {

// Merging weight of token t: sigmoid(G[t mod s] . (c_t * PE_t) + g[t mod s])
// (computed), the supplied value, or 1. Every thread of the block returns it;
// all threads must call it (block reduction inside).
template <typename T>
__device__ float gate_weight(const Shape& sh, int64_t t, const T* c_t, const float* gate_w,
                             const float* gate_b, const float* w_given, float* red) {
    if (sh.gate_mode == 2) return 1.f;
    if (sh.gate_mode == 1) return *w_given;
    const int r = (int)(t % sh.s);
    const float* G = gate_w + (size_t)r * sh.d_c;
    float z = 0.f;
    for (int k = threadIdx.x; k < sh.d_c / 2; k += blockDim.x) {
        float sn, cs;
        pair_sincos(t, k, sh.d_c, sh.log2_pe_base, &sn, &cs);
        z = fmaf(G[2 * k] * to_f<T>(c_t[2 * k]), sn, z);
        z = fmaf(G[2 * k + 1] * to_f<T>(c_t[2 * k + 1]), cs, z);
    }
    z = block_sum(z, red) + gate_b[r];
    return sigmoidf_(z);
}

// Decode: gate, RoPE and in-place update of sequence b's open slot; writes
// the rounded row into the cache. Returns false (and latches CAPACITY) if
// pos[b] does not fit the cache.
template <typename T>
__device__ bool decode_update_body(const DecodeArgs& a, int b) {
    const Shape& sh = a.sh;
    const int64_t t = a.pos[b];
    if (t < 0 || t >= (int64_t)sh.max_slots * sh.s) {
        if (threadIdx.x == 0) latch_status(a.status, kStatusCapacity);
        return false;
    }
    __shared__ float red[32];
    const T* c = (const T*)a.c_new + (size_t)b * sh.d_c;
    const T* kr = (const T*)a.kr_new + (size_t)b * sh.d_r;
    const float w = gate_weight<T>(sh, t, c, a.gate_w, a.gate_b, a.gate_in ? a.gate_in + b : nullptr, red);
    float* acc = a.open_slot + (size_t)b * sh.D;
    T* row = (T*)a.cache + ((size_t)b * sh.max_slots + (size_t)(t / sh.s)) * sh.D;
    const bool fresh = (t % sh.s) == 0;
    for (int k = threadIdx.x; k < sh.d_c; k += blockDim.x) {
        const float v = (fresh ? 0.f : acc[k]) + w * to_f<T>(c[k]);
        acc[k] = v;
        row[k] = from_f<T>(v);
    }
    for (int k = threadIdx.x; k < sh.d_r / 2; k += blockDim.x) {
        float sn, cs;
        pair_sincos(t, k, sh.d_r, sh.log2_rope_base, &sn, &cs);
        const float x0 = to_f<T>(kr[2 * k]), x1 = to_f<T>(kr[2 * k + 1]);
        const float y0 = x0 * cs - x1 * sn, y1 = x0 * sn + x1 * cs;
        float* ar = acc + sh.d_c;
        const float v0 = (fresh ? 0.f : ar[2 * k]) + w * y0;
        const float v1 = (fresh ? 0.f : ar[2 * k + 1]) + w * y1;
        ar[2 * k] = v0;
        ar[2 * k + 1] = v1;
        row[sh.d_c + 2 * k] = from_f<T>(v0);
        row[sh.d_c + 2 * k + 1] = from_f<T>(v1);
    }
    return true;
}

// Absorbed query of (row, head h) at position t into qt[(row*H + h)*D ...]
// (fp32): q~[j] = sum_i W_UK[h][i][j] qC[i] for j < d_c, then RoPE_t(qR).
template <typename T>
__device__ void absorb_query_body(const Shape& sh, const T* qc, const T* qr, const T* w_uk, int64_t row,
                                  int h, int64_t t, float* qt) {
    __shared__ float q[256];
    const size_t rh = (size_t)row * sh.H + h;
    for (int i = threadIdx.x; i < sh.d_h; i += blockDim.x) q[i] = to_f<T>(qc[rh * sh.d_h + i]);
    __syncthreads();
    const T* W = w_uk + (size_t)h * sh.d_h * sh.d_c;
    float* out = qt + rh * sh.D;
    for (int j = threadIdx.x; j < sh.d_c; j += blockDim.x) {
        float acc = 0.f;
        for (int i = 0; i < sh.d_h; ++i) acc = fmaf(to_f<T>(W[(size_t)i * sh.d_c + j]), q[i], acc);
        out[j] = acc;
    }
    const T* r = qr + rh * sh.d_r;
    for (int k = threadIdx.x; k < sh.d_r / 2; k += blockDim.x) {
        float sn, cs;
        pair_sincos(t, k, sh.d_r, sh.log2_rope_base, &sn, &cs);
        const float x0 = to_f<T>(r[2 * k]), x1 = to_f<T>(r[2 * k + 1]);
        out[sh.d_c + 2 * k] = x0 * cs - x1 * sn;
        out[sh.d_c + 2 * k + 1] = x0 * sn + x1 * cs;
    }
}

// One launch for both: block (b, h < H) absorbs head h of sequence b; block
// (b, H) updates sequence b's open slot. grid (B, H + 1).
template <typename T>
__global__ void __launch_bounds__(128) k_decode_prep(DecodeArgs a, float* qt) {
    const Shape& sh = a.sh;
    const int b = blockIdx.x, h = blockIdx.y;
    if (h == sh.H) {
        decode_update_body<T>(a, b);
        return;
    }
    const int64_t t = a.pos[b];
    if (t < 0 || t >= (int64_t)sh.max_slots * sh.s) return;
    absorb_query_body<T>(sh, (const T*)a.q_c, (const T*)a.q_r, (const T*)a.w_uk, b, h, t, qt);
}

// Prefill absorption: grid (B*T, H); row = b*T + t.
template <typename T>
__global__ void __launch_bounds__(128) k_prefill_absorb(Shape sh, const T* qc, const T* qr, const T* w_uk,
                                                        int T_len, float* qt) {
    const int64_t row = blockIdx.x;
    absorb_query_body<T>(sh, qc, qr, w_uk, row, blockIdx.y, row % T_len, qt);
}

}  // namespace mtla
