// prep.cuh -- per-token work in front of the attention: the merging gate
// ("Multi-head Temporal Latent Attention", Sec. 4.1, Eq. 13), the RoPE of the
// decoupled key (Sec. 4.3), the in-place update of the slot being filled
// (Method (1)), and the query absorption [W_UK^T qC ; RoPE(qR)] (absorption
// kept from MLA). Device functions shared by the CUDA-core and tensor-core
// decode paths and by the prefill.
#pragma once
#include <type_traits>

#include "common.cuh"
#include "mtla_internal.h"

namespace mtla {

constexpr int kUpdMaxPer = 4;     // latent pairs per thread of the slot update (d_c / 2 <= 4 * blockDim)
constexpr int kUpdMaxPairs = 3;   // RoPE pairs per thread (d_r / 2 <= 3 * blockDim)

// Inverse frequencies base^(-2k/d) of this thread's sinusoidal-PE pairs (over
// d_c) and RoPE pairs (over d_R) in the slot update: position independent, so
// a kernel may compute them before it waits for the step's inputs.
struct UpdateFreqs {
    double pe[kUpdMaxPer];
    double rope[kUpdMaxPairs];
};

__device__ __forceinline__ void update_freqs(const Shape& sh, UpdateFreqs& f) {
    const int nt = blockDim.x, tid = threadIdx.x;
#pragma unroll
    for (int i = 0; i < kUpdMaxPer; ++i) {
        const int kp = tid + i * nt;
        f.pe[i] = kp < sh.d_c / 2 ? exp2(-(2.0 * kp / (double)sh.d_c) * sh.log2_pe_base) : 0.0;
    }
#pragma unroll
    for (int i = 0; i < kUpdMaxPairs; ++i) {
        const int kp = tid + i * nt;
        f.rope[i] = kp < sh.d_r / 2 ? exp2(-(2.0 * kp / (double)sh.d_r) * sh.log2_rope_base) : 0.0;
    }
}

// Decode: gate (the merging weight of token t: sigmoid(G[t mod s] .
// (c_t * PE_t) + g[t mod s]) computed, the supplied value, or 1), RoPE and
// in-place update of sequence b's open slot; writes the rounded row into the
// cache. Every thread of the block must call it (block reduction inside).
// Returns false (and latches CAPACITY) if pos[b] does not fit the cache.
// `gate_w` is G [s x d_c] (global memory, or a copy in shared memory) and `f`
// the frequencies from update_freqs.
// Per-channel gate (modes 3 and 4): the D merging weights of token t of
// sequence b into wch, computed as sigmoid((c_t * PE_t) . G[r][:, k] + g[r][k])
// with G [s, d_c, D], g [s, D] (thread k of the block: output channel k, G read
// along k), or read from gate_in [B, D]. vch holds c_t * PE_t; c0/c1 are this
// thread's latent pairs and f its PE frequencies. Every thread calls it.
template <int kMaxPer>
__device__ void channel_gate(const DecodeArgs& a, int b, int64_t t, const float* gate_w, const UpdateFreqs& f,
                             const float* c0, const float* c1, float* vch, float* wch) {
    const Shape& sh = a.sh;
    const int nt = blockDim.x, tid = threadIdx.x;
    __syncthreads();                     // vch / wch of an earlier call of this block are read
    if (sh.gate_mode == 4) {
        for (int k = tid; k < sh.D; k += nt) wch[k] = a.gate_in[(size_t)b * sh.D + k];
    } else {
        const int r = (int)(t % sh.s);
#pragma unroll
        for (int i = 0; i < kMaxPer; ++i) {
            const int kp = tid + i * nt;
            if (kp < sh.d_c / 2) {
                float sn, cs;
                pair_sincos_f(t, f.pe[i], &sn, &cs);
                vch[2 * kp] = c0[i] * sn;
                vch[2 * kp + 1] = c1[i] * cs;
            }
        }
        __syncthreads();
        const float* G = gate_w + (size_t)r * sh.d_c * sh.D;
        for (int k = tid; k < sh.D; k += nt) {
            float z = a.gate_b[(size_t)r * sh.D + k];
            for (int i = 0; i < sh.d_c; ++i) z = fmaf(vch[i], G[(size_t)i * sh.D + k], z);
            wch[k] = sigmoidf_(z);
        }
    }
    __syncthreads();
}

template <typename T>
__device__ bool decode_update_body(const DecodeArgs& a, int b, const float* gate_w, const UpdateFreqs& f) {
    const Shape& sh = a.sh;
    __shared__ float red[32];
    __shared__ float vch[512], wch[576];  // per-channel gate: c_t * PE_t and the D weights
    constexpr int kMaxPer = kUpdMaxPer;
    constexpr int kMaxPairs = kUpdMaxPairs;
    const int nt = blockDim.x, tid = threadIdx.x;
    const T* c = (const T*)a.c_new + (size_t)b * sh.d_c;
    const T* kr = (const T*)a.kr_new + (size_t)b * sh.d_r;
    float* acc = a.open_slot + (size_t)b * sh.D;
    // every load that does not depend on the position first (one round trip
    // with the position itself): latent pairs (2kp, 2kp+1), open-slot values,
    // RoPE key pairs
    const int64_t t = a.pos[b];
    float c0[kMaxPer], c1[kMaxPer], a0[kMaxPer], a1[kMaxPer];
#pragma unroll
    for (int i = 0; i < kMaxPer; ++i) {
        const int kp = tid + i * nt;
        c0[i] = c1[i] = a0[i] = a1[i] = 0.f;
        if (kp < sh.d_c / 2) {
            c0[i] = to_f<T>(c[2 * kp]);
            c1[i] = to_f<T>(c[2 * kp + 1]);
            a0[i] = acc[2 * kp];
            a1[i] = acc[2 * kp + 1];
        }
    }
    float x0[kMaxPairs], x1[kMaxPairs], ar0[kMaxPairs], ar1[kMaxPairs];
#pragma unroll
    for (int i = 0; i < kMaxPairs; ++i) {
        const int kp = tid + i * nt;
        x0[i] = x1[i] = ar0[i] = ar1[i] = 0.f;
        if (kp < sh.d_r / 2) {
            x0[i] = to_f<T>(kr[2 * kp]);
            x1[i] = to_f<T>(kr[2 * kp + 1]);
            ar0[i] = acc[sh.d_c + 2 * kp];
            ar1[i] = acc[sh.d_c + 2 * kp + 1];
        }
    }
    if (t < 0 || t >= (int64_t)sh.max_slots * sh.s) {
        if (threadIdx.x == 0) latch_status(a.status, kStatusCapacity);
        return false;
    }
    T* row = (T*)a.cache + ((size_t)b * sh.max_slots + (size_t)(t / sh.s)) * sh.D;
    const bool fresh = (t % sh.s) == 0;           // a new slot opens: the accumulator restarts
    const int r = (int)(t % sh.s);
    if (fresh) {
#pragma unroll
        for (int i = 0; i < kMaxPer; ++i) a0[i] = a1[i] = 0.f;
#pragma unroll
        for (int i = 0; i < kMaxPairs; ++i) ar0[i] = ar1[i] = 0.f;
    }
    // RoPE of the key at position t (independent of the gate)
    float y0[kMaxPairs], y1[kMaxPairs];
#pragma unroll
    for (int i = 0; i < kMaxPairs; ++i) {
        const int kp = tid + i * nt;
        y0[i] = y1[i] = 0.f;
        if (kp < sh.d_r / 2) {
            float sn, cs;
            pair_sincos_f(t, f.rope[i], &sn, &cs);
            y0[i] = x0[i] * cs - x1[i] * sn;
            y1[i] = x0[i] * sn + x1[i] * cs;
        }
    }
    // gate (Eq. 13): w = sigmoid(G[t mod s] . (c_t * PE_t) + g[t mod s]), or
    // one weight per slot channel (modes 3, 4)
    const bool channel = sh.gate_mode >= 3;
    float w = 1.f;
    if (channel) {
        channel_gate<kMaxPer>(a, b, t, gate_w, f, c0, c1, vch, wch);
    } else if (sh.gate_mode == 2) {
        w = 1.f;
    } else if (sh.gate_mode == 1) {
        w = a.gate_in[b];
    } else {
        float g0[kMaxPer], g1[kMaxPer];
#pragma unroll
        for (int i = 0; i < kMaxPer; ++i) {
            const int kp = tid + i * nt;
            g0[i] = g1[i] = 0.f;
            if (kp < sh.d_c / 2) {
                g0[i] = gate_w[(size_t)r * sh.d_c + 2 * kp];
                g1[i] = gate_w[(size_t)r * sh.d_c + 2 * kp + 1];
            }
        }
        float z = 0.f;
#pragma unroll
        for (int i = 0; i < kMaxPer; ++i) {
            const int kp = tid + i * nt;
            if (kp < sh.d_c / 2) {
                float sn, cs;
                pair_sincos_f(t, f.pe[i], &sn, &cs);   // PE_t[2kp], PE_t[2kp+1]
                z = fmaf(g0[i] * c0[i], sn, z);
                z = fmaf(g1[i] * c1[i], cs, z);
            }
        }
        z = block_sum(z, red) + a.gate_b[r];
        w = sigmoidf_(z);
    }
    // in-place update of the open slot; its bf16 rounding is the cache row
#pragma unroll
    for (int i = 0; i < kMaxPer; ++i) {
        const int kp = tid + i * nt;
        if (kp < sh.d_c / 2) {
            const float w0 = channel ? wch[2 * kp] : w, w1 = channel ? wch[2 * kp + 1] : w;
            const float v0 = a0[i] + w0 * c0[i], v1 = a1[i] + w1 * c1[i];
            acc[2 * kp] = v0;
            acc[2 * kp + 1] = v1;
            row[2 * kp] = from_f<T>(v0);
            row[2 * kp + 1] = from_f<T>(v1);
        }
    }
#pragma unroll
    for (int i = 0; i < kMaxPairs; ++i) {
        const int kp = tid + i * nt;
        if (kp < sh.d_r / 2) {
            const float w0 = channel ? wch[sh.d_c + 2 * kp] : w, w1 = channel ? wch[sh.d_c + 2 * kp + 1] : w;
            const float v0 = ar0[i] + w0 * y0[i], v1 = ar1[i] + w1 * y1[i];
            acc[sh.d_c + 2 * kp] = v0;
            acc[sh.d_c + 2 * kp + 1] = v1;
            row[sh.d_c + 2 * kp] = from_f<T>(v0);
            row[sh.d_c + 2 * kp + 1] = from_f<T>(v1);
        }
    }
    return true;
}

template <typename T>
__device__ bool decode_update_body(const DecodeArgs& a, int b) {
    UpdateFreqs f;
    update_freqs(a.sh, f);
    return decode_update_body<T>(a, b, a.gate_w, f);
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
        for (int i0 = 0; i0 < sh.d_h; i0 += 16) {      // d_h is a multiple of 16
            float wv[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) wv[u] = to_f<T>(W[(size_t)(i0 + u) * sh.d_c + j]);
#pragma unroll
            for (int u = 0; u < 16; ++u) acc = fmaf(wv[u], q[i0 + u], acc);
        }
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

// Prefill absorption: grid (B*T, H); row = b*T + t, position t0 + t.
template <typename T>
__global__ void __launch_bounds__(128) k_prefill_absorb(Shape sh, const T* qc, const T* qr, const T* w_uk,
                                                        int T_len, int t0, float* qt) {
    const int64_t row = blockIdx.x;
    absorb_query_body<T>(sh, qc, qr, w_uk, row, blockIdx.y, t0 + row % T_len, qt);
}

// 8 consecutive values as float (T = float or bf16; 16-byte aligned address).
template <typename T> __device__ __forceinline__ void load8(const T* p, float* v);
template <> __device__ __forceinline__ void load8<float>(const float* p, float* v) {
    const float4 a = *(const float4*)p, c = *(const float4*)(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = c.x; v[5] = c.y; v[6] = c.z; v[7] = c.w;
}
template <> __device__ __forceinline__ void load8<bf16>(const bf16* p, float* v) {
    const uint4 raw = *(const uint4*)p;
    const bf16* h = (const bf16*)&raw;
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __bfloat162float(h[i]);
}
template <> __device__ __forceinline__ void load8<f16>(const f16* p, float* v) {
    const uint4 raw = *(const uint4*)p;
    const f16* h = (const f16*)&raw;
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __half2float(h[i]);
}
template <typename T> __device__ __forceinline__ void store8(T* p, const float* v);
template <> __device__ __forceinline__ void store8<f16>(f16* p, const float* v) {
    uint4 raw;
    f16* h = (f16*)&raw;
#pragma unroll
    for (int i = 0; i < 8; ++i) h[i] = __float2half_rn(v[i]);
    *(uint4*)p = raw;
}
template <> __device__ __forceinline__ void store8<float>(float* p, const float* v) {
    *(float4*)p = make_float4(v[0], v[1], v[2], v[3]);
    *(float4*)(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}
template <> __device__ __forceinline__ void store8<bf16>(bf16* p, const float* v) {
    uint4 raw;
    raw.x = pack_bf16x2(v[0], v[1]);
    raw.y = pack_bf16x2(v[2], v[3]);
    raw.z = pack_bf16x2(v[4], v[5]);
    raw.w = pack_bf16x2(v[6], v[7]);
    *(uint4*)p = raw;
}

// Block-prefix scan (MTLA Sec. 4.2): for slot j of sequence b, the merging
// weights w_u (Sec. 4.1, Eq. 13) of its tokens u and the partial slots
//   P_u = sum_{v = s*j}^{u} w_v [c_v ; RoPE_v(k_v)]
// (stored as PT), the slot itself in the cache (rounded to T: finished, or the
// last one) and, for the slot holding the last token, the unrounded open slot.
// The tokens are t0 .. t0+T-1 (absolute positions; inputs, P and the (cos,
// sin) table are indexed from t0): the slots are floor(t0/s) .. and the one
// open at t0, if t0 is not a multiple of s, starts from open_slot_in (the
// accumulator after t0 tokens) instead of 0.
// One warp per slot: grid (ceil(n / 8), B), n = slots touched, 256 threads.
// With 16-bit partial slots (the tensor-core prefill) the sine and cosine of the
// angle, reduced to [-pi, pi] in double as everywhere, come from the special-
// function unit (absolute error about 2^-21 there, far below the bf16 rounding
// of the slots); the fp32 partial slots of the CUDA-core path keep sincosf.
template <typename T, typename PT>
__global__ void __launch_bounds__(256) k_prefill_scan(PrefillArgs a, PT* P, float2* rope_tab = nullptr,
                                                      float* w_out = nullptr) {
    constexpr bool kFastSinCos = !std::is_same<PT, float>::value;
    auto sincos_at = [](int64_t t, double inv_freq, float* sn, float* cs) {
        if constexpr (kFastSinCos) {
            double ang = (double)t * inv_freq;
            ang = fma(-6.283185307179586476925, rint(ang * 0.15915494309189533577), ang);
            __sincosf((float)ang, sn, cs);
        } else {
            pair_sincos_f(t, inv_freq, sn, cs);
        }
    };
    const Shape sh = a.sh;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.y;
    const int Tn = a.T;
    __shared__ double pe_freq[256];     // PE frequencies, d_c / 2 <= 256
    __shared__ double rope_freq[288];   // RoPE frequencies, d_r / 2 <= 280
    for (int k = threadIdx.x; k < sh.d_c / 2; k += blockDim.x)
        pe_freq[k] = exp2(-(2.0 * k / (double)sh.d_c) * sh.log2_pe_base);
    for (int k = threadIdx.x; k < sh.d_r / 2; k += blockDim.x)
        rope_freq[k] = exp2(-(2.0 * k / (double)sh.d_r) * sh.log2_rope_base);
    __syncthreads();
    const int t0 = a.t0;
    const int j_first = t0 / sh.s, j_end = (t0 + Tn - 1) / sh.s + 1;
    const int j = j_first + blockIdx.x * 8 + warp;
    if (j >= j_end) return;
    // this slot's new tokens: absolute positions ua .. ua + nu - 1, local index lu0 ..
    const int ua = max(j * sh.s, t0), nu = min((j + 1) * sh.s, t0 + Tn) - ua;
    const int lu0 = ua - t0;
    const float* seed = (j * sh.s < t0 && a.open_slot_in) ? a.open_slot_in + (size_t)b * sh.D : nullptr;
    const T* c = (const T*)a.c + ((size_t)b * Tn + lu0) * sh.d_c;
    const T* kr = (const T*)a.kr + ((size_t)b * Tn + lu0) * sh.d_r;
    float wv[8];
#pragma unroll
    for (int uo = 0; uo < 8; ++uo) {
        wv[uo] = 0.f;
        if (uo >= nu) continue;
        const int u = ua + uo;
        if (sh.gate_mode == 2) {
            wv[uo] = 1.f;
        } else if (sh.gate_mode == 1) {
            wv[uo] = a.gate_in[(size_t)b * Tn + lu0 + uo];
        } else {
            const int r = u % sh.s;
            const float* G = a.gate_w + (size_t)r * sh.d_c;
            const T* cu = c + (size_t)uo * sh.d_c;
            float z = 0.f;
            for (int k = lane; k < sh.d_c / 2; k += 32) {
                float sn, cs;
                sincos_at(u, pe_freq[k], &sn, &cs);
                z = fmaf(G[2 * k] * to_f<T>(cu[2 * k]), sn, z);
                z = fmaf(G[2 * k + 1] * to_f<T>(cu[2 * k + 1]), cs, z);
            }
            wv[uo] = sigmoidf_(warp_sum(z) + a.gate_b[r]);
        }
        if (w_out && lane == 0) w_out[(size_t)b * Tn + lu0 + uo] = wv[uo];   // the weights, for the backward
    }
    T* slot = (T*)a.cache_out + ((size_t)b * sh.max_slots + j) * sh.D;
    float* open = (ua + nu == t0 + Tn && a.open_slot_out) ? a.open_slot_out + (size_t)b * sh.D : nullptr;
    PT* Pj = P + ((size_t)b * Tn + lu0) * sh.D;
    for (int k0 = lane * 8; k0 < sh.d_c; k0 += 256) {
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (seed) load8<float>(seed + k0, acc);
#pragma unroll
        for (int uo = 0; uo < 8; ++uo) {
            if (uo >= nu) continue;
            float x[8];
            load8<T>(c + (size_t)uo * sh.d_c + k0, x);
#pragma unroll
            for (int v = 0; v < 8; ++v) acc[v] = fmaf(wv[uo], x[v], acc[v]);
            store8<PT>(Pj + (size_t)uo * sh.D + k0, acc);
        }
        store8<T>(slot + k0, acc);
        if (open) store8<float>(open + k0, acc);
    }
    for (int k = lane; k < sh.d_r / 2; k += 32) {
        float a0 = seed ? seed[sh.d_c + 2 * k] : 0.f, a1 = seed ? seed[sh.d_c + 2 * k + 1] : 0.f;
#pragma unroll
        for (int uo = 0; uo < 8; ++uo) {
            if (uo >= nu) continue;
            float sn, cs;
            sincos_at(ua + uo, rope_freq[k], &sn, &cs);
            // (cos, sin) of every position for the queries' RoPE (sequence 0 writes it)
            if (rope_tab && b == 0) rope_tab[(size_t)(lu0 + uo) * (sh.d_r / 2) + k] = make_float2(cs, sn);
            const float x0 = to_f<T>(kr[(size_t)uo * sh.d_r + 2 * k]);
            const float x1 = to_f<T>(kr[(size_t)uo * sh.d_r + 2 * k + 1]);
            a0 = fmaf(wv[uo], x0 * cs - x1 * sn, a0);
            a1 = fmaf(wv[uo], x0 * sn + x1 * cs, a1);
            PT* pr = Pj + (size_t)uo * sh.D + sh.d_c;
            pr[2 * k] = from_f<PT>(a0);
            pr[2 * k + 1] = from_f<PT>(a1);
        }
        slot[sh.d_c + 2 * k] = from_f<T>(a0);
        slot[sh.d_c + 2 * k + 1] = from_f<T>(a1);
        if (open) {
            open[sh.d_c + 2 * k] = a0;
            open[sh.d_c + 2 * k + 1] = a1;
        }
    }
}

// The block-prefix scan with per-channel gates (modes 3 and 4): the same
// outputs as k_prefill_scan (partial slots P, the slots in the cache, the open
// slot, the (cos, sin) table), with every slot channel k of token u weighted by
// its own w_u[k]. One warp per slot, tokens in order: the warp stages c_u * PE_u
// and then the D weights of token u in shared memory (lane k: channels
// k, k+32, ..., G read along k), and each lane carries its channels' sums.
template <typename T, typename PT>
__global__ void __launch_bounds__(256) k_prefill_scan_channel(PrefillArgs a, PT* P, float2* rope_tab = nullptr) {
    const Shape sh = a.sh;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.y;
    const int Tn = a.T;
    __shared__ double pe_freq[256];
    __shared__ double rope_freq[64];
    __shared__ float vsh[8][512];
    __shared__ float wsh[8][576];
    for (int k = threadIdx.x; k < sh.d_c / 2; k += blockDim.x)
        pe_freq[k] = exp2(-(2.0 * k / (double)sh.d_c) * sh.log2_pe_base);
    for (int k = threadIdx.x; k < sh.d_r / 2; k += blockDim.x)
        rope_freq[k] = exp2(-(2.0 * k / (double)sh.d_r) * sh.log2_rope_base);
    __syncthreads();
    const int t0 = a.t0;
    const int j = t0 / sh.s + blockIdx.x * 8 + warp;
    if (j >= (t0 + Tn - 1) / sh.s + 1) return;
    const int ua = max(j * sh.s, t0), nu = min((j + 1) * sh.s, t0 + Tn) - ua;
    const int lu0 = ua - t0;
    const float* seed = (j * sh.s < t0 && a.open_slot_in) ? a.open_slot_in + (size_t)b * sh.D : nullptr;
    // this lane's channels: latent k0 = 8 lane + 256 q (q < 2), RoPE pairs lane + 32 q (q < 2)
    float al[2][8], ar[2][2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const int k0 = lane * 8 + 256 * q;
#pragma unroll
        for (int v = 0; v < 8; ++v) al[q][v] = (seed && k0 < sh.d_c) ? seed[k0 + v] : 0.f;
        const int kp = lane + 32 * q;
        ar[q][0] = (seed && kp < sh.d_r / 2) ? seed[sh.d_c + 2 * kp] : 0.f;
        ar[q][1] = (seed && kp < sh.d_r / 2) ? seed[sh.d_c + 2 * kp + 1] : 0.f;
    }
    float* vs = vsh[warp];
    float* ws = wsh[warp];
    for (int uo = 0; uo < nu; ++uo) {
        const int u = ua + uo, lu = lu0 + uo;
        const T* cu = (const T*)a.c + ((size_t)b * Tn + lu) * sh.d_c;
        const T* ku = (const T*)a.kr + ((size_t)b * Tn + lu) * sh.d_r;
        if (sh.gate_mode == 4) {
            for (int k = lane; k < sh.D; k += 32) ws[k] = a.gate_in[((size_t)b * Tn + lu) * sh.D + k];
        } else {
            const int r = u % sh.s;
            for (int kp = lane; kp < sh.d_c / 2; kp += 32) {
                float sn, cs;
                pair_sincos_f(u, pe_freq[kp], &sn, &cs);
                vs[2 * kp] = to_f<T>(cu[2 * kp]) * sn;
                vs[2 * kp + 1] = to_f<T>(cu[2 * kp + 1]) * cs;
            }
            __syncwarp();
            const float* G = a.gate_w + (size_t)r * sh.d_c * sh.D;
            for (int k = lane; k < sh.D; k += 32) {
                float z = a.gate_b[(size_t)r * sh.D + k];
                for (int i = 0; i < sh.d_c; ++i) z = fmaf(vs[i], G[(size_t)i * sh.D + k], z);
                ws[k] = sigmoidf_(z);
            }
        }
        __syncwarp();
        PT* Pu = P + ((size_t)b * Tn + lu) * sh.D;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int k0 = lane * 8 + 256 * q;
            if (k0 < sh.d_c) {
                float x[8];
                load8<T>(cu + k0, x);
#pragma unroll
                for (int v = 0; v < 8; ++v) al[q][v] = fmaf(ws[k0 + v], x[v], al[q][v]);
                store8<PT>(Pu + k0, al[q]);
            }
            const int kp = lane + 32 * q;
            if (kp < sh.d_r / 2) {
                float sn, cs;
                pair_sincos_f(u, rope_freq[kp], &sn, &cs);
                if (rope_tab && b == 0) rope_tab[(size_t)lu * (sh.d_r / 2) + kp] = make_float2(cs, sn);
                const float x0 = to_f<T>(ku[2 * kp]), x1 = to_f<T>(ku[2 * kp + 1]);
                ar[q][0] = fmaf(ws[sh.d_c + 2 * kp], x0 * cs - x1 * sn, ar[q][0]);
                ar[q][1] = fmaf(ws[sh.d_c + 2 * kp + 1], x0 * sn + x1 * cs, ar[q][1]);
                Pu[sh.d_c + 2 * kp] = from_f<PT>(ar[q][0]);
                Pu[sh.d_c + 2 * kp + 1] = from_f<PT>(ar[q][1]);
            }
        }
        __syncwarp();                    // vs / ws of this token are read
    }
    T* slot = (T*)a.cache_out + ((size_t)b * sh.max_slots + j) * sh.D;
    float* open = (ua + nu == t0 + Tn && a.open_slot_out) ? a.open_slot_out + (size_t)b * sh.D : nullptr;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        const int k0 = lane * 8 + 256 * q;
        if (k0 < sh.d_c) {
            store8<T>(slot + k0, al[q]);
            if (open) store8<float>(open + k0, al[q]);
        }
        const int kp = lane + 32 * q;
        if (kp < sh.d_r / 2) {
            slot[sh.d_c + 2 * kp] = from_f<T>(ar[q][0]);
            slot[sh.d_c + 2 * kp + 1] = from_f<T>(ar[q][1]);
            if (open) {
                open[sh.d_c + 2 * kp] = ar[q][0];
                open[sh.d_c + 2 * kp + 1] = ar[q][1];
            }
        }
    }
}

}  // namespace mtla
