// simt_kernels.cu -- CUDA-core kernels of the MTLA decode step and prefill.
//
// These are the fp32 path (every product and sum in true fp32 FMA; tensor
// cores would round operands to tf32) and the reference shape of the work the
// tensor-core kernels do for bf16. Steps, in the order of "Multi-head Temporal
// Latent Attention", Method:
//   gate w_t (Sec. 4.1, Eq. 13) -> RoPE of the decoupled key (Sec. 4.3) ->
//   merge into the slot being filled (in place at decode; block-prefix scan at
//   prefill, Sec. 4.2) -> absorbed query [W_UK^T qC ; RoPE(qR)] -> softmax over
//   the finished slots plus the own partial slot -> W_UV on the weighted latent.
#include "common.cuh"
#include "mtla_internal.h"
#include "prep.cuh"

namespace mtla {

namespace {

constexpr int kMaxD = 576;              // d_c + d_r
constexpr int kMaxPerLane = kMaxD / 32; // 18
constexpr int kMaxLatPerLane = 512 / 32;

// Online-softmax state of one (query, head) row held by a warp: lane l owns
// latent entries l, l+32, ...
struct RowState {
    float m, l;
    float o[kMaxLatPerLane];
};

template <typename K>
__device__ __forceinline__ void row_visit(RowState& st, const float* q, const K* key, int D,
                                          int d_c, float scale) {
    const int lane = threadIdx.x & 31;
    float x[kMaxPerLane];
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
        const int idx = lane + 32 * i;
        float v = 0.f;
        if (idx < D) v = to_f<K>(key[idx]);
        x[i] = v;
        dot = fmaf(q[i], v, dot);
    }
    dot = warp_sum(dot) * scale;
    const float m_new = fmaxf(st.m, dot);
    const float corr = (st.m == -INFINITY) ? 0.f : expf(st.m - m_new);
    const float p = expf(dot - m_new);
    st.l = st.l * corr + p;
#pragma unroll
    for (int i = 0; i < kMaxLatPerLane; ++i) {
        const int idx = lane + 32 * i;
        if (idx < d_c) st.o[i] = st.o[i] * corr + p * x[i];
    }
    st.m = m_new;
}

// Split-K attention: block (split, b) covers slots [split*chunk, ...) of the
// n = floor(t/s)+1 slots of sequence b for all heads; writes (o, m, l).
template <typename T>
__global__ void __launch_bounds__(256) k_decode_attn(DecodeArgs a, int chunk, int splits,
                                                     const float* qt, float* part) {
    const Shape sh = a.sh;
    const int split = blockIdx.x, b = blockIdx.y;
    const int64_t t = a.pos[b];
    if (t < 0 || t >= (int64_t)sh.max_slots * sh.s) return;
    const int64_t n = t / sh.s + 1;
    const int64_t j0 = (int64_t)split * chunk;
    const int64_t j1 = min(n, j0 + chunk);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const T* cache = (const T*)a.cache + (size_t)b * sh.max_slots * sh.D;
    for (int h = warp; h < sh.H; h += 8) {
        float q[kMaxPerLane];
        const float* qrow = qt + ((size_t)b * sh.H + h) * sh.D;
#pragma unroll
        for (int i = 0; i < kMaxPerLane; ++i) {
            const int idx = lane + 32 * i;
            q[i] = idx < sh.D ? qrow[idx] : 0.f;
        }
        RowState st;
        st.m = -INFINITY;
        st.l = 0.f;
#pragma unroll
        for (int i = 0; i < kMaxLatPerLane; ++i) st.o[i] = 0.f;
        for (int64_t j = j0; j < j1; ++j)
            row_visit<T>(st, q, cache + (size_t)j * sh.D, sh.D, sh.d_c, sh.scale);
        float* dst = part + (((size_t)b * splits + split) * sh.H + h) * (sh.d_c + 2);
#pragma unroll
        for (int i = 0; i < kMaxLatPerLane; ++i) {
            const int idx = lane + 32 * i;
            if (idx < sh.d_c) dst[idx] = st.o[i];
        }
        if (lane == 0) {
            dst[sh.d_c] = st.m;
            dst[sh.d_c + 1] = st.l;
        }
    }
}

// Merge the splits of (b, h) and apply W_UV. grid (H, B).
template <typename T>
__global__ void __launch_bounds__(256) k_decode_combine(DecodeArgs a, int chunk, int splits,
                                                        const float* part) {
    const Shape sh = a.sh;
    const int h = blockIdx.x, b = blockIdx.y;
    const int64_t t = a.pos[b];
    if (t < 0 || t >= (int64_t)sh.max_slots * sh.s) return;
    const int64_t n = t / sh.s + 1;
    const int used = (int)((n + chunk - 1) / chunk);
    __shared__ float wts[64];
    __shared__ float olat[512];
    __shared__ float inv_l;
    const float* base = part + ((size_t)b * splits * sh.H + h) * (sh.d_c + 2);
    const size_t sstride = (size_t)sh.H * (sh.d_c + 2);
    if (threadIdx.x == 0) {
        float M = -INFINITY;
        for (int k = 0; k < used; ++k) M = fmaxf(M, base[k * sstride + sh.d_c]);
        float L = 0.f;
        for (int k = 0; k < used; ++k) {
            const float mk = base[k * sstride + sh.d_c];
            const float wk = (mk == -INFINITY) ? 0.f : expf(mk - M);
            wts[k] = wk;
            L += wk * base[k * sstride + sh.d_c + 1];
        }
        inv_l = 1.f / L;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < sh.d_c; j += blockDim.x) {
        float acc = 0.f;
        for (int k = 0; k < used; ++k) acc = fmaf(wts[k], base[k * sstride + j], acc);
        olat[j] = acc * inv_l;
    }
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const T* W = (const T*)a.w_uv + (size_t)h * sh.d_h * sh.d_c;
    T* out = (T*)a.out + ((size_t)b * sh.H + h) * sh.d_h;
    for (int i = warp; i < sh.d_h; i += 8) {
        float acc = 0.f;
        for (int j = lane; j < sh.d_c; j += 32) acc = fmaf(to_f<T>(W[(size_t)i * sh.d_c + j]), olat[j], acc);
        acc = warp_sum(acc);
        if (lane == 0) out[i] = from_f<T>(acc);
    }
}

// ----------------------------------------------------------------- prefill

// Masked attention: one warp per (t, h) row; keys are the finished slots
// j < floor(t/s) (rounded cache) plus the own partial slot P_t (rounded).
template <typename T>
__global__ void __launch_bounds__(256) k_prefill_attn(PrefillArgs a, const float* P, const float* qt) {
    const Shape sh = a.sh;
    const int b = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t row = (int64_t)blockIdx.x * 8 + warp;
    if (row >= (int64_t)a.T * sh.H) return;
    const int t = (int)(row / sh.H), h = (int)(row % sh.H);
    const float* qrow = qt + (((size_t)b * a.T + t) * sh.H + h) * sh.D;
    float q[kMaxPerLane];
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
        const int idx = lane + 32 * i;
        q[i] = idx < sh.D ? qrow[idx] : 0.f;
    }
    RowState st;
    st.m = -INFINITY;
    st.l = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxLatPerLane; ++i) st.o[i] = 0.f;
    const T* cache = (const T*)a.cache_out + (size_t)b * sh.max_slots * sh.D;
    const int nf = (a.t0 + t) / sh.s;          // finished slots: the cache's and this chunk's
    for (int j = 0; j < nf; ++j) row_visit<T>(st, q, cache + (size_t)j * sh.D, sh.D, sh.d_c, sh.scale);
    {
        // own partial slot, rounded to the storage type
        const float* pp = P + ((size_t)b * a.T + t) * sh.D;
        float x[kMaxPerLane];
        float dot = 0.f;
#pragma unroll
        for (int i = 0; i < kMaxPerLane; ++i) {
            const int idx = lane + 32 * i;
            float v = 0.f;
            if (idx < sh.D) v = round_to<T>(pp[idx]);
            x[i] = v;
            dot = fmaf(q[i], v, dot);
        }
        dot = warp_sum(dot) * sh.scale;
        const float m_new = fmaxf(st.m, dot);
        const float corr = (st.m == -INFINITY) ? 0.f : expf(st.m - m_new);
        const float p = expf(dot - m_new);
        st.l = st.l * corr + p;
#pragma unroll
        for (int i = 0; i < kMaxLatPerLane; ++i) {
            const int idx = lane + 32 * i;
            if (idx < sh.d_c) st.o[i] = st.o[i] * corr + p * x[i];
        }
        st.m = m_new;
    }
    const float inv_l = 1.f / st.l;
    const T* W = (const T*)a.w_uv + (size_t)h * sh.d_h * sh.d_c;
    T* out = (T*)a.out + (((size_t)b * a.T + t) * sh.H + h) * sh.d_h;
    for (int i = 0; i < sh.d_h; ++i) {
        float acc = 0.f;
#pragma unroll
        for (int k = 0; k < kMaxLatPerLane; ++k) {
            const int idx = lane + 32 * k;
            if (idx < sh.d_c) acc = fmaf(to_f<T>(W[(size_t)i * sh.d_c + idx]), st.o[k], acc);
        }
        acc = warp_sum(acc);
        if (lane == 0) out[i] = from_f<T>(acc * inv_l);
    }
}

void decode_plan(const Shape& sh, int* splits, int* chunk) {
    int sp = (sh.max_slots + 63) / 64;
    if (sp < 1) sp = 1;
    if (sp > 32) sp = 32;
    *splits = sp;
    *chunk = (sh.max_slots + sp - 1) / sp;
}

template <typename T>
cudaError_t decode_impl(const DecodeArgs& a, cudaStream_t st, uint64_t* launches) {
    const Shape& sh = a.sh;
    int splits, chunk;
    decode_plan(sh, &splits, &chunk);
    char* ws = (char*)a.workspace;
    float* qt = (float*)ws;
    float* part = (float*)(ws + align256((size_t)sh.B * sh.H * sh.D * sizeof(float)));
    k_decode_prep<T><<<dim3(sh.B, sh.H + 1), 128, 0, st>>>(a, qt);
    profile_begin(st);
    k_decode_attn<T><<<dim3(splits, sh.B), 256, 0, st>>>(a, chunk, splits, qt, part);
    profile_end(st);
    k_decode_combine<T><<<dim3(sh.H, sh.B), 256, 0, st>>>(a, chunk, splits, part);
    *launches += 3;
    return cudaGetLastError();
}

template <typename T>
cudaError_t prefill_impl(const PrefillArgs& a_in, cudaStream_t st, uint64_t* launches) {
    PrefillArgs a = a_in;
    const Shape& sh = a.sh;
    char* ws = (char*)a.workspace;
    float* P = (float*)ws;
    const size_t p_bytes = align256((size_t)sh.B * a.T * sh.D * sizeof(float));
    float* qt = (float*)(ws + p_bytes);
    cudaError_t e = prefill_seed(a, ws + p_bytes + align256((size_t)sh.B * a.T * sh.H * sh.D * sizeof(float)), st);
    if (e != cudaSuccess) return e;
    const int n_slots = (a.t0 + a.T - 1) / sh.s - a.t0 / sh.s + 1;    // slots the chunk touches
    if (sh.gate_mode >= 3)
        k_prefill_scan_channel<T, float><<<dim3((n_slots + 7) / 8, sh.B), 256, 0, st>>>(a, P);
    else
        k_prefill_scan<T, float><<<dim3((n_slots + 7) / 8, sh.B), 256, 0, st>>>(a, P);
    k_prefill_absorb<T><<<dim3(sh.B * a.T, sh.H), 128, 0, st>>>(sh, (const T*)a.q_c, (const T*)a.q_r,
                                                                 (const T*)a.w_uk, a.T, a.t0, qt);
    const int64_t rows = (int64_t)a.T * sh.H;
    profile_begin(st);
    k_prefill_attn<T><<<dim3((unsigned)((rows + 7) / 8), sh.B), 256, 0, st>>>(a, P, qt);
    profile_end(st);
    *launches += 3;
    return cudaGetLastError();
}

}  // namespace

size_t simt_decode_workspace(const Shape& sh) {
    int splits, chunk;
    decode_plan(sh, &splits, &chunk);
    return align256((size_t)sh.B * sh.H * sh.D * sizeof(float)) +
           align256((size_t)sh.B * splits * sh.H * (sh.d_c + 2) * sizeof(float));
}

size_t simt_prefill_workspace(const Shape& sh, int T) {
    return align256((size_t)sh.B * T * sh.D * sizeof(float)) +
           align256((size_t)sh.B * T * sh.H * sh.D * sizeof(float)) + prefill_seed_bytes(sh);
}

cudaError_t simt_decode(const DecodeArgs& a, int dtype, cudaStream_t st, uint64_t* launches) {
    if (dtype == kDtypeF32) return decode_impl<float>(a, st, launches);
    if (dtype == kDtypeF16) return decode_impl<f16>(a, st, launches);
    return decode_impl<bf16>(a, st, launches);
}

cudaError_t simt_prefill(const PrefillArgs& a, int dtype, cudaStream_t st, uint64_t* launches) {
    if (dtype == kDtypeF32) return prefill_impl<float>(a, st, launches);
    if (dtype == kDtypeF16) return prefill_impl<f16>(a, st, launches);
    return prefill_impl<bf16>(a, st, launches);
}

}  // namespace mtla
