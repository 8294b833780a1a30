// backward.cu -- training backward of the parallel (prefill) forward from
// position 0 ("Multi-head Temporal Latent Attention", Results: the models are
// trained from scratch; Key claims: the stride-aware mask lets the parallel
// training pass match incremental decoding). Two paths behind one entry:
// bf16 at the tensor-core prefill's widths runs the masked attention's
// gradients on the tensor cores (tc_backward.cu) around the CUDA-core kernels
// here; every other shape and storage type runs the CUDA-core path below,
// in fp32 arithmetic.
//
// Forward, per sequence: x_u = [c_u ; R_u k_u], P_t = sum_{u in block(t), u <= t}
// w_u x_u (w_u the merging weight of Eq. 13); query i of head h attends the
// finished slots F_j = P_{js+s-1}, j < floor(i/s), and its own partial P_i with
// the absorbed query qt = [W_UK[h]^T qC ; R_i qR] and scale; a_ij the softmax
// weights, obar = sum_j a_ij key_j[0:d_c], out = W_UV[h] obar.
// Backward from dout (the gradient of the loss with respect to out):
//   dobar = W_UV[h]^T dout, delta = dobar . obar,
//   de_ij = a_ij (dobar . key_j[0:d_c] - delta),
//   dqt = scale sum_j de_ij key_j, dkey_j += scale de_ij qt + a_ij [dobar ; 0],
//   dqC = W_UK[h] dqt[0:d_c], dqR = R_i^T dqt[d_c:],
//   dW_UK[h] += qC dqt[0:d_c]^T, dW_UV[h] += dout obar^T,
//   through the scan: S_u = sum over t >= u in u's block of dP_t (dP_t the
//   gradient of P_t, from its roles as an own partial and as a finished slot),
//   dx_u = w_u S_u, dw_u = x_u . S_u; dc_u = dx_u[0:d_c], dk_u = R_u^T dx_u[d_c:];
//   the gate: dz = dw w (1 - w), dG[r] += dz (c_u * PE_u), dg[r] += dz,
//   dc_u += dz (G[r] * PE_u), r = u mod s; a supplied gate gets dgate_in = dw.
// CUDA-core path, kernels in launch order:
//   k_prefill_scan    the forward scan (P in fp32, the weights w)
//   k_prefill_absorb  the absorbed queries qt (fp32)
//   k_bwd_rows        block (i, b), a warp per head: the row's softmax (two
//                     passes over its keys), dobar, delta, dqt and the own
//                     partial's key gradient summed over the heads (in a
//                     fixed order: dP, dF and what follows from them are
//                     the same bytes on every call)
//   k_bwd_columns     block (j, b), a warp per head: the finished slot F_j's
//                     key gradient over every query that sees it
//   k_bwd_query       dqC, dqR
//   k_bwd_wpart/wsum  dW_UK, dW_UV (per row chunk, then the chunks in order)
//   k_bwd_scan        a warp per slot: the scan and gate backward
// Tensor-core path (backward_tc): the forward on the tensor cores keeping each
// row's log-sum-exp, O / l and absorbed query; dobar and U (GEMMs), delta
// (k_bwd_delta); the finished-slot gradients (k_bwd_dq_tc, k_bwd_dk_tc); the
// own-partial term with dqR (k_bwd_own); dqC (GEMM); dW_UK and dW_UV as two
// products on the tensor cores (k_wgrad_tc, tc_wgrad.cu) summed over row chunks
// in order (k_bwd_wsum); k_bwd_scan as above, the heads' dF summed in a fixed
// order.
#include <type_traits>

#include "common.cuh"
#include "mtla_internal.h"
#include "prep.cuh"

namespace mtla {

namespace {

constexpr int kMaxD = 576;             // slot width the kernels hold (d_c + d_R)
constexpr int kPer = kMaxD / 32;       // a lane's channels: lane + 32 k
constexpr int kWChunk = 1024;          // token rows per block of k_bwd_wpart

struct BwdArgs {
    Shape sh;
    int T, n_slots;
    const void* qc;        // [B,T,H,d_h]
    const void* w_uk;      // [H,d_h,d_c]
    const void* w_uv;      // [H,d_h,d_c]
    const void* dout;      // [B,T,H,d_h]
    const float* P;        // [B,T,D] partial slots
    const float* qt;       // [B,T,H,D] absorbed queries
    const float* w;        // [B,T] merging weights
    float* mrow;           // [B,T,H] scaled row maximum
    float* lrow;           // [B,T,H] row sum
    float* delta;          // [B,T,H]
    float* dob;            // [B,T,H,d_c] dobar
    void* obar;            // [B,T,H,d_c] fp32 (CUDA-core path) or bf16 (tensor-core path)
    float* dqt;            // [B,T,H,D]
    float* dP;             // [B,T,D] own-partial key gradients
    float* dF;             // [n_parts][B,n_slots,D] finished-slot key gradients (summed over parts)
    int n_parts;
};

template <typename T> __device__ __forceinline__ float ldf(const void* p, size_t i) {
    return to_f<T>(((const T*)p)[i]);
}

// Row pass. Keys of query i: finished slots 0 .. nf-1 (nf = floor(i/s)), then
// the own partial P_i.
template <typename T>
__global__ void __launch_bounds__(256) k_bwd_rows(BwdArgs a) {
    const Shape sh = a.sh;
    const int i = blockIdx.x, b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const int D = sh.D, d_c = sh.d_c, s = sh.s;
    __shared__ float dkey_own[8][kMaxD];   // a warp's heads, summed in a fixed order below
    float* own = dkey_own[warp];
    for (int q = lane; q < D; q += 32) own[q] = 0.f;
    const float* Pb = a.P + (size_t)b * a.T * D;
    const int nf = i / s;
    for (int h = warp; h < sh.H; h += nw) {
        const size_t row = ((size_t)b * a.T + i) * sh.H + h;
        float qv[kPer], dv[kPer], ob[kPer], dq[kPer];
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            const int c = lane + 32 * k;
            qv[k] = c < D ? a.qt[row * D + c] : 0.f;
            float acc = 0.f;
            if (c < d_c)
                for (int r = 0; r < sh.d_h; ++r)
                    acc = fmaf(ldf<T>(a.w_uv, ((size_t)h * sh.d_h + r) * d_c + c), ldf<T>(a.dout, row * sh.d_h + r),
                               acc);
            dv[k] = acc;   // dobar = W_UV[h]^T dout (0 past d_c)
            ob[k] = 0.f;
            dq[k] = 0.f;
        }
        // pass 1: the row's maximum, sum and obar
        float m = -INFINITY, l = 0.f;
        for (int j = 0; j <= nf; ++j) {
            const float* key = Pb + (size_t)(j < nf ? j * s + s - 1 : i) * D;
            float kv[kPer], dot = 0.f;
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
                const int c = lane + 32 * k;
                kv[k] = c < D ? key[c] : 0.f;
                dot = fmaf(qv[k], kv[k], dot);
            }
            const float e = warp_sum(dot) * sh.scale;
            const float mn = fmaxf(m, e), corr = expf(m - mn), p = expf(e - mn);
            l = l * corr + p;
#pragma unroll
            for (int k = 0; k < kPer; ++k)
                if (lane + 32 * k < d_c) ob[k] = fmaf(p, kv[k], ob[k] * corr);
            m = mn;
        }
        const float inv = 1.f / l;
        float dl = 0.f;
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            ob[k] *= inv;
            dl = fmaf(dv[k], ob[k], dl);
        }
        const float delta = warp_sum(dl);
        // pass 2: dqt and the own partial's key gradient
        for (int j = 0; j <= nf; ++j) {
            const float* key = Pb + (size_t)(j < nf ? j * s + s - 1 : i) * D;
            float kv[kPer], dot = 0.f, da = 0.f;
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
                const int c = lane + 32 * k;
                kv[k] = c < D ? key[c] : 0.f;
                dot = fmaf(qv[k], kv[k], dot);
                da = fmaf(dv[k], kv[k], da);
            }
            const float e = warp_sum(dot) * sh.scale;
            da = warp_sum(da);
            const float p = expf(e - m) * inv;
            const float sde = sh.scale * p * (da - delta);
#pragma unroll
            for (int k = 0; k < kPer; ++k) dq[k] = fmaf(sde, kv[k], dq[k]);
            if (j == nf) {
#pragma unroll
                for (int k = 0; k < kPer; ++k) {
                    const int c = lane + 32 * k;
                    if (c < D) own[c] += fmaf(sde, qv[k], p * dv[k]);
                }
            }
        }
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            const int c = lane + 32 * k;
            if (c < D) a.dqt[row * D + c] = dq[k];
            if (c < d_c) {
                a.dob[row * d_c + c] = dv[k];
                ((float*)a.obar)[row * d_c + c] = ob[k];
            }
        }
        if (lane == 0) {
            a.mrow[row] = m;
            a.lrow[row] = l;
            a.delta[row] = delta;
        }
    }
    __syncthreads();
    for (int q = threadIdx.x; q < D; q += blockDim.x) {
        float acc = 0.f;
        for (int v = 0; v < nw; ++v) acc += dkey_own[v][q];
        a.dP[((size_t)b * a.T + i) * D + q] = acc;
    }
}

// Column pass: F_j = P_{js+s-1} is a key of every query i >= (j+1)s.
__global__ void __launch_bounds__(256) k_bwd_columns(BwdArgs a) {
    const Shape sh = a.sh;
    const int j = blockIdx.x, b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const int D = sh.D, d_c = sh.d_c, s = sh.s;
    __shared__ float dkey[8][kMaxD];       // a warp's heads, summed in a fixed order below
    for (int q = lane; q < D; q += 32) dkey[warp][q] = 0.f;
    const int t = j * s + s - 1;
    if (t < a.T) {
        const float* key = a.P + ((size_t)b * a.T + t) * D;
        float kv[kPer];
#pragma unroll
        for (int k = 0; k < kPer; ++k) kv[k] = lane + 32 * k < D ? key[lane + 32 * k] : 0.f;
        for (int h = warp; h < sh.H; h += nw) {
            float g[kPer];
#pragma unroll
            for (int k = 0; k < kPer; ++k) g[k] = 0.f;
            for (int i = (j + 1) * s; i < a.T; ++i) {
                const size_t row = ((size_t)b * a.T + i) * sh.H + h;
                const float* q = a.qt + row * D;
                const float* dv = a.dob + row * d_c;
                float qv[kPer], dvv[kPer], dot = 0.f, da = 0.f;
#pragma unroll
                for (int k = 0; k < kPer; ++k) {
                    const int c = lane + 32 * k;
                    qv[k] = c < D ? q[c] : 0.f;
                    dvv[k] = c < d_c ? dv[c] : 0.f;
                    dot = fmaf(qv[k], kv[k], dot);
                    da = fmaf(dvv[k], kv[k], da);
                }
                const float e = warp_sum(dot) * sh.scale;
                da = warp_sum(da);
                const float p = expf(e - a.mrow[row]) / a.lrow[row];
                const float sde = sh.scale * p * (da - a.delta[row]);
#pragma unroll
                for (int k = 0; k < kPer; ++k) g[k] = fmaf(sde, qv[k], fmaf(p, dvv[k], g[k]));
            }
#pragma unroll
            for (int k = 0; k < kPer; ++k)
                if (lane + 32 * k < D) dkey[warp][lane + 32 * k] += g[k];
        }
    }
    __syncthreads();
    for (int q = threadIdx.x; q < D; q += blockDim.x) {
        float acc = 0.f;
        for (int v = 0; v < nw; ++v) acc += dkey[v][q];
        a.dF[((size_t)b * a.n_slots + j) * D + q] = acc;
    }
}

// dqC = W_UK[h] dqt[0:d_c] and dqR = R_i^T dqt[d_c:]: block (i, b), a warp per head.
template <typename T>
__global__ void __launch_bounds__(256) k_bwd_query(BwdArgs a, float* dqc, float* dqr) {
    const Shape sh = a.sh;
    const int i = blockIdx.x, b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    for (int h = warp; h < sh.H; h += nw) {
        const size_t row = ((size_t)b * a.T + i) * sh.H + h;
        const float* g = a.dqt + row * sh.D;
        for (int r = 0; r < sh.d_h; ++r) {
            float acc = 0.f;
            for (int c = lane; c < sh.d_c; c += 32)
                acc = fmaf(ldf<T>(a.w_uk, ((size_t)h * sh.d_h + r) * sh.d_c + c), g[c], acc);
            acc = warp_sum(acc);
            if (lane == 0) dqc[row * sh.d_h + r] = acc;
        }
        for (int k = lane; k < sh.d_r / 2; k += 32) {
            float sn, cs;
            pair_sincos(i, k, sh.d_r, sh.log2_rope_base, &sn, &cs);
            const float g0 = g[sh.d_c + 2 * k], g1 = g[sh.d_c + 2 * k + 1];
            dqr[row * sh.d_r + 2 * k] = fmaf(g0, cs, g1 * sn);          // R_i^T: rotation by -angle
            dqr[row * sh.d_r + 2 * k + 1] = fmaf(-g0, sn, g1 * cs);
        }
    }
}

// Weight gradients in two deterministic stages. k_bwd_wpart: block (row chunk,
// h, output tile), the tile a [64 r x 256 c] block of
//   partK[chunk][h][r][c] = sum_m qC[m,h,r] g[m,h,c],  g = dqt[0:d_c]    (z even)
//   partV[chunk][h][r][c] = sum_m dout[m,h,r] obar[m,h,c]                 (z odd)
// over the chunk's token rows m (g and obar rows g_pitch / d_c elements
// apart, of type GT / OT). Rows are staged 32 at a time in shared memory as
// fp32; each thread keeps an 8 r x 8 c register tile (64 FMAs per row against
// four 16-byte shared loads). Then k_bwd_wsum adds the chunks in order.
template <typename T, typename GT, typename OT>
__global__ void __launch_bounds__(256) k_bwd_wpart(BwdArgs a, const void* g, int g_pitch, float* part_k,
                                                   float* part_v) {
    const Shape sh = a.sh;
    const int chunk = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
    const bool uv = blockIdx.z & 1;
    const int n_ct = (sh.d_c + 255) / 256;
    const int r0 = (int)(blockIdx.z >> 1) / n_ct * 64, c0 = (int)(blockIdx.z >> 1) % n_ct * 256;
    const int64_t M = (int64_t)sh.B * a.T;
    const int64_t m0 = (int64_t)chunk * kWChunk, m1 = m0 + kWChunk < M ? m0 + kWChunk : M;
    const void* asrc = uv ? a.dout : a.qc;
    const void* bsrc = uv ? (const void*)a.obar : g;
    const int bpitch = uv ? sh.d_c : g_pitch;
    __shared__ __align__(16) float As[32][64];
    __shared__ __align__(16) float Bs[32][256];
    const int tr = tid >> 5, tc = tid & 31;          // r = r0 + 8 tr + i, c = c0 + 8 tc + j
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
    constexpr bool kVec = std::is_same<T, bf16>::value && std::is_same<GT, bf16>::value &&
                          std::is_same<OT, bf16>::value;
    if constexpr (kVec) {
        // bf16 operands: 16-byte loads (8 values), the next 32-row stage fetched
        // into registers while this one is multiplied
        const bf16* A = (const bf16*)asrc;
        const bf16* Bm = (const bf16*)bsrc;
        uint4 ra, rb[4];
        auto fetch = [&](int64_t mb) {
            {
                const int mm = tid >> 3, rr = (tid & 7) * 8;       // 32 rows x 8 groups of 8 r
                const int64_t m = mb + mm;
                ra = (m < m1 && r0 + rr < sh.d_h) ? *(const uint4*)(A + ((size_t)m * sh.H + h) * sh.d_h + r0 + rr)
                                                  : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int q = tid + 256 * k, mm = q >> 5, cc = (q & 31) * 8;   // 32 rows x 32 groups of 8 c
                const int64_t m = mb + mm;
                rb[k] = (m < m1 && c0 + cc < sh.d_c) ? *(const uint4*)(Bm + ((size_t)m * sh.H + h) * bpitch + c0 + cc)
                                                     : make_uint4(0, 0, 0, 0);
            }
        };
        auto put = [&]() {
            float v[8];
            const bf16* e = (const bf16*)&ra;
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = __bfloat162float(e[u]);
            *(float4*)&As[tid >> 3][(tid & 7) * 8] = make_float4(v[0], v[1], v[2], v[3]);
            *(float4*)&As[tid >> 3][(tid & 7) * 8 + 4] = make_float4(v[4], v[5], v[6], v[7]);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int q = tid + 256 * k;
                const bf16* f = (const bf16*)&rb[k];
#pragma unroll
                for (int u = 0; u < 8; ++u) v[u] = __bfloat162float(f[u]);
                *(float4*)&Bs[q >> 5][(q & 31) * 8] = make_float4(v[0], v[1], v[2], v[3]);
                *(float4*)&Bs[q >> 5][(q & 31) * 8 + 4] = make_float4(v[4], v[5], v[6], v[7]);
            }
        };
        if (m0 < m1) fetch(m0);
        for (int64_t mb = m0; mb < m1; mb += 32) {
            __syncthreads();
            put();
            __syncthreads();
            if (mb + 32 < m1) fetch(mb + 32);
            const int nm = (int)(m1 - mb < 32 ? m1 - mb : 32);
            for (int mm = 0; mm < nm; ++mm) {
                const float4 a0 = *(const float4*)&As[mm][8 * tr], a1 = *(const float4*)&As[mm][8 * tr + 4];
                const float4 b0 = *(const float4*)&Bs[mm][8 * tc], b1 = *(const float4*)&Bs[mm][8 * tc + 4];
                const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
            }
        }
    } else
    for (int64_t mb = m0; mb < m1; mb += 32) {
        __syncthreads();
        for (int q = tid; q < 32 * 64; q += 256) {
            const int mm = q >> 6, rr = q & 63;
            const int64_t m = mb + mm;
            As[mm][rr] = (m < m1 && r0 + rr < sh.d_h) ? ldf<T>(asrc, ((size_t)m * sh.H + h) * sh.d_h + r0 + rr) : 0.f;
        }
        for (int q = tid; q < 32 * 256; q += 256) {
            const int mm = q >> 8, cc = q & 255;
            const int64_t m = mb + mm;
            float v = 0.f;
            if (m < m1 && c0 + cc < sh.d_c) {
                const size_t o = ((size_t)m * sh.H + h) * bpitch + c0 + cc;
                v = uv ? ldf<OT>(bsrc, o) : ldf<GT>(bsrc, o);
            }
            Bs[mm][cc] = v;
        }
        __syncthreads();
        const int nm = (int)(m1 - mb < 32 ? m1 - mb : 32);
        for (int mm = 0; mm < nm; ++mm) {
            const float4 a0 = *(const float4*)&As[mm][8 * tr], a1 = *(const float4*)&As[mm][8 * tr + 4];
            const float4 b0 = *(const float4*)&Bs[mm][8 * tc], b1 = *(const float4*)&Bs[mm][8 * tc + 4];
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
    }
    float* part = uv ? part_v : part_k;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int r = r0 + 8 * tr + i;
        if (r >= sh.d_h) continue;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int c = c0 + 8 * tc + j;
            if (c < sh.d_c) part[(((size_t)chunk * sh.H + h) * sh.d_h + r) * sh.d_c + c] = acc[i][j];
        }
    }
}

__global__ void __launch_bounds__(256) k_bwd_wsum(int n_chunks, size_t n, const float* part_k, const float* part_v,
                                                  float* dw_uk, float* dw_uv) {
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    float k = 0.f, v = 0.f;
    for (int q = 0; q < n_chunks; ++q) {
        k += part_k[(size_t)q * n + i];
        v += part_v[(size_t)q * n + i];
    }
    dw_uk[i] = k;
    dw_uv[i] = v;
}

// Scan and gate backward: a warp per slot j of sequence b, its tokens from the
// block's end down (the suffix sum S_u), grid (ceil(n_slots / 8), B). The gate
// gradients of the block's warps meet in shared memory, then one atomic per
// element goes to the zeroed dG / dg.
template <typename T>
__global__ void __launch_bounds__(256) k_bwd_scan(BwdArgs a, const void* c_in, const void* kr_in,
                                                  const float* gate_w, float* dc, float* dkr, float* dG,
                                                  float* dg, float* dgate_in) {
    const Shape sh = a.sh;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.y, j = blockIdx.x * 8 + warp;
    const int D = sh.D, d_c = sh.d_c, s = sh.s, Tn = a.T;
    __shared__ float Ss[8][kMaxD];
    __shared__ float gG[8 * 512];          // s * d_c <= 8 * 512
    __shared__ float gg[8];
    __shared__ double pe_freq[256], rope_freq[288];
    const bool computed = sh.gate_mode == 0;
    for (int k = threadIdx.x; k < d_c / 2; k += blockDim.x)
        pe_freq[k] = exp2(-(2.0 * k / (double)d_c) * sh.log2_pe_base);
    for (int k = threadIdx.x; k < sh.d_r / 2; k += blockDim.x)
        rope_freq[k] = exp2(-(2.0 * k / (double)sh.d_r) * sh.log2_rope_base);
    if (computed) {
        for (int k = threadIdx.x; k < s * d_c; k += blockDim.x) gG[k] = 0.f;
        if (threadIdx.x < s) gg[threadIdx.x] = 0.f;
    }
    __syncthreads();
    if (j < a.n_slots) {
        float* S = Ss[warp];
        for (int c = lane; c < D; c += 32) S[c] = 0.f;
        const int u0 = j * s, u1 = min(u0 + s, Tn);
        const bool finished = u0 + s - 1 < Tn;   // F_j exists as a key
        const float* dF = a.dF + ((size_t)b * a.n_slots + j) * D;
        for (int u = u1 - 1; u >= u0; --u) {
            const size_t bu = (size_t)b * Tn + u;
            const float* dPu = a.dP + bu * D;
            const bool end = finished && u == u0 + s - 1;
            __syncwarp();
            for (int c = lane; c < D; c += 32) {
                float f = 0.f;
                if (end)
                    for (int q = 0; q < a.n_parts; ++q) f += dF[(size_t)q * sh.B * a.n_slots * D + c];
                S[c] += dPu[c] + f;
            }
            __syncwarp();
            const float wu = a.w[bu];
            float dw = 0.f;
            for (int c = lane; c < d_c; c += 32) dw = fmaf(ldf<T>(c_in, bu * d_c + c), S[c], dw);
            for (int k = lane; k < sh.d_r / 2; k += 32) {
                float sn, cs;
                pair_sincos_f(u, rope_freq[k], &sn, &cs);
                const float x0 = ldf<T>(kr_in, bu * sh.d_r + 2 * k), x1 = ldf<T>(kr_in, bu * sh.d_r + 2 * k + 1);
                const float s0 = S[d_c + 2 * k], s1 = S[d_c + 2 * k + 1];
                dw = fmaf(x0 * cs - x1 * sn, s0, fmaf(x0 * sn + x1 * cs, s1, dw));
                const float dx0 = wu * s0, dx1 = wu * s1;
                dkr[bu * sh.d_r + 2 * k] = fmaf(dx0, cs, dx1 * sn);        // R_u^T
                dkr[bu * sh.d_r + 2 * k + 1] = fmaf(-dx0, sn, dx1 * cs);
            }
            dw = warp_sum(dw);
            if (sh.gate_mode == 1 && lane == 0) dgate_in[bu] = dw;
            if (computed) {
                const int r = u % s;
                const float dz = dw * wu * (1.f - wu);
                if (lane == 0) atomicAdd(&gg[r], dz);
                const float* G = gate_w + (size_t)r * d_c;
                for (int k = lane; k < d_c / 2; k += 32) {
                    float sn, cs;
                    pair_sincos_f(u, pe_freq[k], &sn, &cs);   // PE_u[2k], PE_u[2k+1]
                    const float c0 = ldf<T>(c_in, bu * d_c + 2 * k), c1 = ldf<T>(c_in, bu * d_c + 2 * k + 1);
                    dc[bu * d_c + 2 * k] = fmaf(wu, S[2 * k], dz * G[2 * k] * sn);
                    dc[bu * d_c + 2 * k + 1] = fmaf(wu, S[2 * k + 1], dz * G[2 * k + 1] * cs);
                    atomicAdd(&gG[r * d_c + 2 * k], dz * c0 * sn);
                    atomicAdd(&gG[r * d_c + 2 * k + 1], dz * c1 * cs);
                }
            } else {
                for (int c = lane; c < d_c; c += 32) dc[bu * d_c + c] = wu * S[c];
            }
        }
    }
    if (computed) {
        __syncthreads();
        for (int k = threadIdx.x; k < s * d_c; k += blockDim.x) atomicAdd(&dG[k], gG[k]);
        if (threadIdx.x < s) atomicAdd(&dg[threadIdx.x], gg[threadIdx.x]);
    }
}

// Tensor-core path: W_UV^T [H][d_c][d_h] (the B operand of the dobar GEMM).
__global__ void __launch_bounds__(256) k_transpose_wuv(Shape sh, const bf16* w, bf16* wt) {
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t n = (size_t)sh.H * sh.d_h * sh.d_c;
    if (i >= n) return;
    const int c = (int)(i % sh.d_c);
    const size_t hr = i / sh.d_c;
    const int r = (int)(hr % sh.d_h), h = (int)(hr / sh.d_h);
    wt[((size_t)h * sh.d_c + c) * sh.d_h + r] = w[i];
}

// Tensor-core path: delta = dobar . obar per row from the bf16 values the
// tensor-core kernels read, in the [B, H, pitch] layout; a warp per row
// (b, t, h), 8 channels a lane.
__global__ void __launch_bounds__(256) k_bwd_delta(Shape sh, int T, const bf16* dob, const bf16* obar, float* delta) {
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    const int64_t rows = (int64_t)sh.B * T * sh.H;
    if (row >= rows) return;
    float acc = 0.f;
    for (int c0 = lane * 8; c0 < sh.d_c; c0 += 256) {
        float x[8], y[8];
        load8<bf16>(dob + row * sh.d_c + c0, x);
        load8<bf16>(obar + row * sh.d_c + c0, y);
#pragma unroll
        for (int u = 0; u < 8; ++u) acc = fmaf(x[u], y[u], acc);
    }
    acc = warp_sum(acc);
    if (lane == 0) {
        const int h = (int)(row % sh.H);
        const int64_t bt = row / sh.H;
        const int t = (int)(bt % T), b = (int)(bt / T);
        delta[((size_t)b * sh.H + h) * stats_pitch(T) + t] = acc;
    }
}

// Tensor-core path: the own-partial term of every row (one key, P_i) added to
// the finished-slot part of dqt; then the row's query gradients leave: the
// latent part as bf16 (the operand of the dqC GEMM and the weight gradients)
// and dqR = R_i^T dqt[d_c:] (fp32, the output); dP_i = the heads' own-partial
// key gradients, summed in a fixed order. Block (i, b), a warp per head, 8
// channels a lane (16-byte loads).
constexpr int kOwnGroups = 2;          // 8-channel groups a lane takes: D <= 512 (the tensor-core widths)
__device__ __forceinline__ float bf_at(const uint4& r, int u) { return __bfloat162float(((const bf16*)&r)[u]); }
__global__ void __launch_bounds__(256) k_bwd_own(BwdArgs a, const bf16* qt, const bf16* P, const bf16* dob,
                                                    const float* lse, const float* delta, bf16* dqtl, float* dq_r) {
    const Shape sh = a.sh;
    const int i = blockIdx.x, b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const int D = sh.D, d_c = sh.d_c;
    const float scale_log2 = sh.scale * 1.4426950408889634f;
    __shared__ float dkey_own[8][kMaxD];
    __shared__ float2 rcs[kMaxD / 2];               // (sin, cos) of position i's RoPE pairs
    float* own = dkey_own[warp];
    const bf16* Pi = P + ((size_t)b * a.T + i) * D;
    const uint4 z4 = make_uint4(0, 0, 0, 0);
    uint4 pr4[kOwnGroups];                          // P_i, 8 bf16 a group, kept packed
#pragma unroll
    for (int k = 0; k < kOwnGroups; ++k) {
        const int c0 = 8 * (lane + 32 * k);
        pr4[k] = c0 < D ? *(const uint4*)(Pi + c0) : z4;
    }
    // every load of a head's row first (their latencies overlap), then the sums;
    // the warp's first head is loaded before the block waits for the RoPE table
    uint4 q4[kOwnGroups], d4[kOwnGroups];
    float gv[kOwnGroups][8];
    float lse_r = 0.f, delta_r = 0.f;
    auto load_row = [&](int h) {
        const size_t row = ((size_t)b * a.T + i) * sh.H + h;
        const size_t srow = ((size_t)b * sh.H + h) * stats_pitch(a.T) + i;
#pragma unroll
        for (int k = 0; k < kOwnGroups; ++k) {
            const int c0 = 8 * (lane + 32 * k);
            q4[k] = c0 < D ? *(const uint4*)(qt + row * D + c0) : z4;
            d4[k] = c0 < d_c ? *(const uint4*)(dob + row * d_c + c0) : z4;
            if (c0 < D) load8<float>(a.dqt + row * D + c0, gv[k]);
            else
#pragma unroll
                for (int u = 0; u < 8; ++u) gv[k][u] = 0.f;
        }
        lse_r = lse[srow];
        delta_r = delta[srow];
    };
    if (warp < sh.H) load_row(warp);
    for (int q = lane; q < D; q += 32) own[q] = 0.f;
    for (int kp = threadIdx.x; kp < sh.d_r / 2; kp += blockDim.x) {
        float sn, cs;
        pair_sincos(i, kp, sh.d_r, sh.log2_rope_base, &sn, &cs);
        rcs[kp] = make_float2(sn, cs);
    }
    __syncthreads();
    for (int h = warp; h < sh.H; h += nw) {
        const size_t row = ((size_t)b * a.T + i) * sh.H + h;
        float e = 0.f, da = 0.f;
#pragma unroll
        for (int k = 0; k < kOwnGroups; ++k)
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float pu = bf_at(pr4[k], u);
                e = fmaf(bf_at(q4[k], u), pu, e);
                da = fmaf(bf_at(d4[k], u), pu, da);
            }
        e = warp_sum(e);
        da = warp_sum(da);
        const float pr = exp2f(fmaf(e, scale_log2, -lse_r));
        const float sde = sh.scale * pr * (da - delta_r);
#pragma unroll
        for (int k = 0; k < kOwnGroups; ++k) {
            const int c0 = 8 * (lane + 32 * k);
            if (c0 >= D) continue;
            float* g = gv[k];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                g[u] = fmaf(sde, bf_at(pr4[k], u), g[u]);
                own[c0 + u] += fmaf(sde, bf_at(q4[k], u), pr * bf_at(d4[k], u));
            }
            if (c0 < d_c) {
                store8<bf16>(dqtl + row * d_c + c0, g);
            } else {
#pragma unroll
                for (int u = 0; u < 8; u += 2) {
                    const int kp = (c0 - d_c + u) / 2;        // RoPE pair
                    const float sn = rcs[kp].x, cs = rcs[kp].y;
                    dq_r[row * sh.d_r + 2 * kp] = fmaf(g[u], cs, g[u + 1] * sn);        // R_i^T
                    dq_r[row * sh.d_r + 2 * kp + 1] = fmaf(-g[u], sn, g[u + 1] * cs);
                }
            }
        }
        if (h + nw < sh.H) load_row(h + nw);
    }
    __syncthreads();
    for (int q = threadIdx.x; q < D; q += blockDim.x) {
        float acc = 0.f;
        for (int v = 0; v < nw; ++v) acc += dkey_own[v][q];
        a.dP[((size_t)b * a.T + i) * D + q] = acc;
    }
}

struct BwdWs {
    size_t P, w, cache, qt, mrow, lrow, delta, dob, obar, dqt, dP, dF, part_k, part_v, total;
};

int weight_chunks(const Shape& sh, int T) { return (int)(((int64_t)sh.B * T + kWChunk - 1) / kWChunk); }
size_t weight_part_bytes(const Shape& sh, int T) {
    return (size_t)weight_chunks(sh, T) * sh.H * sh.d_h * sh.d_c * sizeof(float);
}

// dW_UK, dW_UV from the rows' latent query gradients g (rows g_pitch apart, type GT)
template <typename T, typename GT, typename OT>
cudaError_t weight_grads(const BwdArgs& a, const void* g, int g_pitch, float* part_k, float* part_v, float* dw_uk,
                         float* dw_uv, cudaStream_t st) {
    const Shape& sh = a.sh;
    const int nc = weight_chunks(sh, a.T);
    const int tiles = ((sh.d_h + 63) / 64) * ((sh.d_c + 255) / 256);
    k_bwd_wpart<T, GT, OT><<<dim3(nc, sh.H, 2 * tiles), 256, 0, st>>>(a, g, g_pitch, part_k, part_v);
    const size_t n = (size_t)sh.H * sh.d_h * sh.d_c;
    k_bwd_wsum<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(nc, n, part_k, part_v, dw_uk, dw_uv);
    return cudaGetLastError();
}

BwdWs bwd_layout(const Shape& sh, int T, size_t elem) {
    const size_t BT = (size_t)sh.B * T, rows = BT * sh.H;
    const size_t n_slots = (T + sh.s - 1) / sh.s;
    BwdWs l;
    size_t o = 0;
    auto take = [&](size_t bytes) { size_t at = o; o += align256(bytes); return at; };
    l.P = take(BT * sh.D * 4);
    l.w = take(BT * 4);
    l.cache = take((size_t)sh.B * n_slots * sh.D * elem);
    l.qt = take(rows * sh.D * 4);
    l.mrow = take(rows * 4);
    l.lrow = take(rows * 4);
    l.delta = take(rows * 4);
    l.dob = take(rows * sh.d_c * 4);
    l.obar = take(rows * sh.d_c * 4);
    l.dqt = take(rows * sh.D * 4);
    l.dP = take(BT * sh.D * 4);
    l.dF = take((size_t)sh.B * n_slots * sh.D * 4);
    l.part_k = take(weight_part_bytes(sh, T));
    l.part_v = take(weight_part_bytes(sh, T));
    l.total = o;
    return l;
}

template <typename T>
cudaError_t backward_impl(const PrefillArgs& pa_in, const BackwardGrads& g, cudaStream_t st, uint64_t* launches) {
    PrefillArgs pa = pa_in;
    const int T_len = pa.T;
    const int n_slots = (T_len + pa.sh.s - 1) / pa.sh.s;
    pa.sh.max_slots = n_slots;          // the scan's slot rows (a scratch copy)
    const Shape sh = pa.sh;
    char* ws = (char*)pa.workspace;
    const BwdWs l = bwd_layout(sh, T_len, sizeof(T));
    pa.cache_out = ws + l.cache;
    pa.open_slot_out = nullptr;
    pa.open_slot_in = nullptr;
    pa.t0 = 0;
    BwdArgs a;
    a.sh = sh;
    a.T = T_len;
    a.n_slots = n_slots;
    a.qc = pa.q_c;
    a.w_uk = pa.w_uk;
    a.w_uv = pa.w_uv;
    a.dout = g.dout;
    a.P = (const float*)(ws + l.P);
    a.qt = (const float*)(ws + l.qt);
    a.w = (const float*)(ws + l.w);
    a.mrow = (float*)(ws + l.mrow);
    a.lrow = (float*)(ws + l.lrow);
    a.delta = (float*)(ws + l.delta);
    a.dob = (float*)(ws + l.dob);
    a.obar = (float*)(ws + l.obar);
    a.dqt = (float*)(ws + l.dqt);
    a.dP = (float*)(ws + l.dP);
    a.dF = (float*)(ws + l.dF);
    a.n_parts = 1;
    cudaError_t e;
    if (sh.gate_mode == 0) {
        if ((e = cudaMemsetAsync(g.dgate_w, 0, (size_t)sh.s * sh.d_c * sizeof(float), st)) != cudaSuccess)
            return note_error("backward zero dG", e);
        if ((e = cudaMemsetAsync(g.dgate_b, 0, (size_t)sh.s * sizeof(float), st)) != cudaSuccess)
            return note_error("backward zero dg", e);
    }
    const int threads = 32 * (sh.H < 8 ? sh.H : 8);
    k_prefill_scan<T, float><<<dim3((n_slots + 7) / 8, sh.B), 256, 0, st>>>(pa, (float*)(ws + l.P), nullptr,
                                                                           (float*)(ws + l.w));
    k_prefill_absorb<T><<<dim3(sh.B * T_len, sh.H), 128, 0, st>>>(sh, (const T*)pa.q_c, (const T*)pa.q_r,
                                                                  (const T*)pa.w_uk, T_len, 0, (float*)(ws + l.qt));
    profile_begin(st);
    k_bwd_rows<T><<<dim3(T_len, sh.B), threads, 0, st>>>(a);
    k_bwd_columns<<<dim3(n_slots, sh.B), threads, 0, st>>>(a);
    profile_end(st);
    k_bwd_query<T><<<dim3(T_len, sh.B), threads, 0, st>>>(a, g.dq_c, g.dq_r);
    if ((e = weight_grads<T, float, float>(a, a.dqt, sh.D, (float*)(ws + l.part_k), (float*)(ws + l.part_v),
                                           g.dw_uk, g.dw_uv, st)) != cudaSuccess)
        return note_error("backward weight-gradient launch", e);
    k_bwd_scan<T><<<dim3((n_slots + 7) / 8, sh.B), 256, 0, st>>>(a, pa.c, pa.kr, pa.gate_w, g.dc, g.dkr, g.dgate_w,
                                                                 g.dgate_b, g.dgate_in);
    *launches += 8;
    return note_error("backward launch", cudaGetLastError());
}

// ---------------------------------------------------------------- tensor-core path

Shape with_slots(const Shape& sh, int T) {
    Shape s2 = sh;
    s2.max_slots = (T + sh.s - 1) / sh.s;
    return s2;
}

// What the training forward keeps for the backward (tensor-core path): the
// forward's own scratch (its first region the partial slots P, bf16), the
// slots, each row's log2-domain log-sum-exp, O / l, the absorbed query, and
// the merging weights.
struct SavedWs {
    size_t fwd, cache, lse, obar, qt, w, total;
};

SavedWs saved_layout(const Shape& sh_in, int T) {
    const Shape sh = with_slots(sh_in, T);
    const size_t BT = (size_t)sh.B * T, rows = BT * sh.H;
    SavedWs l;
    size_t o = 0;
    auto take = [&](size_t bytes) { size_t at = o; o += align256(bytes); return at; };
    l.fwd = take(tc_prefill_workspace(sh, T));
    l.cache = take((size_t)sh.B * sh.max_slots * sh.D * 2);
    l.lse = take((size_t)sh.B * sh.H * stats_pitch(T) * 4);
    l.obar = take(rows * sh.d_c * 2);
    l.qt = take(rows * sh.D * 2);
    l.w = take(BT * 4);
    l.total = o;
    return l;
}

// The backward's own scratch, after the saved rows when it recomputes them
// (`base` = their size; `out` then takes the recomputed forward's output).
struct BwdTcWs {
    size_t out, delta, dob, dqt, dF, dP, wuvt, dqtl, part_k, part_v, u, total;
};

BwdTcWs bwd_tc_layout(const Shape& sh_in, int T, size_t base, bool recompute) {
    const Shape sh = with_slots(sh_in, T);
    const size_t BT = (size_t)sh.B * T, rows = BT * sh.H;
    BwdTcWs l;
    size_t o = base;
    auto take = [&](size_t bytes) { size_t at = o; o += align256(bytes); return at; };
    l.out = recompute ? take(rows * sh.d_h * 2) : 0;
    l.delta = take((size_t)sh.B * sh.H * stats_pitch(T) * 4);
    l.dob = take(rows * sh.d_c * 2);
    l.dqt = take(rows * sh.D * 4);
    l.dF = take((size_t)sh.H * sh.B * sh.max_slots * sh.D * 4);
    l.dP = take(BT * sh.D * 4);
    l.wuvt = take((size_t)sh.H * sh.d_h * sh.d_c * 2);
    l.dqtl = take(rows * sh.d_c * 2);
    l.part_k = take(weight_part_bytes(sh, T));
    l.part_v = take(weight_part_bytes(sh, T));
    l.u = take((size_t)sh.B * sh.max_slots * sh.H * sh.d_h * 2);
    l.total = o;
    return l;
}

// The forward on the tensor cores from position 0, keeping the rows the
// backward needs in `sv` (saved_layout); `out` receives the forward's output.
cudaError_t train_forward(const PrefillArgs& pa_in, char* sv, void* out, cudaStream_t st, uint64_t* launches) {
    const int T_len = pa_in.T;
    PrefillArgs pa = pa_in;
    pa.sh = with_slots(pa_in.sh, T_len);
    const SavedWs S = saved_layout(pa.sh, T_len);
    pa.workspace = sv + S.fwd;
    pa.workspace_bytes = tc_prefill_workspace(pa.sh, T_len);
    pa.cache_out = sv + S.cache;
    pa.out = out;
    pa.open_slot_in = nullptr;
    pa.open_slot_out = nullptr;
    pa.t0 = 0;
    PrefillSave keep;
    keep.w = (float*)(sv + S.w);
    keep.lse = (float*)(sv + S.lse);
    keep.obar = sv + S.obar;
    keep.qt = sv + S.qt;
    return tc_prefill_save(pa, keep, st, launches);
}

bool use_tc(const Shape& sh, int dtype) {
    return dtype == kDtypeBF16 && tc_backward_supported(sh) && tc_prefill_supported(sh);
}

// bf16 at the tensor-core prefill's widths: the rows kept by the training
// forward (`saved`; recomputed here into the workspace when it is null), dobar
// and delta, the finished-slot parts on the tensor cores, the own-partial
// term, then the same query, weight and scan/gate backward as the CUDA-core
// path (dF summed over heads).
cudaError_t backward_tc(const PrefillArgs& pa_in, const BackwardGrads& g, const void* saved, cudaStream_t st,
                        uint64_t* launches) {
    const int T_len = pa_in.T;
    PrefillArgs pa = pa_in;
    pa.sh = with_slots(pa_in.sh, T_len);
    const Shape sh = pa.sh;
    const int n_slots = sh.max_slots;
    char* ws = (char*)pa.workspace;
    const SavedWs S = saved_layout(sh, T_len);
    const bool recompute = saved == nullptr;
    const BwdTcWs l = bwd_tc_layout(sh, T_len, recompute ? S.total : 0, recompute);
    char* sv = recompute ? ws : (char*)saved;
    cudaError_t e;
    if (sh.gate_mode == 0) {
        if ((e = cudaMemsetAsync(g.dgate_w, 0, (size_t)sh.s * sh.d_c * sizeof(float), st)) != cudaSuccess)
            return note_error("backward zero dG", e);
        if ((e = cudaMemsetAsync(g.dgate_b, 0, (size_t)sh.s * sizeof(float), st)) != cudaSuccess)
            return note_error("backward zero dg", e);
    }
    if (recompute && (e = train_forward(pa_in, sv, ws + l.out, st, launches)) != cudaSuccess) return e;
    BwdArgs a;
    a.sh = sh;
    a.T = T_len;
    a.n_slots = n_slots;
    a.qc = pa.q_c;
    a.w_uk = pa.w_uk;
    a.w_uv = pa.w_uv;
    a.dout = g.dout;
    a.P = nullptr;
    a.qt = nullptr;
    a.w = (const float*)(sv + S.w);
    a.mrow = a.lrow = a.delta = nullptr;
    a.dob = nullptr;
    a.obar = sv + S.obar;
    a.dqt = (float*)(ws + l.dqt);
    a.dP = (float*)(ws + l.dP);
    a.dF = (float*)(ws + l.dF);
    a.n_parts = sh.H;
    const int threads = 32 * (sh.H < 8 ? sh.H : 8);
    const int M = sh.B * T_len;
    bf16* dob = (bf16*)(ws + l.dob);
    // dobar = dout . W_UV[h] on the tensor cores (W_UV^T as the K-major operand),
    // then delta = dobar . obar
    const size_t nw = (size_t)sh.H * sh.d_h * sh.d_c;
    k_transpose_wuv<<<(unsigned)((nw + 255) / 256), 256, 0, st>>>(sh, (const bf16*)pa.w_uv, (bf16*)(ws + l.wuvt));
    e = gemm_batched(GemmOperand{g.dout, sh.H * sh.d_h, (size_t)sh.d_h},
                     GemmOperand{ws + l.wuvt, sh.d_h, (size_t)sh.d_c * sh.d_h}, dob, sh.H * sh.d_c, (size_t)sh.d_c,
                     false, M, sh.d_c, sh.d_h, sh.H, pa.status, st, launches);
    if (e != cudaSuccess) return e;
    const int64_t rows = (int64_t)M * sh.H;
    k_bwd_delta<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(sh, T_len, dob, (const bf16*)(sv + S.obar),
                                                             (float*)(ws + l.delta));
    if ((e = cudaGetLastError()) != cudaSuccess) return note_error("k_bwd_delta launch", e);
    // U_j[h] = W_UV[h] F_j[0:d_c] for every finished slot and head: one GEMM,
    // [B n_slots, d_c] . W_UV viewed as [H d_h, d_c]
    e = gemm_batched(GemmOperand{sv + S.cache, sh.D, 0}, GemmOperand{pa.w_uv, sh.d_c, 0}, ws + l.u, sh.H * sh.d_h, 0,
                     false, sh.B * n_slots, sh.H * sh.d_h, sh.d_c, 1, pa.status, st, launches);
    if (e != cudaSuccess) return e;
    BwdTCInputs in;
    in.qt = sv + S.qt;
    in.dob = ws + l.dob;
    in.slots = sv + S.cache;
    in.dout = g.dout;
    in.u = ws + l.u;
    in.lse = (const float*)(sv + S.lse);
    in.delta = (const float*)(ws + l.delta);
    in.dqt = a.dqt;
    in.dF = a.dF;
    in.status = pa.status;
    profile_begin(st);
    e = tc_backward_attention(sh, T_len, in, st, launches);
    profile_end(st);
    if (e != cudaSuccess) return e;
    bf16* dqtl = (bf16*)(ws + l.dqtl);
    k_bwd_own<<<dim3(T_len, sh.B), threads, 0, st>>>(a, (const bf16*)(sv + S.qt), (const bf16*)(sv + S.fwd), dob,
                                                      in.lse, in.delta, dqtl, g.dq_r);
    if ((e = cudaGetLastError()) != cudaSuccess) return note_error("k_bwd_own launch", e);
    // dqC = dqt[0:d_c] . W_UK[h]^T on the tensor cores, fp32 out
    e = gemm_batched(GemmOperand{dqtl, sh.H * sh.d_c, (size_t)sh.d_c},
                     GemmOperand{pa.w_uk, sh.d_c, (size_t)sh.d_h * sh.d_c}, g.dq_c, sh.H * sh.d_h, (size_t)sh.d_h,
                     true, M, sh.d_h, sh.d_c, sh.H, pa.status, st, launches);
    if (e != cudaSuccess) return e;
    {
        // dW_UK, dW_UV on the tensor cores: per chunk of rows, then the chunks in order
        float* part_k = (float*)(ws + l.part_k);
        float* part_v = (float*)(ws + l.part_v);
        const int nc = tc_weight_chunks(sh, M, weight_chunks(sh, T_len));
        if ((e = tc_weight_parts(sh, M, pa.q_c, dqtl, g.dout, sv + S.obar, part_k, part_v, nc, pa.status, st)) !=
            cudaSuccess)
            return e;
        const size_t n = (size_t)sh.H * sh.d_h * sh.d_c;
        k_bwd_wsum<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(nc, n, part_k, part_v, g.dw_uk, g.dw_uv);
        if ((e = cudaGetLastError()) != cudaSuccess) return note_error("k_bwd_wsum launch", e);
    }
    k_bwd_scan<bf16><<<dim3((n_slots + 7) / 8, sh.B), 256, 0, st>>>(a, pa.c, pa.kr, pa.gate_w, g.dc, g.dkr,
                                                                    g.dgate_w, g.dgate_b, g.dgate_in);
    *launches += 6;
    return note_error("backward launch", cudaGetLastError());
}

}  // namespace

size_t prefill_backward_workspace(const Shape& sh, int T, int dtype) {
    return use_tc(sh, dtype) ? bwd_tc_layout(sh, T, saved_layout(sh, T).total, true).total
                             : bwd_layout(sh, T, dtype_bytes(dtype)).total;
}

bool prefill_train_supported(const Shape& sh) { return use_tc(sh, sh.dtype); }
size_t prefill_train_saved_bytes(const Shape& sh, int T) { return saved_layout(sh, T).total; }
size_t prefill_backward_saved_workspace(const Shape& sh, int T) { return bwd_tc_layout(sh, T, 0, false).total; }

cudaError_t prefill_train(const PrefillArgs& a, void* saved, cudaStream_t st, uint64_t* launches) {
    return train_forward(a, (char*)saved, a.out, st, launches);
}

cudaError_t prefill_backward_saved(const PrefillArgs& a, const BackwardGrads& g, const void* saved, cudaStream_t st,
                                   uint64_t* launches) {
    return backward_tc(a, g, saved, st, launches);
}

cudaError_t prefill_backward(const PrefillArgs& a, const BackwardGrads& g, int dtype, cudaStream_t st,
                             uint64_t* launches) {
    if (use_tc(a.sh, dtype)) return backward_tc(a, g, nullptr, st, launches);
    if (dtype == kDtypeF32) return backward_impl<float>(a, g, st, launches);
    if (dtype == kDtypeF16) return backward_impl<f16>(a, g, st, launches);
    return backward_impl<bf16>(a, g, st, launches);
}

}  // namespace mtla
