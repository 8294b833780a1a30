// backward.cu -- training backward of the parallel (prefill) forward from
// position 0 ("Multi-head Temporal Latent Attention", Results: the models are
// trained from scratch; Key claims: the stride-aware mask lets the parallel
// training pass match incremental decoding), on the CUDA cores in fp32.
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
// Kernels, in launch order:
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
//   k_bwd_weights     dW_UK, dW_UV (row chunks, atomics into zeroed outputs)
//   k_bwd_scan        a warp per slot: the scan and gate backward
#include "common.cuh"
#include "mtla_internal.h"
#include "prep.cuh"

namespace mtla {

namespace {

constexpr int kMaxD = 576;             // slot width the kernels hold (d_c + d_R)
constexpr int kPer = kMaxD / 32;       // a lane's channels: lane + 32 k
constexpr int kWRows = 16;             // dW rows r per block of k_bwd_weights
constexpr int kWChunk = 512;           // token rows per block of k_bwd_weights

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

// dW_UK[h][r][c] += sum_rows qC[r] dqt[c], dW_UV[h][r][c] += sum_rows dout[r] obar[c]
// over token rows m0 .. m0 + kWChunk - 1: block (row chunk, h, r group), a
// thread per channel c (two when d_c > 256).
template <typename T, typename OT>
__global__ void __launch_bounds__(256) k_bwd_weights(BwdArgs a, float* dw_uk, float* dw_uv) {
    const Shape sh = a.sh;
    const int h = blockIdx.y, r0 = blockIdx.z * kWRows, tid = threadIdx.x;
    const int64_t M = (int64_t)sh.B * a.T;
    const int64_t m0 = (int64_t)blockIdx.x * kWChunk, m1 = m0 + kWChunk < M ? m0 + kWChunk : M;
    __shared__ float qs[kWRows], os[kWRows];
    float gk[2][kWRows], gv[2][kWRows];
#pragma unroll
    for (int cc = 0; cc < 2; ++cc)
#pragma unroll
        for (int r = 0; r < kWRows; ++r) gk[cc][r] = gv[cc][r] = 0.f;
    for (int64_t m = m0; m < m1; ++m) {
        const size_t row = (size_t)m * sh.H + h;
        __syncthreads();
        if (tid < kWRows) qs[tid] = ldf<T>(a.qc, row * sh.d_h + r0 + tid);
        else if (tid < 2 * kWRows) os[tid - kWRows] = ldf<T>(a.dout, row * sh.d_h + r0 + tid - kWRows);
        __syncthreads();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            const int c = tid + 256 * cc;
            if (c < sh.d_c) {
                const float x = a.dqt[row * sh.D + c], y = ldf<OT>(a.obar, row * sh.d_c + c);
#pragma unroll
                for (int r = 0; r < kWRows; ++r) {
                    gk[cc][r] = fmaf(qs[r], x, gk[cc][r]);
                    gv[cc][r] = fmaf(os[r], y, gv[cc][r]);
                }
            }
        }
    }
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
        const int c = tid + 256 * cc;
        if (c < sh.d_c)
#pragma unroll
            for (int r = 0; r < kWRows; ++r) {
                const size_t o = ((size_t)h * sh.d_h + r0 + r) * sh.d_c + c;
                atomicAdd(&dw_uk[o], gk[cc][r]);
                atomicAdd(&dw_uv[o], gv[cc][r]);
            }
    }
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

// Tensor-core path, per (16 positions, head, sequence): dobar = W_UV[h]^T dout
// rounded to bf16 (the operand of the tensor-core kernels) and delta =
// dobar . obar from the same rounded values, in the [B, H, T] layout.
template <typename T>
__global__ void __launch_bounds__(256) k_bwd_dob(BwdArgs a, bf16* dob, float* delta) {
    const Shape sh = a.sh;
    const int t0 = blockIdx.x * 16, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    __shared__ float dsm[16][256];
    __shared__ float red[8][16];
    for (int q = tid; q < 16 * sh.d_h; q += blockDim.x) {
        const int pp = q / sh.d_h, r = q % sh.d_h, t = t0 + pp;
        dsm[pp][r] = t < a.T ? ldf<T>(a.dout, (((size_t)b * a.T + t) * sh.H + h) * sh.d_h + r) : 0.f;
    }
    __syncthreads();
    float dl[16];
#pragma unroll
    for (int pp = 0; pp < 16; ++pp) dl[pp] = 0.f;
    for (int c = tid; c < sh.d_c; c += blockDim.x) {
        float acc[16];
#pragma unroll
        for (int pp = 0; pp < 16; ++pp) acc[pp] = 0.f;
        for (int r = 0; r < sh.d_h; ++r) {
            const float wv = ldf<T>(a.w_uv, ((size_t)h * sh.d_h + r) * sh.d_c + c);
#pragma unroll
            for (int pp = 0; pp < 16; ++pp) acc[pp] = fmaf(dsm[pp][r], wv, acc[pp]);
        }
#pragma unroll
        for (int pp = 0; pp < 16; ++pp) {
            const int t = t0 + pp;
            if (t < a.T) {
                const size_t o = (((size_t)b * a.T + t) * sh.H + h) * sh.d_c + c;
                const bf16 v = __float2bfloat16_rn(acc[pp]);
                dob[o] = v;
                dl[pp] = fmaf(__bfloat162float(v), ldf<bf16>(a.obar, o), dl[pp]);
            }
        }
    }
#pragma unroll
    for (int pp = 0; pp < 16; ++pp) {
        const float v = warp_sum(dl[pp]);
        if (lane == 0) red[warp][pp] = v;
    }
    __syncthreads();
    if (tid < 16 && t0 + tid < a.T) {
        float v = 0.f;
        for (int q = 0; q < (int)(blockDim.x >> 5); ++q) v += red[q][tid];
        delta[((size_t)b * sh.H + h) * stats_pitch(a.T) + t0 + tid] = v;
    }
}

// Tensor-core path: the own-partial term of every row (one key, P_i), added
// to the finished-slot part of dqt; dP_i = the heads' own-partial key
// gradients (summed in a fixed order). Block (i, b), a warp per head.
__global__ void __launch_bounds__(256) k_bwd_own(BwdArgs a, const bf16* qt, const bf16* P, const bf16* dob,
                                                 const float* lse, const float* delta) {
    const Shape sh = a.sh;
    const int i = blockIdx.x, b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const int D = sh.D, d_c = sh.d_c;
    const float scale_log2 = sh.scale * 1.4426950408889634f;
    __shared__ float dkey_own[8][kMaxD];
    float* own = dkey_own[warp];
    for (int q = lane; q < D; q += 32) own[q] = 0.f;
    const bf16* Pi = P + ((size_t)b * a.T + i) * D;
    float pv[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) pv[k] = lane + 32 * k < D ? __bfloat162float(Pi[lane + 32 * k]) : 0.f;
    for (int h = warp; h < sh.H; h += nw) {
        const size_t row = ((size_t)b * a.T + i) * sh.H + h;
        const size_t srow = ((size_t)b * sh.H + h) * stats_pitch(a.T) + i;
        float qv[kPer], dv[kPer], e = 0.f, da = 0.f;
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            const int c = lane + 32 * k;
            qv[k] = c < D ? __bfloat162float(qt[row * D + c]) : 0.f;
            dv[k] = c < d_c ? __bfloat162float(dob[row * d_c + c]) : 0.f;
            e = fmaf(qv[k], pv[k], e);
            da = fmaf(dv[k], pv[k], da);
        }
        e = warp_sum(e);
        da = warp_sum(da);
        const float pr = exp2f(fmaf(e, scale_log2, -lse[srow]));
        const float sde = sh.scale * pr * (da - delta[srow]);
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            const int c = lane + 32 * k;
            if (c < D) {
                a.dqt[row * D + c] += sde * pv[k];
                own[c] += fmaf(sde, qv[k], pr * dv[k]);
            }
        }
    }
    __syncthreads();
    for (int q = threadIdx.x; q < D; q += blockDim.x) {
        float acc = 0.f;
        for (int v = 0; v < nw; ++v) acc += dkey_own[v][q];
        a.dP[((size_t)b * a.T + i) * D + q] = acc;
    }
}

struct BwdWs {
    size_t P, w, cache, qt, mrow, lrow, delta, dob, obar, dqt, dP, dF, total;
};

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
    const size_t wbytes = (size_t)sh.H * sh.d_h * sh.d_c * sizeof(float);
    cudaError_t e;
    if ((e = cudaMemsetAsync(g.dw_uk, 0, wbytes, st)) != cudaSuccess) return note_error("backward zero dW_UK", e);
    if ((e = cudaMemsetAsync(g.dw_uv, 0, wbytes, st)) != cudaSuccess) return note_error("backward zero dW_UV", e);
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
    const int64_t M = (int64_t)sh.B * T_len;
    k_bwd_weights<T, float><<<dim3((unsigned)((M + kWChunk - 1) / kWChunk), sh.H, sh.d_h / kWRows), 256, 0, st>>>(
        a, g.dw_uk, g.dw_uv);
    k_bwd_scan<T><<<dim3((n_slots + 7) / 8, sh.B), 256, 0, st>>>(a, pa.c, pa.kr, pa.gate_w, g.dc, g.dkr, g.dgate_w,
                                                                 g.dgate_b, g.dgate_in);
    *launches += 7;
    return note_error("backward launch", cudaGetLastError());
}

// ---------------------------------------------------------------- tensor-core path

struct BwdTcWs {
    size_t fwd, cache, out, lse, delta, obar, qt, w, dob, dqt, dF, dP, total;
};

Shape with_slots(const Shape& sh, int T) {
    Shape s2 = sh;
    s2.max_slots = (T + sh.s - 1) / sh.s;
    return s2;
}

BwdTcWs bwd_tc_layout(const Shape& sh_in, int T) {
    const Shape sh = with_slots(sh_in, T);
    const size_t BT = (size_t)sh.B * T, rows = BT * sh.H;
    BwdTcWs l;
    size_t o = 0;
    auto take = [&](size_t bytes) { size_t at = o; o += align256(bytes); return at; };
    l.fwd = take(tc_prefill_workspace(sh, T));            // its first region: the partial slots P (bf16)
    l.cache = take((size_t)sh.B * sh.max_slots * sh.D * 2);
    l.out = take(rows * sh.d_h * 2);
    l.lse = take((size_t)sh.B * sh.H * stats_pitch(T) * 4);
    l.delta = take((size_t)sh.B * sh.H * stats_pitch(T) * 4);
    l.obar = take(rows * sh.d_c * 2);
    l.qt = take(rows * sh.D * 2);
    l.w = take(BT * 4);
    l.dob = take(rows * sh.d_c * 2);
    l.dqt = take(rows * sh.D * 4);
    l.dF = take((size_t)sh.H * sh.B * sh.max_slots * sh.D * 4);
    l.dP = take(BT * sh.D * 4);
    l.total = o;
    return l;
}

bool use_tc(const Shape& sh, bool fp32) {
    return !fp32 && tc_backward_supported(sh) && tc_prefill_supported(sh);
}

// bf16 at the tensor-core prefill's widths: the forward recomputed on the
// tensor cores keeping its rows' statistics, dobar and delta, the finished-
// slot parts on the tensor cores, the own-partial term, then the same query,
// weight and scan/gate backward as the CUDA-core path (dF summed over heads).
cudaError_t backward_tc(const PrefillArgs& pa_in, const BackwardGrads& g, cudaStream_t st, uint64_t* launches) {
    const int T_len = pa_in.T;
    PrefillArgs pa = pa_in;
    pa.sh = with_slots(pa_in.sh, T_len);
    const Shape sh = pa.sh;
    const int n_slots = sh.max_slots;
    char* ws = (char*)pa.workspace;
    const BwdTcWs l = bwd_tc_layout(sh, T_len);
    pa.workspace = ws + l.fwd;
    pa.workspace_bytes = tc_prefill_workspace(sh, T_len);
    pa.cache_out = ws + l.cache;
    pa.out = ws + l.out;
    pa.open_slot_in = nullptr;
    pa.open_slot_out = nullptr;
    pa.t0 = 0;
    const size_t wbytes = (size_t)sh.H * sh.d_h * sh.d_c * sizeof(float);
    cudaError_t e;
    if ((e = cudaMemsetAsync(g.dw_uk, 0, wbytes, st)) != cudaSuccess) return note_error("backward zero dW_UK", e);
    if ((e = cudaMemsetAsync(g.dw_uv, 0, wbytes, st)) != cudaSuccess) return note_error("backward zero dW_UV", e);
    if (sh.gate_mode == 0) {
        if ((e = cudaMemsetAsync(g.dgate_w, 0, (size_t)sh.s * sh.d_c * sizeof(float), st)) != cudaSuccess)
            return note_error("backward zero dG", e);
        if ((e = cudaMemsetAsync(g.dgate_b, 0, (size_t)sh.s * sizeof(float), st)) != cudaSuccess)
            return note_error("backward zero dg", e);
    }
    PrefillSave sv;
    sv.w = (float*)(ws + l.w);
    sv.lse = (float*)(ws + l.lse);
    sv.obar = ws + l.obar;
    sv.qt = ws + l.qt;
    if ((e = tc_prefill_save(pa, sv, st, launches)) != cudaSuccess) return e;
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
    a.w = (const float*)(ws + l.w);
    a.mrow = a.lrow = a.delta = nullptr;
    a.dob = nullptr;
    a.obar = ws + l.obar;
    a.dqt = (float*)(ws + l.dqt);
    a.dP = (float*)(ws + l.dP);
    a.dF = (float*)(ws + l.dF);
    a.n_parts = sh.H;
    const int threads = 32 * (sh.H < 8 ? sh.H : 8);
    k_bwd_dob<bf16><<<dim3((T_len + 15) / 16, sh.H, sh.B), 256, 0, st>>>(a, (bf16*)(ws + l.dob),
                                                                          (float*)(ws + l.delta));
    if ((e = cudaGetLastError()) != cudaSuccess) return note_error("k_bwd_dob launch", e);
    BwdTCInputs in;
    in.qt = ws + l.qt;
    in.dob = ws + l.dob;
    in.slots = ws + l.cache;
    in.lse = (const float*)(ws + l.lse);
    in.delta = (const float*)(ws + l.delta);
    in.dqt = a.dqt;
    in.dF = a.dF;
    in.status = pa.status;
    profile_begin(st);
    e = tc_backward_attention(sh, T_len, in, st, launches);
    profile_end(st);
    if (e != cudaSuccess) return e;
    k_bwd_own<<<dim3(T_len, sh.B), threads, 0, st>>>(a, (const bf16*)(ws + l.qt), (const bf16*)(ws + l.fwd),
                                                      (const bf16*)(ws + l.dob), in.lse, in.delta);
    k_bwd_query<bf16><<<dim3(T_len, sh.B), threads, 0, st>>>(a, g.dq_c, g.dq_r);
    const int64_t M = (int64_t)sh.B * T_len;
    k_bwd_weights<bf16, bf16><<<dim3((unsigned)((M + kWChunk - 1) / kWChunk), sh.H, sh.d_h / kWRows), 256, 0, st>>>(
        a, g.dw_uk, g.dw_uv);
    k_bwd_scan<bf16><<<dim3((n_slots + 7) / 8, sh.B), 256, 0, st>>>(a, pa.c, pa.kr, pa.gate_w, g.dc, g.dkr,
                                                                    g.dgate_w, g.dgate_b, g.dgate_in);
    *launches += 5;
    return note_error("backward launch", cudaGetLastError());
}

}  // namespace

size_t prefill_backward_workspace(const Shape& sh, int T, size_t elem_bytes) {
    return use_tc(sh, elem_bytes == 4) ? bwd_tc_layout(sh, T).total : bwd_layout(sh, T, elem_bytes).total;
}

cudaError_t prefill_backward(const PrefillArgs& a, const BackwardGrads& g, bool fp32, cudaStream_t st,
                             uint64_t* launches) {
    if (use_tc(a.sh, fp32)) return backward_tc(a, g, st, launches);
    return fp32 ? backward_impl<float>(a, g, st, launches) : backward_impl<bf16>(a, g, st, launches);
}

}  // namespace mtla
