// tc_decode.cu -- bf16 decode step on the 5th-generation tensor cores.
//
// "Multi-head Temporal Latent Attention", Method: at inference only every
// s-th step opens a slot and the steps in between update the slot being
// filled in place; the query attends all slots 0..floor(t/s) in the absorbed
// form (W_UK folded into the query, W_UV applied after the weighted sum).
// Per-token decode work is O(N/s) slot reads (Sec. 6.1), so this kernel is a
// streaming read of the bf16 latent cache.
//
// Launches per step (the last two with programmatic dependent launch, so their
// prologues overlap the previous kernel's tail):
//   k_dec_prep_tc   gate, RoPE, in-place slot update; absorbed queries written
//                   as a bf16 image already in the attention's SW128 layout
//   k_dec_attn_sh   split-K attention over slot tiles (tcgen05 + TMEM + TMA)
//   k_dec_combine   merge of the split partials and W_UV
//
// k_dec_attn_sh (heads <= 32; "swap-AB" so the 128 slots of a tile are the
// MMA's M dimension and the heads its N):
//   S^T[slot, h]   = K_tile[slot, :] . q~[h, :]         (A = slot tile, K-major)
//   O^T[lat, h]   += V^T[lat, slot] . P^T[slot, h]      (A = same tile, MN-major)
// The slot tile [128 x D] arrives by TMA in 64-column SW128 boxes and serves
// as both operands; S^T and O^T live in TMEM; one thread per slot row runs
// the online softmax (tile max per head across the block, exp2, fp32 sums).
// The grid is balanced over slot tiles: CTA g takes the global tiles
// [g*total/G, (g+1)*total/G), crossing sequence boundaries, and writes one
// partial (o, m, l) per sequence segment at index g + b.
#include <cudaTypedefs.h>

#include <cstdio>
#include <mutex>
#include <utility>

#include "common.cuh"
#include "mtla_internal.h"
#include "prep.cuh"
#include "tc_common.cuh"

namespace mtla {

namespace {

using namespace tc;

constexpr int kTileSlots = 128;
constexpr int kThreads = 128;
constexpr int kMaxGrid = 160;  // >= SMs of any sm_100 part; sizes the partial buffer
constexpr int kMaxB = 2048;
// S^T is accumulated in 4 independent TMEM accumulators (K-steps round robin)
// so that the chain of dependent MMAs is a quarter as long; the softmax adds them.
constexpr int kSAcc = 4;

struct DecTC {
    int B, H, D, d_c, s, max_slots;
    int n_chunks;    // D rounded up to 64, in 64-column chunks
    int lat_blocks;  // d_c / 128
    int G;           // grid size
    float scale_log2;
    const int32_t* pos;
    const uint8_t* qimg;  // [B] x n_chunks x [NH rows x 128 B]: q~ in bf16, SW128, zero padded
    uint32_t qimg_bytes;  // per sequence
    float* part;          // [(kMaxGrid + B), H, d_c + 2]
    int* status;
};

__device__ __forceinline__ int seq_tiles(const DecTC& p, int b) {
    const int64_t t = p.pos[b];
    if (t < 0 || t >= (int64_t)p.max_slots * p.s) return 0;
    const int n = (int)(t / p.s) + 1;
    return (n + kTileSlots - 1) / kTileSlots;
}
__device__ __forceinline__ int seq_slots(const DecTC& p, int b) {
    const int64_t t = p.pos[b];
    if (t < 0 || t >= (int64_t)p.max_slots * p.s) return 0;
    return (int)(t / p.s) + 1;
}

template <int NH>
struct Misc {
    uint64_t full[2];
    uint64_t bar_s;
    uint64_t bar_o;
    uint64_t bar_q;
    uint32_t tmem_base;
    int fail;
    int rescale;
    int total;
    float red[4][NH];
    float m_run[NH];
    float fac[NH];
};

// Decode prep for the tensor-core path. grid (B, H + 1), 128 threads.
// Block (b, h < H): absorbed query of head h, q~ = [W_UK[h]^T qC ; RoPE_t(qR)],
// rounded to bf16 into row h of sequence b's query image (64-column SW128
// chunks of NH rows, zero beyond D). Block (b, H): gate, RoPE and in-place
// update of the open slot (MTLA Method (1)), and zero rows H..NH-1 of the image.
__global__ void __launch_bounds__(128) k_dec_prep_tc(DecodeArgs a, uint8_t* qimg, int n_chunks, int NH) {
    pdl_launch_dependents();   // the attention kernel may start its prologue now
    const Shape& sh = a.sh;
    const int b = blockIdx.x, h = blockIdx.y;
    const uint32_t img_bytes = (uint32_t)n_chunks * NH * 128;
    uint8_t* img = qimg + (size_t)b * img_bytes;
    if (h == sh.H) {
        decode_update_body<bf16>(a, b);
        for (int e = threadIdx.x; e < n_chunks * (NH - sh.H) * 8; e += blockDim.x) {
            const int c = e / ((NH - sh.H) * 8), rr = e % ((NH - sh.H) * 8);
            *(uint4*)(img + (size_t)c * NH * 128 + (size_t)(sh.H + rr / 8) * 128 + (rr % 8) * 16) =
                make_uint4(0, 0, 0, 0);
        }
        return;
    }
    const int64_t t = a.pos[b];
    if (t < 0 || t >= (int64_t)sh.max_slots * sh.s) return;
    __shared__ float q[256];
    __shared__ float part_sum[8][512];     // [i-group][latent column]
    const size_t rh = (size_t)b * sh.H + h;
    const bf16* qc = (const bf16*)a.q_c + rh * sh.d_h;
    for (int i = threadIdx.x; i < sh.d_h; i += blockDim.x) q[i] = __bfloat162float(qc[i]);
    __syncthreads();
    // thread (ig, jg): 8 latent columns [8 jg, 8 jg + 8) over rows i of group ig;
    // all of its 16-byte loads of W_UK are issued before any product
    const bf16* W = (const bf16*)a.w_uk + (size_t)h * sh.d_h * sh.d_c;
    const int n_jg = sh.d_c / 8;
    const int n_ig = max(1, min(8, (int)blockDim.x / n_jg));
    const int rows_per = (sh.d_h + n_ig - 1) / n_ig;
    for (int e = threadIdx.x; e < n_ig * n_jg; e += blockDim.x) {
        const int ig = e / n_jg, jg = e % n_jg;
        const int i0 = ig * rows_per, i1 = min(sh.d_h, i0 + rows_per);
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int ib = i0; ib < i1; ib += 16) {
            uint4 raw[16];
#pragma unroll
            for (int u = 0; u < 16; ++u)
                if (ib + u < i1) raw[u] = *(const uint4*)(W + (size_t)(ib + u) * sh.d_c + jg * 8);
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                if (ib + u < i1) {
                    const bf16* wv = (const bf16*)&raw[u];
                    const float qi = q[ib + u];
#pragma unroll
                    for (int v = 0; v < 8; ++v) acc[v] = fmaf(__bfloat162float(wv[v]), qi, acc[v]);
                }
            }
        }
#pragma unroll
        for (int v = 0; v < 8; ++v) part_sum[ig][jg * 8 + v] = acc[v];
    }
    __syncthreads();
    const bf16* qr = (const bf16*)a.q_r + rh * sh.d_r;
    const int dpad = n_chunks * 64;
    for (int j = threadIdx.x; j < dpad; j += blockDim.x) {
        float v = 0.f;
        if (j < sh.d_c) {
            for (int ig = 0; ig < n_ig; ++ig) v += part_sum[ig][j];
        } else if (j < sh.D) {
            const int e = j - sh.d_c, k = e >> 1;
            float sn, cs;
            pair_sincos(t, k, sh.d_r, sh.log2_rope_base, &sn, &cs);
            const float x0 = __bfloat162float(qr[2 * k]), x1 = __bfloat162float(qr[2 * k + 1]);
            v = (e & 1) ? (x0 * sn + x1 * cs) : (x0 * cs - x1 * sn);
        }
        *(bf16*)(img + (size_t)(j >> 6) * NH * 128 + sw128_offset(h, j & 63)) = __float2bfloat16_rn(v);
    }
}

template <int NH>
__global__ void __launch_bounds__(kThreads, 1)
    k_dec_attn_sh(const __grid_constant__ CUtensorMap tmap, const DecTC p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_chunks = p.n_chunks;
    const uint32_t stage_bytes = (uint32_t)n_chunks * 16384u;
    uint8_t* stage_ptr[2] = {smem, smem + stage_bytes};
    uint8_t* q_s = smem + 2 * stage_bytes;                       // n_chunks x [NH x 128 B]
    uint8_t* p_s = q_s + (size_t)n_chunks * NH * 128;            // 2 x [NH x 128 B]
    Misc<NH>& m = *(Misc<NH>*)(p_s + 2 * NH * 128);
    int* starts = (int*)((uint8_t*)&m + ((sizeof(Misc<NH>) + 15) & ~(size_t)15));   // [B + 1]

    // ---- schedule: tiles per sequence and their exclusive prefix sum
    {
        const int per = (p.B + kThreads - 1) / kThreads;
        const int b0 = tid * per, b1 = min(b0 + per, p.B);
        int local = 0;
        for (int b = b0; b < b1; ++b) local += seq_tiles(p, b);
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        __shared__ int warp_tot[4];
        if (lane == 31) warp_tot[warp] = incl;
        __syncthreads();
        int off = 0;
        for (int w = 0; w < warp; ++w) off += warp_tot[w];
        int run = off + incl - local;
        for (int b = b0; b < b1; ++b) {
            starts[b] = run;
            run += seq_tiles(p, b);
        }
        if (tid == 0) {
            m.total = warp_tot[0] + warp_tot[1] + warp_tot[2] + warp_tot[3];
            starts[p.B] = m.total;
        }
    }
    // ---- barriers and TMEM
    const uint32_t tmem_cols_needed = (uint32_t)NH * (kSAcc + p.lat_blocks);
    uint32_t tmem_cols = 32;
    while (tmem_cols < tmem_cols_needed) tmem_cols <<= 1;
    if (tid == 0) {
        mbar_init(&m.full[0], 1);
        mbar_init(&m.full[1], 1);
        mbar_init(&m.bar_s, 1);
        mbar_init(&m.bar_o, 1);
        mbar_init(&m.bar_q, 1);
        m.fail = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmap);
    }
    pdl_launch_dependents();
    if (warp == 0) {
        tmem_alloc(&m.tmem_base, tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = m.tmem_base;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const uint32_t t_s = tmem;                // S^T: kSAcc partial sums of NH columns each
    const uint32_t t_o = tmem + kSAcc * NH;   // O^T: lat_blocks x NH columns

    const int total = m.total;
    const int g = blockIdx.x;
    const int gt0 = (int)(((int64_t)g * total) / p.G);
    const int gt1 = (int)(((int64_t)(g + 1) * total) / p.G);

    // global tile -> (sequence, tile within the sequence)
    auto locate = [&](int gt, int& b, int& j) {
        int lo = 0, hi = p.B - 1;        // largest b with starts[b] <= gt
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (starts[mid] <= gt) lo = mid; else hi = mid - 1;
        }
        b = lo;
        j = gt - starts[lo];
    };
    auto issue_load = [&](int gt, int stage) {
        int b, j;
        locate(gt, b, j);
        mbar_arrive_expect_tx(&m.full[stage], stage_bytes);
        for (int c = 0; c < n_chunks; ++c)
            tma_load_3d(stage_ptr[stage] + (size_t)c * 16384, &tmap, &m.full[stage], c * 64, j * kTileSlots, b);
    };

    const uint32_t idesc_s = idesc_bf16_f32(128, NH, false, false);
    const uint32_t idesc_o = idesc_bf16_f32(128, NH, true, false);

    // everything above only read pos; the cache row and q~ come from k_dec_prep_tc
    pdl_wait();
    int loads_issued = 0;
    if (tid == 0) {
        for (int k = 0; k < 2 && gt0 + k < gt1; ++k) {
            issue_load(gt0 + k, k);
            ++loads_issued;
        }
    }

    float l_part[NH];
    int seq_b = -1, seq_n = 0, q_phase = 0;
    bool first_o = true;
    bool failed = false;
    int it = 0;
    for (int gt = gt0; gt < gt1; ++gt, ++it) {
        int b, j;
        locate(gt, b, j);
        const int st = it & 1;
        if (b != seq_b) {
            // new segment: this sequence's query image (one bulk copy)
            seq_b = b;
            seq_n = seq_slots(p, b);
            first_o = true;
            if (tid == 0) {
                mbar_arrive_expect_tx(&m.bar_q, p.qimg_bytes);
                bulk_load(q_s, p.qimg + (size_t)b * p.qimg_bytes, p.qimg_bytes, &m.bar_q);
            }
            if (!mbar_wait(&m.bar_q, q_phase & 1)) m.fail = 1;
            ++q_phase;
            if (tid < NH) m.m_run[tid] = -INFINITY;
#pragma unroll
            for (int h = 0; h < NH; ++h) l_part[h] = 0.f;
        }
        // (1) previous PV done: its stage takes the tile after this one
        if (it > 0) {
            if (!mbar_wait(&m.bar_o, (it - 1) & 1)) m.fail = 1;
            if (tid == 0 && !m.fail && gt + 1 < gt1) {
                issue_load(gt + 1, (it + 1) & 1);
                ++loads_issued;
            }
        }
        // (2) this tile's slots
        if (!mbar_wait(&m.full[st], (it >> 1) & 1)) m.fail = 1;
        const int valid = min(kTileSlots, seq_n - j * kTileSlots);
        if (valid < kTileSlots && tid >= valid) {
            // stale rows past the sequence's last slot must not reach P.V
            for (int c = 0; c < n_chunks; ++c) {
                uint4* row = (uint4*)(stage_ptr[st] + (size_t)c * 16384 + (size_t)tid * 128);
#pragma unroll
                for (int u = 0; u < 8; ++u) row[u] = make_uint4(0, 0, 0, 0);
            }
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (m.fail) { failed = true; break; }
        // (3) S^T = K_tile . q~^T
        if (tid == 0) {
            const uint32_t a0 = smem_u32(stage_ptr[st]);
            const uint32_t b0 = smem_u32(q_s);
            for (int c = 0; c < n_chunks; ++c)
                for (int kk = 0; kk < 4; ++kk) {
                    const int step = c * 4 + kk;
                    const uint64_t ad = sdesc_sw128(a0 + c * 16384 + kk * 32, 16, 1024);
                    const uint64_t bd = sdesc_sw128(b0 + c * NH * 128 + kk * 32, 16, 1024);
                    umma_bf16(t_s + (step % kSAcc) * NH, ad, bd, idesc_s, step >= kSAcc);
                }
            umma_commit(&m.bar_s);
        }
        if (!mbar_wait(&m.bar_s, it & 1)) m.fail = 1;
        tc_fence_after();
        // (4) online softmax, thread = slot row
        float sv[NH];
        {
            float part[kSAcc][NH];
#pragma unroll
            for (int q = 0; q < kSAcc; ++q) {
                tmem_ld16(t_s + q * NH + lane_off, part[q]);
                if (NH == 32) tmem_ld16(t_s + q * NH + lane_off + 16, part[q] + 16);
            }
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < NH; ++h) sv[h] = (part[0][h] + part[1][h]) + (part[2][h] + part[3][h]);
        }
        const bool row_ok = tid < valid;
#pragma unroll
        for (int h = 0; h < NH; ++h) sv[h] = row_ok ? sv[h] * p.scale_log2 : -INFINITY;
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            if (h < p.H) {
                const float mx = warp_max(sv[h]);
                if (lane == 0) m.red[warp][h] = mx;
            }
        }
        __syncthreads();
        if (tid < p.H) {
            const float tile_max = fmaxf(fmaxf(m.red[0][tid], m.red[1][tid]), fmaxf(m.red[2][tid], m.red[3][tid]));
            const float old = m.m_run[tid];
            const float nm = fmaxf(old, tile_max);
            m.fac[tid] = (old == -INFINITY) ? 0.f : exp2f(old - nm);
            m.m_run[tid] = nm;
        }
        if (tid == 0) m.rescale = 0;
        __syncthreads();
        if (tid < p.H && m.fac[tid] != 1.f && !first_o) m.rescale = 1;
        float pv[NH];
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            pv[h] = 0.f;
            if (h < p.H) {
                pv[h] = exp2f(sv[h] - m.m_run[h]);
                l_part[h] = l_part[h] * m.fac[h] + pv[h];
            }
        }
        // P^T into shared memory as the K-major B operand [NH x 128 slots]
        {
            uint8_t* pc = p_s + (size_t)(tid >> 6) * NH * 128;
#pragma unroll
            for (int h = 0; h < NH; ++h) *(bf16*)(pc + sw128_offset(h, tid & 63)) = __float2bfloat16_rn(pv[h]);
        }
        fence_proxy_async();
        __syncthreads();
        // (5) rescale the running O^T where a head's max moved
        if (m.rescale) {
            for (int lb = 0; lb < p.lat_blocks; ++lb) {
                float ov[NH];
                const uint32_t ta = t_o + lb * NH + lane_off;
                tmem_ld16(ta, ov);
                if (NH == 32) tmem_ld16(ta + 16, ov + 16);
                tmem_wait_ld();
#pragma unroll
                for (int h = 0; h < NH; ++h) ov[h] *= m.fac[h];
                tmem_st16(ta, ov);
                if (NH == 32) tmem_st16(ta + 16, ov + 16);
            }
            tmem_wait_st();
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // (6) O^T += V^T . P^T
        if (tid == 0) {
            const uint32_t a0 = smem_u32(stage_ptr[st]);
            const uint32_t b0 = smem_u32(p_s);
            for (int lb = 0; lb < p.lat_blocks; ++lb)
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t ad = sdesc_sw128(a0 + (2 * lb) * 16384 + kk * 2048, 16384, 1024);
                    const uint64_t bd = sdesc_sw128(b0 + (kk >> 2) * NH * 128 + (kk & 3) * 32, 16, 1024);
                    umma_bf16(t_o + lb * NH, ad, bd, idesc_o, (first_o && kk == 0) ? 0u : 1u);
                }
            umma_commit(&m.bar_o);
        }
        first_o = false;
        // (7) end of this sequence's segment: write the partial (o, m, l)
        const bool seg_end = (gt + 1 == gt1) || (j + 1 == starts[b + 1] - starts[b]);
        if (seg_end) {
            if (!mbar_wait(&m.bar_o, it & 1)) m.fail = 1;
            tc_fence_after();
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                if (h < p.H) {
                    const float sum = warp_sum(l_part[h]);
                    if (lane == 0) m.red[warp][h] = sum;
                }
            }
            __syncthreads();
            if (m.fail) { failed = true; break; }
            float* dst = p.part + (size_t)(g + b) * p.H * (p.d_c + 2);
            for (int lb = 0; lb < p.lat_blocks; ++lb) {
                float ov[NH];
                const uint32_t ta = t_o + lb * NH + lane_off;
                tmem_ld16(ta, ov);
                if (NH == 32) tmem_ld16(ta + 16, ov + 16);
                tmem_wait_ld();
#pragma unroll
                for (int h = 0; h < NH; ++h)
                    if (h < p.H) dst[(size_t)h * (p.d_c + 2) + lb * 128 + tid] = ov[h];
            }
            if (tid < p.H) {
                dst[(size_t)tid * (p.d_c + 2) + p.d_c] = m.m_run[tid];
                dst[(size_t)tid * (p.d_c + 2) + p.d_c + 1] =
                    m.red[0][tid] + m.red[1][tid] + m.red[2][tid] + m.red[3][tid];
            }
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
        }
    }
    if (failed) {
        // drain what is still in flight (bounded), then report
        if (tid == 0) {
            latch_status(p.status, kStatusTimeout);
            for (int k = it; k < loads_issued && k < it + 2; ++k) mbar_wait(&m.full[k & 1], (k >> 1) & 1);
            mbar_wait(&m.bar_s, it & 1);
            if (it > 0) mbar_wait(&m.bar_o, (it - 1) & 1);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, tmem_cols);
}

// Merge the partials of (b, h) and apply W_UV. grid (H, B), 256 threads.
// W_UV[h] is staged in shared memory before the wait for the attention kernel;
// after it, every partial value this block needs is read in one round.
__global__ void __launch_bounds__(256) k_dec_combine(DecodeArgs a, DecTC p) {
    const int h = blockIdx.x, b = blockIdx.y;
    const Shape& sh = a.sh;
    if (seq_tiles(p, b) == 0) return;
    __shared__ float red[32];
    __shared__ int idx[kMaxGrid];
    __shared__ int n_part;
    __shared__ float olat[512];
    extern __shared__ uint8_t dyn[];
    bf16* Ws = (bf16*)dyn;                            // W_UV[h] [d_h x d_c]
    {
        const uint4* src = (const uint4*)((const bf16*)a.w_uv + (size_t)h * sh.d_h * sh.d_c);
        uint4* dst = (uint4*)Ws;
        const int n16 = sh.d_h * sh.d_c / 8;
        for (int e = threadIdx.x; e < n16; e += blockDim.x) dst[e] = src[e];
    }
    // this sequence's tile range and the total
    int before = 0, all = 0;
    for (int bb = threadIdx.x; bb < p.B; bb += blockDim.x) {
        const int t = seq_tiles(p, bb);
        all += t;
        if (bb < b) before += t;
    }
    const int S_b = (int)block_sum((float)before, red);
    const int total = (int)block_sum((float)all, red);
    const int E_b = S_b + seq_tiles(p, b);
    if (threadIdx.x == 0) {
        // CTA g covers tiles [lo(g), lo(g+1)) with lo(g) = floor(g*total/G). The
        // CTAs touching [S_b, E_b) are g_first..g_last, the largest g with
        // lo(g) <= S_b and lo(g) <= E_b - 1: g = ceil((x+1)*G/total) - 1 for x.
        const int64_t G = p.G, tot = total;
        const int g_first = (int)(((int64_t)(S_b + 1) * G + tot - 1) / tot) - 1;
        const int g_last = (int)(((int64_t)E_b * G + tot - 1) / tot) - 1;
        int n = 0;
        int64_t lo = ((int64_t)g_first * tot) / G;
        for (int g = g_first; g <= g_last; ++g) {
            const int64_t hi = ((int64_t)(g + 1) * tot) / G;
            if (hi > lo) idx[n++] = g + b;
            lo = hi;
        }
        n_part = n;
    }
    __syncthreads();
    pdl_wait();   // the partials come from k_dec_attn_sh
    const int n = n_part;
    const size_t stride = (size_t)p.H * (p.d_c + 2);
    const size_t hoff = (size_t)h * (p.d_c + 2);
    for (int jj = threadIdx.x; jj < p.d_c; jj += blockDim.x) {
        // one round of loads: (m, l, o[jj]) of every partial
        float mk[8], lk[8], ok[8];
        float M = -INFINITY, L = 0.f, acc = 0.f;
        for (int k0 = 0; k0 < n; k0 += 8) {
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (k0 + u < n) {
                    const float* e = p.part + idx[k0 + u] * stride + hoff;
                    mk[u] = e[p.d_c];
                    lk[u] = e[p.d_c + 1];
                    ok[u] = e[jj];
                }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (k0 + u < n) {
                    const float Mn = fmaxf(M, mk[u]);
                    const float c0 = exp2f(M - Mn), c1 = exp2f(mk[u] - Mn);
                    L = L * c0 + lk[u] * c1;
                    acc = acc * c0 + ok[u] * c1;
                    M = Mn;
                }
            }
        }
        olat[jj] = acc / L;
    }
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    bf16* out = (bf16*)a.out + ((size_t)b * sh.H + h) * sh.d_h;
    for (int i = warp; i < sh.d_h; i += 8) {
        float acc = 0.f;
        const bf16* Wi = Ws + (size_t)i * sh.d_c;
        for (int c0 = lane * 8; c0 < sh.d_c; c0 += 256) {
            const uint4 raw = *(const uint4*)(Wi + c0);
            const bf16* wv = (const bf16*)&raw;
#pragma unroll
            for (int v = 0; v < 8; ++v) acc = fmaf(__bfloat162float(wv[v]), olat[c0 + v], acc);
        }
        acc = warp_sum(acc);
        if (lane == 0) out[i] = __float2bfloat16_rn(acc);
    }
}

// ---------------------------------------------------------------- host side

int n_chunks_of(const Shape& sh) { return (sh.D + 63) / 64; }

size_t attn_smem_bytes(const Shape& sh, int NH) {
    const size_t nc = n_chunks_of(sh);
    size_t bytes = 1024;                          // alignment slack
    bytes += 2 * nc * 16384;                      // two stages
    bytes += nc * NH * 128;                       // q~
    bytes += 2 * NH * 128;                        // P^T
    bytes += 256 + 4 * (size_t)NH * 4 + 2 * (size_t)NH * 4;   // barriers, reductions
    bytes += ((size_t)sh.B + 1) * 4 + 16;         // tile prefix sums
    return bytes;
}

// Opt the kernel into `smem` bytes of dynamic shared memory (once per device
// and size); fails if the device cannot give that much next to the kernel's
// static shared memory.
template <typename K>
cudaError_t ensure_smem(K kernel, size_t smem, size_t* done) {
    if (*done >= smem) return cudaSuccess;
    int dev = 0, optin = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return e;
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kernel);
    if (e != cudaSuccess) return e;
    if (smem + fa.sharedSizeBytes > (size_t)optin) return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) *done = smem;
    return e;
}

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel in the stream finishes; it waits (griddepcontrol.wait)
// before it reads that kernel's results.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <int NH>
cudaError_t launch_attn(const CUtensorMap& map, const DecTC& p, size_t smem, cudaStream_t st) {
    static size_t done[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    cudaError_t e = ensure_smem(k_dec_attn_sh<NH>, smem, &done[dev]);
    if (e != cudaSuccess) return note_error("cudaFuncSetAttribute(k_dec_attn_sh)", e);
    return note_error("k_dec_attn_sh launch", launch_pdl(k_dec_attn_sh<NH>, dim3(p.G), dim3(kThreads), smem, st, map, p));
}

}  // namespace

void* tensor_map_encoder() {
    static void* fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = ptr;
    });
    return fn;
}

int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

bool tc_decode_supported(const Shape& sh) {
    return sh.H <= 32 && sh.d_c % 128 == 0 && n_chunks_of(sh) <= 6 && sh.B <= kMaxB &&
           (size_t)sh.d_h * sh.d_c * sizeof(bf16) <= 160 * 1024 &&
           attn_smem_bytes(sh, sh.H <= 16 ? 16 : 32) <= 232448 - 1024;
}

static uint32_t qimg_bytes(const Shape& sh) {
    return (uint32_t)n_chunks_of(sh) * (sh.H <= 16 ? 16 : 32) * 128;
}

size_t tc_decode_workspace(const Shape& sh) {
    return align256((size_t)sh.B * qimg_bytes(sh)) +
           align256((size_t)(kMaxGrid + sh.B) * sh.H * (sh.d_c + 2) * sizeof(float));
}

cudaError_t tc_decode(const DecodeArgs& a, cudaStream_t st, uint64_t* launches) {
    const Shape& sh = a.sh;
    char* ws = (char*)a.workspace;
    uint8_t* qimg = (uint8_t*)ws;
    float* part = (float*)(ws + align256((size_t)sh.B * qimg_bytes(sh)));
    const int NH = sh.H <= 16 ? 16 : 32;

    auto encode = (PFN_cuTensorMapEncodeTiled_v12000)tensor_map_encoder();
    if (!encode) return note_error("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", cudaErrorNotSupported);
    CUtensorMap map;
    cuuint64_t dims[3] = {(cuuint64_t)sh.D, (cuuint64_t)sh.max_slots, (cuuint64_t)sh.B};
    cuuint64_t strides[2] = {(cuuint64_t)sh.D * 2, (cuuint64_t)sh.max_slots * sh.D * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)kTileSlots, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.cache, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        char buf[96];
        snprintf(buf, sizeof(buf), "cuTensorMapEncodeTiled (CUresult %d)", (int)r);
        return note_error(buf, cudaErrorInvalidValue);
    }

    DecTC p;
    p.B = sh.B;
    p.H = sh.H;
    p.D = sh.D;
    p.d_c = sh.d_c;
    p.s = sh.s;
    p.max_slots = sh.max_slots;
    p.n_chunks = n_chunks_of(sh);
    p.lat_blocks = sh.d_c / 128;
    const int64_t max_tiles = (int64_t)sh.B * ((sh.max_slots + kTileSlots - 1) / kTileSlots);
    p.G = (int)std::min<int64_t>(std::min(sm_count(), kMaxGrid), max_tiles);
    p.scale_log2 = sh.scale * 1.4426950408889634f;
    p.pos = a.pos;
    p.qimg = qimg;
    p.qimg_bytes = qimg_bytes(sh);
    p.part = part;
    p.status = a.status;

    {
        // keep the SMs in the max-shared-memory configuration across the
        // three kernels of a step (no carve-out switch between them)
        static bool carve[64] = {false};
        int dev = 0;
        cudaGetDevice(&dev);
        if (dev >= 0 && dev < 64 && !carve[dev]) {
            cudaFuncSetAttribute(k_dec_prep_tc, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
            cudaFuncSetAttribute(k_dec_combine, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
            cudaGetLastError();
            carve[dev] = true;
        }
    }
    k_dec_prep_tc<<<dim3(sh.B, sh.H + 1), 128, 0, st>>>(a, qimg, p.n_chunks, NH);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return note_error("k_dec_prep_tc launch", e);
    const size_t smem = attn_smem_bytes(sh, NH);
    profile_begin(st);
    e = NH == 16 ? launch_attn<16>(map, p, smem, st) : launch_attn<32>(map, p, smem, st);
    profile_end(st);
    if (e != cudaSuccess) return e;
    const size_t comb_smem = (size_t)sh.d_h * sh.d_c * sizeof(bf16);
    {
        static size_t done[64] = {0};
        int dev = 0;
        cudaGetDevice(&dev);
        if (dev < 0 || dev >= 64) dev = 0;
        e = ensure_smem(k_dec_combine, comb_smem, &done[dev]);
        if (e != cudaSuccess) return note_error("cudaFuncSetAttribute(k_dec_combine)", e);
    }
    e = launch_pdl(k_dec_combine, dim3(sh.H, sh.B), dim3(256), comb_smem, st, a, p);
    *launches += 3;
    return note_error("k_dec_combine launch", e);
}

}  // namespace mtla
