// tc_decode_lh.cu -- bf16 decode step for many heads (32 < H <= 128) on the
// tensor cores: all heads form the M = 128 dimension of the contraction.
//
// "Multi-head Temporal Latent Attention", Method (1): one new token per
// sequence updates the slot being filled in place, then the absorbed query of
// every head attends slots 0..floor(t/s) (Sec. 6.1: O(N/s) slot reads). The
// latent cache is streamed once from HBM.
//
// The output accumulator O [128 heads x d_c] fp32 fills the whole tensor
// memory at d_c = 512, so the work of a slot range is split over a cluster of
// two CTAs by slot columns: CTA 0 holds latent columns [0, d_c/2) plus the
// RoPE part, CTA 1 latent columns [d_c/2, d_c). Each CTA
//   - loads only its columns of every 64-slot tile (TMA, no duplication),
//   - computes its partial scores S_c = q~_c . K_c^T       (M=128, N=64),
//   - sends S_c to the peer through distributed shared memory and adds the
//     peer's part, so both hold S and run the same softmax (thread per head),
//   - accumulates its half O_c += P . V_c                 (M=128, N=d_c/2),
// Tensor memory per CTA: O_c (d_c/2 columns) + two S buffers (64 each).
//
// Launches per step:
//   k_lh_prep      gate, RoPE and in-place slot update; absorbed queries for
//                  all heads, written as a bf16 SW128 image per sequence
//   k_lh_attn      the cluster kernel above, grid balanced over slot tiles,
//                  one partial (o, m, l) per sequence segment
//   k_lh_combine   merge of the partials and W_UV, one block per head
#include <cudaTypedefs.h>

#include <cstdio>
#include <utility>

#include <cuda_fp16.h>

#include "common.cuh"
#include "mtla_internal.h"
#include "prep.cuh"
#include "tc_common.cuh"

namespace mtla {

namespace {

using namespace tc;

constexpr int kKT = 64;          // slots per key tile
constexpr int kStages = 2;
constexpr int kThreads = 192;    // warp 0 TMA, warp 1 MMA, warps 2-5 softmax
constexpr int kMaxClusters = 80; // >= SMs/2 of any sm_100 part; sizes the partial buffer
constexpr int kMaxB = 2048;
constexpr float kRescaleLog2 = 8.f;

struct LhArgs {
    int B, H, D, d_c, d_r, s, max_slots;
    int G2;                 // clusters in the grid
    int n_qchunks;          // D / 64
    float scale_log2;
    const int32_t* pos;
    const uint8_t* qimg;    // [B] x n_qchunks x [128 heads x 128 B]
    float* part;            // [(kMaxClusters + B), H, d_c + 2]
    int* status;
};

__device__ __forceinline__ int lh_slots(const LhArgs& p, int b) {
    const int64_t t = p.pos[b];
    if (t < 0 || t >= (int64_t)p.max_slots * p.s) return 0;
    return (int)(t / p.s) + 1;
}
__device__ __forceinline__ int lh_tiles(const LhArgs& p, int b) { return (lh_slots(p, b) + kKT - 1) / kKT; }

// ---------------------------------------------------------------- prep

// Register-blocked product for one head, 32 sequences at a time, CUDA cores:
//   acc[i][jj] = sum_k X[k][b0 + i] * W[k][j0 + jj]     (i < BT, jj < 8)
// with X fp32 [K][32] and W bf16 [K][N] in shared memory. The 256 threads
// tile the [32 x N] output as (32 / BT) sequence groups x (N / 8) column
// groups, BT = N / 64 (N in {64, 128, 256, 512}).
template <int BT>
__device__ __forceinline__ void head_gemm_32(const float* X, const bf16* W, int K, int N, float (&acc)[BT][8],
                                             int& b0, int& j0) {
    const int n_jg = N / 8;
    const int t = threadIdx.x;
    j0 = 8 * (t % n_jg);
    b0 = BT * (t / n_jg);
#pragma unroll
    for (int i = 0; i < BT; ++i)
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) acc[i][jj] = 0.f;
    if (b0 >= 32) return;
    for (int k = 0; k < K; ++k) {
        const uint4 raw = *(const uint4*)(W + (size_t)k * N + j0);
        const bf16* w = (const bf16*)&raw;
        float wf[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) wf[jj] = __bfloat162float(w[jj]);
#pragma unroll
        for (int i = 0; i < BT; ++i) {
            const float x = X[k * 32 + b0 + i];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) acc[i][jj] = fmaf(x, wf[jj], acc[i][jj]);
        }
    }
}

__device__ __forceinline__ bool lh_pos_ok(const Shape& sh, int64_t t) {
    return t >= 0 && t < (int64_t)sh.max_slots * sh.s;
}

// grid (H), 256 threads. Block h: W_UK[h] staged by one bulk copy; for every
// 32 sequences, q~ = W_UK[h]^T qC[b, h] (latent part) by head_gemm_32 and
// RoPE_t(qR[b, h]) (rotated part), rounded to bf16 into row h of sequence b's
// image. Then the in-place slot updates of sequences b = h, h + H, ... (gate,
// RoPE, open slot; MTLA Method (1)) and the zero rows H..127 of their images.
__global__ void __launch_bounds__(256) k_lh_prep(DecodeArgs a, uint8_t* qimg, int n_qchunks) {
    pdl_launch_dependents();
    const Shape& sh = a.sh;
    const int h = blockIdx.x;
    const uint32_t img_bytes = (uint32_t)n_qchunks * 128 * 128;
    extern __shared__ uint8_t dyn[];
    bf16* Ws = (bf16*)dyn;                                                   // [d_h][d_c]
    float* X = (float*)(dyn + (size_t)sh.d_h * sh.d_c * sizeof(bf16));      // [d_h][32]
    uint64_t* bar = (uint64_t*)(X + (size_t)sh.d_h * 32);
    const uint32_t w_bytes = (uint32_t)sh.d_h * sh.d_c * sizeof(bf16);
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(bar, w_bytes);
        const uint8_t* src = (const uint8_t*)((const bf16*)a.w_uk + (size_t)h * sh.d_h * sh.d_c);
        for (uint32_t off = 0; off < w_bytes; off += 32768)
            bulk_load((uint8_t*)Ws + off, src + off, min(32768u, w_bytes - off), bar);
    }
    __syncthreads();
    bool w_ok = mbar_wait(bar, 0);
    if (!w_ok && threadIdx.x == 0) latch_status(a.status, kStatusTimeout);
    for (int c0 = 0; c0 < sh.B && w_ok; c0 += 32) {
        __syncthreads();                                          // X free
        for (int e = threadIdx.x; e < sh.d_h * 32; e += blockDim.x) {
            const int k = e / 32, bb = e % 32, b = c0 + bb;
            X[e] = b < sh.B ? __bfloat162float(((const bf16*)a.q_c)[((size_t)b * sh.H + h) * sh.d_h + k]) : 0.f;
        }
        __syncthreads();
        auto emit = [&](auto& acc, int b0, int j0, int bt) {
            for (int i = 0; i < bt; ++i) {
                const int b = c0 + b0 + i;
                if (b0 >= 32 || b >= sh.B || !lh_pos_ok(sh, a.pos[b])) continue;
                uint4 pk;
                pk.x = pack_bf16x2(acc[i][0], acc[i][1]);
                pk.y = pack_bf16x2(acc[i][2], acc[i][3]);
                pk.z = pack_bf16x2(acc[i][4], acc[i][5]);
                pk.w = pack_bf16x2(acc[i][6], acc[i][7]);
                *(uint4*)(qimg + (size_t)b * img_bytes + (size_t)(j0 >> 6) * 128 * 128 + sw128_offset(h, j0 & 63)) = pk;
            }
        };
        int b0, j0;
        if (sh.d_c == 512) { float acc[8][8]; head_gemm_32<8>(X, Ws, sh.d_h, sh.d_c, acc, b0, j0); emit(acc, b0, j0, 8); }
        else if (sh.d_c == 256) { float acc[4][8]; head_gemm_32<4>(X, Ws, sh.d_h, sh.d_c, acc, b0, j0); emit(acc, b0, j0, 4); }
        else { float acc[2][8]; head_gemm_32<2>(X, Ws, sh.d_h, sh.d_c, acc, b0, j0); emit(acc, b0, j0, 2); }
        // rotated part: columns [d_c, n_qchunks*64), zero past D
        const int nrot = n_qchunks * 64 - sh.d_c;
        for (int e = threadIdx.x; e < 32 * nrot; e += blockDim.x) {
            const int bb = e / nrot, jr = e % nrot, b = c0 + bb;
            if (b >= sh.B) continue;
            const int64_t t = a.pos[b];
            if (!lh_pos_ok(sh, t)) continue;
            float v = 0.f;
            if (jr < sh.d_r) {
                const bf16* qr = (const bf16*)a.q_r + ((size_t)b * sh.H + h) * sh.d_r;
                const int k = jr >> 1;
                float sn, cs;
                pair_sincos(t, k, sh.d_r, sh.log2_rope_base, &sn, &cs);
                const float x0 = __bfloat162float(qr[2 * k]), x1 = __bfloat162float(qr[2 * k + 1]);
                v = (jr & 1) ? (x0 * sn + x1 * cs) : (x0 * cs - x1 * sn);
            }
            const int j = sh.d_c + jr;
            *(bf16*)(qimg + (size_t)b * img_bytes + (size_t)(j >> 6) * 128 * 128 + sw128_offset(h, j & 63)) =
                __float2bfloat16_rn(v);
        }
    }
    for (int b = h; b < sh.B; b += sh.H) {
        __syncthreads();
        decode_update_body<bf16>(a, b);
        uint8_t* img = qimg + (size_t)b * img_bytes;
        const int pad_rows = 128 - sh.H;
        for (int e = threadIdx.x; e < n_qchunks * pad_rows * 8; e += blockDim.x) {
            const int c = e / (pad_rows * 8), rr = e % (pad_rows * 8);
            *(uint4*)(img + (size_t)c * 128 * 128 + (size_t)(sh.H + rr / 8) * 128 + (rr % 8) * 16) =
                make_uint4(0, 0, 0, 0);
        }
    }
}

// ---------------------------------------------------------------- attention

struct LhBars {
    uint64_t full[kStages], empty[kStages];
    uint64_t q_full, q_free;
    uint64_t s_full, s_empty;
    uint64_t p_full, o_done;
    uint64_t x_full, x_empty;
    uint32_t tmem_base;
    volatile int fail;
    int total;
};

__device__ __forceinline__ bool lh_wait(uint64_t* bar, uint32_t parity, LhBars& bs) {
    if (bs.fail) return false;
    if (mbar_wait(bar, parity)) return true;
    bs.fail = 1;
    return false;
}
__device__ __forceinline__ bool lh_wait_cluster(uint64_t* bar, uint32_t parity, LhBars& bs) {
    if (bs.fail) return false;
    if (mbar_wait_cluster(bar, parity)) return true;
    bs.fail = 1;
    return false;
}

// Chunk i of this CTA's slot columns -> 64-column chunk index of the slot.
__device__ __forceinline__ int lh_chunk_id(int rank, int i, int lat_chunks, int rope_first) {
    if (rank == 1) return lat_chunks + i;
    return i < lat_chunks ? i : rope_first + (i - lat_chunks);
}

// Exchange buffer: row r holds the 64 scaled partial scores of head r as fp16
// (128 B), its 16-byte units XOR-swizzled by r mod 8 (conflict-free access).
__device__ __forceinline__ uint32_t xoff(int r, int unit) { return (uint32_t)r * 128 + (((unit ^ r) & 7) << 4); }

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    k_lh_attn(const __grid_constant__ CUtensorMap tmap, const LhArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rank = (int)cluster_rank(), peer = rank ^ 1;
    const int g = blockIdx.x >> 1;                       // cluster index
    const int lat_half = p.d_c / 2, lat_chunks = lat_half / 64;
    const int rope_first = p.d_c / 64;                   // first chunk of the RoPE columns
    const int max_chunks = lat_chunks + (p.n_qchunks - rope_first);
    const int my_chunks = rank == 0 ? max_chunks : lat_chunks;
    const uint32_t stage_bytes = (uint32_t)max_chunks * kKT * 128;
    uint8_t* q_s = smem;                                             // max_chunks x [128 x 128 B]
    uint8_t* ring = q_s + (size_t)max_chunks * 128 * 128;            // kStages x stage_bytes
    uint8_t* p_s = ring + (size_t)kStages * stage_bytes;             // P [128 x 128 B]
    uint8_t* x_out = p_s + 128 * 128;                                // own scores, fp16 [128 x 128 B]
    uint8_t* x_in = x_out + 128 * 128;                               // peer scores, fp16 [128 x 128 B]
    LhBars& bs = *(LhBars*)(x_in + 128 * 128);
    int* starts = (int*)((uint8_t*)&bs + ((sizeof(LhBars) + 15) & ~(size_t)15));   // [B + 1]

    // ---- schedule over 64-slot tiles (reads pos only)
    {
        const int per = (p.B + kThreads - 1) / kThreads;
        const int b0 = tid * per, b1 = min(b0 + per, p.B);
        int local = 0;
        for (int b = b0; b < b1; ++b) local += lh_tiles(p, b);
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        __shared__ int warp_tot[kThreads / 32];
        if (lane == 31) warp_tot[warp] = incl;
        __syncthreads();
        int off = 0, tot = 0;
        for (int w = 0; w < kThreads / 32; ++w) {
            if (w < warp) off += warp_tot[w];
            tot += warp_tot[w];
        }
        int run = off + incl - local;
        for (int b = b0; b < b1; ++b) {
            starts[b] = run;
            run += lh_tiles(p, b);
        }
        if (tid == 0) {
            bs.total = tot;
            starts[p.B] = tot;
        }
    }
    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&bs.full[i], 1);
            mbar_init(&bs.empty[i], 1);
        }
        mbar_init(&bs.q_full, 1);
        mbar_init(&bs.q_free, 1);
        mbar_init(&bs.s_full, 1);
        mbar_init(&bs.s_empty, 4);
        mbar_init(&bs.p_full, 4);
        mbar_init(&bs.o_done, 1);
        mbar_init(&bs.x_full, 1);        // local expect_tx arrive; the peer's copy completes the bytes
        mbar_init(&bs.x_empty, 1);       // one remote arrive per tile from the peer
        bs.fail = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmap);
    }
    if (warp == 1) {
        tmem_alloc(&bs.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_sync();                      // peer barriers exist before any remote operation
    pdl_launch_dependents();
    const uint32_t tmem = bs.tmem_base;
    const uint32_t t_o = tmem;                         // O_c: columns [0, lat_half)
    const uint32_t t_s = tmem + 256;                   // S: 4 accumulators of 64 columns
    const int total = bs.total;
    const int gt0 = (int)(((int64_t)g * total) / p.G2);
    const int gt1 = (int)(((int64_t)(g + 1) * total) / p.G2);
    auto locate = [&](int gt, int& b, int& j) {
        int lo = 0, hi = p.B - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (starts[mid] <= gt) lo = mid; else hi = mid - 1;
        }
        b = lo;
        j = gt - starts[lo];
    };
    pdl_wait();                          // cache row and query image come from k_lh_prep

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int seg = -1, prev_b = -1;
            for (int gt = gt0, it = 0; gt < gt1; ++gt, ++it) {
                int b, j;
                locate(gt, b, j);
                if (b != prev_b) {
                    prev_b = b;
                    ++seg;
                    if (seg >= 1 && !lh_wait(&bs.q_free, (seg - 1) & 1, bs)) break;
                    mbar_arrive_expect_tx(&bs.q_full, (uint32_t)my_chunks * 128 * 128);
                    const uint8_t* src = p.qimg + (size_t)b * p.n_qchunks * 128 * 128;
                    for (int i = 0; i < my_chunks; ++i)
                        bulk_load(q_s + (size_t)i * 128 * 128,
                                  src + (size_t)lh_chunk_id(rank, i, lat_chunks, rope_first) * 128 * 128,
                                  128 * 128, &bs.q_full);
                }
                const int st = it % kStages;
                if (it >= kStages && !lh_wait(&bs.empty[st], ((it / kStages) - 1) & 1, bs)) break;
                mbar_arrive_expect_tx(&bs.full[st], (uint32_t)my_chunks * kKT * 128);
                for (int i = 0; i < my_chunks; ++i)
                    tma_load_3d(ring + st * stage_bytes + (size_t)i * kKT * 128, &tmap, &bs.full[st],
                                lh_chunk_id(rank, i, lat_chunks, rope_first) * 64, j * kKT, b);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issue
        if (lane == 0) {
            const uint32_t id_s = idesc_bf16_f32(128, kKT, false, false);
            const uint32_t id_o = idesc_bf16_f32(128, lat_half, false, true);
            const uint32_t ring_a = smem_u32(ring);
            const uint64_t q_d = sdesc_sw128(smem_u32(q_s), 16, 1024), p_d = sdesc_sw128(smem_u32(p_s), 16, 1024);
            int seg = -1, prev_b = -1;
            bool prev_first = true;          // first tile of its segment (for the pending P.V)
            bool ok = true;
            int it = 0;
            auto issue_pv = [&](int k, bool first) -> bool {
                if (!lh_wait(&bs.p_full, k & 1, bs)) return false;
                tc_fence_after();
                const uint64_t vd = sdesc_sw128(ring_a + (k % kStages) * stage_bytes, kKT * 128, 1024);
#pragma unroll
                for (int kk = 0; kk < kKT / 16; ++kk)
                    umma_bf16(t_o, desc_add(p_d, kk * 32), desc_add(vd, kk * 2048), id_o, (first && kk == 0) ? 0u : 1u);
                umma_commit(&bs.empty[k % kStages]);
                umma_commit(&bs.o_done);
                return true;
            };
            for (int gt = gt0; gt < gt1 && ok; ++gt, ++it) {
                int b, j;
                locate(gt, b, j);
                const bool first = (b != prev_b);
                if (first) {
                    prev_b = b;
                    ++seg;
                    if (!lh_wait(&bs.q_full, seg & 1, bs)) { ok = false; break; }
                }
                const int st = it % kStages;
                if (!lh_wait(&bs.full[st], (it / kStages) & 1, bs)) { ok = false; break; }
                if (it >= 1 && !lh_wait(&bs.s_empty, (it - 1) & 1, bs)) { ok = false; break; }
                tc_fence_after();
                // S_c = q~_c . K_c^T into 4 accumulators (K-steps round robin)
                const uint64_t kd = sdesc_sw128(ring_a + st * stage_bytes, 16, 1024);
                for (int i = 0; i < my_chunks; ++i) {
                    const uint64_t qi = desc_add(q_d, i * 128 * 128), ki = desc_add(kd, i * kKT * 128);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_bf16(t_s + kk * kKT, desc_add(qi, kk * 32), desc_add(ki, kk * 32), id_s, i > 0);
                }
                umma_commit(&bs.s_full);
                const bool last = (gt + 1 == gt1) || (j + 1 == starts[b + 1] - starts[b]);
                if (last) umma_commit(&bs.q_free);
                if (it >= 1 && !issue_pv(it - 1, prev_first)) { ok = false; break; }
                prev_first = first;
            }
            if (ok && it >= 1) issue_pv(it - 1, prev_first);
        }
    } else {
        // ------------------------------------------------------------ softmax (thread = head row)
        // No early exit: every softmax thread passes every named barrier even after a
        // bounded wait gave up (later waits then return at once), so none can hang.
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint32_t x_in_peer = map_to_rank(x_in, peer);
        const uint32_t xfull_peer = map_to_rank(&bs.x_full, peer);
        const uint32_t xempty_peer = map_to_rank(&bs.x_empty, peer);
        const bool leader = (tid == 64);
        float m_ref = -INFINITY, l = 0.f;
        int prev_b = -1, n_b = 0, k_in_seg = 0;
        for (int gt = gt0, it = 0; gt < gt1; ++gt, ++it) {
            int b, j;
            locate(gt, b, j);
            if (b != prev_b) {
                prev_b = b;
                n_b = lh_slots(p, b);
                m_ref = -INFINITY;
                l = 0.f;
                k_in_seg = 0;
            }
            const int st = it % kStages;
            const int valid = min(kKT, n_b - j * kKT);
            if (leader && !bs.fail) mbar_arrive_expect_tx(&bs.x_full, 128 * 128);   // peer's scores, this tile
            lh_wait(&bs.s_full, it & 1, bs);    // on a timeout: keep going, the status is latched
            tc_fence_after();
            float sv[kKT];
            {
                float tmp[32];
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    tmem_ld32(t_s + h2 * 32 + lane_off, sv + h2 * 32);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 1; q < 4; ++q) {
                        tmem_ld32(t_s + q * kKT + h2 * 32 + lane_off, tmp);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) sv[h2 * 32 + i] += tmp[i];
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bs.s_empty);
            // stale rows past the sequence's last slot must not reach P.V
            if (valid < kKT) {
                const int rows = kKT - valid;
                uint8_t* stg = ring + st * stage_bytes;
                for (int e = tid - 64; e < my_chunks * rows * 8; e += 128) {
                    const int i = e / (rows * 8), rr = e % (rows * 8);
                    *(uint4*)(stg + (size_t)i * kKT * 128 + (size_t)(valid + rr / 8) * 128 + (rr % 8) * 16) =
                        make_uint4(0, 0, 0, 0);
                }
            }
            // own scaled partial scores as fp16 (both CTAs use the rounded values)
            if (it >= 1 && leader) bulk_wait_read_all();    // x_out free again
            named_sync(1, 128);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                uint4 pk;
                __half2 h0 = __floats2half2_rn(sv[8 * u + 0] * p.scale_log2, sv[8 * u + 1] * p.scale_log2);
                __half2 h1 = __floats2half2_rn(sv[8 * u + 2] * p.scale_log2, sv[8 * u + 3] * p.scale_log2);
                __half2 h2 = __floats2half2_rn(sv[8 * u + 4] * p.scale_log2, sv[8 * u + 5] * p.scale_log2);
                __half2 h3 = __floats2half2_rn(sv[8 * u + 6] * p.scale_log2, sv[8 * u + 7] * p.scale_log2);
                pk.x = *(uint32_t*)&h0;
                pk.y = *(uint32_t*)&h1;
                pk.z = *(uint32_t*)&h2;
                pk.w = *(uint32_t*)&h3;
                *(uint4*)(x_out + xoff(r, u)) = pk;
            }
            fence_proxy_async();
            named_sync(1, 128);
            if (leader) {
                if (it == 0 || lh_wait_cluster(&bs.x_empty, (it - 1) & 1, bs)) {
                    bulk_copy_to_peer(x_in_peer, x_out, 128 * 128, xfull_peer);
                    bulk_commit_group();
                }
            }
            lh_wait_cluster(&bs.x_full, it & 1, bs);
            float mt = -INFINITY;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const uint4 mine = *(const uint4*)(x_out + xoff(r, u));
                const uint4 theirs = *(const uint4*)(x_in + xoff(r, u));
                const __half2* hm = (const __half2*)&mine;
                const __half2* ht = (const __half2*)&theirs;
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const float2 fm = __half22float2(hm[v]), ft = __half22float2(ht[v]);
                    const int c = 8 * u + 2 * v;
                    const float s0 = rank == 0 ? fm.x + ft.x : ft.x + fm.x;
                    const float s1 = rank == 0 ? fm.y + ft.y : ft.y + fm.y;
                    sv[c] = (c < valid) ? s0 : -INFINITY;
                    sv[c + 1] = (c + 1 < valid) ? s1 : -INFINITY;
                    mt = fmaxf(mt, fmaxf(sv[c], sv[c + 1]));
                }
            }
            named_sync(1, 128);                              // every row of x_in read
            if (leader) mbar_arrive_remote(xempty_peer);
            float m_new = m_ref, fac = 1.f;
            if (mt > m_ref + kRescaleLog2 || m_ref == -INFINITY) {
                m_new = mt;
                fac = (m_ref == -INFINITY) ? 0.f : exp2f(m_ref - mt);
            }
            float rs = 0.f;
#pragma unroll
            for (int c = 0; c < kKT; ++c) {
                sv[c] = exp2f(sv[c] - m_new);
                rs += sv[c];
            }
            l = l * fac + rs;
            if (it >= 1) {
                lh_wait(&bs.o_done, (it - 1) & 1, bs);
                tc_fence_after();
                if (k_in_seg > 0 && __any_sync(0xffffffffu, fac != 1.f)) {
                    float v[32];
                    for (int cc = 0; cc < lat_half / 32; ++cc) {
                        tmem_ld32(t_o + cc * 32 + lane_off, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] *= fac;
                        tmem_st32(t_o + cc * 32 + lane_off, v);
                    }
                    tmem_wait_st();
                }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                uint4 pk;
                pk.x = pack_bf16x2(sv[8 * u + 0], sv[8 * u + 1]);
                pk.y = pack_bf16x2(sv[8 * u + 2], sv[8 * u + 3]);
                pk.z = pack_bf16x2(sv[8 * u + 4], sv[8 * u + 5]);
                pk.w = pack_bf16x2(sv[8 * u + 6], sv[8 * u + 7]);
                *(uint4*)(p_s + sw128_offset(r, 8 * u)) = pk;
            }
            fence_proxy_async();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bs.p_full);
            m_ref = m_new;
            ++k_in_seg;
            const bool last = (gt + 1 == gt1) || (j + 1 == starts[b + 1] - starts[b]);
            if (last) {
                // partial of this sequence segment: this CTA's half of O, plus (m, l)
                lh_wait(&bs.o_done, it & 1, bs);
                tc_fence_after();
                const size_t row = (size_t)p.d_c + 4;
                float* dst = p.part + ((size_t)(g + b) * p.H + r) * row;
                float v[32];
                for (int cc = 0; cc < lat_half / 32; ++cc) {
                    tmem_ld32(t_o + cc * 32 + lane_off, v);
                    tmem_wait_ld();
                    if (r < p.H) {
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            *(float4*)(dst + rank * lat_half + cc * 32 + 4 * u) =
                                make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
                    }
                }
                if (rank == 0 && r < p.H) {
                    dst[p.d_c] = m_ref;
                    dst[p.d_c + 1] = l;
                }
                tc_fence_before();
            }
        }
        if (leader) bulk_wait_read_all();
    }
    if (bs.fail && (tid & 63) == 0) latch_status(p.status, kStatusTimeout);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
    cluster_sync();                      // the peer may still copy into / arrive on us until here
}

// ---------------------------------------------------------------- combine

// Exclusive prefix sum of the 64-slot tile counts of all sequences into
// starts[0..B] (starts[B] = total). All threads of the block call it.
__device__ void lh_tile_starts(const LhArgs& p, int* starts, int* warp_tot) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const int per = (p.B + blockDim.x - 1) / blockDim.x;
    const int b0 = tid * per, b1 = min(b0 + per, p.B);
    int local = 0;
    for (int b = b0; b < b1; ++b) local += lh_tiles(p, b);
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int off = 0, tot = 0;
    for (int w = 0; w < nw; ++w) {
        if (w < warp) off += warp_tot[w];
        tot += warp_tot[w];
    }
    int run = off + incl - local;
    for (int b = b0; b < b1; ++b) {
        starts[b] = run;
        run += lh_tiles(p, b);
    }
    if (tid == 0) starts[p.B] = tot;
    __syncthreads();
}

// grid (H), 256 threads. Block h: W_UV[h] staged transposed ([d_c][d_h]); for
// every 32 sequences, the partials of head h are merged by the online-softmax
// rule into o_lat [d_c][32], then out[b, h] = W_UV[h] o_lat[b] by head_gemm_32.
__global__ void __launch_bounds__(256) k_lh_combine(DecodeArgs a, LhArgs p) {
    const Shape& sh = a.sh;
    const int h = blockIdx.x;
    extern __shared__ uint8_t dyn[];
    bf16* Wt = (bf16*)dyn;                                                    // [d_c][d_h]
    float* X = (float*)(dyn + (size_t)sh.d_h * sh.d_c * sizeof(bf16));       // [d_c][32]
    int* idx = (int*)(X + (size_t)sh.d_c * 32);                               // [32][kMaxClusters]
    int* npart = idx + 32 * kMaxClusters;                                     // [32]
    int* starts = npart + 32;                                                 // [B + 1]
    float* wts = (float*)(starts + sh.B + 1);                                 // [32][kMaxClusters]
    __shared__ int warp_tot[8];
    __shared__ float invl[32];
    __shared__ int maxn_s;
    {
        // transpose W_UV[h] [d_h][d_c] into [d_c][d_h]; 8 loads in flight per thread
        const bf16* src = (const bf16*)a.w_uv + (size_t)h * sh.d_h * sh.d_c;
        const int n16 = sh.d_h * sh.d_c / 8;
        for (int e0 = threadIdx.x; e0 < n16; e0 += 8 * blockDim.x) {
            uint4 raw[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int e = e0 + u * blockDim.x;
                if (e < n16) raw[u] = *(const uint4*)(src + (size_t)e * 8);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int e = e0 + u * blockDim.x;
                if (e < n16) {
                    const int i = (e * 8) / sh.d_c, k0 = (e * 8) % sh.d_c;
                    const bf16* w = (const bf16*)&raw[u];
#pragma unroll
                    for (int v = 0; v < 8; ++v) Wt[(size_t)(k0 + v) * sh.d_h + i] = w[v];
                }
            }
        }
    }
    lh_tile_starts(p, starts, warp_tot);
    pdl_wait();                          // the partials come from k_lh_attn
    const int total = starts[p.B];
    const size_t row = (size_t)p.d_c + 4;
    for (int c0 = 0; c0 < sh.B; c0 += 32) {
        __syncthreads();                 // X, idx free
        if (threadIdx.x < 32) {
            const int b = c0 + threadIdx.x;
            int n = 0;
            if (b < sh.B && starts[b + 1] > starts[b] && total > 0) {
                const int S_b = starts[b], E_b = starts[b + 1];
                const int64_t G = p.G2, tot = total;
                const int g_first = (int)(((int64_t)(S_b + 1) * G + tot - 1) / tot) - 1;
                const int g_last = (int)(((int64_t)E_b * G + tot - 1) / tot) - 1;
                int64_t lo = ((int64_t)g_first * tot) / G;
                for (int gg = g_first; gg <= g_last; ++gg) {
                    const int64_t hi = ((int64_t)(gg + 1) * tot) / G;
                    if (hi > lo && n < kMaxClusters) idx[threadIdx.x * kMaxClusters + n++] = gg + b;
                    lo = hi;
                }
            }
            npart[threadIdx.x] = n;
            // merge weights 2^(m_i - M) and 1 / sum_i 2^(m_i - M) l_i
            float M = -INFINITY;
            for (int i = 0; i < n; ++i)
                M = fmaxf(M, p.part[((size_t)idx[threadIdx.x * kMaxClusters + i] * p.H + h) * row + p.d_c]);
            float L = 0.f;
            for (int i = 0; i < n; ++i) {
                const float* ep = p.part + ((size_t)idx[threadIdx.x * kMaxClusters + i] * p.H + h) * row;
                const float w = exp2f(ep[p.d_c] - M);
                wts[threadIdx.x * kMaxClusters + i] = w;
                L += w * ep[p.d_c + 1];
            }
            invl[threadIdx.x] = n > 0 ? 1.f / L : 0.f;
            int mx = n;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            if (threadIdx.x == 0) maxn_s = mx;
        }
        __syncthreads();
        // o_lat[k][bb] = sum_i w_i o_i[k] / L: 32 partial values in flight per round
        for (int k = threadIdx.x; k < sh.d_c; k += blockDim.x) {
            for (int g8 = 0; g8 < 4; ++g8) {
                float acc8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                for (int kk0 = 0; kk0 < maxn_s; kk0 += 4) {
                    float o[8][4];
#pragma unroll
                    for (int i = 0; i < 8; ++i)
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int bb = 8 * g8 + i;
                            o[i][u] = (kk0 + u < npart[bb])
                                          ? p.part[((size_t)idx[bb * kMaxClusters + kk0 + u] * p.H + h) * row + k]
                                          : 0.f;
                        }
#pragma unroll
                    for (int i = 0; i < 8; ++i)
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int bb = 8 * g8 + i;
                            if (kk0 + u < npart[bb]) acc8[i] = fmaf(wts[bb * kMaxClusters + kk0 + u], o[i][u], acc8[i]);
                        }
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) X[(size_t)k * 32 + 8 * g8 + i] = acc8[i] * invl[8 * g8 + i];
            }
        }
        __syncthreads();
        auto emit = [&](auto& acc, int b0, int j0, int bt) {
            for (int i = 0; i < bt; ++i) {
                const int b = c0 + b0 + i;
                if (b0 >= 32 || b >= sh.B || npart[b0 + i] == 0) continue;
                uint4 pk;
                pk.x = pack_bf16x2(acc[i][0], acc[i][1]);
                pk.y = pack_bf16x2(acc[i][2], acc[i][3]);
                pk.z = pack_bf16x2(acc[i][4], acc[i][5]);
                pk.w = pack_bf16x2(acc[i][6], acc[i][7]);
                *(uint4*)((bf16*)a.out + ((size_t)b * sh.H + h) * sh.d_h + j0) = pk;
            }
        };
        int b0, j0;
        if (sh.d_h == 512) { float acc[8][8]; head_gemm_32<8>(X, Wt, sh.d_c, sh.d_h, acc, b0, j0); emit(acc, b0, j0, 8); }
        else if (sh.d_h == 256) { float acc[4][8]; head_gemm_32<4>(X, Wt, sh.d_c, sh.d_h, acc, b0, j0); emit(acc, b0, j0, 4); }
        else if (sh.d_h == 128) { float acc[2][8]; head_gemm_32<2>(X, Wt, sh.d_c, sh.d_h, acc, b0, j0); emit(acc, b0, j0, 2); }
        else { float acc[1][8]; head_gemm_32<1>(X, Wt, sh.d_c, sh.d_h, acc, b0, j0); emit(acc, b0, j0, 1); }
    }
}

// ---------------------------------------------------------------- host side

size_t lh_attn_smem(const Shape& sh) {
    const int lat_chunks = sh.d_c / 128;
    const int max_chunks = lat_chunks + (sh.D / 64 - sh.d_c / 64);
    size_t bytes = 1024;
    bytes += (size_t)max_chunks * 128 * 128;            // q~ chunks
    bytes += (size_t)kStages * max_chunks * kKT * 128;  // key tiles
    bytes += 128 * 128;                                 // P
    bytes += 2 * 128 * 128;                             // exchanged scores (own, peer), fp16
    bytes += ((sizeof(LhBars) + 15) & ~(size_t)15) + ((size_t)sh.B + 1) * 4;
    return bytes;
}

size_t lh_stage_smem(const Shape& sh) { return (size_t)sh.d_h * sh.d_c * sizeof(bf16); }
size_t lh_prep_smem(const Shape& sh) { return lh_stage_smem(sh) + (size_t)sh.d_h * 32 * 4 + 16; }
size_t lh_comb_smem(const Shape& sh) {
    return lh_stage_smem(sh) + (size_t)sh.d_c * 32 * 4 + (2 * 32 * kMaxClusters + 32 + (size_t)sh.B + 1) * 4;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_lh(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
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

template <typename K>
cudaError_t lh_set_smem(K kernel, size_t smem, size_t* done) {
    if (*done >= smem) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) *done = smem;
    return e;
}

}  // namespace

bool tc_decode_lh_supported(const Shape& sh) {
    return sh.H > 32 && sh.H <= 128 && sh.d_c % 128 == 0 && sh.d_c <= 512 && sh.D % 64 == 0 &&
           (sh.d_h == 64 || sh.d_h == 128 || sh.d_h == 256 || sh.d_h == 512) &&
           (sh.d_c == 128 || sh.d_c == 256 || sh.d_c == 512) && sh.B <= kMaxB && lh_comb_smem(sh) <= 227 * 1024 &&
           lh_prep_smem(sh) <= 227 * 1024 &&
           lh_attn_smem(sh) <= 232448 - 1024;
}

size_t tc_decode_lh_workspace(const Shape& sh) {
    return align256((size_t)sh.B * (sh.D / 64) * 128 * 128) +
           align256((size_t)(kMaxClusters + sh.B) * sh.H * (sh.d_c + 4) * sizeof(float));
}

cudaError_t tc_decode_lh(const DecodeArgs& a, cudaStream_t st, uint64_t* launches) {
    const Shape& sh = a.sh;
    uint8_t* qimg = (uint8_t*)a.workspace;
    float* part = (float*)((char*)a.workspace + align256((size_t)sh.B * (sh.D / 64) * 128 * 128));
    auto encode = (PFN_cuTensorMapEncodeTiled_v12000)tensor_map_encoder();
    if (!encode) return note_error("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", cudaErrorNotSupported);
    CUtensorMap map;
    cuuint64_t dims[3] = {(cuuint64_t)sh.D, (cuuint64_t)sh.max_slots, (cuuint64_t)sh.B};
    cuuint64_t strides[2] = {(cuuint64_t)sh.D * 2, (cuuint64_t)sh.max_slots * sh.D * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)kKT, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.cache, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        char buf[96];
        snprintf(buf, sizeof(buf), "cuTensorMapEncodeTiled (CUresult %d)", (int)r);
        return note_error(buf, cudaErrorInvalidValue);
    }
    LhArgs p;
    p.B = sh.B;
    p.H = sh.H;
    p.D = sh.D;
    p.d_c = sh.d_c;
    p.d_r = sh.d_r;
    p.s = sh.s;
    p.max_slots = sh.max_slots;
    p.n_qchunks = sh.D / 64;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    static size_t done_prep[64] = {0}, done_attn[64] = {0}, done_comb[64] = {0};
    static int co_resident[64] = {0};
    const size_t prep_smem = lh_prep_smem(sh);
    const size_t attn_smem = lh_attn_smem(sh);
    const size_t comb_smem = lh_comb_smem(sh);
    cudaError_t e = lh_set_smem(k_lh_prep, prep_smem, &done_prep[dev]);
    if (e == cudaSuccess) e = lh_set_smem(k_lh_attn, attn_smem, &done_attn[dev]);
    if (e == cudaSuccess) e = lh_set_smem(k_lh_combine, comb_smem, &done_comb[dev]);
    if (e != cudaSuccess) return note_error("cudaFuncSetAttribute(large-head decode)", e);
    if (!co_resident[dev]) {
        // clusters that can be resident at once: the balanced split assumes one wave
        cudaLaunchConfig_t oc = {};
        oc.gridDim = dim3(2 * kMaxClusters);
        oc.blockDim = dim3(kThreads);
        oc.dynamicSmemBytes = attn_smem;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, k_lh_attn, &oc) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = sm_count() / 2;
        }
        co_resident[dev] = n;
    }
    const int64_t max_tiles = (int64_t)sh.B * ((sh.max_slots + kKT - 1) / kKT);
    p.G2 = (int)std::min<int64_t>(std::min(co_resident[dev], kMaxClusters), max_tiles);
    p.scale_log2 = sh.scale * 1.4426950408889634f;
    p.pos = a.pos;
    p.qimg = qimg;
    p.part = part;
    p.status = a.status;

    k_lh_prep<<<sh.H, 256, prep_smem, st>>>(a, qimg, p.n_qchunks);
    e = cudaGetLastError();
    if (e != cudaSuccess) return note_error("k_lh_prep launch", e);
    profile_begin(st);
    e = launch_pdl_lh(k_lh_attn, dim3(2 * p.G2), dim3(kThreads), attn_smem, st, map, p);
    profile_end(st);
    if (e != cudaSuccess) return note_error("k_lh_attn launch", e);
    e = launch_pdl_lh(k_lh_combine, dim3(sh.H), dim3(256), comb_smem, st, a, p);
    *launches += 3;
    return note_error("k_lh_combine launch", e);
}

}  // namespace mtla
