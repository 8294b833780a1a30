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
#include <algorithm>
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
constexpr int kStages = 3;
constexpr int kMaxSq = 4;         // query chunks in shared memory: at most 4 latent + 2 RoPE - 2 in TMEM
constexpr int kThreads = 352;    // warp 0 TMA, 1 score MMAs, 2-9 softmax, 10 P.V MMAs
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

__device__ __forceinline__ bool lh_pos_ok(const Shape& sh, int64_t t) {
    return t >= 0 && t < (int64_t)sh.max_slots * sh.s;
}

// Decode prep for many heads on the tensor cores. grid (H, ceil(B / 32)),
// 256 threads. Block (h, group of 32 sequences):
//   q~^T [d_c x 32] = W_UK[h]^T [d_c x d_h] . qC^T [d_h x 32]   (tcgen05,
//   M = 128 latent columns per block, N = 32, A = W_UK[h] by TMA, MN-major)
// rounded to bf16 into row h of each sequence's query image; the RoPE part
// RoPE_t(qR) and the zero tail on the CUDA cores; then the in-place slot
// updates (gate, RoPE key, open slot; MTLA Method (1)) of the group's
// sequences b with b mod H = h, and the zero rows H..127 of their images.
constexpr int kPrepThreads = 256;
__global__ void __launch_bounds__(kPrepThreads, 1)
    k_lh_prep(const __grid_constant__ CUtensorMap wuk_map, DecodeArgs a, uint8_t* qimg, int n_qchunks) {
    pdl_launch_dependents();
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const Shape& sh = a.sh;
    const int h = blockIdx.x, c0 = blockIdx.y * 32;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t img_bytes = (uint32_t)n_qchunks * 128 * 128;
    const int n_kc = sh.d_c / 64;                          // 64-column chunks of W_UK rows (= latent)
    const int n_kb = (sh.d_h + 127) / 128;                 // 128-row blocks of W_UK (= K)
    const int n_qc = (sh.d_h + 63) / 64;                   // 64-column chunks of qC
    uint8_t* w_s = smem;                                   // n_kc x [128 k-rows x 128 B]
    uint8_t* x_s = w_s + (size_t)n_kc * 16384;             // n_qc x [32 sequences x 128 B]: qC rows
    uint64_t* bars = (uint64_t*)(x_s + (size_t)n_qc * 4096);   // [0] W landed, [1] MMAs done
    uint32_t* tmem_slot = (uint32_t*)(bars + 2);
    const uint32_t w_bytes = (uint32_t)n_kc * 16384;
    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(&bars[0], w_bytes);
        for (int kc = 0; kc < n_kc; ++kc) tma_load_2d(w_s + kc * 16384, &wuk_map, &bars[0], kc * 64, h * sh.d_h);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 128);
        tmem_relinquish();
    }
    __shared__ double rope_freq[64];                      // base^(-2k / d_r), d_r / 2 <= 64
    for (int k = tid; k < sh.d_r / 2; k += kPrepThreads)
        rope_freq[k] = exp2(-(2.0 * k / (double)sh.d_r) * sh.log2_rope_base);
    // qC rows of the 32 sequences (zero past B) as the K-major B operand
    for (int e = tid; e < 32 * n_qc * 8; e += kPrepThreads) {
        const int bb = e / (n_qc * 8), rem = e % (n_qc * 8), c = rem >> 3, u = rem & 7;
        const int b = c0 + bb, col = c * 64 + u * 8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (b < sh.B && col < sh.d_h) v = *(const uint4*)((const bf16*)a.q_c + ((size_t)b * sh.H + h) * sh.d_h + col);
        *(uint4*)(x_s + (size_t)c * 4096 + sw128_offset(bb, u * 8)) = v;
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t t_d = *tmem_slot;
    if (tid == 0) {
        bool ok = true;
        const uint32_t idesc = idesc_bf16_f32(128, 32, true, false);
        const uint64_t ad = sdesc_sw128(smem_u32(w_s), 16384, 1024), bd = sdesc_sw128(smem_u32(x_s), 16, 1024);
        for (int kb = 0; kb < n_kb && ok; ++kb) {
            if (kb > 0) {
                // the next 128 rows of W_UK[h] into the same buffer once the MMAs read it
                ok = mbar_wait(&bars[1], (kb - 1) & 1);
                if (!ok) break;
                mbar_arrive_expect_tx(&bars[0], w_bytes);
                for (int kc = 0; kc < n_kc; ++kc)
                    tma_load_2d(w_s + kc * 16384, &wuk_map, &bars[0], kc * 64, h * sh.d_h + kb * 128);
            }
            ok = mbar_wait(&bars[0], kb & 1);
            if (!ok) break;
            tc_fence_after();
            const int ksteps = min(128, sh.d_h - kb * 128) / 16;
            for (int mb = 0; mb < n_kc / 2; ++mb) {
                // A = W_UK[h]^T block mb: latent 128 mb.. as M (two 64-column chunks), k rows as K
                const uint64_t am = desc_add(ad, mb * 2 * 16384);
                for (int kk = 0; kk < ksteps; ++kk) {
                    const int kg = kb * 8 + kk;                // global 16-row K step
                    umma_bf16(t_d + mb * 32, desc_add(am, kk * 2048),
                              desc_add(bd, (kg >> 2) * 4096 + (kg & 3) * 32), idesc, (kg > 0) ? 1u : 0u);
                }
            }
            umma_commit(&bars[1]);
        }
        if (!ok) latch_status(a.status, kStatusTimeout);
    }
    // RoPE part of q~ and the zero tail (columns d_c .. n_qchunks * 64) meanwhile:
    // every load of a thread's (up to 4) pairs first, frequencies from a table
    {
        const int nrot = n_qchunks * 64 - sh.d_c;            // even, <= 128
        const int npair = nrot / 2;
        constexpr int kPer = 8;                              // 32 * 64 pairs / 256 threads
        int64_t tv[kPer];
        uint32_t qv[kPer];
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int e = tid + i * kPrepThreads, bb = e / npair, k = e % npair, b = c0 + bb;
            tv[i] = -1;
            qv[i] = 0;
            if (bb < 32 && b < sh.B) {
                tv[i] = a.pos[b];
                if (2 * k < sh.d_r) qv[i] = *(const uint32_t*)((const bf16*)a.q_r + ((size_t)b * sh.H + h) * sh.d_r + 2 * k);
            }
        }
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int e = tid + i * kPrepThreads, bb = e / npair, k = e % npair, b = c0 + bb;
            if (bb >= 32 || b >= sh.B || !lh_pos_ok(sh, tv[i])) continue;
            float v0 = 0.f, v1 = 0.f;
            if (2 * k < sh.d_r) {
                const bf16* xq = (const bf16*)&qv[i];
                const float x0 = __bfloat162float(xq[0]), x1 = __bfloat162float(xq[1]);
                float sn, cs;
                pair_sincos_f(tv[i], rope_freq[k], &sn, &cs);
                v0 = x0 * cs - x1 * sn;
                v1 = x0 * sn + x1 * cs;
            }
            const int j = sh.d_c + 2 * k;
            *(uint32_t*)(qimg + (size_t)b * img_bytes + (size_t)(j >> 6) * 128 * 128 + sw128_offset(h, j & 63)) =
                pack_bf16x2(v0, v1);
        }
    }
    // latent part: warp w reads TMEM lane quarter w mod 4 (latent rows), sequences
    // 16 (w / 4) .. 16 (w / 4) + 15
    const bool done = mbar_wait(&bars[1], (n_kb - 1) & 1);
    tc_fence_after();
    {
        const int quarter = warp & 3, half = warp >> 2;
        for (int mb = 0; mb < n_kc / 2; ++mb) {
            float v[16];
            tmem_ld16(t_d + mb * 32 + half * 16 + ((uint32_t)(quarter * 32) << 16), v);
            tmem_wait_ld();
            const int j = mb * 128 + quarter * 32 + lane;      // latent column
#pragma unroll
            for (int s = 0; s < 16; ++s) {
                const int b = c0 + half * 16 + s;
                if (done && b < sh.B && lh_pos_ok(sh, a.pos[b]))
                    *(bf16*)(qimg + (size_t)b * img_bytes + (size_t)(j >> 6) * 128 * 128 + sw128_offset(h, j & 63)) =
                        __float2bfloat16_rn(v[s]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(t_d, 128);
    // in-place slot updates of this group's sequences b with b mod H = h
    for (int b = c0 + ((h - c0 % sh.H) % sh.H + sh.H) % sh.H; b < min(sh.B, c0 + 32); b += sh.H) {
        __syncthreads();
        decode_update_body<bf16>(a, b);
        uint8_t* img = qimg + (size_t)b * img_bytes;
        const int pad_rows = 128 - sh.H;
        for (int e = tid; e < n_qchunks * pad_rows * 8; e += kPrepThreads) {
            const int c = e / (pad_rows * 8), rr = e % (pad_rows * 8);
            *(uint4*)(img + (size_t)c * 128 * 128 + (size_t)(sh.H + rr / 8) * 128 + (rr % 8) * 16) =
                make_uint4(0, 0, 0, 0);
        }
    }
}

// ---------------------------------------------------------------- attention

struct LhBars {
    uint64_t full[kStages], empty[kStages];   // slot-tile ring
    uint64_t q_full, q_free;                  // query image of the current segment
    uint64_t s_full[2], s_empty[2];           // partial scores in TMEM, by tile parity
    uint64_t p_full[2], o_done[2];            // P in TMEM; P.V of tiles with this parity completed
    uint64_t x_full[2];                       // peer's partial scores landed in x_in[parity] (bulk copy)
    uint64_t x_free[2];                       // peer has read the scores this CTA sent into its x_in[parity]
    uint64_t qt_full;                         // query chunks of the segment written to TMEM (8 warps)
    uint64_t drain[2];                        // MMAs in flight when a wait gave up (per issuing thread)
    uint32_t tmem_base;
    volatile int fail;
    int total;
    float red[2][2][128];                     // [tile parity][column half][row]: half-row maxima
    float lsum[2][128];                       // [column half][row]: half-row sums at a segment end
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

// Attention over 64-slot tiles for one cluster of two CTAs (see the top of the
// file). Warp 0: TMA; warp 1: MMA issue and TMEM; warps 2-9: softmax, two
// threads per head row (one per 32-slot half of a tile). The softmax of tile it
// is split in two halves:
//   A(it)  read this CTA's partial scores from TMEM, round them (scaled) to
//          fp16 and send them to the peer (one bulk copy into its x_in);
//   B(it)  add the peer's partial scores, online softmax, P into TMEM.
// The order A(it+1), B(it) lets both copies of tile it+1 fly while the CTAs
// do B(it). Scores, P and x_in are double-buffered; the ring has three stages.
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
    // the last n_tq of this CTA's query chunks live in TMEM (the MMA's A from
    // tensor memory), the first n_sq in shared memory
    const int n_tq = min(2, my_chunks), n_sq = my_chunks - n_tq;
    const uint32_t stage_bytes = (uint32_t)max_chunks * kKT * 128;
    uint8_t* q_s = smem;                                             // (max_chunks - 2) x [128 x 128 B]
    uint8_t* ring = q_s + (size_t)max(0, max_chunks - 2) * 128 * 128;   // kStages x stage_bytes
    uint8_t* x_out = ring + (size_t)kStages * stage_bytes;           // own scores, fp16 [128 x 128 B]
    uint8_t* x_in = x_out + 128 * 128;                               // peer's scores, 2 x [128 x 128 B]
    LhBars& bs = *(LhBars*)(x_in + 2 * 128 * 128);
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
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bs.s_full[i], 1);
            mbar_init(&bs.s_empty[i], 8);
            mbar_init(&bs.p_full[i], 8);
            mbar_init(&bs.o_done[i], 1);
        }
        mbar_init(&bs.q_full, 1);
        mbar_init(&bs.q_free, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bs.x_full[i], 1);     // local expect_tx arrive; the peer's copy completes the bytes
            mbar_init(&bs.x_free[i], 1);     // one remote arrive from the peer
        }
        mbar_init(&bs.qt_full, 8);
        mbar_init(&bs.drain[0], 1);
        mbar_init(&bs.drain[1], 1);
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
    const uint32_t t_s = tmem + 256;                   // partial scores: 2 x 64 columns
    const uint32_t t_p = tmem + 384;                   // P (bf16 pairs): 2 x 32 columns
    const uint32_t t_q = tmem + 448;                   // query chunks (bf16 pairs): 2 x 32 columns
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

    int loads_issued = 0, q_loads = 0;   // producer's copies, for the drain on failure
    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int prev_b = -1;
            for (int gt = gt0, it = 0; gt < gt1; ++gt, ++it) {
                int b, j;
                locate(gt, b, j);
                if (b != prev_b) {
                    prev_b = b;
                    if (q_loads >= 1 && !lh_wait(&bs.q_free, (q_loads - 1) & 1, bs)) break;
                    mbar_arrive_expect_tx(&bs.q_full, (uint32_t)n_sq * 128 * 128);
                    const uint8_t* src = p.qimg + (size_t)b * p.n_qchunks * 128 * 128;
                    for (int i = 0; i < n_sq; ++i)
                        bulk_load(q_s + (size_t)i * 128 * 128,
                                  src + (size_t)lh_chunk_id(rank, i, lat_chunks, rope_first) * 128 * 128,
                                  128 * 128, &bs.q_full);
                    ++q_loads;
                }
                const int st = it % kStages;
                if (it >= kStages && !lh_wait(&bs.empty[st], ((it / kStages) - 1) & 1, bs)) break;
                mbar_arrive_expect_tx(&bs.full[st], (uint32_t)my_chunks * kKT * 128);
                for (int i = 0; i < my_chunks; ++i)
                    tma_load_3d(ring + st * stage_bytes + (size_t)i * kKT * 128, &tmap, &bs.full[st],
                                lh_chunk_id(rank, i, lat_chunks, rope_first) * 64, j * kKT, b);
                ++loads_issued;

            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ score MMAs
        if (lane == 0) {
            const uint32_t id_s = idesc_bf16_f32(128, kKT, false, false);
            const uint32_t ring_a = smem_u32(ring);
            const uint64_t q_d = sdesc_sw128(smem_u32(q_s), 16, 1024);
            int seg = -1, prev_b = -1, it = 0;
            for (int gt = gt0; gt < gt1; ++gt, ++it) {
                int b, j;
                locate(gt, b, j);
                if (b != prev_b) {
                    prev_b = b;
                    ++seg;
                    if (!lh_wait(&bs.q_full, seg & 1, bs)) break;    // q~ chunks in smem
                    if (!lh_wait(&bs.qt_full, seg & 1, bs)) break;   // q~ chunks in TMEM
                }
                const int st = it % kStages;
                if (!lh_wait(&bs.full[st], (it / kStages) & 1, bs)) break;
                if (it >= 2 && !lh_wait(&bs.s_empty[it & 1], ((it >> 1) - 1) & 1, bs)) break;
                tc_fence_after();
                // S_c = q~_c . K_c^T (M = 128 heads, N = 64 slots)
                const uint64_t kd = sdesc_sw128(ring_a + st * stage_bytes, 16, 1024);
                const uint32_t ts = t_s + (it & 1) * kKT;
                // Straight-line groups of four MMAs with one test per group (a
                // runtime loop or a test per MMA halves their issue rate). Every
                // chunk is a full 64 columns (D is a multiple of 64).
#pragma unroll
                for (int i = 0; i < kMaxSq; ++i) {
                    if (i < n_sq) {
                        const uint64_t qi = desc_add(q_d, i * 128 * 128), ki = desc_add(kd, i * kKT * 128);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_bf16(ts, desc_add(qi, kk * 32), desc_add(ki, kk * 32), id_s, (i | kk) != 0);
                    }
                }
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    if (i < n_tq) {
                        const uint64_t ki = desc_add(kd, (n_sq + i) * kKT * 128);
                        const uint32_t acc0 = (n_sq + i) != 0 ? 1u : 0u;
                        umma_bf16_ts(ts, t_q + i * 32, ki, id_s, acc0);
#pragma unroll
                        for (int kk = 1; kk < 4; ++kk)
                            umma_bf16_ts(ts, t_q + i * 32 + kk * 8, desc_add(ki, kk * 32), id_s, 1u);
                    }
                }
                umma_commit(&bs.s_full[it & 1]);
                const bool last = (gt + 1 == gt1) || (j + 1 == starts[b + 1] - starts[b]);
                if (last) umma_commit(&bs.q_free);
            }
        }
    } else if (warp == 10) {
        // ------------------------------------------------------------ P.V MMAs
        // A second issuing thread, so that P.V (which frees ring stages) never
        // waits behind score MMAs that wait for a load.
        if (lane == 0) {
            const uint32_t id_o = idesc_bf16_f32(128, lat_half, false, true);
            const uint32_t ring_a = smem_u32(ring);
            int prev_b = -1, it = 0;
            for (int gt = gt0; gt < gt1; ++gt, ++it) {
                int b, j;
                locate(gt, b, j);
                const bool first = (b != prev_b);
                prev_b = b;
                if (!lh_wait(&bs.p_full[it & 1], (it >> 1) & 1, bs)) break;
                tc_fence_after();
                // O_c += P . V_c: A = P in TMEM, B = the tile's latent columns (MN-major)
                const uint64_t vd = sdesc_sw128(ring_a + (it % kStages) * stage_bytes, kKT * 128, 1024);
#pragma unroll
                for (int kk = 0; kk < kKT / 16; ++kk)
                    umma_bf16_ts(t_o, t_p + (it & 1) * 32 + kk * 8, desc_add(vd, kk * 2048), id_o,
                                 (first && kk == 0) ? 0u : 1u);
                umma_commit(&bs.empty[it % kStages]);
                umma_commit(&bs.o_done[it & 1]);
            }
        }
    } else {
        // ------------------------------------------------------------ softmax (two threads per head row)
        // Warps 2-9: row r = (warp mod 4) * 32 + lane (the TMEM lane quarter a warp
        // may access), column half hc = (warp - 2) / 4 of each 64-slot tile.
        // The partial scores travel by one bulk copy per tile from x_out into the
        // peer's x_in[tile parity]; the copy completes the bytes on the peer's
        // x_full[parity]. No early exit from the loop: after a bounded wait gave
        // up, later waits return at once, so no thread is left waiting.
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const int hc = (warp - 2) >> 2;
        const int sidx = tid - 64;                     // 0..255 over the softmax warps
        const bool leader = sidx == 0;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint32_t x_in_peer = map_to_rank(x_in, peer);
        const uint32_t xfull_peer = map_to_rank(&bs.x_full[0], peer);
        const uint32_t xfree_peer = map_to_rank(&bs.x_free[0], peer);
        uint32_t own[16];        // this thread's 32 scaled partial scores of the newest tile, fp16 pairs
        uint32_t own_prev[16];   // ... of the tile B works on
        // Query chunks n_sq.. of sequence b into TMEM: the thread of row r and
        // half hc writes chunk n_sq + hc of row r (de-swizzled from the image).
        auto load_qt = [&](int b) {
            if (hc < n_tq) {
                const uint8_t* src = p.qimg + (size_t)b * p.n_qchunks * 128 * 128 +
                                     (size_t)lh_chunk_id(rank, n_sq + hc, lat_chunks, rope_first) * 128 * 128 +
                                     (size_t)r * 128;
                uint32_t w[32];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const uint4 v = *(const uint4*)(src + (((u ^ r) & 7) << 4));
                    w[4 * u] = v.x;
                    w[4 * u + 1] = v.y;
                    w[4 * u + 2] = v.z;
                    w[4 * u + 3] = v.w;
                }
                tmem_st32_u(t_q + hc * 32 + lane_off, w);
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bs.qt_full);
        };
        // A(k): partial scores of tile k -> own[], x_out, and the peer's x_in[k & 1]
        auto half_a = [&](int k) {
            lh_wait(&bs.s_full[k & 1], (k >> 1) & 1, bs);
            tc_fence_after();
            float sv[32];
            tmem_ld32(t_s + (k & 1) * kKT + hc * 32 + lane_off, sv);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bs.s_empty[k & 1]);
            if (gt0 + k + 1 < gt1) {
                // S(k) is complete, so every score MMA that read the TMEM query chunks
                // is done; if tile k+1 opens a new segment, bring in its query
                int b1, j1;
                locate(gt0 + k + 1, b1, j1);
                if (j1 == 0) load_qt(b1);
            }
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const __half2 h2 = __floats2half2_rn(sv[2 * c] * p.scale_log2, sv[2 * c + 1] * p.scale_log2);
                own[c] = *(const uint32_t*)&h2;
            }
            if (leader) {
                bulk_wait_read_all();                               // the copy of tile k-1 has read x_out
                if (!bs.fail) mbar_arrive_expect_tx(&bs.x_full[k & 1], 128 * 128);   // the peer's tile k
            }
            named_sync(1, 256);
#pragma unroll
            for (int u = 0; u < 4; ++u)
                *(uint4*)(x_out + xoff(r, 4 * hc + u)) =
                    make_uint4(own[4 * u], own[4 * u + 1], own[4 * u + 2], own[4 * u + 3]);
            fence_proxy_async();
            named_sync(1, 256);
            if (leader) {
                // the peer's x_in[k & 1] was read by its B(k - 2)
                if (k < 2 || lh_wait_cluster(&bs.x_free[k & 1], ((k >> 1) - 1) & 1, bs)) {
                    bulk_copy_to_peer(x_in_peer + (k & 1) * 128 * 128, x_out, 128 * 128, xfull_peer + (k & 1) * 8);
                    bulk_commit_group();
                }
            }
        };
        float m_ref = -INFINITY, l = 0.f;              // l: this thread's half of the row sum
        int prev_b = -1, n_b = 0, k_in_seg = 0;
        if (gt0 < gt1) {
            int b0, j0;
            locate(gt0, b0, j0);
            load_qt(b0);
            half_a(0);
        }
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
#pragma unroll
            for (int c = 0; c < 16; ++c) own_prev[c] = own[c];
            if (gt + 1 < gt1) half_a(it + 1);       // the peer's copy of tile it+1 overlaps B(it)
            const int st = it % kStages;
            const int valid = min(kKT, n_b - j * kKT) - hc * 32;   // valid columns of this half
            // B(it): add the peer's partial scores of this tile (a + b = b + a
            // exactly, so both CTAs hold the same scores)
            lh_wait(&bs.x_full[it & 1], (it >> 1) & 1, bs);
            const uint8_t* xin = x_in + (it & 1) * 128 * 128;
            uint4 th[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) th[u] = *(const uint4*)(xin + xoff(r, 4 * hc + u));
            float sv[32];
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};   // four independent chains
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const uint32_t tw[4] = {th[u].x, th[u].y, th[u].z, th[u].w};
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const float2 fm = __half22float2(*(const __half2*)&own_prev[4 * u + v]);
                    const float2 ft = __half22float2(*(const __half2*)&tw[v]);
                    const int c = 8 * u + 2 * v;
                    sv[c] = c < valid ? fm.x + ft.x : -INFINITY;
                    sv[c + 1] = c + 1 < valid ? fm.y + ft.y : -INFINITY;
                    m4[v] = fmaxf(m4[v], fmaxf(sv[c], sv[c + 1]));
                }
            }
            float mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
            bs.red[it & 1][hc][r] = mt;
            named_sync(1, 256);                        // also: every thread has read x_in[it & 1]
            if (leader) mbar_arrive_remote_relaxed(xfree_peer + (it & 1) * 8);
            mt = fmaxf(mt, bs.red[it & 1][hc ^ 1][r]);
            // lazy rescale: the reference maximum moves only when the tile's maximum
            // exceeds it by more than 2^8 (P stays <= 256); both halves decide alike
            const bool upd = mt > m_ref + kRescaleLog2;
            const float nm = upd ? mt : m_ref;
            const float fac = ex2_approx(m_ref - nm);    // 0 when m_ref was -inf, 1 when kept
            float rs4[4] = {0.f, 0.f, 0.f, 0.f};
            uint32_t pk[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const float p0 = ex2_approx(sv[2 * c] - nm), p1 = ex2_approx(sv[2 * c + 1] - nm);
                rs4[c & 3] += p0 + p1;
                pk[c] = pack_bf16x2(p0, p1);
            }
            l = fmaf(l, fac, (rs4[0] + rs4[1]) + (rs4[2] + rs4[3]));
            m_ref = nm;
            const bool need = upd && k_in_seg > 0;
            if (__any_sync(0xffffffffu, need)) {
                // this warp's rows of its half of O_c move to their new reference maxima
                lh_wait(&bs.o_done[(it - 1) & 1], ((it - 1) >> 1) & 1, bs);
                tc_fence_after();
                const float f = need ? fac : 1.f;
                const int cols = lat_half / 2;
                float v[32];
                for (int cc = 0; cc < cols / 32; ++cc) {
                    const uint32_t ta = t_o + hc * cols + cc * 32 + lane_off;
                    tmem_ld32(ta, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] *= f;
                    tmem_st32(ta, v);
                }
                tmem_wait_st();
            }
            if (valid + hc * 32 < kKT) {
                // stale rows past the sequence's last slot must not reach P.V
                const int v0 = valid + hc * 32, rows = kKT - v0;
                uint8_t* stg = ring + st * stage_bytes;
                for (int e = sidx; e < my_chunks * rows * 8; e += 256) {
                    const int i = e / (rows * 8), rr = e % (rows * 8);
                    *(uint4*)(stg + (size_t)i * kKT * 128 + (size_t)(v0 + rr / 8) * 128 + (rr % 8) * 16) =
                        make_uint4(0, 0, 0, 0);
                }
            }
            if (it >= 2) lh_wait(&bs.o_done[it & 1], ((it >> 1) - 1) & 1, bs);   // P.V of tile it-2 read this P buffer
            tmem_st16_u(t_p + (it & 1) * 32 + hc * 16 + lane_off, pk);
            tmem_wait_st();
            fence_proxy_async();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bs.p_full[it & 1]);
            ++k_in_seg;
            const bool last = (gt + 1 == gt1) || (j + 1 == starts[b + 1] - starts[b]);
            if (last) {
                // partial of this sequence segment: this CTA's half of O, plus (m, l)
                bs.lsum[hc][r] = l;
                lh_wait(&bs.o_done[it & 1], (it >> 1) & 1, bs);
                tc_fence_after();
                named_sync(1, 256);
                const size_t row = (size_t)p.d_c + 4;
                float* dst = p.part + ((size_t)(g + b) * p.H + r) * row;
                const int cols = lat_half / 2;
                float v[32];
                for (int cc = 0; cc < cols / 32; ++cc) {
                    tmem_ld32(t_o + hc * cols + cc * 32 + lane_off, v);
                    tmem_wait_ld();
                    if (r < p.H) {
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            *(float4*)(dst + rank * lat_half + hc * cols + cc * 32 + 4 * u) =
                                make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
                    }
                }
                if (rank == 0 && hc == 0 && r < p.H) {
                    dst[p.d_c] = m_ref;
                    dst[p.d_c + 1] = l + bs.lsum[1][r];
                }
                tc_fence_before();
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (bs.fail) {
        // a bounded wait gave up: let this CTA's copies and MMAs land (bounded
        // again) before shared memory and TMEM are released, then report
        if (warp == 0 && lane == 0) {
            for (int k = max(0, loads_issued - kStages); k < loads_issued; ++k)
                mbar_wait(&bs.full[k % kStages], (k / kStages) & 1);
            if (q_loads > 0) mbar_wait(&bs.q_full, (q_loads - 1) & 1);
        }
        if ((warp == 1 || warp == 10) && lane == 0) {
            uint64_t* d = &bs.drain[warp == 1 ? 0 : 1];
            umma_commit(d);              // arrives when this thread's MMAs are done
            mbar_wait(d, 0);
        }
        if (tid == 64) {
            // the peer's score copies into this CTA, and this CTA's own copies
            const int n = gt1 - gt0;
            for (int k = max(0, n - 2); k < n; ++k) mbar_wait(&bs.x_full[k & 1], (k >> 1) & 1);
            bulk_wait_read_all();
        }
        if (tid == 0) latch_status(p.status, kStatusTimeout);
        __syncthreads();
    }
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
    cluster_sync();                      // the peer may still store into / arrive on us until here
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

// Merge and W_UV on the tensor cores. grid (H, ceil(B / 32)), 512 threads.
// Block (h, group of 32 sequences):
//   A. per sequence, one warp turns the partial maxima and sums (m_i, l_i)
//      into merge weights 2^(m_i - M) / L (lane i: partial i);
//   B. thread (column quad, sequence octet) sums the weighted partial rows,
//      writing o_lat as bf16 into a K-major operand;
//   C. out^T [d_h x 32] = W_UV[h] [d_h x d_c] . o_lat^T  (tcgen05, M = 128, N = 32)
//      with W_UV[h] brought in by TMA before the wait for the attention kernel.
constexpr int kCombThreads = 512;
__global__ void __launch_bounds__(kCombThreads, 1)
    k_lh_combine(const __grid_constant__ CUtensorMap wuv_map, DecodeArgs a, LhArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const Shape& sh = a.sh;
    const int h = blockIdx.x, c0 = blockIdx.y * 32;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_kc = p.d_c / 64, n_mb = (sh.d_h + 127) / 128;
    uint8_t* w_s = smem;                                  // n_kc x [128 W_UV rows x 128 B]
    uint8_t* o_s = w_s + (size_t)n_kc * 16384;            // n_kc x [32 sequences x 128 B]
    float* wts = (float*)(o_s + (size_t)n_kc * 4096);     // [32][kMaxClusters] merge weights
    int* pidx = (int*)(wts + 32 * kMaxClusters);          // [32][kMaxClusters] partial index or -1
    int* npart = pidx + 32 * kMaxClusters;                // [32]
    uint64_t* bars = (uint64_t*)(npart + 32);             // [0] W landed, [1] MMAs done
    uint32_t* tmem_slot = (uint32_t*)(bars + 2);
    int* starts = (int*)(bars + 4);                       // [B + 1]
    __shared__ int warp_tot[kCombThreads / 32];
    const uint32_t w_bytes = (uint32_t)n_kc * 16384;
    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_mbar_init();
        tma_prefetch_desc(&wuv_map);
        mbar_arrive_expect_tx(&bars[0], w_bytes);
        for (int kc = 0; kc < n_kc; ++kc) tma_load_2d(w_s + kc * 16384, &wuv_map, &bars[0], kc * 64, h * sh.d_h);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 128);
        tmem_relinquish();
    }
    lh_tile_starts(p, starts, warp_tot);                  // reads pos only; ends with a block barrier
    tc_fence_after();
    const uint32_t t_d = *tmem_slot;
    const int total = starts[p.B];
    const size_t row = (size_t)p.d_c + 4;
    pdl_wait();                                           // the partials come from k_lh_attn
    // ---- A: merge weights
    for (int bb = warp; bb < 32; bb += kCombThreads / 32) {
        const int b = c0 + bb;
        int n = 0;
        if (b < sh.B && starts[b + 1] > starts[b] && total > 0) {
            // the clusters g_first..g_last touching this sequence's tiles [S_b, E_b)
            const int S_b = starts[b], E_b = starts[b + 1];
            const int64_t G = p.G2, tot = total;
            const int g_first = (int)(((int64_t)(S_b + 1) * G + tot - 1) / tot) - 1;
            const int g_last = (int)(((int64_t)E_b * G + tot - 1) / tot) - 1;
            n = min(g_last - g_first + 1, kMaxClusters);
            float mv[3], lv[3];                           // n <= kMaxClusters <= 96 = 3 x 32
            float M = -INFINITY;
#pragma unroll
            for (int r = 0; r < 3; ++r) {
                const int i = r * 32 + lane, g = g_first + i;
                mv[r] = -INFINITY;
                lv[r] = 0.f;
                if (i < n) {
                    const int64_t lo = ((int64_t)g * tot) / G, hi = ((int64_t)(g + 1) * tot) / G;
                    if (hi > lo) {
                        const float* e = p.part + ((size_t)(g + b) * p.H + h) * row;
                        mv[r] = e[p.d_c];
                        lv[r] = e[p.d_c + 1];
                    }
                }
                M = fmaxf(M, mv[r]);
            }
            M = warp_max(M);
            float L = 0.f;
#pragma unroll
            for (int r = 0; r < 3; ++r) L += (mv[r] == -INFINITY) ? 0.f : exp2f(mv[r] - M) * lv[r];
            const float inv = 1.f / warp_sum(L);
#pragma unroll
            for (int r = 0; r < 3; ++r) {
                const int i = r * 32 + lane;
                if (i < n) {
                    const bool live = mv[r] != -INFINITY;
                    wts[bb * kMaxClusters + i] = live ? exp2f(mv[r] - M) * inv : 0.f;
                    pidx[bb * kMaxClusters + i] = live ? g_first + i + b : -1;
                }
            }
        }
        if (lane == 0) npart[bb] = n;
    }
    __syncthreads();
    // ---- B: weighted sums, thread = (column quad cq, octet of sequences so)
    {
        const int cq = tid & 127, so = tid >> 7;
        const int k = cq * 4;
        for (int bb = so * 8; bb < so * 8 + 8; bb += 2) {
            float o[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            const int nmax = max(npart[bb], npart[bb + 1]);
            for (int i0 = 0; i0 < nmax; i0 += 4) {
                float4 v[2][4];
                float wv[2][4];
#pragma unroll
                for (int s2 = 0; s2 < 2; ++s2)
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int i = i0 + u, q = bb + s2;
                        v[s2][u] = make_float4(0.f, 0.f, 0.f, 0.f);
                        wv[s2][u] = 0.f;
                        if (k < p.d_c && i < npart[q]) {
                            const int pi = pidx[q * kMaxClusters + i];
                            if (pi >= 0) {
                                wv[s2][u] = wts[q * kMaxClusters + i];
                                v[s2][u] = *(const float4*)(p.part + ((size_t)pi * p.H + h) * row + k);
                            }
                        }
                    }
#pragma unroll
                for (int s2 = 0; s2 < 2; ++s2)
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        o[s2][0] = fmaf(wv[s2][u], v[s2][u].x, o[s2][0]);
                        o[s2][1] = fmaf(wv[s2][u], v[s2][u].y, o[s2][1]);
                        o[s2][2] = fmaf(wv[s2][u], v[s2][u].z, o[s2][2]);
                        o[s2][3] = fmaf(wv[s2][u], v[s2][u].w, o[s2][3]);
                    }
            }
            if (k < p.d_c) {
#pragma unroll
                for (int s2 = 0; s2 < 2; ++s2) {
                    uint2 pk;
                    pk.x = pack_bf16x2(o[s2][0], o[s2][1]);
                    pk.y = pack_bf16x2(o[s2][2], o[s2][3]);
                    *(uint2*)(o_s + (size_t)(k >> 6) * 4096 + sw128_offset(bb + s2, k & 63)) = pk;
                }
            }
        }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // ---- C: out^T = W_UV[h] . o_lat^T, 128 output rows at a time
    if (tid == 0) {
        bool ok = true;
        for (int mb = 0; mb < n_mb && ok; ++mb) {
            if (mb > 0) {
                // the next 128 rows of W_UV[h] into the same buffer, once the previous
                // block's MMAs have read it
                ok = mbar_wait(&bars[1], (mb - 1) & 1);
                if (!ok) break;
                mbar_arrive_expect_tx(&bars[0], w_bytes);
                for (int kc = 0; kc < n_kc; ++kc)
                    tma_load_2d(w_s + kc * 16384, &wuv_map, &bars[0], kc * 64, h * sh.d_h + mb * 128);
            }
            ok = mbar_wait(&bars[0], mb & 1);
            if (!ok) break;
            tc_fence_after();
            const uint32_t idesc = idesc_bf16_f32(128, 32, false, false);
            const uint64_t ad = sdesc_sw128(smem_u32(w_s), 16, 1024), bd = sdesc_sw128(smem_u32(o_s), 16, 1024);
            for (int kc = 0; kc < n_kc; ++kc) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_bf16(t_d + mb * 32, desc_add(ad, kc * 16384 + kk * 32), desc_add(bd, kc * 4096 + kk * 32),
                              idesc, (kc | kk) != 0);
            }
            umma_commit(&bars[1]);
        }
        if (!ok) latch_status(a.status, kStatusTimeout);
    }
    // every thread: the last block's MMAs (they complete in order); warp w reads
    // TMEM lane quarter w mod 4, sequences 8 (w / 4) .. 8 (w / 4) + 7
    const bool done = mbar_wait(&bars[1], (n_mb - 1) & 1);
    tc_fence_after();
    const int quarter = warp & 3, oct = warp >> 2;
    for (int mb = 0; mb < n_mb; ++mb) {
        float v[8];
        tmem_ld8(t_d + mb * 32 + oct * 8 + ((uint32_t)(quarter * 32) << 16), v);
        tmem_wait_ld();
        const int i = mb * 128 + quarter * 32 + lane;       // output dimension (W_UV row)
        if (done && i < sh.d_h) {
#pragma unroll
            for (int s8 = 0; s8 < 8; ++s8) {
                const int b = c0 + oct * 8 + s8;
                if (b < sh.B && starts[b + 1] > starts[b])
                    ((bf16*)a.out)[((size_t)b * sh.H + h) * sh.d_h + i] = __float2bfloat16_rn(v[s8]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(t_d, 128);
}

// ---------------------------------------------------------------- host side

size_t lh_attn_smem(const Shape& sh) {
    const int lat_chunks = sh.d_c / 128;
    const int max_chunks = lat_chunks + (sh.D / 64 - sh.d_c / 64);
    size_t bytes = 1024;
    bytes += (size_t)std::max(0, max_chunks - 2) * 128 * 128;   // q~ chunks in shared memory
    bytes += (size_t)kStages * max_chunks * kKT * 128;  // key tiles
    bytes += 3 * 128 * 128;                             // exchanged scores (own; peer's x 2), fp16
    bytes += ((sizeof(LhBars) + 15) & ~(size_t)15) + ((size_t)sh.B + 1) * 4;
    return bytes;
}

size_t lh_prep_smem(const Shape& sh) {
    return 1024 + (size_t)(sh.d_c / 64) * 16384 + (size_t)((sh.d_h + 63) / 64) * 4096 + 32;
}
size_t lh_comb_smem(const Shape& sh) {
    const size_t n_kc = sh.d_c / 64;
    return 1024 + n_kc * 16384 + n_kc * 4096 + (2 * 32 * kMaxClusters + 32) * 4 + 32 + ((size_t)sh.B + 1) * 4;
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
    return sh.H > 32 && sh.H <= 128 && sh.d_c % 128 == 0 && sh.d_c <= 512 && sh.D % 64 == 0 && sh.d_r <= 128 &&
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
    // W_UK and W_UV as [H * d_h rows][d_c] bf16, 128-row x 64-column boxes
    // (rows past the last head read as zero)
    CUtensorMap wuk_map, wuv_map;
    for (int w = 0; w < 2; ++w) {
        cuuint64_t d2[2] = {(cuuint64_t)sh.d_c, (cuuint64_t)sh.H * sh.d_h};
        cuuint64_t s2[1] = {(cuuint64_t)sh.d_c * 2};
        cuuint32_t b2[2] = {64, 128};
        cuuint32_t e2[2] = {1, 1};
        r = encode(w == 0 ? &wuk_map : &wuv_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(w == 0 ? a.w_uk : a.w_uv), d2, s2, b2, e2, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            char buf[96];
            snprintf(buf, sizeof(buf), "cuTensorMapEncodeTiled %s (CUresult %d)", w == 0 ? "W_UK" : "W_UV", (int)r);
            return note_error(buf, cudaErrorInvalidValue);
        }
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

    k_lh_prep<<<dim3(sh.H, (sh.B + 31) / 32), kPrepThreads, prep_smem, st>>>(wuk_map, a, qimg, p.n_qchunks);
    e = cudaGetLastError();
    if (e != cudaSuccess) return note_error("k_lh_prep launch", e);
    profile_begin(st);
    e = launch_pdl_lh(k_lh_attn, dim3(2 * p.G2), dim3(kThreads), attn_smem, st, map, p);
    profile_end(st);
    if (e != cudaSuccess) return note_error("k_lh_attn launch", e);
    e = launch_pdl_lh(k_lh_combine, dim3(sh.H, (sh.B + 31) / 32), dim3(kCombThreads), comb_smem, st, wuv_map, a, p);
    *launches += 3;
    return note_error("k_lh_combine launch", e);
}

}  // namespace mtla
