// tc_decode_lh.cu -- bf16 decode step for many heads (32 < H <= 128) on the
// tensor cores: all heads form the M = 128 dimension of the contraction.
//
// "Multi-head Temporal Latent Attention", Method (1): one new token per
// sequence updates the slot being filled in place, then the absorbed query of
// every head attends slots 0..floor(t/s) (Sec. 6.1: O(N/s) slot reads). The
// latent cache is streamed once from HBM.
//
// The output accumulator O [128 heads x d_c] fp32 fills the whole tensor
// memory at d_c = 512, so a cluster of two CTAs splits the work by role:
//   - rank 0 holds the absorbed queries in tensor memory and computes the
//     scores of every 128-slot tile over the whole slot width (M = 128 heads,
//     N = 128 slots), runs the online softmax and writes P (bf16) straight
//     into rank 1's shared memory;
//   - rank 1 holds O and accumulates O += P . V over the latent columns
//     (M = 128 heads, N = 256 columns), reading each tile a second time (from
//     L2: the two CTAs stream the same tiles a few microseconds apart).
// No partial scores are exchanged; the tensor pipes of the two CTAs take
// about the same time per tile (36 score MMAs of N = 128 against 16 P.V MMAs
// of N = 256).
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
#include <type_traits>
#include <utility>

#include <cuda_fp16.h>

#include "common.cuh"
#include "mtla_internal.h"
#include "prep.cuh"
#include "tc_common.cuh"

namespace mtla {

namespace {

using namespace tc;

constexpr int kKT = 128;          // slots per tile
constexpr int kHalf = 64;         // slots per half tile (one P buffer, one P.V block)
constexpr int kMaxRing = 8;       // ring stages of either CTA
constexpr int kMaxQChunks = 10;   // 64-column chunks of a slot (D <= 640)
constexpr int kChunksPerStage = 3;  // 64-column chunks per score-ring stage (one TMA box)
constexpr int kThreads = 320;     // warp 0 TMA, 1 MMA issue, 2-9 softmax / events
constexpr int kMaxClusters = 80;  // >= SMs/2 of any sm_100 part; sizes the partial buffer
constexpr int kMaxB = 2048;
constexpr float kRescaleLog2 = 8.f;

struct LhArgs {
    int B, H, D, d_c, d_r, s, max_slots;
    int G2;                 // clusters in the grid
    int n_qchunks;          // D / 64
    int unit_cols;          // latent columns per P.V MMA (N): min(256, d_c)
    uint32_t smem_bytes;    // dynamic shared memory of the attention kernel
    float scale_log2;
    const int32_t* pos;
    const uint8_t* qimg;    // [B] x n_qchunks x [128 heads x 128 B]
    float* part;            // [(kMaxClusters + B), H, d_c + 4]
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
template <typename E>
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
    // everything above reads weights only; the step's inputs (and the cache this
    // step updates) only once the previous kernel in the stream has completed
    pdl_wait();
    // qC rows of the 32 sequences (zero past B) as the K-major B operand
    for (int e = tid; e < 32 * n_qc * 8; e += kPrepThreads) {
        const int bb = e / (n_qc * 8), rem = e % (n_qc * 8), c = rem >> 3, u = rem & 7;
        const int b = c0 + bb, col = c * 64 + u * 8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (b < sh.B && col < sh.d_h) v = *(const uint4*)((const E*)a.q_c + ((size_t)b * sh.H + h) * sh.d_h + col);
        *(uint4*)(x_s + (size_t)c * 4096 + sw128_offset(bb, u * 8)) = v;
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t t_d = *tmem_slot;
    if (tid == 0) {
        bool ok = true;
        const uint32_t idesc = idesc_f32<E>(128, 32, true, false);
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
                if (2 * k < sh.d_r) qv[i] = *(const uint32_t*)((const E*)a.q_r + ((size_t)b * sh.H + h) * sh.d_r + 2 * k);
            }
        }
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int e = tid + i * kPrepThreads, bb = e / npair, k = e % npair, b = c0 + bb;
            if (bb >= 32 || b >= sh.B || !lh_pos_ok(sh, tv[i])) continue;
            float v0 = 0.f, v1 = 0.f;
            if (2 * k < sh.d_r) {
                const E* xq = (const E*)&qv[i];
                const float x0 = to_f<E>(xq[0]), x1 = to_f<E>(xq[1]);
                float sn, cs;
                pair_sincos_f(tv[i], rope_freq[k], &sn, &cs);
                v0 = x0 * cs - x1 * sn;
                v1 = x0 * sn + x1 * cs;
            }
            const int j = sh.d_c + 2 * k;
            *(uint32_t*)(qimg + (size_t)b * img_bytes + (size_t)(j >> 6) * 128 * 128 + sw128_offset(h, j & 63)) =
                pack2<E>(v0, v1);
        }
    }
    // latent part: warp w reads TMEM lane quarter w mod 4 (latent rows), sequences
    // 16 (w / 4) .. 16 (w / 4) + 15. Each sequence's row h of every 64-column
    // chunk is one 128-byte run of its image: the rows are assembled in shared
    // memory (the W_UK buffer, free once the MMAs are done) with the image's
    // swizzle and leave as 16-byte stores.
    const bool done = mbar_wait(&bars[1], (n_kb - 1) & 1);
    tc_fence_after();
    uint8_t* stage = w_s;                                  // [32 sequences][n_kc chunks][128 B]
    {
        const int quarter = warp & 3, half = warp >> 2;
        const uint32_t hx = (uint32_t)(h & 7);
        for (int mb = 0; mb < n_kc / 2; ++mb) {
            float v[16];
            tmem_ld16(t_d + mb * 32 + half * 16 + ((uint32_t)(quarter * 32) << 16), v);
            tmem_wait_ld();
            const int j = mb * 128 + quarter * 32 + lane;      // latent column
            const uint32_t in_row = ((((uint32_t)(j & 63) >> 3) ^ hx) << 4) + ((j & 7) << 1);
#pragma unroll
            for (int s = 0; s < 16; ++s) {
                const int bb = half * 16 + s;
                *(E*)(stage + ((size_t)bb * n_kc + (j >> 6)) * 128 + in_row) = from_f<E>(v[s]);
            }
        }
    }
    __syncthreads();
    for (int e = tid; e < 32 * n_kc * 8; e += kPrepThreads) {
        const int row = e >> 3, u = e & 7, bb = row / n_kc, c = row % n_kc, b = c0 + bb;
        if (done && b < sh.B && lh_pos_ok(sh, a.pos[b]))
            *(uint4*)(qimg + (size_t)b * img_bytes + (size_t)c * 128 * 128 + (size_t)h * 128 + u * 16) =
                *(const uint4*)(stage + (size_t)row * 128 + u * 16);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(t_d, 128);
    // in-place slot updates of this group's sequences b with b mod H = h
    for (int b = c0 + ((h - c0 % sh.H) % sh.H + sh.H) % sh.H; b < min(sh.B, c0 + 32); b += sh.H) {
        __syncthreads();
        decode_update_body<E>(a, b);
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

// Per-tile side information rank 0 sends with P half 0: the factor each row
// of O must be scaled by before this tile adds to it (1 if none), and whether
// any row of a TMEM lane quarter needs it.
struct __align__(16) LhSide {
    float fac[128];
    int flag[4];
};

// Shared-memory control block at the (1024-aligned) start of both CTAs' shared
// memory. The barriers a peer arrives on and the side information sit at the
// same offset in both CTAs.
struct LhCtl {
    uint64_t full[kMaxRing], empty[kMaxRing];   // this CTA's ring of landed tiles
    uint64_t s_full, s_empty, qt_full;          // rank 0: scores in TMEM; query chunks in TMEM
    uint64_t p_free[2];                         // rank 0: rank 1's P.V has read P half h
    uint64_t p_full[2];                         // rank 1: P half h (and the side information) copied in
    uint64_t o_done, ev_full, ev_done;          // rank 1: P.V complete; event posted / handled
    uint64_t drain;                             // MMAs in flight when a wait gave up
    uint32_t tmem_base;
    volatile int fail;
    int b0, j0, n_tiles;                        // the cluster's first tile and tile count
    volatile int ev[2];                         // rank 1: event type and argument
    volatile int ev_arg[2];
    LhSide side;                                // rank 0: staged for the copy; rank 1: received
};
constexpr uint32_t kCtlBytes = 1024;
static_assert(sizeof(LhCtl) <= kCtlBytes, "control block");

enum { kEvEnd = 0, kEvRescale = 1, kEvZero = 2, kEvSegEnd = 3 };

__device__ __forceinline__ bool lh_wait(uint64_t* bar, uint32_t parity, LhCtl& cs) {
    if (cs.fail) return false;
    if (mbar_wait(bar, parity)) return true;
    cs.fail = 1;
    return false;
}
__device__ __forceinline__ bool lh_wait_cluster(uint64_t* bar, uint32_t parity, LhCtl& cs) {
    if (cs.fail) return false;
    if (mbar_wait_cluster(bar, parity)) return true;
    cs.fail = 1;
    return false;
}

// Walk over the cluster's tiles in order: sequence b, tile j of nt, nb slots.
struct LhWalk {
    int b, j, nb, nt;
    __device__ void start(const LhArgs& p, int b0, int j0) {
        b = b0;
        j = j0;
        nb = b < p.B ? lh_slots(p, b) : 0;
        nt = (nb + kKT - 1) / kKT;
    }
    __device__ void next(const LhArgs& p) {
        if (++j < nt) return;
        j = 0;
        do {
            ++b;
            nb = b < p.B ? lh_slots(p, b) : 0;
        } while (b < p.B && nb == 0);
        nt = (nb + kKT - 1) / kKT;
    }
    __device__ bool last_of_seq() const { return j == nt - 1; }
};

// Decode attention for one cluster of two CTAs over a contiguous range of
// 128-slot tiles (the grid is balanced over all tiles of the batch):
//   rank 0 (scorer): the absorbed queries of all heads in TMEM as the MMA's A
//     operand; S = q~ K^T over the whole slot width (M = 128 heads, N = 128
//     slots) from 64-column chunks of the tile streamed through a 14-stage
//     ring; online softmax (two threads per head row, one per 64-slot half);
//     P (bf16) written straight into rank 1's shared memory;
//   rank 1 (accumulator): O [128 heads x d_c] fp32 in all of its TMEM;
//     O += P V from the tile's latent columns (N = 256) streamed through its
//     own ring (the second read of each tile, served by L2).
// Warp 0: TMA; warp 1: MMA issue; warps 2-9: softmax (rank 0) or the event
// handlers of rank 1 (rescale of O when a row's reference maximum moves,
// zeroing of cache rows past a sequence's last slot, writing O at the end of a
// sequence segment). One partial (O, m, l) per sequence segment.
template <typename E>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    k_lh_attn(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v, const LhArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const uint32_t pad = (uint32_t)(base - smem_raw);
    LhCtl& cs = *(LhCtl*)base;
    uint8_t* region = base + kCtlBytes;
    const uint32_t region_bytes = p.smem_bytes - pad - kCtlBytes;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rank = (int)cluster_rank();
    const int g = blockIdx.x >> 1;                        // cluster index
    const int nq = p.n_qchunks;                           // 64-column chunks of a slot
    const uint32_t unit_bytes = (uint32_t)p.unit_cols * kHalf * 2;
    const int n_units = p.d_c / p.unit_cols;              // P.V units per 64-slot half
    const int n_kst = (nq + kChunksPerStage - 1) / kChunksPerStage;   // score stages per tile
    // both CTAs: two P halves [128 heads x 64 slots] bf16 (rank 0 stages them,
    // rank 1 receives them), then the ring: rank 0 stages of three 64-column
    // chunks [128 slots x 64 columns] each, rank 1 units [64 slots x unit_cols]
    const uint32_t stage_bytes = rank == 0 ? (uint32_t)kChunksPerStage * 16384 : unit_bytes;
    const int ring = min(kMaxRing, (int)((region_bytes - 2 * 16384) / stage_bytes));
    uint8_t* ring_base = region + 2 * 16384;

    // ---- the cluster's tile range (reads pos only)
    if (warp == 0) {
        int total = 0;
        for (int c = 0; c < p.B; c += 32) {
            const int b = c + lane;
            int t = b < p.B ? (lh_slots(p, b) + kKT - 1) / kKT : 0;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
            total += t;
        }
        const int gt0 = (int)(((int64_t)g * total) / p.G2);
        const int gt1 = (int)(((int64_t)(g + 1) * total) / p.G2);
        // the sequence holding tile gt0: first b whose inclusive tile prefix exceeds gt0
        int run = 0, b0 = p.B, j0 = 0;
        for (int c = 0; c < p.B && b0 == p.B; c += 32) {
            const int b = c + lane;
            const int t = b < p.B ? (lh_slots(p, b) + kKT - 1) / kKT : 0;
            int incl = t;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            const unsigned hit = __ballot_sync(0xffffffffu, run + incl > gt0);
            if (hit) {
                const int l0 = __ffs(hit) - 1;
                const int excl = __shfl_sync(0xffffffffu, incl - t, l0);
                b0 = c + l0;
                j0 = gt0 - (run + excl);
            }
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            cs.b0 = b0;
            cs.j0 = j0;
            cs.n_tiles = gt1 - gt0;
        }
    }
    if (tid == 0) {
        for (int i = 0; i < kMaxRing; ++i) {
            mbar_init(&cs.full[i], 1);
            mbar_init(&cs.empty[i], 1);
        }
        mbar_init(&cs.s_full, 1);
        mbar_init(&cs.s_empty, 8);
        mbar_init(&cs.qt_full, 8);
        for (int h = 0; h < 2; ++h) {
            mbar_init(&cs.p_free[h], 1);
            mbar_init(&cs.p_full[h], 1);
        }
        mbar_init(&cs.o_done, 1);
        mbar_init(&cs.ev_full, 1);
        mbar_init(&cs.ev_done, 1);
        mbar_init(&cs.drain, 1);
        cs.fail = 0;
        fence_mbar_init();
        tma_prefetch_desc(rank == 0 ? &map_k : &map_v);
    }
    if (warp == 1) {
        tmem_alloc(&cs.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_sync();                      // the peer's barriers exist before any remote operation
    pdl_launch_dependents();
    const uint32_t tmem = cs.tmem_base;
    const int n = cs.n_tiles;
    LhWalk w0;
    w0.start(p, cs.b0, cs.j0);

    int loads_issued = 0;                // producer: ring fills, for the drain after a failure
    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        // Tiles before a sequence's last one do not hold the slot k_lh_prep
        // updates, so their loads start before the wait for that kernel.
        if (lane == 0) {
            LhWalk w = w0;
            bool waited = false;
            for (int k = 0; k < n && !cs.fail; ++k, w.next(p)) {
                if (!waited && w.last_of_seq()) {
                    pdl_wait();
                    waited = true;
                }
                if (rank == 0) {
                    // one box per stage: chunks 3i .. 3i+2 of 128 slots (a chunk past
                    // the slot width reads as zero)
                    for (int i = 0; i < n_kst; ++i, ++loads_issued) {
                        const int st = loads_issued % ring;
                        if (loads_issued >= ring && !lh_wait(&cs.empty[st], ((loads_issued / ring) - 1) & 1, cs)) break;
                        mbar_arrive_expect_tx(&cs.full[st], stage_bytes);
                        tma_load_4d(ring_base + (size_t)st * stage_bytes, &map_k, &cs.full[st], 0, w.j * kKT,
                                    i * kChunksPerStage, w.b);
                    }
                } else {
                    for (int h = 0; h < 2; ++h)
                        for (int u = 0; u < n_units; ++u, ++loads_issued) {
                            const int st = loads_issued % ring;
                            if (loads_issued >= ring &&
                                !lh_wait(&cs.empty[st], ((loads_issued / ring) - 1) & 1, cs))
                                break;
                            mbar_arrive_expect_tx(&cs.full[st], unit_bytes);
                            tma_load_4d(ring_base + (size_t)st * unit_bytes, &map_v, &cs.full[st], 0,
                                        w.j * kKT + h * kHalf, u * (p.unit_cols / 64), w.b);
                        }
                }
            }
            if (cs.fail) {
                // let the loads in flight land before shared memory is released
                for (int k = max(0, loads_issued - ring); k < loads_issued; ++k)
                    mbar_wait(&cs.full[k % ring], (k / ring) & 1);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            if (rank == 0) {
                // -------------------------------------------------------- score MMAs
                const uint32_t id_s = idesc_f32<E>(128, kKT, false, false);
                const uint32_t t_s = tmem, t_q = tmem + 128;
                LhWalk w = w0;
                int it = 0, seg = -1;
                for (int k = 0; k < n; ++k, w.next(p)) {
                    if (k == 0 || w.j == 0) {
                        ++seg;
                        if (!lh_wait(&cs.qt_full, seg & 1, cs)) break;    // query chunks in TMEM
                    }
                    if (k >= 1 && !lh_wait(&cs.s_empty, (k - 1) & 1, cs)) break;   // S(k-1) read out
                    tc_fence_after();
                    bool ok = true;
                    // straight-line groups of four MMAs, one wait per stage of three chunks
#pragma unroll
                    for (int c = 0; c < kMaxQChunks; ++c) {
                        if (c < nq && ok) {
                            const int st = it % ring;
                            const int cs3 = c % kChunksPerStage;
                            if (cs3 == 0) {
                                ok = lh_wait(&cs.full[st], (it / ring) & 1, cs);
                                tc_fence_after();
                            }
                            if (ok) {
                                const uint64_t kd = sdesc_sw128(
                                    smem_u32(ring_base + (size_t)st * stage_bytes + cs3 * 16384), 16, 1024);
                                umma_bf16_ts(t_s, t_q + c * 32, kd, id_s, c != 0 ? 1u : 0u);
                                umma_bf16_ts(t_s, t_q + c * 32 + 8, desc_add(kd, 32), id_s, 1u);
                                umma_bf16_ts(t_s, t_q + c * 32 + 16, desc_add(kd, 64), id_s, 1u);
                                umma_bf16_ts(t_s, t_q + c * 32 + 24, desc_add(kd, 96), id_s, 1u);
                                if (cs3 == kChunksPerStage - 1 || c == nq - 1) {
                                    umma_commit(&cs.empty[st]);
                                    ++it;
                                }
                            }
                        }
                    }
                    if (!ok) break;
                    umma_commit(&cs.s_full);
                }
                if (cs.fail) {
                    umma_commit(&cs.drain);
                    mbar_wait(&cs.drain, 0);
                }
            } else {
                // -------------------------------------------------------- P.V MMAs
                const uint32_t id_o = idesc_f32<E>(128, p.unit_cols, false, true);
                LhWalk w = w0;
                int it = 0, ev = 0, ocnt = 0;
                auto post = [&](int type, int arg) -> bool {
                    cs.ev[0] = type;
                    cs.ev_arg[0] = arg;
                    mbar_arrive(&cs.ev_full);
                    const bool ok = lh_wait(&cs.ev_done, ev & 1, cs);
                    ++ev;
                    return ok;
                };
                auto o_settle = [&]() -> bool {      // every P.V issued so far is complete
                    umma_commit(&cs.o_done);
                    ++ocnt;
                    return lh_wait(&cs.o_done, (ocnt - 1) & 1, cs);
                };
                bool ok = true;
                for (int k = 0; k < n && ok; ++k, w.next(p)) {
                    const bool first = (k == 0) || (w.j == 0);
                    for (int h = 0; h < 2 && ok; ++h) {
                        // rank 0's bulk copy of P half h (and, with half 0, the side
                        // information) completes its bytes on p_full[h]
                        mbar_arrive_expect_tx(&cs.p_full[h], h == 0 ? 16384u + (uint32_t)sizeof(LhSide) : 16384u);
                        ok = lh_wait_cluster(&cs.p_full[h], k & 1, cs);
                        if (!ok) break;
                        tc_fence_after();
                        const volatile int* fl = cs.side.flag;
                        if (h == 0 && !first && (fl[0] | fl[1] | fl[2] | fl[3])) {
                            // a row's reference maximum moved: O rows scaled before this tile adds to them
                            ok = o_settle() && post(kEvRescale, 0);
                            if (!ok) break;
                            tc_fence_after();
                        }
                        const int s0 = w.j * kKT + h * kHalf;
                        const int v0 = max(0, min(kHalf, w.nb - s0));          // valid slots of this half
                        const int vend = min(kHalf, p.max_slots - s0);         // rows inside the cache buffer
                        if (v0 < vend) {
                            // rows past the sequence's last slot hold stale bytes: zeroed before P.V
                            ok = post(kEvZero, (it << 8) | v0);
                            if (!ok) break;
                        }
                        const uint64_t pd = sdesc_sw128(smem_u32(region + h * 16384), 16, 1024);
                        for (int u = 0; u < n_units; ++u) {
                            const int st = it % ring;
                            ok = lh_wait(&cs.full[st], (it / ring) & 1, cs);
                            if (!ok) break;
                            tc_fence_after();
                            const uint64_t vd = sdesc_sw128(smem_u32(ring_base + (size_t)st * unit_bytes), 8192, 1024);
                            const uint32_t t_o = tmem + u * p.unit_cols;
                            umma_bf16(t_o, pd, vd, id_o, (first && h == 0) ? 0u : 1u);
                            umma_bf16(t_o, desc_add(pd, 32), desc_add(vd, 2048), id_o, 1u);
                            umma_bf16(t_o, desc_add(pd, 64), desc_add(vd, 4096), id_o, 1u);
                            umma_bf16(t_o, desc_add(pd, 96), desc_add(vd, 6144), id_o, 1u);
                            umma_commit(&cs.empty[st]);
                            ++it;
                        }
                        if (!ok) break;
                        umma_commit_to(&cs.p_free[h], 0x1);                    // rank 0 may write P half h again
                    }
                    if (ok && (k == n - 1 || w.last_of_seq())) {
                        ok = o_settle() && post(kEvSegEnd, g + w.b);
                    }
                }
                cs.ev[0] = kEvEnd;
                mbar_arrive(&cs.ev_full);
                if (cs.fail) {
                    umma_commit(&cs.drain);
                    mbar_wait(&cs.drain, 0);
                }
            }
        }
    } else if (rank == 0) {
        // ------------------------------------------------------------ softmax (two threads per head row)
        // Warps 2-9: row r = (warp mod 4) * 32 + lane (the TMEM lane quarter a
        // warp may access), slot half hc = (warp - 2) / 4 of each tile. No early
        // exit from the loop: after a bounded wait gave up, later waits return
        // at once, so every thread reaches every named barrier.
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const int hc = (warp - 2) >> 2;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint32_t t_s = tmem, t_q = tmem + 128;
        // columns 480..484: the two half-row maxima by tile parity, and the
        // second half's row sum at a segment end, exchanged between the two
        // threads of a row (same TMEM lane quarter)
        const uint32_t t_x = tmem + 480 + lane_off;
        uint8_t* prow = region + hc * 16384 + r * 128;            // staging of P half hc, row r
        const uint32_t p_peer = map_to_rank(region + hc * 16384, 1);
        const uint32_t side_peer = map_to_rank(&cs.side, 1);
        const uint32_t pfull_peer = map_to_rank(&cs.p_full[hc], 1);
        const bool elected = (warp == 2 + 4 * hc) && lane == 0;   // issues the half's copies
        // query chunks c = hc, hc + 2, ... of sequence b into TMEM (row r de-swizzled from the image)
        auto load_qt = [&](int b) {
            const uint8_t* img = p.qimg + (size_t)b * nq * 16384 + (size_t)r * 128;
            for (int c = hc; c < nq; c += 2) {
                uint32_t wv[32];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const uint4 v = *(const uint4*)(img + (size_t)c * 16384 + (((u ^ r) & 7) << 4));
                    wv[4 * u] = v.x;
                    wv[4 * u + 1] = v.y;
                    wv[4 * u + 2] = v.z;
                    wv[4 * u + 3] = v.w;
                }
                tmem_st32_u(t_q + c * 32 + lane_off, wv);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&cs.qt_full);
        };
        pdl_wait();                      // the query images come from k_lh_prep
        if (n > 0) load_qt(w0.b);
        float m_ref = -INFINITY, l = 0.f;   // l: this thread's half of the row sum
        int k_in_seg = 0;
        LhWalk w = w0;
        for (int k = 0; k < n; ++k) {
            if (k > 0 && w.j == 0) {
                m_ref = -INFINITY;
                l = 0.f;
                k_in_seg = 0;
            }
            lh_wait(&cs.s_full, k & 1, cs);
            tc_fence_after();
            float sv[64];
            tmem_ld32(t_s + hc * 64 + lane_off, sv);
            tmem_ld32(t_s + hc * 64 + 32 + lane_off, sv + 32);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&cs.s_empty);
            LhWalk nx = w;
            nx.next(p);
            // S(k) complete: every score MMA that read the query chunks is done
            if (k + 1 < n && nx.j == 0) load_qt(nx.b);
            const int valid = min(kKT, w.nb - w.j * kKT) - hc * kHalf;   // valid slots of this half
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};  // four independent chains
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                sv[c] = c < valid ? sv[c] : -INFINITY;
                m4[c & 3] = fmaxf(m4[c & 3], sv[c]);
            }
            float mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * p.scale_log2;
            tmem_st1(t_x + (k & 1) * 2 + hc, mt);
            tmem_wait_st();
            tc_fence_before();
            named_sync(1, 256);
            tc_fence_after();
            mt = fmaxf(mt, tmem_ld1(t_x + (k & 1) * 2 + (hc ^ 1)));
            tmem_wait_ld();
            // lazy rescale: the reference maximum moves only when the tile's maximum
            // exceeds it by more than 2^8 (P stays <= 256); both halves decide alike
            const bool upd = mt > m_ref + kRescaleLog2;
            const float nm = upd ? mt : m_ref;
            const float fac = ex2_approx(m_ref - nm);    // 0 when m_ref was -inf, 1 when kept
            float rs4[4] = {0.f, 0.f, 0.f, 0.f};
            uint32_t pk[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                const float p0 = ex2_approx(fmaf(sv[2 * c], p.scale_log2, -nm));
                const float p1 = ex2_approx(fmaf(sv[2 * c + 1], p.scale_log2, -nm));
                rs4[c & 3] += p0 + p1;
                pk[c] = pack2<E>(p0, p1);
            }
            l = fmaf(l, fac, (rs4[0] + rs4[1]) + (rs4[2] + rs4[3]));
            m_ref = nm;
            const bool need = upd && k_in_seg > 0;
            // P half hc of tile k: staged here (the copy of tile k-1 has read the
            // staging), then one bulk copy into rank 1 once its P.V of tile k-1
            // has read the destination; the copy completes on rank 1's p_full[hc]
            if (elected) bulk_wait_read_all();
            named_sync(2 + hc, 128);
#pragma unroll
            for (int u = 0; u < 8; ++u)
                *(uint4*)(prow + (((u ^ r) & 7) << 4)) = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
            if (hc == 0) {
                cs.side.fac[r] = need ? fac : 1.f;
                const bool any = __any_sync(0xffffffffu, need);
                if (lane == 0) cs.side.flag[quarter] = any ? 1 : 0;
            }
            fence_proxy_async();
            named_sync(2 + hc, 128);
            if (elected) {
                if (k >= 1) lh_wait(&cs.p_free[hc], (k - 1) & 1, cs);
                if (!cs.fail) {
                    bulk_copy_to_peer(p_peer, region + hc * 16384, 16384, pfull_peer);
                    if (hc == 0) bulk_copy_to_peer(side_peer, &cs.side, (uint32_t)sizeof(LhSide), pfull_peer);
                    bulk_commit_group();
                }
            }
            ++k_in_seg;
            if (k == n - 1 || w.last_of_seq()) {
                // (m, l) of this sequence segment; rank 1 writes its O
                if (hc == 1) {
                    tmem_st1(t_x + 4, l);
                    tmem_wait_st();
                }
                tc_fence_before();
                named_sync(1, 256);
                tc_fence_after();
                if (hc == 0) {
                    const float l1 = tmem_ld1(t_x + 4);
                    tmem_wait_ld();
                    if (r < p.H) {
                        float* dst = p.part + ((size_t)(g + w.b) * p.H + r) * ((size_t)p.d_c + 4);
                        dst[p.d_c] = m_ref;
                        dst[p.d_c + 1] = l + l1;
                    }
                }
            }
            w = nx;
        }
        if (elected) bulk_wait_read_all();
    } else {
        // ------------------------------------------------------------ rank 1 events
        // Warps 2-9 take the events the MMA thread posts, in order: thread
        // (row r, column half hc) of O.
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const int hc = (warp - 2) >> 2;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int cols = p.d_c / 2;
        const int sidx = tid - 64;
        for (int ev = 0;; ++ev) {
            const bool got = mbar_wait(&cs.ev_full, ev & 1);
            if (!named_sync_and(1, 256, got)) break;
            const int type = cs.ev[0], arg = cs.ev_arg[0];
            if (type == kEvEnd) break;
            tc_fence_after();
            if (type == kEvRescale) {
                const float f = cs.side.fac[r];
                if (__any_sync(0xffffffffu, f != 1.f)) {
                    for (int cc = 0; cc < cols / 32; ++cc) {
                        const uint32_t ta = tmem + hc * cols + cc * 32 + lane_off;
                        float v[32];
                        tmem_ld32(ta, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] *= f;
                        tmem_st32(ta, v);
                    }
                    tmem_wait_st();
                }
            } else if (type == kEvZero) {
                // rows v0.. of the units it0 .. it0 + n_units - 1 (one 64-slot half)
                const int it0 = arg >> 8, v0 = arg & 255;
                const int rows = kHalf - v0, per_unit = rows * (p.unit_cols / 8);
                bool landed = true;
                for (int u = 0; u < n_units; ++u)
                    landed &= mbar_wait(&cs.full[(it0 + u) % ring], ((it0 + u) / ring) & 1);
                if (landed) {
                    for (int e = sidx; e < n_units * per_unit; e += 256) {
                        const int u = e / per_unit, rem = e % per_unit;
                        const int row = v0 + rem / (p.unit_cols / 8), q16 = rem % (p.unit_cols / 8);
                        uint8_t* unit = ring_base + (size_t)((it0 + u) % ring) * unit_bytes;
                        *(uint4*)(unit + (size_t)(q16 >> 3) * 8192 + (size_t)row * 128 + (q16 & 7) * 16) =
                            make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async();
                } else {
                    cs.fail = 1;
                }
            } else if (type == kEvSegEnd) {
                // TMEM loads are warp-collective: every lane loads, rows past H drop theirs
                float* dst = p.part + ((size_t)arg * p.H + r) * ((size_t)p.d_c + 4) + hc * cols;
                for (int cc = 0; cc < cols / 32; ++cc) {
                    float v[32];
                    tmem_ld32(tmem + hc * cols + cc * 32 + lane_off, v);
                    tmem_wait_ld();
                    if (r < p.H) {
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            *(float4*)(dst + cc * 32 + 4 * u) = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
                    }
                }
            }
            tc_fence_before();
            named_sync(1, 256);
            if (sidx == 0) mbar_arrive(&cs.ev_done);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (cs.fail && tid == 0) latch_status(p.status, kStatusTimeout);
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
template <typename E>
__global__ void __launch_bounds__(kCombThreads, 1)
    k_lh_combine(const __grid_constant__ CUtensorMap wuv_map, DecodeArgs a, LhArgs p) {
    pdl_launch_dependents();   // the next step's prep may stage its W_UK rows now
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
                    pk.x = pack2<E>(o[s2][0], o[s2][1]);
                    pk.y = pack2<E>(o[s2][2], o[s2][3]);
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
            const uint32_t idesc = idesc_f32<E>(128, 32, false, false);
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
                    ((E*)a.out)[((size_t)b * sh.H + h) * sh.d_h + i] = from_f<E>(v[s8]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(t_d, 128);
}

// ---------------------------------------------------------------- host side

// The attention kernel takes all the shared memory a block may opt into: its
// rings are sized from what it gets (at least two P.V units on rank 1).
size_t lh_attn_smem() {
    static int optin = 0;
    if (!optin) {
        int dev = 0, v = 0;
        if (cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) == cudaSuccess && v > 0)
            optin = v;
        else
            optin = 232448;
    }
    return (size_t)optin;
}
size_t lh_attn_smem_min(const Shape& sh) {
    const size_t unit = (size_t)std::min(256, sh.d_c) * kHalf * 2;
    return 1023 + kCtlBytes + 2 * 16384 + 2 * std::max(unit, (size_t)kChunksPerStage * 16384);
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
           lh_prep_smem(sh) <= 227 * 1024 && sh.D / 64 <= kMaxQChunks && lh_attn_smem_min(sh) <= 232448 - 16384;
}

size_t tc_decode_lh_workspace(const Shape& sh) {
    return align256((size_t)sh.B * (sh.D / 64) * 128 * 128) +
           align256((size_t)(kMaxClusters + sh.B) * sh.H * (sh.d_c + 4) * sizeof(float));
}

template <typename E>
cudaError_t tc_decode_lh_impl(const DecodeArgs& a, cudaStream_t st, uint64_t* launches) {
    const Shape& sh = a.sh;
    uint8_t* qimg = (uint8_t*)a.workspace;
    float* part = (float*)((char*)a.workspace + align256((size_t)sh.B * (sh.D / 64) * 128 * 128));
    auto encode = (PFN_cuTensorMapEncodeTiled_v12000)tensor_map_encoder();
    if (!encode) return note_error("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", cudaErrorNotSupported);
    // the cache viewed as {64 columns, max_slots, D / 64 chunks, B} (chunk
    // stride 128 B), so that one box brings several 64-column chunks, each
    // laid out as its own SW128 operand: three chunks x 128 slots for the
    // scores (rank 0), unit_cols / 64 chunks x 64 slots for P.V (rank 1).
    // Slots past max_slots and chunks past D / 64 read as zero. A TMA engine
    // completes about as many boxes per second whatever their size up to
    // 16 KB, so few large boxes keep one SM at the HBM share it needs.
    CUtensorMap map_k, map_v;
    CUresult r = CUDA_SUCCESS;
    for (int m = 0; m < 2; ++m) {
        cuuint64_t dims[4] = {64, (cuuint64_t)sh.max_slots, (cuuint64_t)(sh.D / 64), (cuuint64_t)sh.B};
        cuuint64_t strides[3] = {(cuuint64_t)sh.D * 2, 128, (cuuint64_t)sh.max_slots * sh.D * 2};
        cuuint32_t box[4] = {64, (cuuint32_t)(m == 0 ? kKT : kHalf),
                             (cuuint32_t)(m == 0 ? kChunksPerStage : std::min(256, sh.d_c) / 64), 1};
        cuuint32_t estr[4] = {1, 1, 1, 1};
        r = encode(m == 0 ? &map_k : &map_v, (std::is_same<E, f16>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16), 4, a.cache, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            char buf[96];
            snprintf(buf, sizeof(buf), "cuTensorMapEncodeTiled cache (CUresult %d)", (int)r);
            return note_error(buf, cudaErrorInvalidValue);
        }
    }
    // W_UK and W_UV as [H * d_h rows][d_c] bf16, 128-row x 64-column boxes
    // (rows past the last head read as zero)
    CUtensorMap wuk_map, wuv_map;
    for (int w = 0; w < 2; ++w) {
        cuuint64_t d2[2] = {(cuuint64_t)sh.d_c, (cuuint64_t)sh.H * sh.d_h};
        cuuint64_t s2[1] = {(cuuint64_t)sh.d_c * 2};
        cuuint32_t b2[2] = {64, 128};
        cuuint32_t e2[2] = {1, 1};
        r = encode(w == 0 ? &wuk_map : &wuv_map, (std::is_same<E, f16>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16), 2,
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
    p.unit_cols = std::min(256, sh.d_c);
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    static size_t done_prep[64] = {0}, done_attn[64] = {0}, done_comb[64] = {0};
    static int co_resident[64] = {0};
    const size_t prep_smem = lh_prep_smem(sh);
    const size_t attn_smem = lh_attn_smem();
    p.smem_bytes = (uint32_t)attn_smem;
    const size_t comb_smem = lh_comb_smem(sh);
    cudaError_t e = lh_set_smem(k_lh_prep<E>, prep_smem, &done_prep[dev]);
    if (e == cudaSuccess) e = lh_set_smem(k_lh_attn<E>, attn_smem, &done_attn[dev]);
    if (e == cudaSuccess) e = lh_set_smem(k_lh_combine<E>, comb_smem, &done_comb[dev]);
    if (e != cudaSuccess) return note_error("cudaFuncSetAttribute(large-head decode)", e);
    if (!co_resident[dev]) {
        // clusters that can be resident at once: the balanced split assumes one wave
        cudaLaunchConfig_t oc = {};
        oc.gridDim = dim3(2 * kMaxClusters);
        oc.blockDim = dim3(kThreads);
        oc.dynamicSmemBytes = attn_smem;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, k_lh_attn<E>, &oc) != cudaSuccess || n <= 0) {
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

    e = launch_pdl_lh(k_lh_prep<E>, dim3(sh.H, (sh.B + 31) / 32), dim3(kPrepThreads), prep_smem, st, wuk_map, a, qimg,
                      p.n_qchunks);
    if (e != cudaSuccess) return note_error("k_lh_prep launch", e);
    profile_begin(st);
    e = launch_pdl_lh(k_lh_attn<E>, dim3(2 * p.G2), dim3(kThreads), attn_smem, st, map_k, map_v, p);
    profile_end(st);
    if (e != cudaSuccess) return note_error("k_lh_attn launch", e);
    e = launch_pdl_lh(k_lh_combine<E>, dim3(sh.H, (sh.B + 31) / 32), dim3(kCombThreads), comb_smem, st, wuv_map, a, p);
    *launches += 3;
    return note_error("k_lh_combine launch", e);
}

cudaError_t tc_decode_lh(const DecodeArgs& a, cudaStream_t st, uint64_t* launches) {
    return a.sh.dtype == kDtypeF16 ? tc_decode_lh_impl<f16>(a, st, launches) : tc_decode_lh_impl<bf16>(a, st, launches);
}

}  // namespace mtla
