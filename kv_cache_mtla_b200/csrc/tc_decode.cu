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
#include <cstring>
#include <mutex>
#include <type_traits>
#include <utility>

#include "common.cuh"
#include "mtla_internal.h"
#include "prep.cuh"
#include "tc_common.cuh"

namespace mtla {

namespace {

using namespace tc;

constexpr int kTileSlots = 128;
constexpr int kAttnThreads = 224;   // warps 0-3 softmax, 4 TMA, 5 score MMAs, 6 P.V MMAs
constexpr float kRescaleLog2 = 8.f;
constexpr int kPrepAbsThreads = 128;   // prep: W_UK product threads (plus one RoPE warp)
constexpr int kMaxGrid = 160;  // >= SMs of any sm_100 part; sizes the partial buffer
constexpr int kMaxB = 2048;
constexpr int kMaxChunks = 6;     // 64-column chunks of the slot width (supported shapes)
constexpr int kMaxLatBlocks = 3;  // 128-column latent blocks (d_c <= 384 follows from the above)

struct DecTC {
    int B, H, D, d_c, s, max_slots;
    int Hp;          // H rounded up to 8: heads per partial row block
    int n_chunks;    // D rounded up to 64, in 64-column chunks
    int n_lat;       // d_c / 64 latent chunks
    int compact;     // the RoPE chunk is 32 columns wide (64-byte rows, SW64)
    uint32_t stage_bytes;   // one slot tile in shared memory
    int lat_blocks;  // d_c / 128
    int G;           // grid size
    float scale_log2;
    const int32_t* pos;
    const uint8_t* qimg;  // [B] x image: q~ in bf16, the slot tile's chunk layout, zero padded
    uint32_t qimg_bytes;  // per sequence
    float* part;          // [(kMaxGrid + B), Hp, d_c + 2]
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

// Decode prep for the tensor-core path. grid (B, H + 1), 160 threads.
// Block (b, h < H): absorbed query of head h, q~ = [W_UK[h]^T qC ; RoPE_t(qR)],
// rounded to bf16 into row h of sequence b's query image: 64-column SW128
// chunks of NH rows, zero beyond D; in the compact layout (d_R = 32) the RoPE
// part is one 32-column chunk of 64-byte SW64 rows after the latent chunks.
// Block (b, H): gate, RoPE and in-place update of the open slot (MTLA Method
// (1)), and zero rows H..NH-1 of the image.
// Launched as a programmatic dependent of the previous kernel in the stream:
// only weights (the W_UK rows, G) are read before the wait for that kernel;
// every input of the step and every write come after it.
// The attention kernel may start at once: it reads the positions and finished
// slots before its own wait. Those are safe to read early because this kernel
// starts before its predecessor ends only when that predecessor triggers its
// dependents early, which the library's own kernels alone do (a step's combine
// kernel, which writes neither); the C-ABI header states this for callers.
template <typename E>
__global__ void __launch_bounds__(kPrepAbsThreads + 32) k_dec_prep_tc(DecodeArgs a, uint8_t* qimg, uint32_t img_bytes, int n_chunks, int NH, int compact) {
    pdl_launch_dependents();   // the attention kernel may start its prologue now
    const Shape& sh = a.sh;
    const int b = blockIdx.x, h = blockIdx.y;
    uint8_t* img = qimg + (size_t)b * img_bytes;
    const int n_wide = compact ? n_chunks - 1 : n_chunks;     // chunks of 128-byte rows
    uint8_t* rope_img = img + (size_t)n_wide * NH * 128;     // compact: [NH x 64 B]
    __shared__ float part_sum[8][512];     // W_UK blocks: [i-group][latent column]; update block: G
    if (h == sh.H) {
        // weights first (G into shared memory, the PE and RoPE frequencies),
        // then the wait, then the step's inputs
        UpdateFreqs f;
        update_freqs(sh, f);
        const float* gw = a.gate_w;
        if (sh.gate_mode == 0 && sh.s * sh.d_c <= 8 * 512) {
            float* gs = &part_sum[0][0];
            for (int e = threadIdx.x; e < sh.s * sh.d_c; e += blockDim.x) gs[e] = a.gate_w[e];
            __syncthreads();
            gw = gs;
        }
        pdl_wait();
        decode_update_body<E>(a, b, gw, f);
        const int pad = NH - sh.H;
        for (int e = threadIdx.x; e < n_wide * pad * 8; e += blockDim.x) {
            const int c = e / (pad * 8), rr = e % (pad * 8);
            *(uint4*)(img + (size_t)c * NH * 128 + (size_t)(sh.H + rr / 8) * 128 + (rr % 8) * 16) =
                make_uint4(0, 0, 0, 0);
        }
        if (compact)
            for (int e = threadIdx.x; e < pad * 4; e += blockDim.x)
                *(uint4*)(rope_img + (size_t)(sh.H + e / 4) * 64 + (e % 4) * 16) = make_uint4(0, 0, 0, 0);
        return;
    }
    const size_t rh = (size_t)b * sh.H + h;
    const E* qc = (const E*)a.q_c + rh * sh.d_h;
    const E* qr = (const E*)a.q_r + rh * sh.d_r;
    const int dpad = compact ? sh.D : n_chunks * 64;
    if (threadIdx.x >= kPrepAbsThreads) {
        // the last warp: RoPE part of q~ (columns d_c .. D-1) and the zero padding
        // up to the chunk boundary, independent of the W_UK product
        pdl_wait();
        const int64_t t = a.pos[b];
        if (t < 0 || t >= (int64_t)sh.max_slots * sh.s) return;
        for (int j = sh.d_c + (int)threadIdx.x - kPrepAbsThreads; j < dpad; j += 32) {
            float v = 0.f;
            if (j < sh.D) {
                const int e = j - sh.d_c, k = e >> 1;
                const float x0 = to_f<E>(qr[2 * k]), x1 = to_f<E>(qr[2 * k + 1]);
                float sn, cs;
                pair_sincos(t, k, sh.d_r, sh.log2_rope_base, &sn, &cs);
                v = (e & 1) ? (x0 * sn + x1 * cs) : (x0 * cs - x1 * sn);
            }
            E* dst = compact ? (E*)(rope_img + sw64_offset(h, j - sh.d_c))
                                : (E*)(img + (size_t)(j >> 6) * NH * 128 + sw128_offset(h, j & 63));
            *dst = from_f<E>(v);
        }
        return;
    }
    // thread (ig, jg): 8 latent columns [8 jg, 8 jg + 8) over rows i of group ig;
    // its 16-byte loads of W_UK and of qC are all issued before any product
    const E* W = (const E*)a.w_uk + (size_t)h * sh.d_h * sh.d_c;
    const int n_jg = sh.d_c / 8;
    const int n_ig = max(1, min(8, kPrepAbsThreads / n_jg));
    const int rows_per = (((sh.d_h + n_ig - 1) / n_ig) + 15) & ~15;   // 16-row batches, aligned
    // this thread's first batch of W_UK rows is in flight before the wait
    uint4 raw[16];
    {
        const int e = threadIdx.x;
        if (e < n_ig * n_jg) {
            const int ig = e / n_jg, jg = e % n_jg;
            const int i0 = ig * rows_per, i1 = min(sh.d_h, i0 + rows_per);
#pragma unroll
            for (int u = 0; u < 16; ++u)
                if (i0 + u < i1) raw[u] = *(const uint4*)(W + (size_t)(i0 + u) * sh.d_c + jg * 8);
        }
    }
    pdl_wait();
    const int64_t t = a.pos[b];
    const bool t_ok = t >= 0 && t < (int64_t)sh.max_slots * sh.s;
    for (int e = threadIdx.x; e < n_ig * n_jg; e += kPrepAbsThreads) {
        const int ig = e / n_jg, jg = e % n_jg;
        const int i0 = ig * rows_per, i1 = min(sh.d_h, i0 + rows_per);
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int ib = i0; ib < i1; ib += 16) {
            uint4 qraw[2];
            if (e != (int)threadIdx.x || ib != i0) {
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    if (ib + u < i1) raw[u] = *(const uint4*)(W + (size_t)(ib + u) * sh.d_c + jg * 8);
            }
#pragma unroll
            for (int u = 0; u < 2; ++u)
                if (ib + 8 * u < i1) qraw[u] = *(const uint4*)(qc + ib + 8 * u);   // d_h % 16 == 0
            const E* qv = (const E*)qraw;
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                if (ib + u < i1) {
                    const E* wv = (const E*)&raw[u];
                    const float qi = to_f<E>(qv[u]);
#pragma unroll
                    for (int v = 0; v < 8; ++v) acc[v] = fmaf(to_f<E>(wv[v]), qi, acc[v]);
                }
            }
        }
#pragma unroll
        for (int v = 0; v < 8; ++v) part_sum[ig][jg * 8 + v] = acc[v];
    }
    named_sync(1, kPrepAbsThreads);      // the W_UK threads only
    if (!t_ok) return;                   // (the loads above do not depend on the position)
    for (int j = threadIdx.x; j < sh.d_c; j += kPrepAbsThreads) {
        float v = 0.f;
        for (int ig = 0; ig < n_ig; ++ig) v += part_sum[ig][j];
        *(E*)(img + (size_t)(j >> 6) * NH * 128 + sw128_offset(h, j & 63)) = from_f<E>(v);
    }
}

// Barriers and small shared state of k_dec_attn_sh.
template <int HV>
struct SmallBars {
    uint64_t full[3], empty[3];          // slot-tile ring (2 or 3 stages)
    uint64_t q_full, q_free;             // query image of the current segment
    uint64_t s_full[2], s_empty[2];      // S^T buffers
    uint64_t p_full[2];                  // P^T buffers (4 softmax warps arrive)
    uint64_t o_done[2];                  // P.V of tiles with this parity completed
    uint64_t drain[2];                   // MMAs in flight when a wait gave up (per issuing thread)
    uint32_t tmem_base;
    volatile int fail;
    int total;
    float4 red[2][HV];                   // per head: the 4 warps' tile maxima, by tile parity
    float4 lsum[HV];                     // per head: the 4 warps' sums at a segment end
    float msave[HV];
};

template <int HV>
__device__ __forceinline__ bool sb_wait(uint64_t* bar, uint32_t parity, SmallBars<HV>& bs) {
    if (bs.fail) return false;
    if (mbar_wait(bar, parity)) return true;
    bs.fail = 1;
    return false;
}

// The slot cache as TMA sees it: 64-column SW128 boxes of 128 slots, and (the
// compact layout) the 32-column RoPE part as one SW64 box.
struct DecMaps {
    CUtensorMap lat, rope;
};

// Split-K attention over 128-slot tiles, heads as the MMA's N (NH = 16 or 32).
// Warps 0-3: online softmax, thread = slot row (its TMEM lane), over HV heads
// (H rounded up to 8; a compile-time count, so every per-head loop is
// straight-line code); warp 4: TMA; warp 5: score MMAs; warp 6: P.V MMAs. S^T
// is double-buffered in TMEM so the scores of the next tile overlap this
// tile's softmax.
// ST = 2: a tile is n_chunks 64-column SW128 chunks (the RoPE part padded to a
// whole chunk) and P^T has two buffers of its own.
// ST = 3 (d_R = 32, NH = 16): the compact layout -- the latent chunks, then the
// RoPE part as 128 rows of 64 bytes (SW64), 72 KB per tile for d_c = 256 -- and
// P^T of a tile is written over its RoPE part, which only the score MMAs read
// and which is free once they are done; that leaves room for a third stage,
// so two loads stay in flight while a tile is worked on.
template <int NH, int HV, int ST, typename E>
__global__ void __launch_bounds__(kAttnThreads, 1)
    k_dec_attn_sh(const __grid_constant__ DecMaps maps, const DecTC p) {
    static_assert(HV % 8 == 0 && HV <= NH, "head count");
    static_assert(ST == 2 || (ST == 3 && NH == 16), "ring");
    constexpr bool kCompact = ST == 3;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_chunks = p.n_chunks, n_lat = p.n_lat;
    const uint32_t stage_bytes = p.stage_bytes;
    const uint32_t pt_off = (uint32_t)n_lat * 16384u;           // compact: P^T over the RoPE part
    uint8_t* ring = smem;                                        // ST stages
    uint8_t* q_s = smem + ST * stage_bytes;                      // the query image (qimg_bytes)
    uint8_t* p_s = q_s + p.qimg_bytes;                           // ST = 2: 2 buffers x 2 chunks x [NH x 128 B]
    SmallBars<HV>& bs = *(SmallBars<HV>*)(p_s + (kCompact ? 0 : 4 * NH * 128));
    int* starts = (int*)((uint8_t*)&bs + ((sizeof(SmallBars<HV>) + 15) & ~(size_t)15));   // [B + 1]

    // ---- schedule: tiles per sequence and their exclusive prefix sum (reads pos only)
    {
        const int per = (p.B + kAttnThreads - 1) / kAttnThreads;
        const int b0 = tid * per, b1 = min(b0 + per, p.B);
        int local = 0;
        for (int b = b0; b < b1; ++b) local += seq_tiles(p, b);
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        __shared__ int warp_tot[kAttnThreads / 32];
        if (lane == 31) warp_tot[warp] = incl;
        __syncthreads();
        int off = 0, tot = 0;
        for (int w = 0; w < kAttnThreads / 32; ++w) {
            if (w < warp) off += warp_tot[w];
            tot += warp_tot[w];
        }
        int run = off + incl - local;
        for (int b = b0; b < b1; ++b) {
            starts[b] = run;
            run += seq_tiles(p, b);
        }
        if (tid == 0) {
            bs.total = tot;
            starts[p.B] = tot;
        }
    }
    const uint32_t tmem_cols_needed = (uint32_t)NH * (2 + p.lat_blocks);
    uint32_t tmem_cols = 32;
    while (tmem_cols < tmem_cols_needed) tmem_cols <<= 1;
    if (tid == 0) {
        for (int i = 0; i < ST; ++i) {
            mbar_init(&bs.full[i], 1);
            mbar_init(&bs.empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bs.s_full[i], 1);
            mbar_init(&bs.s_empty[i], 4);
            mbar_init(&bs.p_full[i], 4);
            mbar_init(&bs.o_done[i], 1);
        }
        mbar_init(&bs.q_full, 1);
        mbar_init(&bs.q_free, 1);
        mbar_init(&bs.drain[0], 1);
        mbar_init(&bs.drain[1], 1);
        bs.fail = 0;
        fence_mbar_init();
        tma_prefetch_desc(&maps.lat);
        if (kCompact) tma_prefetch_desc(&maps.rope);
    }
    if (warp == 5) {
        tmem_alloc(&bs.tmem_base, tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_launch_dependents();
    const uint32_t tmem = bs.tmem_base;
    const uint32_t t_s = tmem;                 // S^T buffers: 2 x NH columns
    const uint32_t t_o = tmem + 2 * NH;        // O^T: lat_blocks x NH columns
    const int total = bs.total;
    const int g = blockIdx.x;
    const int gt0 = (int)(((int64_t)g * total) / p.G);
    const int gt1 = (int)(((int64_t)(g + 1) * total) / p.G);
    auto locate = [&](int gt, int& b, int& j) {
        int lo = 0, hi = p.B - 1;            // largest b with starts[b] <= gt
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (starts[mid] <= gt) lo = mid; else hi = mid - 1;
        }
        b = lo;
        j = gt - starts[lo];
    };
    // Only the producer waits for k_dec_prep_tc (programmatic dependent launch):
    // the query image and each sequence's last tile (which holds the slot the
    // prep kernel updates) come from it; the tiles of finished slots do not,
    // so the first of those are already in flight while the prep kernel runs.
    int loads_issued = 0, q_loads = 0;       // producer's copies, for the drain on failure
    if (warp == 4) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            auto load_tile = [&](int st, int b, int j) {
                uint8_t* dst = ring + st * stage_bytes;
                mbar_arrive_expect_tx(&bs.full[st], stage_bytes);
                for (int c = 0; c < (kCompact ? n_lat : n_chunks); ++c)
                    tma_load_3d(dst + (size_t)c * 16384, &maps.lat, &bs.full[st], c * 64, j * kTileSlots, b);
                if (kCompact)
                    tma_load_3d(dst + pt_off, &maps.rope, &bs.full[st], p.d_c, j * kTileSlots, b);
                ++loads_issued;
            };
            int early = 0;                   // tiles 0..early-1 issued before the wait
            for (int gt = gt0; gt < gt1 && early < ST; ++gt) {
                int b, j;
                locate(gt, b, j);
                if (j + 1 == starts[b + 1] - starts[b]) break;    // holds the open slot
                load_tile(early, b, j);
                ++early;
            }
            pdl_wait();
            int prev_b = -1;
            for (int gt = gt0, it = 0; gt < gt1; ++gt, ++it) {
                int b, j;
                locate(gt, b, j);
                if (b != prev_b) {
                    prev_b = b;
                    if (q_loads >= 1 && !sb_wait(&bs.q_free, (q_loads - 1) & 1, bs)) break;
                    mbar_arrive_expect_tx(&bs.q_full, p.qimg_bytes);
                    bulk_load(q_s, p.qimg + (size_t)b * p.qimg_bytes, p.qimg_bytes, &bs.q_full);
                    ++q_loads;
                }
                if (it < early) continue;
                const int st = it % ST;
                if (it >= ST && !sb_wait(&bs.empty[st], ((it / ST) - 1) & 1, bs)) break;
                load_tile(st, b, j);
            }
        }
    } else if (warp == 5) {
        // ------------------------------------------------------------ score MMAs
        if (lane == 0) {
            const uint32_t id_s = idesc_f32<E>(128, NH, false, false);
            const uint64_t q_d = sdesc_sw128(smem_u32(q_s), 16, 1024);
            const uint32_t ring_a = smem_u32(ring);
            const int last_ksteps = (p.D - 64 * (n_chunks - 1)) / 16;   // D is a multiple of 16
            int seg = -1, prev_b = -1, it = 0;
            for (int gt = gt0; gt < gt1; ++gt, ++it) {
                int b, j;
                locate(gt, b, j);
                if (b != prev_b) {
                    prev_b = b;
                    ++seg;
                    if (!sb_wait(&bs.q_full, seg & 1, bs)) break;
                }
                const int rs = it % ST, sb = it & 1;      // ring stage, S^T buffer
                if (!sb_wait(&bs.full[rs], (it / ST) & 1, bs)) break;
                if (it >= 2 && !sb_wait(&bs.s_empty[sb], ((it >> 1) - 1) & 1, bs)) break;
                tc_fence_after();
                // S^T = K_tile . q~^T (A = slot tile, B = q~ image; both K-major)
                // The MMAs go out in straight-line groups (one test per group of
                // four): a runtime loop or a test per MMA halves their issue rate.
                const uint64_t a0 = sdesc_sw128(ring_a + rs * stage_bytes, 16, 1024);
                const uint32_t ts = t_s + sb * NH;
                if (kCompact) {
                    // the latent chunks, then the two K-steps of the 64-byte RoPE rows
#pragma unroll
                    for (int c = 0; c < kMaxLatBlocks * 2; ++c) {
                        if (c < n_lat) {
                            const uint64_t ac = desc_add(a0, c * 16384), bc = desc_add(q_d, c * NH * 128);
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                umma_bf16(ts, desc_add(ac, kk * 32), desc_add(bc, kk * 32), id_s, (c | kk) != 0);
                        }
                    }
                    const uint64_t ar = sdesc_sw64(ring_a + rs * stage_bytes + pt_off);
                    const uint64_t br = sdesc_sw64(smem_u32(q_s) + n_lat * NH * 128);
                    umma_bf16(ts, ar, br, id_s, 1u);
                    umma_bf16(ts, desc_add(ar, 32), desc_add(br, 32), id_s, 1u);
                    umma_commit(&bs.s_full[sb]);
                    const bool last = (gt + 1 == gt1) || (j + 1 == starts[b + 1] - starts[b]);
                    if (last) umma_commit(&bs.q_free);
                    continue;
                }
#pragma unroll
                for (int c = 0; c < kMaxChunks - 1; ++c) {
                    if (c < n_chunks - 1) {
                        const uint64_t ac = desc_add(a0, c * 16384), bc = desc_add(q_d, c * NH * 128);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_bf16(ts, desc_add(ac, kk * 32), desc_add(bc, kk * 32), id_s, (c | kk) != 0);
                    }
                }
                {
                    // the last chunk: its K-steps up to D (the zero-filled tail is skipped)
                    const int cl = n_chunks - 1;
                    const uint64_t ac = desc_add(a0, cl * 16384), bc = desc_add(q_d, cl * NH * 128);
                    const uint32_t acc0 = cl > 0 ? 1u : 0u;
                    switch (last_ksteps) {
                        case 4:
                            umma_bf16(ts, ac, bc, id_s, acc0);
                            umma_bf16(ts, desc_add(ac, 32), desc_add(bc, 32), id_s, 1u);
                            umma_bf16(ts, desc_add(ac, 64), desc_add(bc, 64), id_s, 1u);
                            umma_bf16(ts, desc_add(ac, 96), desc_add(bc, 96), id_s, 1u);
                            break;
                        case 3:
                            umma_bf16(ts, ac, bc, id_s, acc0);
                            umma_bf16(ts, desc_add(ac, 32), desc_add(bc, 32), id_s, 1u);
                            umma_bf16(ts, desc_add(ac, 64), desc_add(bc, 64), id_s, 1u);
                            break;
                        case 2:
                            umma_bf16(ts, ac, bc, id_s, acc0);
                            umma_bf16(ts, desc_add(ac, 32), desc_add(bc, 32), id_s, 1u);
                            break;
                        default:
                            umma_bf16(ts, ac, bc, id_s, acc0);
                            break;
                    }
                }
                umma_commit(&bs.s_full[sb]);
                const bool last = (gt + 1 == gt1) || (j + 1 == starts[b + 1] - starts[b]);
                if (last) umma_commit(&bs.q_free);
            }
        }
    } else if (warp == 6) {
        // ------------------------------------------------------------ P.V MMAs (own thread: they free
        // ring stages, so they never wait behind a score MMA that waits for a load)
        if (lane == 0) {
            const uint32_t id_o = idesc_f32<E>(128, NH, true, false);
            const uint32_t ring_a = smem_u32(ring), p_a = smem_u32(p_s);
            int prev_b = -1, k = 0;
            for (int gt = gt0; gt < gt1; ++gt, ++k) {
                int b, j;
                locate(gt, b, j);
                const bool first = (b != prev_b);
                prev_b = b;
                if (!sb_wait(&bs.p_full[k & 1], (k >> 1) & 1, bs)) break;
                tc_fence_after();
                // O^T += V^T . P^T (A = the slot tile, MN-major; B = P^T, K-major)
                const uint32_t stage_a = ring_a + (k % ST) * stage_bytes;
                const uint64_t a0 = sdesc_sw128(stage_a, 16384, 1024);
                const uint64_t b0 = sdesc_sw128(kCompact ? stage_a + pt_off : p_a + (k & 1) * 2 * NH * 128, 16, 1024);
#pragma unroll
                for (int lb = 0; lb < kMaxLatBlocks; ++lb) {
                    if (lb < p.lat_blocks) {
                        const uint64_t al = desc_add(a0, 2 * lb * 16384);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            umma_bf16(t_o + lb * NH, desc_add(al, kk * 2048),
                                      desc_add(b0, (kk >> 2) * NH * 128 + (kk & 3) * 32), id_o,
                                      (first && kk == 0) ? 0u : 1u);
                    }
                }
                umma_commit(&bs.empty[k % ST]);
                umma_commit(&bs.o_done[k & 1]);
            }
        }
    } else {
        // ------------------------------------------------------------ softmax (warps 0-3)
        // No early exit: every softmax thread passes every named barrier even after a
        // bounded wait gave up (later waits then return at once), so none can hang.
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        float m_ref[HV], l_part[HV];
        int prev_b = -1, n_b = 0, k_in_seg = 0;
        for (int gt = gt0, it = 0; gt < gt1; ++gt, ++it) {
            int b, j;
            locate(gt, b, j);
            if (b != prev_b) {
                prev_b = b;
                n_b = seq_slots(p, b);
                k_in_seg = 0;
#pragma unroll
                for (int h = 0; h < HV; ++h) {
                    m_ref[h] = -INFINITY;
                    l_part[h] = 0.f;
                }
            }
            const int st = it & 1;                  // S^T and P^T buffer parity
            uint8_t* stage = ring + (it % ST) * stage_bytes;
            const int valid = min(kTileSlots, n_b - j * kTileSlots);
            sb_wait(&bs.s_full[st], (it >> 1) & 1, bs);
            tc_fence_after();
            float sv[HV];
            tmem_ld_cols<HV>(t_s + st * NH + lane_off, sv);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bs.s_empty[st]);
            if (valid < kTileSlots) {
                // stale rows past the sequence's last slot must not reach P.V
                // (whole 128-byte rows of the latent chunks, so the swizzle does
                // not matter)
                for (int c = 0; c < n_lat; ++c) {
                    uint8_t* base = stage + (size_t)c * 16384;
                    for (int off = valid * 128 + tid * 16; off < 16384; off += 128 * 16)
                        *(uint4*)(base + off) = make_uint4(0, 0, 0, 0);
                }
            }
            const bool row_ok = tid < valid;
#pragma unroll
            for (int h = 0; h < HV; ++h) {
                sv[h] = row_ok ? sv[h] * p.scale_log2 : -INFINITY;
                const float mx = warp_max_redux(sv[h]);
                if (lane == 0) reinterpret_cast<float*>(&bs.red[st][h])[warp] = mx;
            }
            named_sync(1, 128);
            // lazy rescale: a head's reference maximum moves only when the tile's
            // maximum exceeds it by more than 2^8 (P stays <= 256 in bf16)
            float fac[HV];
            bool any_rescale = false;
#pragma unroll
            for (int h = 0; h < HV; ++h) {
                const float4 r = bs.red[st][h];
                const float tmax = fmaxf(fmaxf(r.x, r.y), fmaxf(r.z, r.w));
                const bool upd = tmax > m_ref[h] + kRescaleLog2;
                const float nm = upd ? tmax : m_ref[h];
                fac[h] = exp2f(m_ref[h] - nm);     // 0 when m_ref was -inf, 1 when kept
                any_rescale |= upd;
                m_ref[h] = nm;
                sv[h] = exp2f(sv[h] - nm);
                l_part[h] = fmaf(l_part[h], fac[h], sv[h]);
            }
            any_rescale &= (k_in_seg > 0);
            // P.V of tile it-2 is done: it read P^T buffer st (in the compact
            // layout P^T sits in this tile's own stage instead), and the P.V
            // thread has taken p_full[st]'s previous phase, so this tile's
            // arrivals cannot run a whole phase ahead of it
            if (it >= 2) sb_wait(&bs.o_done[st], ((it >> 1) - 1) & 1, bs);
            if (any_rescale) {
                // the running O^T of this segment moves to the new reference maximum
                sb_wait(&bs.o_done[st ^ 1], ((it - 1) >> 1) & 1, bs);
                tc_fence_after();
                for (int lb = 0; lb < p.lat_blocks; ++lb) {
                    float ov[HV];
                    const uint32_t ta = t_o + lb * NH + lane_off;
                    tmem_ld_cols<HV>(ta, ov);
                    tmem_wait_ld();
#pragma unroll
                    for (int h = 0; h < HV; ++h) ov[h] *= fac[h];
                    tmem_st_cols<HV>(ta, ov);
                }
                tmem_wait_st();
            }
            {
                uint8_t* pb = (kCompact ? stage + pt_off : p_s + (size_t)st * 2 * NH * 128) +
                              (size_t)(tid >> 6) * NH * 128;
#pragma unroll
                for (int h = 0; h < HV; ++h) *(E*)(pb + sw128_offset(h, tid & 63)) = from_f<E>(sv[h]);
            }
            fence_proxy_async();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bs.p_full[st]);
            ++k_in_seg;
            const bool last = (gt + 1 == gt1) || (j + 1 == starts[b + 1] - starts[b]);
            if (last) {
                // partial (o, m, l) of this sequence segment: rows of HV heads
                sb_wait(&bs.o_done[st], (it >> 1) & 1, bs);
                tc_fence_after();
#pragma unroll
                for (int h = 0; h < HV; ++h) l_part[h] = warp_sum(l_part[h]);
                if (lane == 0) {
#pragma unroll
                    for (int h = 0; h < HV; ++h) reinterpret_cast<float*>(&bs.lsum[h])[warp] = l_part[h];
                }
                if (tid == 0) {
#pragma unroll
                    for (int h = 0; h < HV; ++h) bs.msave[h] = m_ref[h];
                }
                named_sync(1, 128);
                float* dst = p.part + (size_t)(g + b) * HV * (p.d_c + 2);
                for (int lb = 0; lb < p.lat_blocks; ++lb) {
                    float ov[HV];
                    tmem_ld_cols<HV>(t_o + lb * NH + lane_off, ov);
                    tmem_wait_ld();
#pragma unroll
                    for (int h = 0; h < HV; ++h) dst[(size_t)h * (p.d_c + 2) + lb * 128 + tid] = ov[h];
                }
                if (tid < HV) {
                    const float4 l4 = bs.lsum[tid];
                    dst[(size_t)tid * (p.d_c + 2) + p.d_c] = bs.msave[tid];
                    dst[(size_t)tid * (p.d_c + 2) + p.d_c + 1] = (l4.x + l4.y) + (l4.z + l4.w);
                }
                named_sync(1, 128);          // lsum and msave are free for the next segment
                tc_fence_before();
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (bs.fail) {
        // a bounded wait gave up: let this CTA's copies and MMAs land (bounded
        // again) before the shared memory and TMEM are released, then report
        if (warp == 4 && lane == 0) {
            for (int k = max(0, loads_issued - ST); k < loads_issued; ++k) mbar_wait(&bs.full[k % ST], (k / ST) & 1);
            if (q_loads > 0) mbar_wait(&bs.q_full, (q_loads - 1) & 1);
        }
        if ((warp == 5 || warp == 6) && lane == 0) {
            uint64_t* d = &bs.drain[warp - 5];
            umma_commit(d);              // arrives when this thread's MMAs are done
            mbar_wait(d, 0);
        }
        if (tid == 0) latch_status(p.status, kStatusTimeout);
        __syncthreads();
    }
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tmem, tmem_cols);
}

// Merge the partials of (b, h) and apply W_UV. grid (H, B), 256 threads.
// W_UV[h] is staged in shared memory before the wait for the attention kernel;
// after it, every partial value this block needs is read in one round.
template <typename E>
__global__ void __launch_bounds__(256) k_dec_combine(DecodeArgs a, DecTC p) {
    pdl_launch_dependents();   // the next step's prep may stage its W_UK rows now
    const int h = blockIdx.x, b = blockIdx.y;
    const Shape& sh = a.sh;
    if (seq_tiles(p, b) == 0) return;
    __shared__ float red[32];
    __shared__ int idx[kMaxGrid];
    __shared__ int n_part;
    __shared__ __align__(16) float olat[512];
    extern __shared__ uint8_t dyn[];
    E* Ws = (E*)dyn;                            // W_UV[h] [d_h x d_c]
    {
        // eight 16-byte loads in flight per thread before any store
        const uint4* src = (const uint4*)((const E*)a.w_uv + (size_t)h * sh.d_h * sh.d_c);
        uint4* dst = (uint4*)Ws;
        const int n16 = sh.d_h * sh.d_c / 8;
        for (int e0 = threadIdx.x; e0 < n16; e0 += 8 * blockDim.x) {
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (e0 + u * (int)blockDim.x < n16) v[u] = src[e0 + u * blockDim.x];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (e0 + u * (int)blockDim.x < n16) dst[e0 + u * blockDim.x] = v[u];
        }
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
    const size_t stride = (size_t)p.Hp * (p.d_c + 2);
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
    // o = W_UV[h] o_lat: warp w takes rows w, w + 8, ... in groups of 8 rows whose
    // dot products run side by side (8 independent chains, one reduction round)
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    E* out = (E*)a.out + ((size_t)b * sh.H + h) * sh.d_h;
    for (int i0 = warp; i0 < sh.d_h; i0 += 64) {
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int c0 = lane * 8; c0 < sh.d_c; c0 += 256) {
            const float4 o0 = *(const float4*)(olat + c0), o1 = *(const float4*)(olat + c0 + 4);
            const float ov[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const int i = i0 + r * 8;
                if (i < sh.d_h) {
                    const uint4 raw = *(const uint4*)(Ws + (size_t)i * sh.d_c + c0);
                    const E* wv = (const E*)&raw;
#pragma unroll
                    for (int v = 0; v < 8; ++v) acc[r] = fmaf(to_f<E>(wv[v]), ov[v], acc[r]);
                }
            }
        }
#pragma unroll
        for (int r = 0; r < 8; ++r) acc[r] = warp_sum(acc[r]);
        if (lane < 8 && i0 + lane * 8 < sh.d_h) {
            float mine = acc[0];
#pragma unroll
            for (int r = 1; r < 8; ++r) mine = lane == r ? acc[r] : mine;
            out[i0 + lane * 8] = from_f<E>(mine);
        }
    }
}

// ---------------------------------------------------------------- host side

int n_chunks_of(const Shape& sh) { return (sh.D + 63) / 64; }

int heads_padded(const Shape& sh) { return (sh.H + 7) & ~7; }
int nh_of(const Shape& sh) { return sh.H <= 16 ? 16 : 32; }

// One slot tile in shared memory: whole 64-column chunks, or (compact) the
// latent chunks and 128 RoPE rows of 64 bytes.
uint32_t stage_bytes_of(const Shape& sh, bool compact) {
    return compact ? (uint32_t)(sh.d_c / 64) * 16384u + (uint32_t)kTileSlots * 64u
                   : (uint32_t)n_chunks_of(sh) * 16384u;
}

// The query image of one sequence in the tile's chunk layout (NH rows).
uint32_t qimg_bytes_of(const Shape& sh, bool compact) {
    const uint32_t nh = (uint32_t)nh_of(sh);
    return compact ? (uint32_t)(sh.d_c / 64) * nh * 128u + nh * 64u : (uint32_t)n_chunks_of(sh) * nh * 128u;
}

size_t small_bars_bytes(int HV) {
    switch (HV) {
        case 8: return sizeof(SmallBars<8>);
        case 16: return sizeof(SmallBars<16>);
        case 24: return sizeof(SmallBars<24>);
        default: return sizeof(SmallBars<32>);
    }
}

// Dynamic shared memory of k_dec_attn_sh with `stages` ring stages (3 means
// the compact layout); the kernel's static shared memory comes on top.
size_t attn_smem_bytes(const Shape& sh, int stages) {
    const bool compact = stages == 3;
    size_t bytes = 1024;                                   // alignment slack
    bytes += (size_t)stages * stage_bytes_of(sh, compact); // the ring
    bytes += qimg_bytes_of(sh, compact);                   // q~
    if (!compact) bytes += 4 * (size_t)nh_of(sh) * 128;    // P^T (2 buffers)
    bytes += (small_bars_bytes(heads_padded(sh)) + 15) & ~(size_t)15;
    bytes += ((size_t)sh.B + 1) * 4 + 16;                  // tile prefix sums
    return bytes;
}

constexpr size_t kSmemOptin = 232448;      // per-block opt-in limit of sm_100
constexpr size_t kStaticMargin = 64;       // >= the kernel's static shared memory (32 B)

// The compact three-stage ring: 32 RoPE columns, at most 16 heads, room for
// it, and CTAs that may get more than two tiles (with two or fewer, both sit
// in a two-stage ring at once, and the smaller kernel leaves room on its SM
// for the prep and combine kernels that overlap it).
bool use_three_stages(const Shape& sh, int grid) {
    const int64_t max_tiles = (int64_t)sh.B * ((sh.max_slots + kTileSlots - 1) / kTileSlots);
    return sh.d_r == 32 && sh.d_c % 64 == 0 && sh.H <= 16 && max_tiles > 2 * (int64_t)grid &&
           attn_smem_bytes(sh, 3) + kStaticMargin <= kSmemOptin;
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

template <int NH, int HV, int ST, typename E>
cudaError_t launch_attn(const DecMaps& maps, const DecTC& p, size_t smem, cudaStream_t st) {
    static size_t done[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    cudaError_t e = ensure_smem(k_dec_attn_sh<NH, HV, ST, E>, smem, &done[dev]);
    if (e != cudaSuccess) return note_error("cudaFuncSetAttribute(k_dec_attn_sh)", e);
    return note_error("k_dec_attn_sh launch",
                      launch_pdl(k_dec_attn_sh<NH, HV, ST, E>, dim3(p.G), dim3(kAttnThreads), smem, st, maps, p));
}

template <typename E>
cudaError_t launch_attn_any(const DecMaps& maps, const DecTC& p, size_t smem, cudaStream_t st) {
    if (p.compact) {
        if (p.Hp == 8) return launch_attn<16, 8, 3, E>(maps, p, smem, st);
        return launch_attn<16, 16, 3, E>(maps, p, smem, st);
    }
    switch (p.Hp) {
        case 8: return launch_attn<16, 8, 2, E>(maps, p, smem, st);
        case 16: return launch_attn<16, 16, 2, E>(maps, p, smem, st);
        case 24: return launch_attn<32, 24, 2, E>(maps, p, smem, st);
        default: return launch_attn<32, 32, 2, E>(maps, p, smem, st);
    }
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
           attn_smem_bytes(sh, 2) + kStaticMargin <= kSmemOptin;
}

// Workspace layout: the query images (sized for the larger, padded layout),
// then the split partials.
static size_t qimg_region(const Shape& sh) { return align256((size_t)sh.B * qimg_bytes_of(sh, false)); }

size_t tc_decode_workspace(const Shape& sh) {
    return qimg_region(sh) +
           align256((size_t)(kMaxGrid + sh.B) * ((sh.H + 7) & ~7) * (sh.d_c + 2) * sizeof(float));
}

template <typename E>
cudaError_t tc_decode_impl(const DecodeArgs& a, cudaStream_t st, uint64_t* launches) {
    const Shape& sh = a.sh;
    char* ws = (char*)a.workspace;
    uint8_t* qimg = (uint8_t*)ws;
    float* part = (float*)(ws + qimg_region(sh));
    const int NH = nh_of(sh);
    const int grid = (int)std::min<int64_t>(std::min(sm_count(), kMaxGrid),
                                            (int64_t)sh.B * ((sh.max_slots + kTileSlots - 1) / kTileSlots));
    const bool compact = use_three_stages(sh, grid);

    auto encode = (PFN_cuTensorMapEncodeTiled_v12000)tensor_map_encoder();
    if (!encode) return note_error("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", cudaErrorNotSupported);
    DecMaps maps;
    memset(&maps, 0, sizeof(maps));
    cuuint64_t dims[3] = {(cuuint64_t)sh.D, (cuuint64_t)sh.max_slots, (cuuint64_t)sh.B};
    cuuint64_t strides[2] = {(cuuint64_t)sh.D * 2, (cuuint64_t)sh.max_slots * sh.D * 2};
    cuuint32_t estr[3] = {1, 1, 1};
    for (int m = 0; m < (compact ? 2 : 1); ++m) {
        // the latent map (64-column SW128 boxes), then the RoPE map (one
        // 32-column SW64 box starting at column d_c: 2 * d_c bytes, 16-aligned)
        cuuint32_t box[3] = {m == 0 ? 64u : 32u, (cuuint32_t)kTileSlots, 1};
        CUresult r = encode(m == 0 ? &maps.lat : &maps.rope,
                            std::is_same<E, f16>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.cache, dims,
                            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            m == 0 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            char buf[96];
            snprintf(buf, sizeof(buf), "cuTensorMapEncodeTiled (CUresult %d)", (int)r);
            return note_error(buf, cudaErrorInvalidValue);
        }
    }

    DecTC p;
    p.B = sh.B;
    p.H = sh.H;
    p.Hp = (sh.H + 7) & ~7;
    p.D = sh.D;
    p.d_c = sh.d_c;
    p.s = sh.s;
    p.max_slots = sh.max_slots;
    p.n_chunks = n_chunks_of(sh);
    p.n_lat = sh.d_c / 64;
    p.compact = compact ? 1 : 0;
    p.stage_bytes = stage_bytes_of(sh, compact);
    p.lat_blocks = sh.d_c / 128;
    p.G = grid;
    p.scale_log2 = sh.scale * 1.4426950408889634f;
    p.pos = a.pos;
    p.qimg = qimg;
    p.qimg_bytes = qimg_bytes_of(sh, compact);
    p.part = part;
    p.status = a.status;

    {
        // keep the SMs in the max-shared-memory configuration across the
        // three kernels of a step (no carve-out switch between them)
        static bool carve[64] = {false};
        int dev = 0;
        cudaGetDevice(&dev);
        if (dev >= 0 && dev < 64 && !carve[dev]) {
            cudaFuncSetAttribute(k_dec_prep_tc<E>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
            cudaFuncSetAttribute(k_dec_combine<E>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
            cudaGetLastError();
            carve[dev] = true;
        }
    }
    cudaError_t e = launch_pdl(k_dec_prep_tc<E>, dim3(sh.B, sh.H + 1), dim3(kPrepAbsThreads + 32), 0, st, a, qimg,
                               p.qimg_bytes, p.n_chunks, NH, p.compact);
    if (e != cudaSuccess) return note_error("k_dec_prep_tc launch", e);
    const size_t smem = attn_smem_bytes(sh, compact ? 3 : 2);
    profile_begin(st);
    e = launch_attn_any<E>(maps, p, smem, st);
    profile_end(st);
    if (e != cudaSuccess) return e;
    const size_t comb_smem = (size_t)sh.d_h * sh.d_c * sizeof(bf16);
    {
        static size_t done[64] = {0};
        int dev = 0;
        cudaGetDevice(&dev);
        if (dev < 0 || dev >= 64) dev = 0;
        e = ensure_smem(k_dec_combine<E>, comb_smem, &done[dev]);
        if (e != cudaSuccess) return note_error("cudaFuncSetAttribute(k_dec_combine)", e);
    }
    e = launch_pdl(k_dec_combine<E>, dim3(sh.H, sh.B), dim3(256), comb_smem, st, a, p);
    *launches += 3;
    return note_error("k_dec_combine launch", e);
}

cudaError_t tc_decode(const DecodeArgs& a, cudaStream_t st, uint64_t* launches) {
    return a.sh.dtype == kDtypeF16 ? tc_decode_impl<f16>(a, st, launches) : tc_decode_impl<bf16>(a, st, launches);
}

}  // namespace mtla
