// tc_prefill.cu -- bf16 parallel (training-form) forward on the tensor cores.
//
// "Multi-head Temporal Latent Attention", Method (2)-(3), Sec. 4.2-4.3: with
// the stride-aware causal mask, position t attends every finished slot
// j < floor(t/s) plus its own block's partial slot
//   P_t = sum_{u = s*floor(t/s)}^{t} w_u [c_u ; RoPE_u(k_u)],
// which reproduces incremental decoding; W_UK is folded into the query and
// W_UV applied to the weighted latent (absorption kept from MLA).
//
// Launches:
//   k_prefill_scan<bf16, bf16>  gates, partial slots P (bf16, scratch),
//                               finished slots (cache_out), open slot
//   k_prefill_tc                persistent, one CTA per SM walking work items
//                               (query tile of 128 positions, sequence, head),
//                               heaviest first:
//     absorption   q~ = qC . W_UK[h]          tcgen05 M=128 N=d_c K=d_h
//     own partial  the rows' partial slots P_t arrive as one tile; each row's
//                  score q~ . P_t is one dot product on the CUDA cores and the
//                  softmax's starting point; O starts as P_t's latent part
//     finished     128-slot tiles of cache_out  staircase mask on the last
//                  S = q~ . K^T (M=128 N=128 K=D), online softmax (two threads
//                  per row, exp2, rescale only when a row max grows by > 2^8),
//                  O += P . V (M=128 N=d_c K=128, P in TMEM, V = the same tile)
//     epilogue     out = (O / l) . W_UV[h]^T   tcgen05 M=128 N=d_h K=d_c, with
//                  O / l as bf16 in TMEM (the MMA's A operand)
// Warp roles: warp 0 TMA, warp 1 absorption / score / output MMAs and TMEM,
// warps 2-9 softmax, warp 10 P.V MMAs (so P.V, which frees ring stages, never
// waits behind a score MMA that waits for a load). S is double-buffered in
// TMEM beside O and P (bf16) is written over its own tile's scores. The query
// image and the keys are shared-memory operands: the latent columns in 64-
// column chunks with the 128-byte swizzle, the 32 RoPE columns as one chunk
// with the 64-byte swizzle, so that a 128-slot key tile takes 72 KB and two
// of them fit beside the query image. 128-slot tiles (N=128 score MMAs, K=128
// P.V MMAs) halve the per-tile costs of the pipeline (commits, barrier round
// trips) against 64-slot tiles.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdio>

#include "common.cuh"
#include "mtla_internal.h"
#include "prep.cuh"
#include "tc_common.cuh"

namespace mtla {

namespace {

using namespace tc;

constexpr int kQ = 128;         // query positions per CTA
constexpr int kKT = 128;        // keys per tile
constexpr int kStages = 2;
constexpr int kDr = 32;         // RoPE width d_R of this kernel (one 64-byte-swizzled chunk)
constexpr int kThreads = 352;   // warp 0 TMA, 1 score MMAs, 2-9 softmax, 10 P.V MMAs
constexpr float kRescaleLog2 = 8.f;
constexpr int kDh = 64;         // head width d_h of this kernel

struct PreTC {
    int B, T, H, d_h, d_c, d_r, D, s;
    int n_qtiles;     // ceil(T / 128)
    int t0;           // position of the first query (tokens already cached)
    int n_items;      // n_qtiles * B * H
    float scale_log2;
    double log2_rope_base;
    const void* q_r;  // [B, T, H, d_r], storage type
    const float2* rope_tab;   // [T, d_r / 2]: (cos, sin) of every position, from the scan
    void* out;        // [B, T, H, d_h], storage type
    // kept for the training backward when not null (t0 = 0): per row the
    // log2-domain log-sum-exp [B, H, T], O / l [B, T, H, d_c] and the absorbed
    // query as the score MMAs used it [B, T, H, D], bf16
    float* lse;
    void* obar;       // bf16
    void* qt;         // bf16
    int* status;
};

struct Bars {
    uint64_t full[kStages], empty[kStages];      // ring: key tiles and each item's W_UV
    uint64_t abs_full, abs_done, q_ready, q_free;
    uint64_t s_full[2], s_empty[2];
    uint64_t p_full[2], o_done[2];
    uint64_t olat_ready, out_done, tail_free;
    uint64_t drain[2];
    uint32_t tmem_base;
    volatile int fail;
    float red[2][2][kQ];      // [tile parity][column half][row]: half-row maxima
    float xs[2][kQ];          // [column half][row]: own-slot score halves, then row-sum halves
};

struct Maps {
    CUtensorMap qc;     // (d_h, H, T, B)   box (64, 1, 128, 1)
    CUtensorMap wuk;    // (d_c, d_h, H)    box (64, d_h, 1)
    CUtensorMap wuv;    // (d_c, d_h, H)    box (64, d_h, 1)
    CUtensorMap slots;  // (D, n_slots, B)  box (64, 128, 1), 128-byte swizzle: latent chunks
    CUtensorMap slots_r;  // (D, n_slots, B)  box (32, 128, 1), 64-byte swizzle: the RoPE chunk
    CUtensorMap prow;   // (D, T, B)        box (64, 128, 1): the scan's partial slots, latent chunks
    CUtensorMap prow_r; // (D, T, B)        box (32, 128, 1): their RoPE chunk
};

__device__ __forceinline__ bool waitb(uint64_t* bar, uint32_t parity, Bars& bs) {
    if (bs.fail) return false;
    if (mbar_wait(bar, parity)) return true;
    bs.fail = 1;
    return false;
}

// Store 16 packed bf16 pairs (32 columns from `col`) into row `row` of a K-major
// SW128 operand made of [rows x 64] chunks spaced chunk_bytes apart, or of the
// 64-byte-swizzled chunk when sw64 (col is then relative to that chunk).
__device__ __forceinline__ void st_row32_packed(uint8_t* base, uint32_t chunk_bytes, int row, int col,
                                                const uint32_t* pk, bool sw64) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const uint4 q = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
        if (sw64) *(uint4*)(base + sw64_offset(row, col + 8 * u)) = q;
        else *(uint4*)(base + (size_t)(col >> 6) * chunk_bytes + sw128_offset(row, (col & 63) + 8 * u)) = q;
    }
}

// bf16 halves of a packed pair as fp32 (exact: bf16 is the top half of fp32).


// Work item idx (heaviest first): query tile qt = n_qtiles - 1 - idx / (B H),
// then sequence and head.
struct Item {
    int b, h, p0, nft;    // nft: finished-slot tiles of 128 slots this query tile attends
};
__device__ __forceinline__ Item decode_item(const PreTC& p, int idx) {
    const int per_qt = p.B * p.H;
    const int qt = p.n_qtiles - 1 - idx / per_qt;
    const int rem = idx % per_qt;
    Item it;
    it.b = rem / p.H;
    it.h = rem % p.H;
    it.p0 = qt * kQ;
    const int last = min(it.p0 + kQ - 1, p.T - 1);
    it.nft = ((p.t0 + last) / p.s + kKT - 1) / kKT;
    return it;
}
// The j-th item of this CTA, or -1 past the end: round j of gridDim.x items,
// walked forwards on even rounds and backwards on odd ones.
__device__ __forceinline__ int item_at(const PreTC& p, int j) {
    const int g = (int)gridDim.x, c = (int)blockIdx.x;
    const int idx = j * g + ((j & 1) ? g - 1 - c : c);
    return idx < p.n_items ? idx : -1;
}

// One work item = (128 query positions, sequence, head), heaviest first. The
// own partial slots of the item's rows come into the ring as one tile; each
// row's score against its own slot is one dot product on the CUDA cores, and O
// starts as that slot's latent part (weight 1 at the starting reference
// maximum); the finished slots stream through the tensor cores in 128-slot
// tiles. DC = d_c (d_h = 64 and d_R = 32 are fixed): every MMA sequence is
// unrolled at compile time (a runtime loop or branch between tcgen05.mma
// instructions halves their issue rate).
//
// Persistent: CTA c takes items c, 2G-1-c, 2G+c, ... (a snake over rounds of G
// = gridDim.x items, so the heavy and light items of each round spread evenly),
// and the next item's set-up overlaps this one's end:
//   - qC and W_UK of item j+1 load into the query region once the score MMAs
//     of item j are done (q_free);
//   - the ring carries, per item, its own partial slots (one tile, read by the
//     softmax warps), its key tiles and its W_UV (one more position), so the
//     ring's empty/full barriers order each with the tiles around it;
//   - O_lat of item j goes to TMEM (bf16, the output MMA's A operand), so the
//     absorption of item j+1 into the O columns starts as soon as O is read;
//   - item j+1's key tiles load as soon as the P.V of item j frees the stages.
template <int DC, typename E>
__global__ void __launch_bounds__(kThreads, 1) k_prefill_tc(const __grid_constant__ Maps maps, const PreTC p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    constexpr int NL = DC / 64;                                          // latent chunks
    constexpr uint32_t chunk_k = kKT * 128;                              // one latent chunk of a key tile
    constexpr uint32_t rope_k = kKT * 64;                                // its RoPE chunk (64-byte rows)
    constexpr uint32_t stage_bytes = NL * chunk_k + rope_k;
    constexpr uint32_t q_bytes = NL * kQ * 128 + kQ * 64;
    constexpr int dc_chunks = DC / 64;
    constexpr uint32_t wchunk = (uint32_t)kDh * 128;                     // one 64-column chunk of W
    static_assert(kQ * 128 + dc_chunks * wchunk <= q_bytes, "qC and W_UK staging fits the query region");
    static_assert(dc_chunks * wchunk <= stage_bytes, "W_UV fits a ring stage");
    uint8_t* ring = smem;                                                // kStages key tiles
    uint8_t* q_s = ring + kStages * stage_bytes;                         // the query image, same layout
    // qC and W_UK of the next item are staged in the query region (free once the
    // score MMAs of the current item are done)
    uint8_t* qc_s = q_s;
    uint8_t* wk_s = q_s + kQ * 128;
    Bars& bs = *(Bars*)(q_s + q_bytes);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&bs.full[i], 1);
            mbar_init(&bs.empty[i], 1);
        }
        mbar_init(&bs.abs_full, 1);
        mbar_init(&bs.abs_done, 1);
        mbar_init(&bs.q_ready, 8);
        mbar_init(&bs.q_free, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bs.s_full[i], 1);
            mbar_init(&bs.s_empty[i], 1);    // P.V of the tile two back is done (P lives in S)
            mbar_init(&bs.p_full[i], 8);
            mbar_init(&bs.o_done[i], 1);
            mbar_init(&bs.drain[i], 1);
        }
        mbar_init(&bs.olat_ready, 8);
        mbar_init(&bs.out_done, 1);
        mbar_init(&bs.tail_free, 8);
        bs.fail = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&bs.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bs.tmem_base;
    const uint32_t t_s0 = tmem;            // S buffers: columns [0, 128) and [128, 256)
    const uint32_t t_o = tmem + 256;       // q~ (absorption), then O: columns [256, 256 + d_c)
    // P (bf16 pairs) of a tile overwrites the first 64 columns of its S buffer;
    // at an item's end O_lat (bf16 pairs) takes columns [0, d_c / 2) and the
    // output columns [128, 128 + d_h)
    const uint32_t t_olat = tmem, t_out = tmem + 128;

    // every role walks the same items and counts ring positions R (key tiles
    // plus one W_UV position per item) and key tiles G (S buffers) alike
    int loads_R = 0, loads_q = 0;          // the producer's copies, for the drain on failure

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&maps.qc);
            tma_prefetch_desc(&maps.slots);
            tma_prefetch_desc(&maps.slots_r);
            auto load_qw = [&](const Item& it) {
                mbar_arrive_expect_tx(&bs.abs_full, kQ * 128 + dc_chunks * wchunk);
                tma_load_4d(qc_s, &maps.qc, &bs.abs_full, 0, it.h, it.p0, it.b);
                for (int n = 0; n < dc_chunks; ++n)
                    tma_load_3d(wk_s + n * wchunk, &maps.wuk, &bs.abs_full, n * 64, 0, it.h);
                ++loads_q;
            };
            // ring position `pos` is free once the consumer of position pos - 2 released it
            auto ring_free = [&](int pos) {
                return pos < kStages || waitb(&bs.empty[pos & 1], ((pos >> 1) - 1) & 1, bs);
            };
            int R = 0;
            int idx = item_at(p, 0);
            if (idx >= 0) load_qw(decode_item(p, idx));
            for (int j = 0; idx >= 0 && !bs.fail; ++j) {
                const Item it = decode_item(p, idx);
                const int nidx = item_at(p, j + 1);
                {
                    // the item's own partial slots P[b, p0 .. p0+127] as one ring position
                    // (same layout as a key tile; rows past T read as zeros)
                    const int pos = R++;
                    if (!ring_free(pos)) break;
                    uint8_t* dst = ring + (pos & 1) * stage_bytes;
                    mbar_arrive_expect_tx(&bs.full[pos & 1], stage_bytes);
#pragma unroll
                    for (int c = 0; c < NL; ++c)
                        tma_load_3d(dst + c * chunk_k, &maps.prow, &bs.full[pos & 1], c * 64, it.p0, it.b);
                    tma_load_3d(dst + NL * chunk_k, &maps.prow_r, &bs.full[pos & 1], DC, it.p0, it.b);
                    loads_R = R;
                }
                bool ok = true;
                for (int k = 0; k < it.nft && ok; ++k) {
                    const int pos = R++;
                    if (!(ok = ring_free(pos))) break;
                    uint8_t* dst = ring + (pos & 1) * stage_bytes;
                    mbar_arrive_expect_tx(&bs.full[pos & 1], stage_bytes);
#pragma unroll
                    for (int c = 0; c < NL; ++c)
                        tma_load_3d(dst + c * chunk_k, &maps.slots, &bs.full[pos & 1], c * 64, kKT * k, it.b);
                    tma_load_3d(dst + NL * chunk_k, &maps.slots_r, &bs.full[pos & 1], DC, kKT * k, it.b);
                    loads_R = R;
                }
                if (!ok) break;
                // the next item's qC and W_UK into the query region once this item's
                // score MMAs have read it
                if (nidx >= 0) {
                    if (!waitb(&bs.q_free, j & 1, bs)) break;
                    load_qw(decode_item(p, nidx));
                }
                // this item's W_UV as one more ring position
                const int pos = R++;
                if (!ring_free(pos)) break;
                mbar_arrive_expect_tx(&bs.full[pos & 1], dc_chunks * wchunk);
                for (int n = 0; n < dc_chunks; ++n)
                    tma_load_3d(ring + (pos & 1) * stage_bytes + n * wchunk, &maps.wuv, &bs.full[pos & 1], n * 64, 0,
                                it.h);
                loads_R = R;
                idx = nidx;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ absorption, score and output MMAs
        if (lane == 0) {
            const uint32_t id_abs = idesc_f32<E>(128, DC, false, true);
            const uint32_t id_s = idesc_f32<E>(128, kKT, false, false);
            const uint32_t id_out = idesc_f32<E>(128, kDh, false, false);
            const uint32_t ring_a = smem_u32(ring), q_a = smem_u32(q_s);
            const uint64_t q_d = sdesc_sw128(q_a, 16, 1024), q_r = sdesc_sw64(q_a + NL * kQ * 128);
            const uint64_t qc_d = sdesc_sw128(smem_u32(qc_s), 16, 1024);
            const uint64_t wd = sdesc_sw128(smem_u32(wk_s), wchunk, 1024);
            int R = 0, G = 0, wpos = -1;     // wpos: ring position of the previous item's W_UV
            for (int j = 0; !bs.fail; ++j) {
                const int idx = item_at(p, j);
                if (j > 0) {
                    // out = O_lat . W_UV[h]^T of the previous item: A = O_lat [128 x d_c]
                    // (bf16 pairs in TMEM), B = W_UV[h] [d_h x d_c] K-major (ring)
                    if (!waitb(&bs.olat_ready, (j - 1) & 1, bs)) break;
                    if (!waitb(&bs.full[wpos & 1], (wpos >> 1) & 1, bs)) break;
                    tc_fence_after();
                    const uint64_t wv_d = sdesc_sw128(ring_a + (wpos & 1) * stage_bytes, 16, 1024);
#pragma unroll
                    for (int kk = 0; kk < DC / 16; ++kk)
                        umma_bf16_ts(t_out, t_olat + kk * 8, desc_add(wv_d, (kk >> 2) * wchunk + (kk & 3) * 32),
                                     id_out, kk > 0);
                    umma_commit(&bs.out_done);
                    umma_commit(&bs.empty[wpos & 1]);   // the W_UV position of the ring is free
                }
                if (idx < 0) break;
                const Item it = decode_item(p, idx);
                // q~ = qC . W_UK[h]: A = qC [128 x d_h] K-major, B = W_UK[h] [d_h x d_c]
                // MN-major; into the O columns, free since the previous item's O was read
                if (!waitb(&bs.abs_full, j & 1, bs)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kDh / 16; ++kk)
                    umma_bf16(t_o, desc_add(qc_d, kk * 32), desc_add(wd, kk * 2048), id_abs, kk > 0);
                umma_commit(&bs.abs_done);
                if (!waitb(&bs.q_ready, j & 1, bs)) break;
                // the S columns held the previous item's O_lat and output until read
                if (j > 0 && !waitb(&bs.tail_free, (j - 1) & 1, bs)) break;
                ++R;                                 // the item's own partial slots (the softmax reads them)
                bool ok = true;
                for (int k = 0; k < it.nft; ++k, ++G) {
                    const int pos = R++;
                    if (!(ok = waitb(&bs.full[pos & 1], (pos >> 1) & 1, bs))) break;
                    if (G >= 2 && !(ok = waitb(&bs.s_empty[G & 1], ((G >> 1) - 1) & 1, bs))) break;
                    tc_fence_after();
                    // S = q~ . K^T (M = 128 queries, N = 128 slots, K = D): the latent
                    // chunks, then the two K-steps of the RoPE chunk
                    const uint32_t stage_a = ring_a + (pos & 1) * stage_bytes;
                    const uint64_t kd = sdesc_sw128(stage_a, 16, 1024), kr = sdesc_sw64(stage_a + NL * chunk_k);
                    const uint32_t ts = t_s0 + (G & 1) * kKT;
#pragma unroll
                    for (int c = 0; c < NL; ++c) {
                        const uint64_t qc = desc_add(q_d, c * kQ * 128), kc = desc_add(kd, c * chunk_k);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_bf16(ts, desc_add(qc, kk * 32), desc_add(kc, kk * 32), id_s, (c | kk) != 0);
                    }
#pragma unroll
                    for (int kk = 0; kk < kDr / 16; ++kk)
                        umma_bf16(ts, desc_add(q_r, kk * 32), desc_add(kr, kk * 32), id_s, 1u);
                    umma_commit(&bs.s_full[G & 1]);
                }
                if (!ok) break;
                umma_commit(&bs.q_free);             // the query region may take the next item's qC
                wpos = R++;
            }
        }
    } else if (warp == 10) {
        // ------------------------------------------------------------ P.V MMAs (own thread: they free
        // ring stages, so they never wait behind a score MMA that waits for a load)
        if (lane == 0) {
            const uint32_t id_o = idesc_f32<E>(128, DC, false, true);
            const uint32_t ring_a = smem_u32(ring);
            int R = 0, G = 0;
            bool ok = true;
            for (int j = 0; ok; ++j) {
                const int idx = item_at(p, j);
                if (idx < 0) break;
                const Item it = decode_item(p, idx);
                ++R;                                   // the item's own partial slots
                for (int k = 0; k < it.nft; ++k, ++G) {
                    const int pos = R++;
                    if (!(ok = waitb(&bs.p_full[G & 1], (G >> 1) & 1, bs))) break;
                    tc_fence_after();
                    // O += P . V: A = P [128 x 128] in TMEM, B = V = key tile latent [128 x d_c] MN-major
                    const uint64_t vd = sdesc_sw128(ring_a + (pos & 1) * stage_bytes, chunk_k, 1024);
#pragma unroll
                    for (int kk = 0; kk < kKT / 16; ++kk)
                        umma_bf16_ts(t_o, t_s0 + (G & 1) * kKT + kk * 8, desc_add(vd, kk * 2048), id_o, 1u);
                    umma_commit(&bs.empty[pos & 1]);
                    umma_commit(&bs.o_done[G & 1]);
                    umma_commit(&bs.s_empty[G & 1]);   // S buffer G & 1 (which held P) is free
                }
                ++R;                                   // the item's W_UV position
            }
        }
    } else {
        // ------------------------------------------------------------ softmax warps (2-9)
        // Row r = (warp mod 4) * 32 + lane (the TMEM lane quarter a warp may
        // access); hc = (warp - 2) / 4 picks the column half of every tile. No
        // early exit: after a bounded wait gave up, later waits return at once and
        // every thread still meets every named barrier.
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const int hc = (warp - 2) >> 2;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        constexpr int half = DC / 2;
        float v[32];
        uint32_t w[32];
        int G = 0, R = 0;
        for (int j = 0;; ++j) {
            const int idx = item_at(p, j);
            if (idx < 0) break;
            const Item it = decode_item(p, idx);
            const int b = it.b, h = it.h, p0 = it.p0, nft = it.nft;
            const int pos = p0 + r;
            const bool row_ok = pos < p.T;
            // ring positions of this item: own partial slots, key tiles, W_UV
            const int ppos = R;
            R += nft + 2;
            const uint8_t* pst = ring + (ppos & 1) * stage_bytes;   // row r: this row's own partial slot
            // q~ row block of 32 columns into the query image: latent columns into the
            // 128-byte-swizzled chunks, the RoPE block into the 64-byte-swizzled one
            // (v holds the block in fp32; it is rounded once, into packed pairs w)
            auto put_q = [&](int col) {
#pragma unroll
                for (int i = 0; i < 16; ++i) w[i] = pack2<E>(v[2 * i], v[2 * i + 1]);
                if (col < DC) st_row32_packed(q_s, kQ * 128, r, col, w, false);
                else st_row32_packed(q_s + NL * kQ * 128, 0, r, col - DC, w, true);
                if (p.qt && row_ok) {
                    uint4* g = (uint4*)((bf16*)p.qt + (((size_t)b * p.T + pos) * p.H + h) * p.D + col);
#pragma unroll
                    for (int u = 0; u < 4; ++u) g[u] = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
                }
            };
            float e_own = 0.f;
            // 8 columns [c, c + 8) of this row's own partial slot, from the ring
            auto own8 = [&](int c) -> uint4 {
                return c < DC ? *(const uint4*)(pst + (c >> 6) * chunk_k + sw128_offset(r, c & 63))
                              : *(const uint4*)(pst + NL * chunk_k + sw64_offset(r, c - DC));
            };
            // q~ row in 32-column blocks, the first half of the blocks for hc = 0 and
            // the rest for hc = 1 (which therefore holds the RoPE block): latent blocks
            // from TMEM, the RoPE block rotated with the scan's (cos, sin) table; all
            // rounded to bf16 into the query image. The own-slot score q~ . P_pos uses
            // the same rounded values.
            constexpr int n_blk = NL * 2 + 1, nb0 = (n_blk + 1) / 2;
            const int blk0 = hc == 0 ? 0 : nb0, blk1 = hc == 0 ? nb0 : n_blk;   // <= 5 blocks each
            const E* qr = (const E*)p.q_r + (((size_t)b * p.T + min(pos, p.T - 1)) * p.H + h) * p.d_r;
            const float2* cs_row = p.rope_tab + (size_t)min(pos, p.T - 1) * (p.d_r / 2);
            waitb(&bs.abs_done, j & 1, bs);
            waitb(&bs.full[ppos & 1], (ppos >> 1) & 1, bs);
            tc_fence_after();
#pragma unroll
            for (int q = 0; q < 5; ++q) {
                const int c0 = (blk0 + q) * 32;
                if (blk0 + q < blk1) {
                    if (c0 < DC) {
                        tmem_ld32(t_o + c0 + lane_off, v);
                        tmem_wait_ld();
                    } else {
                        // RoPE columns (zero past d_r): qR and the (cos, sin) pairs as vectors
                        const int e0 = c0 - DC;
                        uint4 qv[4];
                        float4 cs4[8];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            qv[u] = make_uint4(0, 0, 0, 0);
                            if (e0 + 8 * u < p.d_r) qv[u] = *(const uint4*)(qr + e0 + 8 * u);
                        }
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            cs4[u] = make_float4(1.f, 0.f, 1.f, 0.f);
                            if (e0 + 4 * u < p.d_r) cs4[u] = *(const float4*)(cs_row + e0 / 2 + 2 * u);
                        }
                        const E* qe = (const E*)qv;
                        const float* csv = (const float*)cs4;      // cos, sin of pair i / 2
#pragma unroll
                        for (int i = 0; i < 32; i += 2) {
                            v[i] = v[i + 1] = 0.f;
                            if (row_ok && e0 + i < p.d_r) {
                                const float cs = csv[i], sn = csv[i + 1];
                                const float x0 = to_f<E>(qe[i]), x1 = to_f<E>(qe[i + 1]);
                                v[i] = x0 * cs - x1 * sn;
                                v[i + 1] = x0 * sn + x1 * cs;
                            }
                        }
                    }
                    put_q(c0);
                    float e2[2] = {0.f, 0.f};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint4 raw = own8(c0 + 8 * u);
                        const uint32_t rw[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            e2[0] = fmaf(lo_of<E>(w[4 * u + i]), lo_of<E>(rw[i]), e2[0]);
                            e2[1] = fmaf(hi_of<E>(w[4 * u + i]), hi_of<E>(rw[i]), e2[1]);
                        }
                    }
                    e_own += e2[0] + e2[1];
                }
            }
            fence_proxy_async();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bs.q_ready);
            bs.xs[hc][r] = e_own;
            named_sync(1, 256);                           // also: every q~ read of TMEM is done
            tc_fence_after();
            const float es = row_ok ? (bs.xs[0][r] + bs.xs[1][r]) * p.scale_log2 : 0.f;
            // O starts as the own slot's latent part, with weight 1 at the starting
            // reference maximum es (its TMEM columns held q~, read above)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int cc = hc * half + 32 * q;
                if (32 * q < half) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint4 raw = own8(cc + 8 * u);
                        const E* pe = (const E*)&raw;
#pragma unroll
                        for (int i = 0; i < 8; ++i) v[8 * u + i] = to_f<E>(pe[i]);
                    }
                    tmem_st32(t_o + cc + lane_off, v);
                }
            }
            tmem_wait_st();
            fence_proxy_async();
            named_sync(1, 256);                           // xs is free again; the own slots are read
            if (tid == 64) mbar_arrive(&bs.empty[ppos & 1]);   // their ring position is free
            // online softmax over the finished-slot tiles; the own slot is the
            // starting point (reference maximum es, weight 1 in the row sum)
            float m_ref = es, l = hc == 0 ? 1.f : 0.f;    // l: this thread's half of the row sum
            const int fin_lim = (p.t0 + pos) / p.s;       // finished slots this row may see
            const int min_fin = (p.t0 + p0) / p.s;        // ... and the first row of the tile
            for (int k = 0; k < nft; ++k, ++G) {
                waitb(&bs.s_full[G & 1], (G >> 1) & 1, bs);
                tc_fence_after();
                float sv[64];
                tmem_ld32(t_s0 + (G & 1) * kKT + hc * 64 + lane_off, sv);
                tmem_ld32(t_s0 + (G & 1) * kKT + hc * 64 + 32 + lane_off, sv + 32);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                // raw scores: the scale is folded into the exponent below. The slot mask
                // only matters on tiles that reach past the first row's limit (a test
                // uniform across the CTA). Maxima and sums in four independent chains.
                const int j0 = kKT * k + 64 * hc;
                if (kKT * (k + 1) > min_fin) {
#pragma unroll
                    for (int c = 0; c < 64; ++c)
                        if (j0 + c >= fin_lim) sv[c] = -INFINITY;
                }
                float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int c = 0; c < 64; ++c) m4[c & 3] = fmaxf(m4[c & 3], sv[c]);
                float mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * p.scale_log2;
                bs.red[G & 1][hc][r] = mt;
                named_sync(1, 256);
                tc_fence_after();                         // the other half's TMEM reads are done
                mt = fmaxf(mt, bs.red[G & 1][hc ^ 1][r]);
                // lazy rescale: the reference maximum moves only when the tile's maximum
                // exceeds it by more than 2^8 (P stays <= 256); both halves decide alike
                const bool upd = mt > m_ref + kRescaleLog2;
                const float nm = upd ? mt : m_ref;
                const float fac = ex2_approx(m_ref - nm);
                float rs4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const float q0 = ex2_approx(fmaf(sv[2 * c], p.scale_log2, -nm));
                    const float q1 = ex2_approx(fmaf(sv[2 * c + 1], p.scale_log2, -nm));
                    rs4[c & 3] += q0 + q1;
                    w[c] = pack2<E>(q0, q1);
                }
                l = fmaf(l, fac, (rs4[0] + rs4[1]) + (rs4[2] + rs4[3]));
                // O holds the own slot and this item's tiles 0..k-1
                if (__any_sync(0xffffffffu, upd)) {
                    if (k > 0) waitb(&bs.o_done[(G - 1) & 1], ((G - 1) >> 1) & 1, bs);
                    tc_fence_after();
                    const float f = upd ? fac : 1.f;
                    for (int cc = hc * half; cc < (hc + 1) * half; cc += 32) {
                        tmem_ld32(t_o + cc + lane_off, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] *= f;
                        tmem_st32(t_o + cc + lane_off, v);
                    }
                    tmem_wait_st();
                }
                // P over the first 64 columns of this tile's S buffer (both halves have
                // read their scores: the barrier above)
                tmem_st32_u(t_s0 + (G & 1) * kKT + hc * 32 + lane_off, w);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bs.p_full[G & 1]);
                m_ref = nm;
            }
            // epilogue: O_lat = O / l as bf16 pairs into the S columns (the output
            // MMA's A operand), then out = O_lat . W_UV^T
            if (nft > 0) waitb(&bs.o_done[(G - 1) & 1], ((G - 1) >> 1) & 1, bs);
            tc_fence_after();
            bs.xs[hc][r] = l;
            named_sync(1, 256);
            const float l_row = bs.xs[0][r] + bs.xs[1][r];
            const float inv = 1.f / l_row;
            named_sync(1, 256);                           // xs is free again
            if (p.lse && row_ok && hc == 0)
                p.lse[((size_t)b * p.H + h) * stats_pitch(p.T) + pos] = m_ref + log2f(l_row);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int cc = hc * half + 32 * q;
                if (32 * q < half) {
                    tmem_ld32(t_o + cc + lane_off, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) w[i] = pack2<E>(v[2 * i] * inv, v[2 * i + 1] * inv);
                    tmem_st16_u(t_olat + cc / 2 + lane_off, w);
                    if (p.obar && row_ok) {
                        uint4* g = (uint4*)((bf16*)p.obar + (((size_t)b * p.T + pos) * p.H + h) * DC + cc);
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            g[u] = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
                    }
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bs.olat_ready);   // also: O has been read
            waitb(&bs.out_done, j & 1, bs);
            tc_fence_after();
            for (int cc = hc * (kDh / 2); cc < (hc + 1) * (kDh / 2); cc += 32) {
                tmem_ld32(t_out + cc + lane_off, v);
                tmem_wait_ld();
                if (row_ok) {
                    E* o = (E*)p.out + (((size_t)b * p.T + pos) * p.H + h) * kDh + cc;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        uint4 pk;
                        pk.x = pack2<E>(v[8 * u + 0], v[8 * u + 1]);
                        pk.y = pack2<E>(v[8 * u + 2], v[8 * u + 3]);
                        pk.z = pack2<E>(v[8 * u + 4], v[8 * u + 5]);
                        pk.w = pack2<E>(v[8 * u + 6], v[8 * u + 7]);
                        *(uint4*)(o + 8 * u) = pk;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bs.tail_free);    // the S columns are free
        }
    }
    tc_fence_before();
    __syncthreads();
    if (bs.fail) {
        // a bounded wait gave up: let the copies and MMAs in flight land (bounded
        // again) before shared memory and TMEM are released, then report
        if ((warp == 1 || warp == 10) && lane == 0) {
            uint64_t* d = &bs.drain[warp == 1 ? 0 : 1];
            umma_commit(d);
            mbar_wait(d, 0);
        }
        if (warp == 0 && lane == 0) {
            for (int pos = max(0, loads_R - kStages); pos < loads_R; ++pos)
                mbar_wait(&bs.full[pos & 1], (pos >> 1) & 1);
            if (loads_q > 0) mbar_wait(&bs.abs_full, (loads_q - 1) & 1);
        }
        if (tid == 0) latch_status(p.status, kStatusTimeout);
        __syncthreads();
    }
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- host side

// Key tile and query image: d_c / 64 latent chunks of 128 rows x 128 B plus a
// RoPE chunk of 128 rows x 64 B.
size_t prefill_smem_bytes(const Shape& sh) {
    const size_t tile = (size_t)(sh.d_c / 64) * kKT * 128 + kKT * 64;
    return 1024 + (kStages + 1) * tile + ((sizeof(Bars) + 15) & ~(size_t)15);
}

cudaError_t make_map(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* m, const void* base, int rank,
                     const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box, const char* what,
                     CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B,
                     CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = enc(m, dt, rank, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        char buf[128];
        snprintf(buf, sizeof(buf), "cuTensorMapEncodeTiled(%s) (CUresult %d)", what, (int)r);
        return note_error(buf, cudaErrorInvalidValue);
    }
    return cudaSuccess;
}

// The compiled instances: d_h = 64, d_R = 32, d_c = 256 or 128, bf16 or fp16
// storage. Other widths take the CUDA-core prefill.
using PrefillKernel = void (*)(Maps, PreTC);
PrefillKernel prefill_kernel(const Shape& sh) {
    if (sh.d_h != kDh || sh.d_r != kDr) return nullptr;
    const bool h16 = sh.dtype == kDtypeF16;
    if (sh.dtype != kDtypeBF16 && !h16) return nullptr;
    if (sh.d_c == 256) return h16 ? k_prefill_tc<256, f16> : k_prefill_tc<256, bf16>;
    if (sh.d_c == 128) return h16 ? k_prefill_tc<128, f16> : k_prefill_tc<128, bf16>;
    return nullptr;
}

}  // namespace

bool tc_prefill_supported(const Shape& sh) {
    return prefill_kernel(sh) != nullptr && prefill_smem_bytes(sh) <= 232448 - 1024;
}

size_t tc_prefill_workspace(const Shape& sh, int T) {
    return align256((size_t)sh.B * T * sh.D * sizeof(bf16)) + align256((size_t)T * (sh.d_r / 2) * sizeof(float2)) +
           prefill_seed_bytes(sh);
}

static cudaError_t tc_prefill_impl(const PrefillArgs& a_in, const PrefillSave* sv, cudaStream_t st,
                                   uint64_t* launches) {
    PrefillArgs a = a_in;
    const Shape& sh = a.sh;
    const int T = a.T;
    void* P = a.workspace;                  // the partial slots, storage type (2 bytes)
    {
        const size_t off = align256((size_t)sh.B * T * sh.D * sizeof(bf16)) +
                           align256((size_t)T * (sh.d_r / 2) * sizeof(float2));
        cudaError_t e = prefill_seed(a, (char*)a.workspace + off, st);
        if (e != cudaSuccess) return e;
    }
    auto enc = (PFN_cuTensorMapEncodeTiled_v12000)tensor_map_encoder();
    const CUtensorMapDataType DT =
        sh.dtype == kDtypeF16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const auto S128 = CU_TENSOR_MAP_SWIZZLE_128B;
    if (!enc) return note_error("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", cudaErrorNotSupported);
    Maps maps;
    const cuuint64_t E = 2;
    {
        cuuint64_t d[4] = {(cuuint64_t)sh.d_h, (cuuint64_t)sh.H, (cuuint64_t)T, (cuuint64_t)sh.B};
        cuuint64_t s[3] = {E * sh.d_h, E * sh.H * sh.d_h, E * T * sh.H * sh.d_h};
        cuuint32_t bx[4] = {64, 1, kQ, 1};
        cudaError_t e = make_map(enc, &maps.qc, a.q_c, 4, d, s, bx, "q_c", S128, DT);
        if (e != cudaSuccess) return e;
    }
    {
        cuuint64_t d[3] = {(cuuint64_t)sh.d_c, (cuuint64_t)sh.d_h, (cuuint64_t)sh.H};
        cuuint64_t s[2] = {E * sh.d_c, E * sh.d_h * sh.d_c};
        cuuint32_t bx[3] = {64, (cuuint32_t)sh.d_h, 1};
        cudaError_t e = make_map(enc, &maps.wuk, a.w_uk, 3, d, s, bx, "w_uk", S128, DT);
        if (e == cudaSuccess) e = make_map(enc, &maps.wuv, a.w_uv, 3, d, s, bx, "w_uv", S128, DT);
        if (e != cudaSuccess) return e;
    }
    {
        // the cache through slot ceil((t0 + T) / s) - 1: the earlier chunks' and this one's
        const int n_slots = (a.t0 + T + sh.s - 1) / sh.s;
        cuuint64_t d[3] = {(cuuint64_t)sh.D, (cuuint64_t)n_slots, (cuuint64_t)sh.B};
        cuuint64_t s[2] = {E * sh.D, E * sh.max_slots * sh.D};
        cuuint32_t bx[3] = {64, kKT, 1};
        cudaError_t e = make_map(enc, &maps.slots, a.cache_out, 3, d, s, bx, "cache_out", S128, DT);
        cuuint32_t bxr[3] = {kDr, kKT, 1};
        if (e == cudaSuccess)
            e = make_map(enc, &maps.slots_r, a.cache_out, 3, d, s, bxr, "cache_out RoPE", CU_TENSOR_MAP_SWIZZLE_64B, DT);
        if (e != cudaSuccess) return e;
    }
    {
        // the own partial slots P [B, T, D] as 128-row tiles of the same layout
        cuuint64_t d[3] = {(cuuint64_t)sh.D, (cuuint64_t)T, (cuuint64_t)sh.B};
        cuuint64_t s[2] = {E * sh.D, E * T * sh.D};
        cuuint32_t bx[3] = {64, kQ, 1};
        cuuint32_t bxr[3] = {kDr, kQ, 1};
        cudaError_t e = make_map(enc, &maps.prow, P, 3, d, s, bx, "partial slots", S128, DT);
        if (e == cudaSuccess)
            e = make_map(enc, &maps.prow_r, P, 3, d, s, bxr, "partial slots RoPE", CU_TENSOR_MAP_SWIZZLE_64B, DT);
        if (e != cudaSuccess) return e;
    }
    PreTC p;
    p.B = sh.B;
    p.T = T;
    p.H = sh.H;
    p.d_h = sh.d_h;
    p.d_c = sh.d_c;
    p.d_r = sh.d_r;
    p.D = sh.D;
    p.s = sh.s;
    p.n_qtiles = (T + kQ - 1) / kQ;
    p.t0 = a.t0;
    p.n_items = p.n_qtiles * sh.B * sh.H;
    p.scale_log2 = sh.scale * 1.4426950408889634f;
    p.log2_rope_base = sh.log2_rope_base;
    p.q_r = a.q_r;
    p.rope_tab = (const float2*)((char*)a.workspace + align256((size_t)sh.B * T * sh.D * sizeof(bf16)));
    p.out = a.out;
    p.lse = sv ? sv->lse : nullptr;
    p.obar = sv ? sv->obar : nullptr;
    p.qt = sv ? sv->qt : nullptr;
    p.status = a.status;

    const int n_slots = (a.t0 + T - 1) / sh.s - a.t0 / sh.s + 1;    // slots the chunk touches
    const dim3 sg((n_slots + 7) / 8, sh.B);
    if (sh.dtype == kDtypeF16) {
        if (sh.gate_mode >= 3) k_prefill_scan_channel<f16, f16><<<sg, 256, 0, st>>>(a, (f16*)P, (float2*)p.rope_tab);
        else k_prefill_scan<f16, f16><<<sg, 256, 0, st>>>(a, (f16*)P, (float2*)p.rope_tab, sv ? sv->w : nullptr);
    } else {
        if (sh.gate_mode >= 3) k_prefill_scan_channel<bf16, bf16><<<sg, 256, 0, st>>>(a, (bf16*)P, (float2*)p.rope_tab);
        else k_prefill_scan<bf16, bf16><<<sg, 256, 0, st>>>(a, (bf16*)P, (float2*)p.rope_tab, sv ? sv->w : nullptr);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return note_error("k_prefill_scan launch", e);

    const size_t smem = prefill_smem_bytes(sh);
    const PrefillKernel kern = prefill_kernel(sh);
    if (!kern) return note_error("tc_prefill: no compiled instance for these widths", cudaErrorInvalidValue);
    // the attribute is set on every call: it is per kernel instance and device
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return note_error("cudaFuncSetAttribute(k_prefill_tc)", e);
    // persistent: one CTA per SM (the shared memory allows no second), each
    // walking its share of the items
    const unsigned grid = (unsigned)std::min(p.n_items, sm_count());
    // the attention kernel's event pair (not inside the training backward,
    // whose own pair brackets its tensor-core kernels)
    if (!sv) profile_begin(st);
    kern<<<grid, kThreads, smem, st>>>(maps, p);
    if (!sv) profile_end(st);
    *launches += 2;
    return note_error("k_prefill_tc launch", cudaGetLastError());
}

cudaError_t tc_prefill(const PrefillArgs& a, cudaStream_t st, uint64_t* launches) {
    return tc_prefill_impl(a, nullptr, st, launches);
}

cudaError_t tc_prefill_save(const PrefillArgs& a, const PrefillSave& sv, cudaStream_t st, uint64_t* launches) {
    if (a.t0 != 0 || a.sh.gate_mode >= 3) return note_error("tc_prefill_save: t0 = 0, scalar gates", cudaErrorInvalidValue);
    return tc_prefill_impl(a, &sv, st, launches);
}

}  // namespace mtla
