// tc_backward.cu -- the masked-attention part of the training backward on the
// tensor cores (bf16 operands, fp32 accumulation), for the widths of the
// tensor-core prefill (d_h = 64, d_R = 32, d_c = 128 or 256).
//
// "Multi-head Temporal Latent Attention", Results (trained from scratch) and
// Key claims (the stride-aware mask in training): query i of head h attends
// the finished slots F_j, j < floor(i/s), and its own partial P_i. With the
// forward's row statistics kept (lse in the log2 domain, obar = O / l) and
//   dobar_i = W_UV[h]^T dout_i,  delta_i = dobar_i . obar_i,
//   p_ij = 2^(S_ij scale log2(e) - lse_i),  S_ij = qt_i . F_j,
//   dPa_ij = dobar_i . F_j[0:d_c],  dS_ij = scale p_ij (dPa_ij - delta_i),
// the finished-slot part of the gradients is two contractions:
//   dqt_i += sum_j dS_ij F_j                 (k_bwd_dq_tc, one CTA per query tile;
//                                             dPa there as dout_i . U_j, U_j = W_UV[h] F_j)
//   dF_j  += sum_i dS_ij qt_i + p_ij [dobar_i ; 0]   (k_bwd_dk_tc, one CTA per slot tile)
// The own-partial term (one key per row) runs on the CUDA cores.
//
// Both kernels: warp 0 issues the TMA loads, warp 1 the MMAs, warps 2-9 turn
// scores into the bf16 A operand of the accumulating MMAs (two threads per TMEM
// lane, 32 columns each). Per tile the two score-shaped MMAs (S and dPa, 64
// columns each: N = 64, so that two ring stages, the resident operand image and
// the 288-column accumulator fit shared memory and TMEM) write TMEM; the
// elementwise warps read them and release the columns (so the next tile's
// score MMAs start at once), then write dS (and P) as packed bf16 into TMEM,
// where the accumulating MMAs read their A operand. Shared-memory operands: the
// latent columns in 64-column chunks with the 128-byte swizzle, the 32 RoPE
// columns as one chunk with the 64-byte swizzle; the same tile serves as a
// K-major operand of the score MMAs and as an MN-major operand of the
// accumulating ones.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdio>

#include "common.cuh"
#include "mtla_internal.h"
#include "tc_common.cuh"

namespace mtla {

namespace {

using namespace tc;

constexpr int kM = 128;         // rows of every MMA: query positions (dQ) or slots (dK)
constexpr int kN = 64;          // keys (dQ) or query positions (dK) per tile
constexpr int kDr = 32;         // d_R of these kernels (one 64-byte-swizzled chunk)
constexpr int kDh = 64;         // d_h of these kernels
constexpr int kThreads = 320;   // warp 0 TMA, 1 MMA, 2-9 elementwise
constexpr int kBand = 8;        // slot tiles per scheduling band of k_bwd_dk_tc

struct BwdTC {
    int B, T, H, D, s, n_slots;
    int n_qtiles, n_ktiles;     // ceil(T / 128), ceil(n_slots / 128)
    float scale, scale_log2;
    const float* lse;           // [B, H, stats_pitch(T)] log2-domain log-sum-exp of every row
    const float* delta;         // [B, H, stats_pitch(T)]
    float* dqt;                 // [B, T, H, D] finished-slot part of dqt
    float* dF;                  // [H, B, n_slots, D] per-head finished-slot key gradients
    int* status;
};

struct MapsQ {
    CUtensorMap q, q_r;         // qt (D, H, T, B): boxes (64, 1, 128, 1) and (32, 1, 128, 1)
    CUtensorMap dout;           // dout (d_h, H, T, B): box (64, 1, 128, 1)
    CUtensorMap k, k_r;         // slots (D, n_slots, B): boxes (64, 64, 1) and (32, 64, 1)
    CUtensorMap u;              // U (H d_h, n_slots, B): box (64, 64, 1)
};
struct MapsK {
    CUtensorMap k, k_r;         // slots: boxes (64, 128, 1) and (32, 128, 1)
    CUtensorMap q, q_r;         // qt: boxes (64, 1, 64, 1) and (32, 1, 64, 1)
    CUtensorMap dob;            // dobar: box (64, 1, 64, 1)
    CUtensorMap lse, delta;     // (T, H, B) fp32: box (64, 1, 1)
};

constexpr int kQStages = 3;     // key-tile ring of k_bwd_dq_tc

struct BarsQ {
    uint64_t full[kQStages], empty[kQStages], q_full, sd_full, sd_free, ds_ready[2], ds_free[2], done, drain[2];
    uint32_t tmem_base;
    volatile int fail;
};
struct BarsK {
    uint64_t full[2], empty[2], k_full, sd_full, sd_free, a_ready, a_free, done, drain[2];
    uint32_t tmem_base;
    volatile int fail;
};

template <typename Bars>
__device__ __forceinline__ bool waitb(uint64_t* bar, uint32_t parity, Bars& bs) {
    if (bs.fail) return false;
    if (mbar_wait(bar, parity)) return true;
    bs.fail = 1;
    return false;
}

// MN-major operand in the 64-byte swizzle: 32 contiguous MN elements per 64-B
// row, 8 K-rows per 512-B atom; SBO = byte distance between 8-row K groups
// (LBO, the distance between 32-element MN chunks, is unused at N = 32).
__device__ __forceinline__ uint64_t sdesc_sw64_mn(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(512u >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)4 << 61;
    return d;
}

// ---------------------------------------------------------------- dQ

// One CTA per (query tile of 128 positions, sequence, head), heaviest first.
// Keys: the finished slots j < floor(pos / s) in tiles of 64.
template <int DC>
__global__ void __launch_bounds__(kThreads, 1) k_bwd_dq_tc(const __grid_constant__ MapsQ maps, const BwdTC p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    constexpr int NL = DC / 64;
    constexpr uint32_t q_bytes = NL * kM * 128 + kM * 64;      // query image: latent chunks + RoPE chunk
    constexpr uint32_t do_bytes = kM * 128;                    // dout image [128 rows x d_h = 64]
    constexpr uint32_t kchunk = kN * 128;                      // one latent chunk of a key tile
    constexpr uint32_t u_off = NL * kchunk + kN * 64;          // the tile's U rows [64 x d_h]
    constexpr uint32_t stage_bytes = u_off + kN * 128;
    uint8_t* q_s = smem;
    uint8_t* do_s = q_s + q_bytes;
    uint8_t* ring = do_s + do_bytes;
    BarsQ& bs = *(BarsQ*)(ring + kQStages * stage_bytes);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int per_qt = p.B * p.H;
    const int qt = p.n_qtiles - 1 - (int)blockIdx.x / per_qt;
    const int b = ((int)blockIdx.x % per_qt) / p.H, h = (int)blockIdx.x % p.H;
    const int p0 = qt * kM;
    const int last = min(p0 + kM - 1, p.T - 1);
    const int nkt = (last / p.s + kN - 1) / kN;               // key tiles (finished slots of the last row)

    if (tid == 0) {
        for (int i = 0; i < kQStages; ++i) {
            mbar_init(&bs.full[i], 1);
            mbar_init(&bs.empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bs.ds_ready[i], 8);
            mbar_init(&bs.ds_free[i], 1);
            mbar_init(&bs.drain[i], 1);
        }
        mbar_init(&bs.q_full, 1);
        mbar_init(&bs.sd_full, 1);
        mbar_init(&bs.sd_free, 8);
        mbar_init(&bs.done, 1);
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
    const uint32_t t_s = tmem, t_dp = tmem + 64;               // S, dPa (fp32, 64 columns each)
    const uint32_t t_ds = tmem + 128;                          // dS (bf16 pairs), two buffers of 32 columns
    const uint32_t t_dq = tmem + 192;                          // dqt accumulator, D columns
    int loads = 0;

    if (warp == 0) {
        if (lane == 0 && nkt > 0) {
            mbar_arrive_expect_tx(&bs.q_full, q_bytes + do_bytes);
#pragma unroll
            for (int c = 0; c < NL; ++c) tma_load_4d(q_s + c * kM * 128, &maps.q, &bs.q_full, c * 64, h, p0, b);
            tma_load_4d(q_s + NL * kM * 128, &maps.q_r, &bs.q_full, DC, h, p0, b);
            tma_load_4d(do_s, &maps.dout, &bs.q_full, 0, h, p0, b);
            for (int k = 0; k < nkt; ++k) {
                const int sg = k % kQStages;
                if (k >= kQStages && !waitb(&bs.empty[sg], ((k / kQStages) - 1) & 1, bs)) break;
                uint8_t* dst = ring + sg * stage_bytes;
                mbar_arrive_expect_tx(&bs.full[sg], stage_bytes);
#pragma unroll
                for (int c = 0; c < NL; ++c) tma_load_3d(dst + c * kchunk, &maps.k, &bs.full[sg], c * 64, kN * k, b);
                tma_load_3d(dst + NL * kchunk, &maps.k_r, &bs.full[sg], DC, kN * k, b);
                tma_load_3d(dst + u_off, &maps.u, &bs.full[sg], h * kDh, kN * k, b);
                loads = k + 1;
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && nkt > 0) {
            const uint32_t id_s = idesc_bf16_f32(kM, kN, false, false);
            const uint32_t id_lat = idesc_bf16_f32(kM, DC, false, true);
            const uint32_t id_rope = idesc_bf16_f32(kM, kDr, false, true);
            const uint32_t q_a = smem_u32(q_s), do_a = smem_u32(do_s), ring_a = smem_u32(ring);
            const uint64_t qd = sdesc_sw128(q_a, 16, 1024), qr = sdesc_sw64(q_a + NL * kM * 128);
            const uint64_t dd = sdesc_sw128(do_a, 16, 1024);
            // dqt += dS . K of tile t: A = dS [128 x 64] in TMEM, B = the key tile
            // MN-major (latent chunks, then the RoPE chunk)
            auto dq_mma = [&](int t) -> bool {
                if (!waitb(&bs.ds_ready[t & 1], (t >> 1) & 1, bs)) return false;
                tc_fence_after();
                const uint32_t st_a = ring_a + (t % kQStages) * stage_bytes;
                const uint64_t bl = sdesc_sw128(st_a, kchunk, 1024), br = sdesc_sw64_mn(st_a + NL * kchunk);
#pragma unroll
                for (int kk = 0; kk < kN / 16; ++kk) {
                    const uint32_t acc = (t > 0 || kk > 0) ? 1u : 0u;
                    umma_bf16_ts(t_dq, t_ds + (t & 1) * 32 + kk * 8, desc_add(bl, kk * 2048), id_lat, acc);
                    umma_bf16_ts(t_dq + DC, t_ds + (t & 1) * 32 + kk * 8, desc_add(br, kk * 1024), id_rope, acc);
                }
                umma_commit(&bs.empty[t % kQStages]);
                umma_commit(&bs.ds_free[t & 1]);
                return true;
            };
            if (waitb(&bs.q_full, 0, bs)) {
                bool ok = true;
                for (int k = 0; k < nkt && ok; ++k) {
                    if (!(ok = waitb(&bs.full[k % kQStages], (k / kQStages) & 1, bs))) break;
                    if (k >= 1 && !(ok = waitb(&bs.sd_free, (k - 1) & 1, bs))) break;
                    tc_fence_after();
                    const uint32_t st_a = ring_a + (k % kQStages) * stage_bytes;
                    const uint64_t kd = sdesc_sw128(st_a, 16, 1024), kr = sdesc_sw64(st_a + NL * kchunk);
                    // S = qt . K^T (K = D); dPa = dobar . V^T = dout . U^T (K = d_h), U_j = W_UV[h] F_j
#pragma unroll
                    for (int c = 0; c < NL; ++c)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_bf16(t_s, desc_add(qd, c * kM * 128 + kk * 32), desc_add(kd, c * kchunk + kk * 32),
                                      id_s, (c | kk) != 0);
#pragma unroll
                    for (int kk = 0; kk < kDr / 16; ++kk)
                        umma_bf16(t_s, desc_add(qr, kk * 32), desc_add(kr, kk * 32), id_s, 1u);
                    const uint64_t ud = sdesc_sw128(st_a + u_off, 16, 1024);
#pragma unroll
                    for (int kk = 0; kk < kDh / 16; ++kk)
                        umma_bf16(t_dp, desc_add(dd, kk * 32), desc_add(ud, kk * 32), id_s, kk != 0);
                    umma_commit(&bs.sd_full);
                    if (k >= 1) ok = dq_mma(k - 1);
                }
                if (ok && dq_mma(nkt - 1)) umma_commit(&bs.done);
            }
        }
    } else {
        // ------------------------------------------------------------ elementwise warps (2-9)
        const int quarter = warp & 3, hc = (warp - 2) >> 2;
        const int r = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int pos = p0 + r;
        const bool row_ok = pos < p.T;
        const int fin_lim = pos / p.s;                         // finished slots this row sees
        const size_t srow = ((size_t)b * p.H + h) * stats_pitch(p.T) + (row_ok ? pos : 0);
        const float lse = row_ok ? p.lse[srow] : 0.f, delta = row_ok ? p.delta[srow] : 0.f;
        float sv[32], dv[32];
        uint32_t w[16];
        for (int k = 0; k < nkt; ++k) {
            waitb(&bs.sd_full, k & 1, bs);
            tc_fence_after();
            tmem_ld32(t_s + hc * 32 + lane_off, sv);
            tmem_ld32(t_dp + hc * 32 + lane_off, dv);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bs.sd_free);
            const int j0 = kN * k + 32 * hc;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                float d2[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int cc = 2 * c + e;
                    const float pr = ex2_approx(fmaf(sv[cc], p.scale_log2, -lse));
                    d2[e] = (row_ok && j0 + cc < fin_lim) ? p.scale * pr * (dv[cc] - delta) : 0.f;
                }
                w[c] = pack_bf16x2(d2[0], d2[1]);
            }
            if (k >= 2) waitb(&bs.ds_free[k & 1], ((k >> 1) - 1) & 1, bs);
            tc_fence_after();
            tmem_st16_u(t_ds + (k & 1) * 32 + hc * 16 + lane_off, w);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bs.ds_ready[k & 1]);
        }
        // epilogue: the accumulator (D = DC + 32 columns, 32-column blocks split
        // between the two threads of a row) to dqt
        constexpr int n_blk = (DC + kDr) / 32, nb0 = (n_blk + 1) / 2;
        if (nkt > 0) waitb(&bs.done, 0, bs);
        tc_fence_after();
        float* out = p.dqt + (((size_t)b * p.T + (row_ok ? pos : 0)) * p.H + h) * p.D;
        for (int q = hc == 0 ? 0 : nb0; q < (hc == 0 ? nb0 : n_blk); ++q) {
            if (nkt > 0) {
                tmem_ld32(t_dq + q * 32 + lane_off, sv);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) sv[i] = 0.f;
            }
            if (row_ok && !bs.fail) {
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    *(float4*)(out + q * 32 + 4 * u) = make_float4(sv[4 * u], sv[4 * u + 1], sv[4 * u + 2], sv[4 * u + 3]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (bs.fail) {
        if (warp == 1 && lane == 0) {
            umma_commit(&bs.drain[0]);
            mbar_wait(&bs.drain[0], 0);
        }
        if (warp == 0 && lane == 0) {
            if (loads > 0) mbar_wait(&bs.q_full, 0);
            for (int k = max(0, loads - kQStages); k < loads; ++k)
                mbar_wait(&bs.full[k % kQStages], (k / kQStages) & 1);
        }
        if (tid == 0) latch_status(p.status, kStatusTimeout);
        __syncthreads();
    }
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- dK

// One CTA per (slot tile of 128, sequence, head). The query positions that
// see any slot of the tile, from the first multiple of 64 at or below
// (j0 + 1) s, in tiles of 64 taken from the last down; positions past T read
// as zeros and are masked.
template <int DC>
__global__ void __launch_bounds__(kThreads, 1) k_bwd_dk_tc(const __grid_constant__ MapsK maps, const BwdTC p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    constexpr int NL = DC / 64;
    constexpr uint32_t k_bytes = NL * kM * 128 + kM * 64;      // slot image
    constexpr uint32_t qchunk = kN * 128;                      // one latent chunk of a query tile
    constexpr uint32_t qt_bytes = NL * qchunk + kN * 64;       // query tile
    constexpr uint32_t dob_bytes = NL * qchunk;                // dobar tile
    constexpr uint32_t stats_off = qt_bytes + dob_bytes;       // lse[64], delta[64]
    constexpr uint32_t stage_bytes = (stats_off + 512 + 1023) & ~1023u;
    uint8_t* k_s = smem;
    uint8_t* ring = k_s + k_bytes;
    BarsK& bs = *(BarsK*)(ring + 2 * stage_bytes);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // items in bands of kBand slot tiles, the heaviest (earliest) band first;
    // inside a band the items of one (sequence, head) are consecutive and walk
    // their query tiles from the top down, so they start on the same tile and
    // share its query rows in L2
    const int BH = p.B * p.H, full = p.n_ktiles / kBand;
    const int idx = blockIdx.x;
    int kt, bh;
    if (idx < full * kBand * BH) {
        const int band = idx / (kBand * BH), rem = idx % (kBand * BH);
        bh = rem / kBand;
        kt = band * kBand + rem % kBand;
    } else {
        const int rem = idx - full * kBand * BH, last = p.n_ktiles - full * kBand;
        bh = rem / last;
        kt = full * kBand + rem % last;
    }
    const int b = bh / p.H, h = bh % p.H;
    const int j0 = kt * kM;
    const int pbase = (((j0 + 1) * p.s) / kN) * kN;
    const int ntl = pbase < p.T ? (p.T - pbase + kN - 1) / kN : 0;

    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bs.full[i], 1);
            mbar_init(&bs.empty[i], 1);
            mbar_init(&bs.drain[i], 1);
        }
        mbar_init(&bs.k_full, 1);
        mbar_init(&bs.sd_full, 1);
        mbar_init(&bs.sd_free, 8);
        mbar_init(&bs.a_ready, 8);
        mbar_init(&bs.a_free, 1);
        mbar_init(&bs.done, 1);
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
    const uint32_t t_s = tmem, t_dp = tmem + 64;               // S^T, dPa^T (fp32, 64 columns each)
    const uint32_t t_p = tmem + 128, t_ds = tmem + 160;        // P^T, dS^T (bf16 pairs, 32 columns each)
    const uint32_t t_dk = tmem + 192;                          // dF accumulator, D columns
    int loads = 0;

    if (warp == 0) {
        if (lane == 0 && ntl > 0) {
            mbar_arrive_expect_tx(&bs.k_full, k_bytes);
#pragma unroll
            for (int c = 0; c < NL; ++c) tma_load_3d(k_s + c * kM * 128, &maps.k, &bs.k_full, c * 64, j0, b);
            tma_load_3d(k_s + NL * kM * 128, &maps.k_r, &bs.k_full, DC, j0, b);
            for (int k = 0; k < ntl; ++k) {
                if (k >= 2 && !waitb(&bs.empty[k & 1], ((k >> 1) - 1) & 1, bs)) break;
                uint8_t* dst = ring + (k & 1) * stage_bytes;
                const int pk = pbase + kN * (ntl - 1 - k);
                mbar_arrive_expect_tx(&bs.full[k & 1], qt_bytes + dob_bytes + 512);
#pragma unroll
                for (int c = 0; c < NL; ++c) {
                    tma_load_4d(dst + c * qchunk, &maps.q, &bs.full[k & 1], c * 64, h, pk, b);
                    tma_load_4d(dst + NL * qchunk + kN * 64 + c * qchunk, &maps.dob, &bs.full[k & 1], c * 64, h, pk, b);
                }
                tma_load_4d(dst + NL * qchunk, &maps.q_r, &bs.full[k & 1], DC, h, pk, b);
                tma_load_3d(dst + stats_off, &maps.lse, &bs.full[k & 1], pk, h, b);
                tma_load_3d(dst + stats_off + 256, &maps.delta, &bs.full[k & 1], pk, h, b);
                loads = k + 1;
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && ntl > 0) {
            const uint32_t id_s = idesc_bf16_f32(kM, kN, false, false);
            const uint32_t id_lat = idesc_bf16_f32(kM, DC, false, true);
            const uint32_t id_rope = idesc_bf16_f32(kM, kDr, false, true);
            const uint32_t k_a = smem_u32(k_s), ring_a = smem_u32(ring);
            const uint64_t kd = sdesc_sw128(k_a, 16, 1024), kr = sdesc_sw64(k_a + NL * kM * 128);
            // dF += dS^T . qt + P^T . [dobar ; 0] of tile t: A = dS^T / P^T [128 x 64]
            // in TMEM, B = the query and dobar tiles MN-major
            auto dk_mma = [&](int t) -> bool {
                if (!waitb(&bs.a_ready, t & 1, bs)) return false;
                tc_fence_after();
                const uint32_t st_a = ring_a + (t & 1) * stage_bytes;
                const uint64_t ql = sdesc_sw128(st_a, qchunk, 1024), qrr = sdesc_sw64_mn(st_a + NL * qchunk);
                const uint64_t dl = sdesc_sw128(st_a + NL * qchunk + kN * 64, qchunk, 1024);
#pragma unroll
                for (int kk = 0; kk < kN / 16; ++kk) {
                    const uint32_t acc = (t > 0 || kk > 0) ? 1u : 0u;
                    umma_bf16_ts(t_dk, t_ds + kk * 8, desc_add(ql, kk * 2048), id_lat, acc);
                    umma_bf16_ts(t_dk + DC, t_ds + kk * 8, desc_add(qrr, kk * 1024), id_rope, acc);
                    umma_bf16_ts(t_dk, t_p + kk * 8, desc_add(dl, kk * 2048), id_lat, 1u);
                }
                umma_commit(&bs.empty[t & 1]);
                umma_commit(&bs.a_free);
                return true;
            };
            if (waitb(&bs.k_full, 0, bs)) {
                bool ok = true;
                for (int k = 0; k < ntl && ok; ++k) {
                    // the accumulating MMAs of tile k - 1 first: they release its ring
                    // stage, so the load of tile k + 1 overlaps this tile's score MMAs
                    // (with two stages, issuing them after S_k would leave every score
                    // MMA waiting for a full load)
                    if (k >= 1 && !(ok = dk_mma(k - 1))) break;
                    if (!(ok = waitb(&bs.full[k & 1], (k >> 1) & 1, bs))) break;
                    if (k >= 1 && !(ok = waitb(&bs.sd_free, (k - 1) & 1, bs))) break;
                    tc_fence_after();
                    const uint32_t st_a = ring_a + (k & 1) * stage_bytes;
                    const uint64_t qd = sdesc_sw128(st_a, 16, 1024), qrd = sdesc_sw64(st_a + NL * qchunk);
                    const uint64_t dd = sdesc_sw128(st_a + NL * qchunk + kN * 64, 16, 1024);
                    // S^T = F . qt^T (K = D), dPa^T = F[0:d_c] . dobar^T (K = d_c)
#pragma unroll
                    for (int c = 0; c < NL; ++c)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_bf16(t_s, desc_add(kd, c * kM * 128 + kk * 32), desc_add(qd, c * qchunk + kk * 32),
                                      id_s, (c | kk) != 0);
#pragma unroll
                    for (int kk = 0; kk < kDr / 16; ++kk)
                        umma_bf16(t_s, desc_add(kr, kk * 32), desc_add(qrd, kk * 32), id_s, 1u);
#pragma unroll
                    for (int c = 0; c < NL; ++c)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_bf16(t_dp, desc_add(kd, c * kM * 128 + kk * 32), desc_add(dd, c * qchunk + kk * 32),
                                      id_s, (c | kk) != 0);
                    umma_commit(&bs.sd_full);
                }
                if (ok && dk_mma(ntl - 1)) umma_commit(&bs.done);
            }
        }
    } else {
        // ------------------------------------------------------------ elementwise warps (2-9)
        const int quarter = warp & 3, hc = (warp - 2) >> 2;
        const int r = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int j = j0 + r;                                  // this lane's slot
        const int first_pos = (j + 1) * p.s;                   // the first query that sees it
        float sv[32], dv[32];
        uint32_t wp[16], wd[16];
        for (int k = 0; k < ntl; ++k) {
            waitb(&bs.sd_full, k & 1, bs);
            tc_fence_after();
            tmem_ld32(t_s + hc * 32 + lane_off, sv);
            tmem_ld32(t_dp + hc * 32 + lane_off, dv);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bs.sd_free);
            // the stage's statistics (TMA): observe its landing here too (the stage
            // is refilled only after this tile's accumulating MMAs, below)
            waitb(&bs.full[k & 1], (k >> 1) & 1, bs);
            const float* st = (const float*)(ring + (k & 1) * stage_bytes + stats_off);
            const int pk = pbase + kN * (ntl - 1 - k) + 32 * hc;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                float p2[2], d2[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int cc = 2 * c + e, pos = pk + cc;
                    const bool vis = pos < p.T && pos >= first_pos;
                    const float lse = st[32 * hc + cc], delta = st[64 + 32 * hc + cc];
                    const float pr = vis ? ex2_approx(fmaf(sv[cc], p.scale_log2, -lse)) : 0.f;
                    p2[e] = pr;
                    d2[e] = p.scale * pr * (dv[cc] - delta);
                }
                wp[c] = pack_bf16x2(p2[0], p2[1]);
                wd[c] = pack_bf16x2(d2[0], d2[1]);
            }
            if (k >= 1) waitb(&bs.a_free, (k - 1) & 1, bs);
            tc_fence_after();
            tmem_st16_u(t_p + hc * 16 + lane_off, wp);
            tmem_st16_u(t_ds + hc * 16 + lane_off, wd);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bs.a_ready);
        }
        constexpr int n_blk = (DC + kDr) / 32, nb0 = (n_blk + 1) / 2;
        if (ntl > 0) waitb(&bs.done, 0, bs);
        tc_fence_after();
        const bool slot_ok = j < p.n_slots;
        float* out = p.dF + (((size_t)h * p.B + b) * p.n_slots + (slot_ok ? j : 0)) * p.D;
        for (int q = hc == 0 ? 0 : nb0; q < (hc == 0 ? nb0 : n_blk); ++q) {
            if (ntl > 0) {
                tmem_ld32(t_dk + q * 32 + lane_off, sv);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) sv[i] = 0.f;
            }
            if (slot_ok && !bs.fail) {
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    *(float4*)(out + q * 32 + 4 * u) = make_float4(sv[4 * u], sv[4 * u + 1], sv[4 * u + 2], sv[4 * u + 3]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (bs.fail) {
        if (warp == 1 && lane == 0) {
            umma_commit(&bs.drain[0]);
            mbar_wait(&bs.drain[0], 0);
        }
        if (warp == 0 && lane == 0) {
            if (loads > 0) mbar_wait(&bs.k_full, 0);
            for (int k = max(0, loads - 2); k < loads; ++k) mbar_wait(&bs.full[k & 1], (k >> 1) & 1);
        }
        if (tid == 0) latch_status(p.status, kStatusTimeout);
        __syncthreads();
    }
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- host side

template <int DC>
constexpr size_t dq_smem() {
    return 1024 + (size_t)(DC / 64) * kM * 128 + kM * 64 + kM * 128 +
           kQStages * ((DC / 64) * kN * 128 + kN * 64 + kN * 128) + ((sizeof(BarsQ) + 15) & ~(size_t)15);
}
template <int DC>
constexpr size_t dk_smem() {
    return 1024 + (size_t)(DC / 64) * kM * 128 + kM * 64 +
           2 * ((((DC / 64) * kN * 128 * 2 + kN * 64 + 512) + 1023) & ~(size_t)1023) +
           ((sizeof(BarsK) + 15) & ~(size_t)15);
}
static_assert(dq_smem<256>() <= 232448 && dk_smem<256>() <= 232448, "one CTA per SM fits");

cudaError_t map_(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* m, const void* base, int rank,
                 const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box, const char* what,
                 CUtensorMapDataType dt, CUtensorMapSwizzle swz) {
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = enc(m, dt, rank, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        char buf[128];
        snprintf(buf, sizeof(buf), "cuTensorMapEncodeTiled(%s) (CUresult %d)", what, (int)r);
        return note_error(buf, cudaErrorInvalidValue);
    }
    return cudaSuccess;
}

template <int DC>
cudaError_t launch(const Shape& sh, const BwdTCInputs& in, const BwdTC& p, cudaStream_t st, uint64_t* launches) {
    auto enc = (PFN_cuTensorMapEncodeTiled_v12000)tensor_map_encoder();
    if (!enc) return note_error("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", cudaErrorNotSupported);
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const auto S128 = CU_TENSOR_MAP_SWIZZLE_128B, S64 = CU_TENSOR_MAP_SWIZZLE_64B;
    const cuuint64_t E = 2, T = p.T, H = sh.H, B = sh.B, D = sh.D, ns = p.n_slots;
    const cuuint64_t dq[4] = {D, H, T, B}, sq[3] = {E * D, E * H * D, E * T * H * D};
    const cuuint64_t dd[4] = {(cuuint64_t)DC, H, T, B}, sd[3] = {E * DC, E * H * DC, E * T * H * DC};
    const cuuint64_t dk[3] = {D, ns, B}, sk[2] = {E * D, E * ns * D};
    const cuuint64_t Tp = stats_pitch(p.T);
    const cuuint64_t ds[3] = {T, H, B}, ss[2] = {4 * Tp, 4 * Tp * H};
    cudaError_t e = cudaSuccess;
    MapsQ mq;
    MapsK mk;
    {
        const cuuint32_t bq[4] = {64, 1, kM, 1}, bqr[4] = {kDr, 1, kM, 1}, bk[3] = {64, kN, 1}, bkr[3] = {kDr, kN, 1};
        if (e == cudaSuccess) e = map_(enc, &mq.q, in.qt, 4, dq, sq, bq, "qt", BF, S128);
        if (e == cudaSuccess) e = map_(enc, &mq.q_r, in.qt, 4, dq, sq, bqr, "qt RoPE", BF, S64);
        const cuuint64_t dh[4] = {(cuuint64_t)kDh, H, T, B}, sh4[3] = {E * kDh, E * H * kDh, E * T * H * kDh};
        const cuuint64_t du[3] = {H * kDh, ns, B}, su[2] = {E * H * kDh, E * ns * H * kDh};
        const cuuint32_t bu[3] = {64, kN, 1};
        if (e == cudaSuccess) e = map_(enc, &mq.dout, in.dout, 4, dh, sh4, bq, "dout", BF, S128);
        if (e == cudaSuccess) e = map_(enc, &mq.u, in.u, 3, du, su, bu, "U", BF, S128);
        if (e == cudaSuccess) e = map_(enc, &mq.k, in.slots, 3, dk, sk, bk, "slots", BF, S128);
        if (e == cudaSuccess) e = map_(enc, &mq.k_r, in.slots, 3, dk, sk, bkr, "slots RoPE", BF, S64);
    }
    {
        const cuuint32_t bk[3] = {64, kM, 1}, bkr[3] = {kDr, kM, 1}, bq[4] = {64, 1, kN, 1}, bqr[4] = {kDr, 1, kN, 1};
        const cuuint32_t bs[3] = {kN, 1, 1};
        if (e == cudaSuccess) e = map_(enc, &mk.k, in.slots, 3, dk, sk, bk, "slots", BF, S128);
        if (e == cudaSuccess) e = map_(enc, &mk.k_r, in.slots, 3, dk, sk, bkr, "slots RoPE", BF, S64);
        if (e == cudaSuccess) e = map_(enc, &mk.q, in.qt, 4, dq, sq, bq, "qt", BF, S128);
        if (e == cudaSuccess) e = map_(enc, &mk.q_r, in.qt, 4, dq, sq, bqr, "qt RoPE", BF, S64);
        if (e == cudaSuccess) e = map_(enc, &mk.dob, in.dob, 4, dd, sd, bq, "dobar", BF, S128);
        if (e == cudaSuccess)
            e = map_(enc, &mk.lse, p.lse, 3, ds, ss, bs, "lse", CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                     CU_TENSOR_MAP_SWIZZLE_NONE);
        if (e == cudaSuccess)
            e = map_(enc, &mk.delta, p.delta, 3, ds, ss, bs, "delta", CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                     CU_TENSOR_MAP_SWIZZLE_NONE);
    }
    if (e != cudaSuccess) return e;
    constexpr size_t sq_bytes = dq_smem<DC>(), sk_bytes = dk_smem<DC>();
    e = cudaFuncSetAttribute(k_bwd_dq_tc<DC>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sq_bytes);
    if (e != cudaSuccess) return note_error("cudaFuncSetAttribute(k_bwd_dq_tc)", e);
    e = cudaFuncSetAttribute(k_bwd_dk_tc<DC>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sk_bytes);
    if (e != cudaSuccess) return note_error("cudaFuncSetAttribute(k_bwd_dk_tc)", e);
    k_bwd_dq_tc<DC><<<p.n_qtiles * sh.B * sh.H, kThreads, sq_bytes, st>>>(mq, p);
    k_bwd_dk_tc<DC><<<p.n_ktiles * sh.B * sh.H, kThreads, sk_bytes, st>>>(mk, p);
    *launches += 2;
    return note_error("backward tensor-core launch", cudaGetLastError());
}

}  // namespace

bool tc_backward_supported(const Shape& sh) {
    return sh.d_h == kDh && sh.d_r == kDr && (sh.d_c == 256 || sh.d_c == 128) && sh.gate_mode <= 2;
}

cudaError_t tc_backward_attention(const Shape& sh, int T, const BwdTCInputs& in, cudaStream_t st,
                                  uint64_t* launches) {
    BwdTC p;
    p.B = sh.B;
    p.T = T;
    p.H = sh.H;
    p.D = sh.D;
    p.s = sh.s;
    p.n_slots = (T + sh.s - 1) / sh.s;
    p.n_qtiles = (T + kM - 1) / kM;
    p.n_ktiles = (p.n_slots + kM - 1) / kM;
    p.scale = sh.scale;
    p.scale_log2 = sh.scale * 1.4426950408889634f;
    p.lse = in.lse;
    p.delta = in.delta;
    p.dqt = in.dqt;
    p.dF = in.dF;
    p.status = in.status;
    return sh.d_c == 256 ? launch<256>(sh, in, p, st, launches) : launch<128>(sh, in, p, st, launches);
}

}  // namespace mtla
