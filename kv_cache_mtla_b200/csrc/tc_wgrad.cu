// tc_wgrad.cu -- the weight gradients of the training backward on the tensor
// cores. With m running over the B*T token rows of one head h,
//   dW_UK[h] = sum_m qC[m, h, :]^T g[m, h, :]        g: the rows' latent query gradients
//   dW_UV[h] = sum_m dout[m, h, :]^T obar[m, h, :]   obar = O / l of the forward
// ("Multi-head Temporal Latent Attention", Method (2)-(3): the absorbed query
// is W_UK^T applied to qC and the output W_UV applied to the weighted latent,
// so these are the two products' weight gradients).
//
// One CTA per (chunk of 128-row tiles, head, product) accumulates
//   D^T [d_c x d_h] += Y^T [d_c x 128 rows] . X [128 rows x d_h]
// tile by tile in tensor memory (M = 128 latent columns per half, N = d_h =
// 64, K = 16 token rows per instruction). Both operands are TMA tiles of 128
// token rows in the 128-byte swizzle, read MN-major: Y = g or obar in 64-column
// chunks, X = qC or dout. The chunk's partial goes to part[chunk][h][r][c];
// the chunks are added in order afterwards, so the result does not depend on
// the schedule. Warp 0 loads (two ring stages), warp 1 issues the MMAs, all
// four warps write the partial.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdio>

#include "common.cuh"
#include "mtla_internal.h"
#include "tc_common.cuh"

namespace mtla {

namespace {

using namespace tc;

constexpr int kRows = 128;       // token rows per tile: the K extent of one ring stage
constexpr int kDh = 64;          // d_h of the compiled instances (N of every MMA)
constexpr int kStages = 2;
constexpr int kThreads = 128;

struct WgArgs {
    int H, n_tiles, tiles_per_chunk;
    float* part[2];              // [chunk][H][d_h][d_c]: dW_UK parts, dW_UV parts
    int* status;
};

struct WgMaps {
    CUtensorMap y[2];            // g, obar  (d_c, H, M)  box (64, 1, 128)
    CUtensorMap x[2];            // qC, dout (d_h, H, M)  box (64, 1, 128)
};

template <int DC>
constexpr uint32_t wg_stage_bytes() { return (uint32_t)(DC / 64 + 1) * kRows * 128; }

template <int DC>
__global__ void __launch_bounds__(kThreads, 1) k_wgrad_tc(const __grid_constant__ WgMaps maps, const WgArgs p) {
    constexpr int NL = DC / 64;                          // 64-column chunks of Y
    constexpr uint32_t chunk = kRows * 128;              // one [128 rows x 64 columns] chunk
    constexpr uint32_t stage_bytes = wg_stage_bytes<DC>();
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t* full = (uint64_t*)(smem + kStages * stage_bytes);
    uint64_t* empty = full + kStages;
    uint64_t* done = empty + kStages;
    uint32_t* tmem_slot = (uint32_t*)(done + 1);
    volatile int* fail = (volatile int*)(tmem_slot + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ci = blockIdx.x, h = blockIdx.y, which = blockIdx.z;
    const int t0 = ci * p.tiles_per_chunk;
    const int n = min(t0 + p.tiles_per_chunk, p.n_tiles) - t0;   // >= 1 (the grid covers the tiles exactly)

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init(done, 1);
        *fail = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t t_d = *tmem_slot;                     // D^T half mh in columns [64 mh, 64 mh + 64)

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------------------ TMA producer
        tma_prefetch_desc(&maps.y[which]);
        tma_prefetch_desc(&maps.x[which]);
        int issued = 0;
        for (int k = 0; k < n; ++k) {
            const int st = k % kStages;
            if (k >= kStages && !mbar_wait(&empty[st], ((k / kStages) - 1) & 1)) {
                *fail = 1;
                break;
            }
            uint8_t* dst = smem + st * stage_bytes;
            const int m = (t0 + k) * kRows;              // rows past B*T read as zeros
            mbar_arrive_expect_tx(&full[st], stage_bytes);
#pragma unroll
            for (int c = 0; c < NL; ++c) tma_load_3d(dst + c * chunk, &maps.y[which], &full[st], c * 64, h, m);
            tma_load_3d(dst + NL * chunk, &maps.x[which], &full[st], 0, h, m);
            issued = k + 1;
        }
        if (*fail) {
            // the copies in flight land before shared memory is released
            for (int k = max(0, issued - kStages); k < issued; ++k) mbar_wait(&full[k % kStages], (k / kStages) & 1);
        }
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------------------ MMA issue
        const uint32_t idesc = idesc_f32<bf16>(128, kDh, true, true);
        for (int k = 0; k < n && !*fail; ++k) {
            const int st = k % kStages;
            if (!mbar_wait(&full[st], (k / kStages) & 1)) {
                *fail = 1;
                break;
            }
            tc_fence_after();
            const uint32_t base = smem_u32(smem + st * stage_bytes);
            // B = X [128 rows x 64] MN-major (one 64-column chunk); A = Y^T, the
            // latent columns as M in two 64-column chunks per half
            const uint64_t bd = sdesc_sw128(base + NL * chunk, chunk, 1024);
#pragma unroll
            for (int mh = 0; mh < NL / 2; ++mh) {
                const uint64_t ad = sdesc_sw128(base + mh * 2 * chunk, chunk, 1024);
#pragma unroll
                for (int kk = 0; kk < kRows / 16; ++kk)
                    umma_bf16(t_d + mh * kDh, desc_add(ad, kk * 2048), desc_add(bd, kk * 2048), idesc,
                              (k | kk) != 0 ? 1u : 0u);
            }
            umma_commit(&empty[st]);                     // the stage may take the next tile
        }
        umma_commit(done);                               // every MMA issued above has completed
    }
    __syncwarp();

    // ---------------------------------------------------------------- the partial
    // warp w reads TMEM lanes 32 w .. 32 w + 31, i.e. latent columns
    // c = 128 mh + 32 w + lane; a warp's stores of one r are 32 consecutive c
    const bool got = mbar_wait(done, 0);
    tc_fence_after();
    float* part = (which ? p.part[1] : p.part[0]) + ((size_t)ci * p.H + h) * kDh * DC;
#pragma unroll 1
    for (int mh = 0; mh < NL / 2; ++mh) {
        float v[64];
        const uint32_t ta = t_d + mh * kDh + ((uint32_t)(warp * 32) << 16);
        tmem_ld32(ta, v);
        tmem_ld32(ta + 32, v + 32);
        tmem_wait_ld();
        const int c = mh * 128 + warp * 32 + lane;
        if (got && !*fail) {
#pragma unroll
            for (int r = 0; r < kDh; ++r) part[(size_t)r * DC + c] = v[r];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && (!got || *fail)) latch_status(p.status, kStatusTimeout);
    tc_fence_after();
    if (warp == 0) tmem_dealloc(t_d, 128);
}

cudaError_t wg_map(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* m, const void* base, int cols, int H, int M,
                   const char* what) {
    const cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)H, (cuuint64_t)M};
    const cuuint64_t strides[2] = {(cuuint64_t)cols * 2, (cuuint64_t)H * cols * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)kRows};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        char buf[128];
        snprintf(buf, sizeof(buf), "cuTensorMapEncodeTiled(weight gradients, %s) (CUresult %d)", what, (int)r);
        return note_error(buf, cudaErrorInvalidValue);
    }
    return cudaSuccess;
}

}  // namespace

int tc_weight_chunks(const Shape& sh, int M, int max_chunks) {
    const int n_tiles = (M + kRows - 1) / kRows;
    // about four CTAs per SM over both products and all heads, at least 8 tiles a chunk
    const int target = std::max(1, (4 * sm_count() + 2 * sh.H - 1) / (2 * sh.H));
    int per = std::max(8, (n_tiles + target - 1) / target);
    int nc = (n_tiles + per - 1) / per;
    while (nc > max_chunks) {
        ++per;
        nc = (n_tiles + per - 1) / per;
    }
    return nc;
}

cudaError_t tc_weight_parts(const Shape& sh, int M, const void* qc, const void* g, const void* dout,
                            const void* obar, float* part_k, float* part_v, int n_chunks, int* status,
                            cudaStream_t st) {
    if (sh.d_h != kDh || (sh.d_c != 128 && sh.d_c != 256) || M <= 0 || n_chunks <= 0)
        return note_error("tc_weight_parts: d_h = 64, d_c = 128 or 256", cudaErrorInvalidValue);
    auto enc = (PFN_cuTensorMapEncodeTiled_v12000)tensor_map_encoder();
    if (!enc) return note_error("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", cudaErrorNotSupported);
    WgMaps maps;
    cudaError_t e = wg_map(enc, &maps.y[0], g, sh.d_c, sh.H, M, "g");
    if (e == cudaSuccess) e = wg_map(enc, &maps.y[1], obar, sh.d_c, sh.H, M, "obar");
    if (e == cudaSuccess) e = wg_map(enc, &maps.x[0], qc, kDh, sh.H, M, "qC");
    if (e == cudaSuccess) e = wg_map(enc, &maps.x[1], dout, kDh, sh.H, M, "dout");
    if (e != cudaSuccess) return e;
    WgArgs p;
    p.H = sh.H;
    p.n_tiles = (M + kRows - 1) / kRows;
    p.tiles_per_chunk = (p.n_tiles + n_chunks - 1) / n_chunks;
    if ((p.n_tiles + p.tiles_per_chunk - 1) / p.tiles_per_chunk != n_chunks)
        return note_error("tc_weight_parts: chunk count does not cover the tiles exactly", cudaErrorInvalidValue);
    p.part[0] = part_k;
    p.part[1] = part_v;
    p.status = status;
    auto kern = sh.d_c == 256 ? k_wgrad_tc<256> : k_wgrad_tc<128>;
    const size_t smem = 1024 + (size_t)kStages * (sh.d_c == 256 ? wg_stage_bytes<256>() : wg_stage_bytes<128>()) + 64;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return note_error("cudaFuncSetAttribute(k_wgrad_tc)", e);
    kern<<<dim3(n_chunks, sh.H, 2), kThreads, smem, st>>>(maps, p);
    return note_error("k_wgrad_tc launch", cudaGetLastError());
}

}  // namespace mtla
