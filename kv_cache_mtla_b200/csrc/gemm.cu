// gemm.cu -- the dense projections around the MTLA path on the tensor cores:
// y[M, N] = x[M, K] . W[N, K]^T with bf16 operands, fp32 accumulation in TMEM
// and a bf16 result ("Multi-head Temporal Latent Attention", Method: the layer
// keeps MLA's low-rank compression, the input h_t projected to the shared
// latent c_t, the decoupled key and the queries, and the attention output
// projected back by W_O; "Multi-Head Latent Attention and Sparse Indexers",
// "Latent attention changes the representation").
//
// Persistent kernel, one CTA per SM walking output tiles of 128 x BN:
//   warp 0     TMA producer: x and W tiles of 64 columns of K (128-byte rows,
//              128-byte swizzle) into a ring of kStages stages
//   warp 1     MMA issue (M = 128, N = BN, K = 16 per instruction), TMEM owner
//   warps 2-5  epilogue: TMEM -> registers -> bf16 -> global, one lane quarter
//              each, while the MMAs of the next tile run into the other of
//              two TMEM accumulators
// Rows of x past M, rows of W past N and columns past K read as zero; the
// epilogue writes only inside [M, N). A batch of such products (the heads of
// a per-head projection) runs as one launch: x and W are 3-D tensor maps with
// the batch index as one coordinate, and y advances by a batch stride.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdio>

#include "common.cuh"
#include "mtla_internal.h"
#include "tc_common.cuh"

namespace mtla {

namespace {

using namespace tc;

constexpr int kBM = 128, kBK = 64;
constexpr int kGemmThreads = 192;

struct GemmArgs {
    int M, N, K, ldc;
    int tiles_n, tiles_mn, n_tiles;
    int x_batch_dim, w_batch_dim;   // which tensor-map coordinate (1 or 2) is the batch index
    size_t y_batch;                 // elements between the batch's outputs
    int out_f32;                    // y is float (else bf16)
    void* y;
    int* status;
};

// coordinates (k, rows, batch) in the map's dimension order
__device__ __forceinline__ void gemm_load(void* dst, const CUtensorMap* m, uint64_t* bar, int k, int row, int bt,
                                          int batch_dim) {
    if (batch_dim == 1) tma_load_3d(dst, m, bar, k, bt, row);
    else tma_load_3d(dst, m, bar, k, row, bt);
}

template <int BN>
struct GemmCfg {
    static constexpr uint32_t a_bytes = kBM * kBK * 2;            // 16 KB
    static constexpr uint32_t b_bytes = BN * kBK * 2;             // 8 / 16 / 32 KB
    static constexpr uint32_t stage_bytes = a_bytes + b_bytes;
    static constexpr int stages = (200 * 1024) / stage_bytes > 8 ? 8 : (200 * 1024) / stage_bytes;
    static constexpr uint32_t smem = 1024 + stages * stage_bytes + 256;
};

template <int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    k_gemm(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w, const GemmArgs g) {
    using C = GemmCfg<BN>;
    constexpr int S = C::stages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t* full = (uint64_t*)(smem + S * C::stage_bytes);
    uint64_t* empty = full + S;
    uint64_t* acc_full = empty + S;        // [2]: a tile's MMAs are done
    uint64_t* acc_empty = acc_full + 2;    // [2]: the epilogue has read the accumulator
    uint64_t* drain = acc_empty + 2;       // MMAs in flight when a wait gave up
    uint32_t* tmem_slot = (uint32_t*)(drain + 1);
    volatile int* fail = (volatile int*)(tmem_slot + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int kb_n = (g.K + kBK - 1) / kBK;
    if (tid == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 4);
        }
        mbar_init(drain, 1);
        *fail = 0;
        fence_mbar_init();
        tma_prefetch_desc(&map_x);
        tma_prefetch_desc(&map_w);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 2 * BN >= 32 ? 2 * BN : 32);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
        if (*fail) return false;
        if (mbar_wait(bar, parity)) return true;
        *fail = 1;
        return false;
    };
    if (warp == 0) {
        if (lane == 0) {
            int it = 0;
            for (int t = blockIdx.x; t < g.n_tiles && !*fail; t += gridDim.x) {
                const int bt = t / g.tiles_mn, tr = t % g.tiles_mn;
                const int m0 = (tr / g.tiles_n) * kBM, n0 = (tr % g.tiles_n) * BN;
                for (int kb = 0; kb < kb_n; ++kb, ++it) {
                    const int st = it % S;
                    if (it >= S && !wait(&empty[st], ((it / S) - 1) & 1)) break;
                    uint8_t* dst = smem + (size_t)st * C::stage_bytes;
                    mbar_arrive_expect_tx(&full[st], C::stage_bytes);
                    gemm_load(dst, &map_x, &full[st], kb * kBK, m0, bt, g.x_batch_dim);
                    gemm_load(dst + C::a_bytes, &map_w, &full[st], kb * kBK, n0, bt, g.w_batch_dim);
                }
            }
            if (*fail)
                for (int k = max(0, it - S); k < it; ++k) mbar_wait(&full[k % S], (k / S) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(kBM, BN, false, false);
            int it = 0, i = 0;
            for (int t = blockIdx.x; t < g.n_tiles; t += gridDim.x, ++i) {
                const int a = i & 1;
                if (i >= 2 && !wait(&acc_empty[a], ((i >> 1) - 1) & 1)) break;
                tc_fence_after();
                const uint32_t d = tmem + a * BN;
                bool ok = true;
                for (int kb = 0; kb < kb_n; ++kb, ++it) {
                    const int st = it % S;
                    if (!(ok = wait(&full[st], (it / S) & 1))) break;
                    tc_fence_after();
                    const uint32_t base = smem_u32(smem + (size_t)st * C::stage_bytes);
                    const uint64_t ad = sdesc_sw128(base, 16, 1024), bd = sdesc_sw128(base + C::a_bytes, 16, 1024);
                    umma_bf16(d, ad, bd, idesc, kb > 0 ? 1u : 0u);
                    umma_bf16(d, desc_add(ad, 32), desc_add(bd, 32), idesc, 1u);
                    umma_bf16(d, desc_add(ad, 64), desc_add(bd, 64), idesc, 1u);
                    umma_bf16(d, desc_add(ad, 96), desc_add(bd, 96), idesc, 1u);
                    umma_commit(&empty[st]);
                }
                if (!ok) break;
                umma_commit(&acc_full[a]);
            }
            if (*fail) {
                umma_commit(drain);
                mbar_wait(drain, 0);
            }
        }
    } else {
        // epilogue: warps 2-5, lane quarter q = warp mod 4 (rows q*32 + lane)
        const int q = warp & 3;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        int i = 0;
        for (int t = blockIdx.x; t < g.n_tiles; t += gridDim.x, ++i) {
            const int a = i & 1;
            const bool ok = wait(&acc_full[a], (i >> 1) & 1);
            tc_fence_after();
            const int bt = t / g.tiles_mn, tr = t % g.tiles_mn;
            const int m0 = (tr / g.tiles_n) * kBM, n0 = (tr % g.tiles_n) * BN;
            const int row = m0 + q * 32 + lane;
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 32) {
                float v[32];
                tmem_ld32(tmem + a * BN + c0 + lane_off, v);
                tmem_wait_ld();
                const int nvalid = g.N - (n0 + c0);
                const size_t off = (size_t)bt * g.y_batch + (size_t)row * g.ldc + n0 + c0;
                if (ok && row < g.M && g.out_f32) {
                    float* dst = (float*)g.y + off;
                    if (nvalid >= 32 && ((((uintptr_t)dst) & 15) == 0)) {
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            *(float4*)(dst + 4 * u) = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
                    } else {
                        for (int cc = 0; cc < 32 && cc < nvalid; ++cc) dst[cc] = v[cc];
                    }
                } else if (ok && row < g.M) {
                    bf16* dst = (bf16*)g.y + off;
                    if (nvalid >= 32 && ((((uintptr_t)dst) & 15) == 0)) {
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            *(uint4*)(dst + 8 * u) =
                                make_uint4(pack_bf16x2(v[8 * u], v[8 * u + 1]), pack_bf16x2(v[8 * u + 2], v[8 * u + 3]),
                                           pack_bf16x2(v[8 * u + 4], v[8 * u + 5]), pack_bf16x2(v[8 * u + 6], v[8 * u + 7]));
                    } else {
                        for (int cc = 0; cc < 32 && cc < nvalid; ++cc) dst[cc] = __float2bfloat16_rn(v[cc]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[a]);
            if (!ok) break;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (*fail) {
        if (tid == 0) latch_status(g.status, kStatusTimeout);
    }
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 2 * BN >= 32 ? 2 * BN : 32);
}

template <int BN>
cudaError_t gemm_launch(const CUtensorMap& mx, const CUtensorMap& mw, const GemmArgs& g, cudaStream_t st) {
    static size_t done[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (done[dev] < GemmCfg<BN>::smem) {
        cudaError_t e = cudaFuncSetAttribute(k_gemm<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)GemmCfg<BN>::smem);
        if (e != cudaSuccess) return note_error("cudaFuncSetAttribute(k_gemm)", e);
        done[dev] = GemmCfg<BN>::smem;
    }
    const int grid = std::min(g.n_tiles, sm_count());
    k_gemm<BN><<<grid, kGemmThreads, GemmCfg<BN>::smem, st>>>(mx, mw, g);
    return note_error("k_gemm launch", cudaGetLastError());
}

}  // namespace

cudaError_t gemm_batched(const GemmOperand& x, const GemmOperand& w, void* y, int ldy, size_t y_batch, bool y_f32,
                         int M, int N, int K, int batch, int* status, cudaStream_t st, uint64_t* launches) {
    auto encode = (PFN_cuTensorMapEncodeTiled_v12000)tensor_map_encoder();
    if (!encode) return note_error("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", cudaErrorNotSupported);
    const int BN = N <= 64 ? 64 : (N <= 128 ? 128 : 256);
    // 3-D map of one operand: (K, rows, batch) when the batch stride exceeds the
    // row pitch, else (K, batch, rows), so that the strides grow with the dimension
    auto make = [&](CUtensorMap* m, const GemmOperand& o, int rows, int box_rows, int* batch_dim,
                    const char* what) -> cudaError_t {
        const bool rows_first = o.batch_stride >= (size_t)o.ld * rows || batch == 1;
        *batch_dim = rows_first ? 2 : 1;
        cuuint64_t d[3], s[2];
        d[0] = (cuuint64_t)K;
        if (rows_first) {
            d[1] = (cuuint64_t)rows;
            d[2] = (cuuint64_t)batch;
            s[0] = (cuuint64_t)o.ld * 2;
            s[1] = (cuuint64_t)(batch == 1 ? (size_t)o.ld * rows : o.batch_stride) * 2;
        } else {
            d[1] = (cuuint64_t)batch;
            d[2] = (cuuint64_t)rows;
            s[0] = (cuuint64_t)o.batch_stride * 2;
            s[1] = (cuuint64_t)o.ld * 2;
        }
        const cuuint32_t bx[3] = {kBK, rows_first ? (cuuint32_t)box_rows : 1u, rows_first ? 1u : (cuuint32_t)box_rows};
        const cuuint32_t e[3] = {1, 1, 1};
        CUresult r = encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(o.p), d, s, bx, e,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            char buf[96];
            snprintf(buf, sizeof(buf), "cuTensorMapEncodeTiled (gemm %s, CUresult %d)", what, (int)r);
            return note_error(buf, cudaErrorInvalidValue);
        }
        return cudaSuccess;
    };
    GemmArgs g;
    CUtensorMap mx, mw;
    cudaError_t e = make(&mx, x, M, kBM, &g.x_batch_dim, "x");
    if (e == cudaSuccess) e = make(&mw, w, N, BN, &g.w_batch_dim, "w");
    if (e != cudaSuccess) return e;
    g.M = M;
    g.N = N;
    g.K = K;
    g.ldc = ldy;
    g.tiles_n = (N + BN - 1) / BN;
    g.tiles_mn = ((M + kBM - 1) / kBM) * g.tiles_n;
    g.n_tiles = g.tiles_mn * batch;
    g.y_batch = y_batch;
    g.out_f32 = y_f32 ? 1 : 0;
    g.y = y;
    g.status = status;
    *launches += 1;
    if (BN == 64) return gemm_launch<64>(mx, mw, g, st);
    if (BN == 128) return gemm_launch<128>(mx, mw, g, st);
    return gemm_launch<256>(mx, mw, g, st);
}

cudaError_t gemm_bf16(const void* x, int ldx, const void* w, int ldw, void* y, int ldy, int M, int N, int K,
                      int* status, cudaStream_t st, uint64_t* launches) {
    return gemm_batched(GemmOperand{x, ldx, 0}, GemmOperand{w, ldw, 0}, y, ldy, 0, false, M, N, K, 1, status, st,
                        launches);
}

}  // namespace mtla
