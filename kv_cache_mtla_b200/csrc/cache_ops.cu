// cache_ops.cu -- operations on the slot cache between decode steps.
//
// Beam-search reorder. The authors' toolkit decodes with parallel beam search
// (the toolkit's project page on sourcepulse.org, "Highlighted Details").
// After each step the surviving beams continue from chosen parent beams, so
// every sequence's cache -- its finished and open slots (MTLA Method (1)) and
// the fp32 accumulator of the slot being filled -- must become a copy of its
// parent's:
//   cache_out[b, 0:n) = cache_in[src[b], 0:n),  n = ceil(n_tokens[src[b]] / s)
//   open_out[b]       = open_in[src[b]]
// Only the n slots the parent has filled are copied; the copy is byte exact
// (no rounding). A plain HBM-bound gather: every byte is read once and
// written once, in 16-byte accesses, with streaming cache hints (the cache is
// larger than L2 at the sizes where the copy takes time).
#include <algorithm>

#include "common.cuh"
#include "mtla_internal.h"

namespace mtla {

namespace {

constexpr int kStatusInvalidArg = 1;   // device status word value of MTLA_ERR_INVALID_ARG
constexpr int kReorderThreads = 256;
constexpr int kRowsPerBlock = 16;   // slot rows of one sequence per block
constexpr int kUnroll = 4;          // 16-byte loads in flight per thread before its stores

// grid (ceil(max_slots / kRowsPerBlock), min(B, 65535)); block (x, y) copies
// slot rows [16x, 16x + 16) of destinations b = y, y + gridDim.y, ... (those
// rows below the parent's slot count); blocks with x = 0 also copy the open
// slot. The rows of one sequence are consecutive in memory, so a block's
// rows are one contiguous run of row16 * rows 16-byte units.
__global__ void __launch_bounds__(kReorderThreads)
    k_reorder_cache(const int32_t* __restrict__ src, const int32_t* __restrict__ n_tokens,
                    const uint4* __restrict__ cin, const float* __restrict__ oin, uint4* __restrict__ cout,
                    float* __restrict__ oout, int B, int max_slots, int s, int row16, int D, int* status) {
    for (int b = blockIdx.y; b < B; b += gridDim.y) {
        const int j = src[b];
        if (j < 0 || j >= B) {
            if (blockIdx.x == 0 && threadIdx.x == 0) latch_status(status, kStatusInvalidArg);
            continue;
        }
        const int64_t n_tok = n_tokens[j];
        if (n_tok < 0 || n_tok > (int64_t)max_slots * s) {
            if (blockIdx.x == 0 && threadIdx.x == 0) latch_status(status, kStatusCapacity);
            continue;
        }
        if (blockIdx.x == 0)
            for (int e = threadIdx.x; e < D; e += blockDim.x) oout[(size_t)b * D + e] = oin[(size_t)j * D + e];
        const int n_slots = (int)((n_tok + s - 1) / s);
        const int r0 = blockIdx.x * kRowsPerBlock;
        const int rows = min(kRowsPerBlock, n_slots - r0);
        if (rows <= 0) continue;
        const uint4* from = cin + ((size_t)j * max_slots + r0) * row16;
        uint4* to = cout + ((size_t)b * max_slots + r0) * row16;
        const int n16 = rows * row16;
        for (int e0 = threadIdx.x; e0 < n16; e0 += kUnroll * kReorderThreads) {
            uint4 v[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int e = e0 + u * kReorderThreads;
                if (e < n16) v[u] = __ldcs(from + e);
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int e = e0 + u * kReorderThreads;
                if (e < n16) __stcs(to + e, v[u]);
            }
        }
    }
}

}  // namespace

cudaError_t reorder_cache(const Shape& sh, size_t elem_bytes, const int32_t* src, const int32_t* n_tokens,
                          const void* cache_in, const float* open_in, void* cache_out, float* open_out,
                          int* status, cudaStream_t st, uint64_t* launches) {
    const int row16 = (int)((size_t)sh.D * elem_bytes / 16);   // D % 16 == 0, so whole 16-byte units
    const dim3 grid((unsigned)((sh.max_slots + kRowsPerBlock - 1) / kRowsPerBlock),
                    (unsigned)std::min(sh.B, 65535));
    k_reorder_cache<<<grid, kReorderThreads, 0, st>>>(src, n_tokens, (const uint4*)cache_in, open_in,
                                                       (uint4*)cache_out, open_out, sh.B, sh.max_slots, sh.s,
                                                       row16, sh.D, status);
    *launches += 1;
    return note_error("k_reorder_cache launch", cudaGetLastError());
}

}  // namespace mtla
