// wait_probe.cu -- a test hook for the bounded-wait path every kernel of the
// library shares: one CTA lands a TMA load on one mbarrier, then waits with a
// caller-chosen limit on a second mbarrier that nothing ever arrives on, so the
// wait runs out. It latches MTLA_ERR_TIMEOUT in the device status word, lets
// its load complete (nothing is left in flight), and returns: the GPU never
// hangs or faults, and the context stays usable for the calls that follow.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "mtla_internal.h"
#include "tc_common.cuh"

namespace mtla {

namespace {

using namespace tc;

__global__ void __launch_bounds__(32, 1) k_wait_probe(const __grid_constant__ CUtensorMap map, uint64_t limit_ns,
                                                      int* status) {
    __shared__ __align__(1024) uint8_t buf[2048];
    __shared__ uint64_t landed, never;
    if (threadIdx.x != 0) return;
    mbar_init(&landed, 1);
    mbar_init(&never, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&landed, 2048);
    tma_load_2d(buf, &map, &landed, 0, 0);
    if (!mbar_wait_for(&never, 0, limit_ns)) {
        latch_status(status, kStatusTimeout);
        mbar_wait(&landed, 0);           // the load in flight lands before the CTA ends
        return;
    }
    mbar_wait(&landed, 0);
}

}  // namespace

cudaError_t wait_probe(uint64_t limit_ns, void* scratch, int* status, cudaStream_t st, uint64_t* launches) {
    auto encode = (PFN_cuTensorMapEncodeTiled_v12000)tensor_map_encoder();
    if (!encode) return note_error("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", cudaErrorNotSupported);
    CUtensorMap map;
    cuuint64_t d[2] = {64, 16};
    cuuint64_t s[1] = {128};
    cuuint32_t b[2] = {64, 16};
    cuuint32_t e[2] = {1, 1};
    CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, scratch, d, s, b, e, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return note_error("cuTensorMapEncodeTiled (wait probe)", cudaErrorInvalidValue);
    k_wait_probe<<<1, 32, 0, st>>>(map, limit_ns, status);
    *launches += 1;
    return note_error("k_wait_probe launch", cudaGetLastError());
}

}  // namespace mtla
