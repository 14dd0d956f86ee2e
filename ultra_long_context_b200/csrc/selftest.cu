// selftest.cu -- hsa_selftest_bounded_wait: runs the error path of the kernels' bounded device waits.
//
// Every kernel of the library waits on mbarriers (TMA copies landing, tensor-core products completing,
// one warp role handing a buffer to another) with a bounded number of probes. A wait that runs out
// records the failure in the status flag at the start of the call's workspace, lets the kernel unwind
// (its own copies finish, its TMEM is freed) and returns; hsa_workspace_status() then reports
// HSA_ERR_TIMEOUT. In a healthy run no wait ever runs out, so this entry point makes one run out on
// purpose, safely: one warp allocates TMEM as the operator kernels do, waits with the same helper on
// an mbarrier whose single expected arrival is never made (a short probe limit instead of the
// kernels' seconds-long one), records the timeout exactly as they do, frees its TMEM and exits. No
// copy is in flight, nothing faults, and the context stays usable.
#include "../../include/hsa.h"
#include "launch.h"
#include "tc.cuh"

namespace {

__global__ void __launch_bounds__(32) bounded_wait_selftest_kernel(int32_t *err, unsigned probes) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t tmem_slot;
    const uint32_t mbar = hsa::smem_u32(&bar);
    hsa::tc::tmem_alloc(hsa::smem_u32(&tmem_slot), 32);  // the whole warp, as the operator kernels do
    if (threadIdx.x == 0) {
        hsa::tc::mbar_init(mbar, 1);  // one arrival expected; none is ever made
        hsa::tc::fence_mbar_init();
    }
    hsa::tc::fence_before();
    __syncwarp();
    hsa::tc::fence_after();
    const uint32_t tmem = tmem_slot;
    bool ok = true;
    if (threadIdx.x == 0) ok = hsa::tc::mbar_wait_n(mbar, 0, probes);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    if (!ok && threadIdx.x == 0) atomicOr(err, 1);  // the operator kernels' error record
    hsa::tc::fence_before();
    __syncwarp();
    hsa::tc::fence_after();
    hsa::tc::tmem_dealloc(tmem, 32);
}

}  // namespace

extern "C" hsa_status hsa_selftest_bounded_wait(void *workspace, size_t workspace_bytes, unsigned probes,
                                                void *stream) {
    hsa::set_last_error("");
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < 256) {
        hsa::set_last_error("hsa_selftest_bounded_wait: workspace must be non-NULL, 256-byte aligned, >= 256 bytes");
        return HSA_ERR_WORKSPACE;
    }
    if (probes < 1 || probes > (1u << 20)) {
        hsa::set_last_error("hsa_selftest_bounded_wait: probes must be in [1, 2^20]");
        return HSA_ERR_INVALID_ARG;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t *err = static_cast<int32_t *>(workspace);
    // like every operator call: the flag is cleared first, so a status query reports this call
    cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int32_t), s);
    if (e == cudaSuccess) {
        bounded_wait_selftest_kernel<<<1, 32, 0, s>>>(err, probes);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) {
        hsa::set_last_error(cudaGetErrorString(e));
        return HSA_ERR_CUDA;
    }
    return HSA_OK;
}
