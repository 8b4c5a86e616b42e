// Failure-detection self-test of the bounded waits.
//
// Every mbarrier wait in the library's kernels is bounded in wall time: a wait
// that runs out raises the timeout device flag, sets the CTA's abort flag and
// returns, so the kernel ends and the CUDA context stays usable.  This kernel
// exercises exactly that path without faulting anything: one thread waits,
// through the same bounded wait the kernels use, on a barrier that nothing
// ever completes, with a short limit.
#include "qlora_internal.cuh"
#include "tc_ptx.cuh"

namespace qlora {
namespace {

__global__ void bounded_wait_probe(uint64_t limit_ns, uint32_t* err, uint32_t* result) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x != 0) return;
    const uint32_t b = ptx::smem_addr(&bar);
    ptx::mbar_init(b, 1);                                     // one arrival expected, none will come
    abort_flag = 0;
    ptx::fence_barrier_init();
    volatile int* abort = &abort_flag;
    const bool completed = ptx::mbar_wait(b, 0, abort, err, limit_ns);
    result[0] = completed ? 1u : 0u;
    result[1] = (uint32_t)*abort;
}

}  // namespace

qlora_status launch_bounded_wait_probe(uint64_t limit_ns, uint32_t* result, cudaStream_t s) {
    uint32_t* err = device_error_word();
    if (!err) return QLORA_ERR_CUDA;
    bounded_wait_probe<<<1, 32, 0, s>>>(limit_ns, err, result);
    QLORA_CHECK_LAUNCH();
    return QLORA_OK;
}

}  // namespace qlora
