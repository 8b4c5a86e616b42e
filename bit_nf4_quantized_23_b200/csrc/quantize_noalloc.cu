// NF4 + Double Quantization without a caller-supplied workspace.
//
// Some callers cannot allocate device memory at the point where they quantize:
// for example a plugin whose host framework owns every device allocation and
// hands the plugin only its input and output pointers, or a latency-critical
// path where a cudaMalloc/cudaFree (which may synchronize the device) is not
// acceptable.  qlora_quantize_nf4_dq_noalloc serves them: it runs the same
// kernels as qlora_quantize_nf4_dq, but its scratch (the fp32 block absmax
// values and the fp64 partial sums of the mean) lives in the static device
// array below, which is part of the library image.  Every GPU that loads the
// library holds this array until the process exits.
//
// Limits and sharing:
//  - At most kNoAllocMaxWeights weights per call (for example W[8192,8192]);
//    larger tensors get QLORA_ERR_TOO_LARGE and nothing is launched.
//  - Every call shares the one array of its device and it keeps the last
//    call's contents.  The quantize kernels overwrite every scratch word they
//    read before reading it, so nothing has to start at zero.  Calls that
//    overlap on the GPU (different streams, or different host threads on the
//    same device without ordering) race on the array and give wrong results.
//  - The first call on a device looks up the device address of the array with
//    cudaGetSymbolAddress (once per device, with that device current).  Make
//    that first call before any stream capture.
#include <mutex>

#include "qlora_internal.cuh"
#include "timing.cuh"

namespace qlora {

size_t quantize_workspace_bytes(int64_t nb1);
qlora_status launch_quantize(const void* W, int64_t N, int64_t K, const qlora_nf4_weight* out,
                             void* workspace, cudaStream_t stream);

namespace {

constexpr int64_t kNoAllocMaxWeights = int64_t(1) << 26;          // 67,108,864
constexpr size_t kNoAllocScratchBytes = (size_t(1) << 22) + (size_t(3) << 18);   // 4.75 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Host-side lookup of the array's device address, once per device.
void* scratch_address(qlora_status* st) {
    static std::mutex mu;
    static void* addr[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        *st = QLORA_ERR_CUDA;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            (void)cudaGetLastError();
            *st = QLORA_ERR_CUDA;
            return nullptr;
        }
        addr[dev] = p;
    }
    *st = QLORA_OK;
    return addr[dev];
}

}  // namespace
}  // namespace qlora

extern "C" qlora_status qlora_quantize_nf4_dq_noalloc(const void* W, int64_t N, int64_t K,
                                                      int32_t blocksize, int32_t blocksize2,
                                                      const qlora_nf4_weight* out, void* stream) {
    using namespace qlora;
    // the same checks as qlora_quantize_nf4_dq, with the size limit ahead of the pointer checks
    QLORA_TRY(check_blocks(blocksize, blocksize2));
    if (N < 1 || K < 1 || K % 64 != 0) return QLORA_ERR_SHAPE;
    if (N > kNoAllocMaxWeights / K) return QLORA_ERR_TOO_LARGE;
    QLORA_TRY(check_shape(N, K));
    QLORA_TRY(check_dev(W));
    QLORA_TRY(check_weight(out));
    if (out->N != N || out->K != K) return QLORA_ERR_SHAPE;
    if (quantize_workspace_bytes(N * K / 64) > kNoAllocScratchBytes) return QLORA_ERR_TOO_LARGE;
    qlora_status st = QLORA_OK;
    void* scratch = scratch_address(&st);
    if (st != QLORA_OK) return st;
    TimerScope t(QLORA_TIMER_QUANTIZE, static_cast<cudaStream_t>(stream));
    return launch_quantize(W, N, K, out, scratch, static_cast<cudaStream_t>(stream));
}
