// Internal declarations shared by the translation units of libqlora.so.
// Device helpers here use only IEEE basic operations with explicit rounding
// (__fmul_rn, __fadd_rn, __fdiv_rn, __float2bfloat16_rn) so that no FMA
// contraction or approximate division changes a bit-exact result.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include <utility>

#include "../../include/qlora.h"

namespace qlora {

// NF4 code values (ascending) and the 15 decision thresholds, passed to
// kernels by value (they land in the kernel-parameter constant bank).
struct NF4Tables {
    float q[16];
    float t[15];
};

// Bucketed code search for the quantize kernel.  For x in [-1, 1] the bucket
// is k = RNE(64*x + 64) in [0, 128] (one FMA with a round-to-integer magic
// constant).  Every gap between decision thresholds exceeds the bucket width
// 1/64, so a bucket holds at most one threshold and
//     code(x) = base[k] + (x > thr[k]),   thr[k] = +inf when the bucket has none.
constexpr int kCodeBuckets = 129;
struct QuantBuckets {
    float2 e[kCodeBuckets];   // (.x = threshold, .y = base code as int bits)
};

// Host side: the tables of a codebook (qlora_codebook), built once (codebook.cu).
const NF4Tables& host_tables(int codebook = QLORA_CODEBOOK_NF4);
const QuantBuckets& host_buckets(int codebook = QLORA_CODEBOOK_NF4);

// Host side: count of kernels launched by this library (api.cu).
void note_launches(int n);

// Host side: argument checks of the entry points (api.cu).  Each returns QLORA_OK or the status
// the entry point reports: blocksizes (UNSUPPORTED), shape (SHAPE), a weight descriptor (pointers,
// alignment, codebook, compute dtype), a device pointer (non-null, 16-byte aligned).
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
qlora_status check_blocks(int32_t bs, int32_t bs2);
qlora_status check_shape(int64_t N, int64_t K);
qlora_status check_weight(const qlora_nf4_weight* w);
qlora_status check_dev(const void* p);

// Device error flag word (one per device that loaded the library).  Kernels in
// quantize.cu set it directly; other kernels get its address as an argument.
enum : uint32_t { ERR_FLAG_TIMEOUT = 1u, ERR_FLAG_NONFINITE = 2u, ERR_FLAG_BOUNDS = 4u };

// Host side: when the environment variable QLORA_SYNC_CHECK is set, every
// library launch is followed by a device synchronization and a failing kernel
// is named on stderr (debugging aid; off by default).
bool sync_check_enabled();
bool sync_check(const char* kernel);

// Host side: device address of the error word of the current device (cached
// per device; nullptr on failure).
uint32_t* device_error_word();

// Bounded mbarrier/flag waits give up after this many polls (well above any
// legitimate wait, far below a GPU hang).
constexpr uint32_t kSpinLimit = 1u << 26;

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) {
    return __uint_as_float(b << 16);
}

__device__ __forceinline__ uint32_t f32_to_bf16_bits_rn(float x) {
    __nv_bfloat16 h = __float2bfloat16_rn(x);
    return (uint32_t)(*reinterpret_cast<unsigned short*>(&h));
}

// Two fp32 -> packed bf16x2 (low half = a), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2_rn(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

// The 16-bit compute types: bf16 (the default) or IEEE fp16, chosen per weight
// (a warp-uniform flag in the kernels).  Round to nearest even in both.
__device__ __forceinline__ uint32_t f32_to_f16_bits_rn(float x) {
    return (uint32_t)__half_as_ushort(__float2half_rn(x));
}
__device__ __forceinline__ float f16_bits_to_f32(uint32_t b) {
    return __half2float(__ushort_as_half((unsigned short)b));
}
__device__ __forceinline__ uint32_t pack_f16x2_rn(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t to16_rn(float x, bool f16) { return f16 ? f32_to_f16_bits_rn(x) : f32_to_bf16_bits_rn(x); }
__device__ __forceinline__ float from16(uint32_t b, bool f16) { return f16 ? f16_bits_to_f32(b) : bf16_bits_to_f32(b); }
__device__ __forceinline__ uint32_t pack16x2_rn(float a, float b, bool f16) {
    return f16 ? pack_f16x2_rn(a, b) : pack_bf16x2_rn(a, b);
}

// Packed fp32 pairs (sm_100 .f32x2 arithmetic): each element is rounded to nearest even on its
// own, exactly as the scalar __fmul_rn / __fmaf_rn, but one instruction serves two elements.
__device__ __forceinline__ float2 mul2_rn(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 fma2_rn(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

// Exact value of an FP8 E4M3 (finite-only) code: sign, 4-bit exponent with
// bias 7, 3-bit mantissa; exponent field 0 holds the subnormals m * 2^-9.
__device__ __forceinline__ float e4m3_to_f32(uint32_t c) {
    const uint32_t s = (c & 0x80u) << 24;
    const uint32_t e = (c >> 3) & 0xFu;
    const uint32_t m = c & 0x7u;
    const float v = (e == 0u) ? (float)m * 0.001953125f
                              : __uint_as_float(((e + 120u) << 23) | (m << 20));
    return __uint_as_float(__float_as_uint(v) | s);
}

// fp32 -> FP8 E4M3 code, round to nearest even, saturating to +-448.
__device__ __forceinline__ uint32_t f32_to_e4m3_rn_sat(float x) {
    return (uint32_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
}

// Rebuilt block constant c1' = fp32(fp32(v8 * c2) + mu), two roundings, no FMA.
__device__ __forceinline__ float rebuild_c1(uint32_t c1_code, float c2, float mu) {
    return __fadd_rn(__fmul_rn(e4m3_to_f32(c1_code), c2), mu);
}

// The dequantized weight value in bf16 bits: bf16_rn(fp32(q * c1')), or fp16 bits.
__device__ __forceinline__ uint32_t dequant_bits(float q, float c1p, bool f16 = false) {
    return to16_rn(__fmul_rn(q, c1p), f16);
}

}  // namespace qlora

// Launch helpers (host).  Every launch in the library goes through these so
// that the launch counter is exact and launch errors map to QLORA_ERR_CUDA.
#define QLORA_CHECK_LAUNCH()                                   \
    do {                                                       \
        qlora::note_launches(1);                               \
        if (cudaPeekAtLastError() != cudaSuccess) {            \
            (void)cudaGetLastError();                          \
            return QLORA_ERR_CUDA;                             \
        }                                                      \
        if (qlora::sync_check_enabled() && !qlora::sync_check(__func__)) return QLORA_ERR_CUDA; \
    } while (0)

// Programmatic dependent launch.  A kernel launched with launch_dependent()
// may start while the previous kernel on the stream still runs; it calls
// grid_dependency_wait() before it touches anything the previous kernel
// writes (or, when it reads nothing of it, before it exits, so that its own
// completion still implies the previous kernel's).  A kernel calls
// allow_dependents() once the next kernel may be scheduled.  Both are no-ops
// when the kernel was launched normally.
namespace qlora {
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" :::); }

template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                             Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
}  // namespace qlora

#define QLORA_TRY(expr)                                        \
    do {                                                       \
        qlora_status _s = (expr);                              \
        if (_s != QLORA_OK) return _s;                         \
    } while (0)
