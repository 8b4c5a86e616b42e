// Blockwise absmax INT8 quantization and its dequantization ("Ch.09 QLoRA 与量化：
// 缩得更小再微调", section "2. INT8 量化": find the block's largest magnitude,
// choose the scale alpha that maps it to 127, store round(x * alpha), and
// recover x as code / alpha before the matrix product).
//
// Arithmetic, all fp32 with round-to-nearest-even unless stated:
//   amax      = max |x| over the block (exact; x is bf16)
//   alpha     = 127 / amax (IEEE division), alpha = 0 for an all-zero block;
//               +inf when amax < 127 / FLT_MAX
//   code      = round half away from zero of (x * alpha) clamped to [-127, 127],
//               0 for x = 0 (the clamp acts only when alpha = +inf:
//               otherwise |x * alpha| <= 127 (1 + 2^-23))
//   x_hat     = code / alpha (correctly rounded: Markstein's division, see
//               int8_value), 0 when alpha = 0, then rounded to the output dtype.
// A block holding Inf or NaN raises the non-finite device flag and gets
// alpha = 0 and zero codes.
// HBM-bound: quantize reads 2 B and writes 1 + 4/blocksize B per element;
// dequantize reads 1 + 4/blocksize B and writes 2 (or 4) B.  Each thread
// handles groups of 8 consecutive elements (one 16-byte load of bf16, one 8-byte
// code word); the blocksize / 8 threads of a block are consecutive lanes of a
// warp and combine their maxima with xor shuffles.
#include "qlora_internal.cuh"

namespace qlora {
namespace {

constexpr int kI8Threads = 256;

// alpha is +inf when amax < 127 / FLT_MAX (tiny bf16 magnitudes): a zero element
// still codes to 0 (not 0 * inf), every other element to +-127.  alpha = 0 (an
// all-zero or a non-finite block) codes everything to 0.
__device__ __forceinline__ int8_t int8_code(float x, float alpha) {
    const float s = (x == 0.f || alpha == 0.f) ? 0.f : __fmul_rn(x, alpha);
    return (int8_t)(int)roundf(fminf(fmaxf(s, -127.f), 127.f));   // roundf: half away from zero
}

// A CTA covers kI8Unroll x 256 groups of 8 elements; thread t takes groups t + 256 u
// (u < kI8Unroll) and issues all their loads before any arithmetic, so each
// thread keeps 64 bytes of reads in flight.  The lanes of a block keep their
// lane positions in every group, so the shuffles never mix blocks.
constexpr int kI8Unroll = 4;

__global__ void __launch_bounds__(kI8Threads)
int8_absmax_quantize(const uint4* __restrict__ W, int64_t n8, int lane_shift, uint2* __restrict__ codes,
                     float* __restrict__ alpha_out, uint32_t* __restrict__ err) {
    const int lanes_per_block = 1 << lane_shift;
    grid_dependency_wait();
    allow_dependents();
    const int64_t g0 = (int64_t)blockIdx.x * (kI8Threads * kI8Unroll) + threadIdx.x;
    uint4 v[kI8Unroll];
#pragma unroll
    for (int u = 0; u < kI8Unroll; ++u) {     // groups past the end carry zeros (whole blocks of lanes)
        const int64_t i = g0 + (int64_t)u * kI8Threads;
        v[u] = i < n8 ? W[i] : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kI8Unroll; ++u) {
        const int64_t i = g0 + (int64_t)u * kI8Threads;
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
        uint32_t mbits = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) mbits = max(mbits, max(w[j] & 0x7FFFu, (w[j] >> 16) & 0x7FFFu));
        for (int o = 1; o < lanes_per_block; o <<= 1) mbits = max(mbits, __shfl_xor_sync(0xffffffffu, mbits, o));
        if (i >= n8) continue;
        if (mbits >= 0x7F80u && err) atomicOr(err, ERR_FLAG_NONFINITE);
        const float amax = bf16_bits_to_f32(mbits);
        const float alpha = (amax > 0.f && mbits < 0x7F80u) ? __fdiv_rn(127.f, amax) : 0.f;
        uint32_t out[2] = {0u, 0u};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t b = (j & 1) ? (w[j >> 1] >> 16) : (w[j >> 1] & 0xFFFFu);
            const uint32_t c = (uint32_t)(uint8_t)int8_code(bf16_bits_to_f32(b), alpha);
            out[j >> 2] |= c << (8 * (j & 3));
        }
        codes[i] = make_uint2(out[0], out[1]);
        if ((threadIdx.x & (lanes_per_block - 1)) == 0) alpha_out[i >> lane_shift] = alpha;
    }
}

// x_hat = RN(code / alpha).  For alpha in [2^-100, 2^100] by Markstein's division
// (P. Markstein, "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990): with y = RN(1/alpha) and
// q0 = RN(code * y), the remainder code - alpha * q0 is exact in one FMA and
// RN(q0 + r * y) is the correctly rounded quotient (no overflow or underflow can
// occur there for |code| <= 128).  Other scales take the IEEE division intrinsic.
__device__ __forceinline__ bool markstein_range(float alpha) {
    return alpha >= 7.8886091e-31f && alpha <= 1.2676506e30f;   // 2^-100 .. 2^100
}

__device__ __forceinline__ float int8_value(uint32_t byte, float alpha, float y, bool fast) {
    const float a = (float)(int8_t)byte;
    if (fast) {
        const float q0 = __fmul_rn(a, y);
        return __fmaf_rn(__fmaf_rn(-alpha, q0, a), y, q0);
    }
    return alpha == 0.f ? 0.f : __fdiv_rn(a, alpha);
}

__global__ void __launch_bounds__(kI8Threads)
int8_absmax_dequantize(const uint2* __restrict__ codes, const float* __restrict__ alpha_in, int64_t n8,
                       int lane_shift, void* __restrict__ out, int out_dtype) {
    grid_dependency_wait();
    allow_dependents();
    const int64_t g0 = (int64_t)blockIdx.x * (kI8Threads * kI8Unroll) + threadIdx.x;
    uint2 c[kI8Unroll];
    float alpha[kI8Unroll];
#pragma unroll
    for (int u = 0; u < kI8Unroll; ++u) {
        const int64_t i = g0 + (int64_t)u * kI8Threads;
        c[u] = i < n8 ? codes[i] : make_uint2(0, 0);
        alpha[u] = i < n8 ? alpha_in[i >> lane_shift] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kI8Unroll; ++u) {
        const int64_t i = g0 + (int64_t)u * kI8Threads;
        if (i >= n8) break;
        const bool fast = markstein_range(alpha[u]);
        const float y = fast ? __frcp_rn(alpha[u]) : 0.f;
        float x[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
            x[j] = int8_value(((j < 4 ? c[u].x : c[u].y) >> (8 * (j & 3))) & 0xFFu, alpha[u], y, fast);
        if (out_dtype == QLORA_DTYPE_F32) {
            uint4* o = static_cast<uint4*>(out) + 2 * i;
            o[0] = make_uint4(__float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]),
                              __float_as_uint(x[3]));
            o[1] = make_uint4(__float_as_uint(x[4]), __float_as_uint(x[5]), __float_as_uint(x[6]),
                              __float_as_uint(x[7]));
        } else {
            const bool h = out_dtype == QLORA_DTYPE_F16;
            static_cast<uint4*>(out)[i] = make_uint4(pack16x2_rn(x[0], x[1], h), pack16x2_rn(x[2], x[3], h),
                                                     pack16x2_rn(x[4], x[5], h), pack16x2_rn(x[6], x[7], h));
        }
    }
}

inline unsigned i8_grid(int64_t n8) {
    return (unsigned)((n8 + kI8Threads * kI8Unroll - 1) / (kI8Threads * kI8Unroll));
}
inline int lane_shift(int blocksize) { return blocksize == 64 ? 3 : blocksize == 128 ? 4 : 5; }

}  // namespace

qlora_status launch_int8_quantize(const void* W, int64_t n, int blocksize, int8_t* codes, float* alpha,
                                  cudaStream_t s) {
    const int64_t n8 = n / 8;
    (void)launch_dependent(int8_absmax_quantize, dim3(i8_grid(n8)), dim3(kI8Threads), 0, s,
                           static_cast<const uint4*>(W), n8, lane_shift(blocksize), reinterpret_cast<uint2*>(codes),
                           alpha, device_error_word());
    QLORA_CHECK_LAUNCH();
    return QLORA_OK;
}

qlora_status launch_int8_dequantize(const int8_t* codes, const float* alpha, int64_t n, int blocksize, void* out,
                                    int out_dtype, cudaStream_t s) {
    const int64_t n8 = n / 8;
    (void)launch_dependent(int8_absmax_dequantize, dim3(i8_grid(n8)), dim3(kI8Threads), 0, s,
                           reinterpret_cast<const uint2*>(codes), alpha, n8, lane_shift(blocksize), out, out_dtype);
    QLORA_CHECK_LAUNCH();
    return QLORA_OK;
}

}  // namespace qlora
