// NF4 + Double Quantization of a frozen bf16 weight ("Science Depth M5-131:
// PEFT (LoRA / QLoRA / Prefix Tuning)", section 3: NF4 with absmax blocks of
// B = 64, nearest-code rule, Double Quantization of the block constants to
// 8-bit floats with second-level block 256).
//
// Kernels, in launch order:
//   nf4_quantize_blocks  one pass over W: per 64-block absmax (4 threads per
//                        block, warp shuffles), IEEE division, 15-threshold
//                        code count, nibble packing; writes the packed codes,
//                        the fp32 absmax c1 per block, and the fp64 sum of the
//                        CTA's 64 c1 values over a fixed pairwise tree.
//   tree_sum_pass        fp64 pairwise-tree sums of 1024 partials per CTA,
//                        repeated until one value is left.
//   dq_blocks            per group of 256 blocks: mu from the tree sum,
//                        d = c1 - mu, c2 = max|d|, E4M3 code of d / c2.
// Every tree is over aligned power-of-two ranges with zero padding, so the
// total equals a pairwise tree over all c1 padded to a power of two.
#include <mutex>

#include "qlora_internal.cuh"

namespace qlora {

// The device error word of this library (zero-initialised at module load).
__device__ uint32_t g_error_flags = 0;

uint32_t* device_error_word() {
    static std::mutex mu;
    static uint32_t* cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!cache[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_error_flags) != cudaSuccess) return nullptr;
        cache[dev] = static_cast<uint32_t*>(p);
    }
    return cache[dev];
}

namespace {

constexpr int kQuantThreads = 256;                   // 64 blocks of 64 weights per CTA
constexpr int kBlocksPerCta = kQuantThreads / 4;
constexpr int kTreeThreads = 1024;
constexpr int kDqThreads = 256;                      // one group of 256 blocks per CTA

__device__ __forceinline__ uint32_t nf4_code(float x, const NF4Tables& tb) {
    uint32_t c = 0;
#pragma unroll
    for (int j = 0; j < 15; ++j) c += (x > tb.t[j]) ? 1u : 0u;
    return c;
}

__global__ void __launch_bounds__(kQuantThreads)
nf4_quantize_blocks(const uint4* __restrict__ W, int64_t nb1, uint2* __restrict__ codes,
                    float* __restrict__ c1_out, double* __restrict__ cta_sums, NF4Tables tb) {
    const int64_t blk = (int64_t)blockIdx.x * kBlocksPerCta + (threadIdx.x >> 2);
    const int sub = threadIdx.x & 3;
    const bool valid = blk < nb1;

    uint32_t w[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (valid) {
        const uint4 a = W[(blk * 64 + sub * 16) / 8];
        const uint4 b = W[(blk * 64 + sub * 16) / 8 + 1];
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
        w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    }
    float v[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        v[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
        v[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
    }
    float m = 0.f;
    bool finite = true;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float a = fabsf(v[i]);
        finite &= (a <= 3.402823466e38f);
        m = fmaxf(m, a);
    }
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    if (!finite) atomicOr(&g_error_flags, ERR_FLAG_NONFINITE);

    if (valid) {
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float x = (m > 0.f) ? __fdiv_rn(v[i], m) : 0.f;
            const uint32_t c = nf4_code(x, tb);
            const int byte = i >> 1;
            const int shift = 8 * (byte & 3) + ((i & 1) ? 0 : 4);   // element 2j -> high nibble
            if (byte < 4) lo |= c << shift; else hi |= c << shift;
        }
        codes[blk * 4 + sub] = make_uint2(lo, hi);
        if (sub == 0) c1_out[blk] = m;
    }

    // fp64 tree over the CTA's 64 block constants: lanes 0,4,...,28 hold blocks
    // 8w..8w+7 of warp w; xor-shuffles by 4, 8, 16 pair neighbours level by level.
    double s = valid ? (double)m : 0.0;
    s += __shfl_xor_sync(0xffffffffu, s, 4);
    s += __shfl_xor_sync(0xffffffffu, s, 8);
    s += __shfl_xor_sync(0xffffffffu, s, 16);
    __shared__ double warp_sums[kQuantThreads / 32];
    if ((threadIdx.x & 31) == 0) warp_sums[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        const double* ws = warp_sums;
        cta_sums[blockIdx.x] = ((ws[0] + ws[1]) + (ws[2] + ws[3])) + ((ws[4] + ws[5]) + (ws[6] + ws[7]));
    }
}

__global__ void __launch_bounds__(kTreeThreads)
tree_sum_pass(const double* __restrict__ in, int64_t n, double* __restrict__ out) {
    const int64_t i = (int64_t)blockIdx.x * kTreeThreads + threadIdx.x;
    double s = i < n ? in[i] : 0.0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    __shared__ double ws[32];
    if ((threadIdx.x & 31) == 0) ws[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x < 32) {
        s = ws[threadIdx.x];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (threadIdx.x == 0) out[blockIdx.x] = s;
    }
}

__global__ void __launch_bounds__(kDqThreads)
dq_blocks(const float* __restrict__ c1, int64_t nb1, const double* __restrict__ total,
          uint8_t* __restrict__ c1_codes, float* __restrict__ c2_out, float* __restrict__ mu_out) {
    const int64_t i = (int64_t)blockIdx.x * kDqThreads + threadIdx.x;
    const bool valid = i < nb1;
    const float mu = __double2float_rn(__ddiv_rn(*total, (double)nb1));
    const float d = valid ? __fsub_rn(c1[i], mu) : 0.f;
    float a = fabsf(d);
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
    __shared__ float wm[kDqThreads / 32];
    if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = a;
    __syncthreads();
    float c2 = wm[0];
#pragma unroll
    for (int k = 1; k < kDqThreads / 32; ++k) c2 = fmaxf(c2, wm[k]);
    if (valid) {
        const float x2 = (c2 > 0.f) ? __fdiv_rn(d, c2) : 0.f;
        c1_codes[i] = (uint8_t)f32_to_e4m3_rn_sat(x2);
    }
    if (threadIdx.x == 0) {
        c2_out[blockIdx.x] = c2;
        if (blockIdx.x == 0) *mu_out = mu;
    }
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace

// Scratch layout of the quantize: fp32 c1[nb1], then the fp64 partial sums of
// every tree level (P1 = ceil(nb1/64), then ceil(P/1024) until 1).
size_t quantize_workspace_bytes(int64_t nb1) {
    size_t bytes = align_up((size_t)nb1 * sizeof(float), 256);
    int64_t p = (nb1 + kBlocksPerCta - 1) / kBlocksPerCta;
    bytes += align_up((size_t)p * sizeof(double), 256);
    while (p > 1) {
        p = (p + kTreeThreads - 1) / kTreeThreads;
        bytes += align_up((size_t)p * sizeof(double), 256);
    }
    return bytes;
}

qlora_status launch_quantize(const void* W, int64_t N, int64_t K, const qlora_nf4_weight* out,
                             void* workspace, cudaStream_t stream) {
    const int64_t nb1 = N * K / 64;
    const NF4Tables& tb = host_tables();
    char* ws = static_cast<char*>(workspace);
    float* c1 = reinterpret_cast<float*>(ws);
    ws += align_up((size_t)nb1 * sizeof(float), 256);
    int64_t p = (nb1 + kBlocksPerCta - 1) / kBlocksPerCta;
    double* level = reinterpret_cast<double*>(ws);
    ws += align_up((size_t)p * sizeof(double), 256);

    nf4_quantize_blocks<<<(unsigned)p, kQuantThreads, 0, stream>>>(
        static_cast<const uint4*>(W), nb1, reinterpret_cast<uint2*>(out->codes), c1, level, tb);
    QLORA_CHECK_LAUNCH();
    while (p > 1) {
        const int64_t np = (p + kTreeThreads - 1) / kTreeThreads;
        double* next = reinterpret_cast<double*>(ws);
        ws += align_up((size_t)np * sizeof(double), 256);
        tree_sum_pass<<<(unsigned)np, kTreeThreads, 0, stream>>>(level, p, next);
        QLORA_CHECK_LAUNCH();
        level = next;
        p = np;
    }
    const int64_t nb2 = (nb1 + 255) / 256;
    dq_blocks<<<(unsigned)nb2, kDqThreads, 0, stream>>>(c1, nb1, level, out->c1_codes, out->c2, out->mu);
    QLORA_CHECK_LAUNCH();
    return QLORA_OK;
}

}  // namespace qlora
