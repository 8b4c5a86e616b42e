// NF4 + Double Quantization of a frozen bf16 weight ("Science Depth M5-131:
// PEFT (LoRA / QLoRA / Prefix Tuning)", section 3: NF4 with absmax blocks of
// B = 64, nearest-code rule, Double Quantization of the block constants to
// 8-bit floats with second-level block 256).
//
// Kernels, in launch order:
//   nf4_quantize_blocks  one pass over W: per 64-block absmax (2 threads per
//                        block, packed 16-bit max), correctly rounded
//                        division, bucketed code search with one compare,
//                        nibble packing; writes the packed codes, the fp32
//                        absmax c1 per block, and the fp64 sum of each
//                        warp's 16 c1 values over a fixed pairwise tree.
//   tree_sum_pass        fp64 pairwise-tree sums of 1024 partials per CTA,
//                        repeated until one value is left.
//   dq_blocks            per group of 256 blocks: mu from the tree sum,
//                        d = c1 - mu, c2 = max|d|, E4M3 code of d / c2.
// Every tree is over aligned power-of-two ranges with zero padding, so the
// total equals a pairwise tree over all c1 padded to a power of two.
#include <algorithm>
#include <mutex>

#include "qlora_internal.cuh"

namespace qlora {

// The device error words of this library (zero-initialised at module load):
// [0] error flags, [1] location code of the last failed self-check or wait.
__device__ uint32_t g_error_flags[2] = {0, 0};

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

constexpr int kQuantThreads = 256;                   // 2 threads per block of 64 weights
constexpr int kBlocksPerCta = kQuantThreads / 2;     // 128 blocks per chunk (one CTA iteration)
constexpr int kCtasPerSm = 3;
constexpr int kTableWords = kCodeBuckets * 32;       // bank-private copies: entry e of lane l at e*32 + l
constexpr int kTreeThreads = 1024;
constexpr int kDqThreads = 256;                      // one group of 256 blocks per CTA

// x = fp32(w / m), correctly rounded, for |w| <= m with m in [2^-100, 2^100]:
// Markstein's division (P. Markstein, "Computation of elementary functions on
// the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990): with
// y = RN(1/m) and q0 = RN(w*y), the remainder r = w - m*q0 is exact in one
// FMA and RN(q0 + r*y) is the correctly rounded quotient.  Outside that scale
// range the IEEE division intrinsic is used.
__device__ __forceinline__ float div_markstein(float w, float m, float y) {
    const float q0 = __fmul_rn(w, y);
    const float r = __fmaf_rn(-m, q0, w);
    return __fmaf_rn(r, y, q0);
}

// NF4 code of x in [-1, 1].  bucket k = RNE(64x + 64) comes from one FMA that
// rounds to an integer (1.5 * 2^23 makes the fp32 ulp 1); the table keeps one
// copy of every entry per lane (entry k of lane l at k*32 + l), so the 32 lanes
// of a warp never meet in a shared-memory bank.
__device__ __forceinline__ uint32_t nf4_code(float x, const float2* __restrict__ lane_table) {
    const float y = __fmaf_rn(x, 64.f, 12582976.f);               // 1.5 * 2^23 + 64
    const uint32_t k = __float_as_uint(y) - 0x4B400000u;          // RNE(64x + 64), 0..128
    const float2 e = lane_table[k * 32u];
    return (uint32_t)__float_as_int(e.y) + (x > e.x ? 1u : 0u);
}

// One pass over W.  Persistent CTAs loop over chunks of 128 consecutive NF4
// blocks (the next chunk's weights are loaded while the current one is coded);
// two threads share a block (32 weights each).  Per chunk: packed codes, fp32
// block absmax, and per warp the fp64 pairwise-tree sum of its 16 blocks' c1
// (aligned subtrees of the global tree, combined by tree_sum_pass).
__global__ void __launch_bounds__(kQuantThreads, kCtasPerSm)
nf4_quantize_blocks(const uint4* __restrict__ W, int64_t nb1, uint4* __restrict__ codes,
                    float* __restrict__ c1_out, double* __restrict__ warp_sums_out, int64_t n_chunks,
                    QuantBuckets qb) {
    __shared__ float2 table[kTableWords];
    for (int i = threadIdx.x; i < kTableWords; i += kQuantThreads) table[i] = qb.e[i >> 5];
    __syncthreads();
    const float2* lane_table = table + (threadIdx.x & 31);
    const int sub = threadIdx.x & 1;

    uint4 nxt[4];
    auto load_chunk = [&](int64_t chunk) {
        const int64_t blk = chunk * kBlocksPerCta + (threadIdx.x >> 1);
#pragma unroll
        for (int j = 0; j < 4; ++j)
            nxt[j] = (chunk < n_chunks && blk < nb1) ? W[blk * 8 + sub * 4 + j] : make_uint4(0, 0, 0, 0);
    };
    load_chunk(blockIdx.x);
    for (int64_t chunk = blockIdx.x; chunk < n_chunks; chunk += gridDim.x) {
        const int64_t blk = chunk * kBlocksPerCta + (threadIdx.x >> 1);
        const bool valid = blk < nb1;
        const uint32_t w[16] = {nxt[0].x, nxt[0].y, nxt[0].z, nxt[0].w, nxt[1].x, nxt[1].y, nxt[1].z, nxt[1].w,
                                nxt[2].x, nxt[2].y, nxt[2].z, nxt[2].w, nxt[3].x, nxt[3].y, nxt[3].z, nxt[3].w};
        load_chunk(chunk + gridDim.x);
        // block absmax on the bf16 bit patterns: |w| orders like the unsigned 15-bit magnitude
        uint32_t mx = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) mx = __vmaxu2(mx, w[i] & 0x7FFF7FFFu);
        uint32_t mbits = max(mx & 0xFFFFu, mx >> 16);
        mbits = max(mbits, (uint32_t)__shfl_xor_sync(0xffffffffu, mbits, 1));
        const float m = bf16_bits_to_f32(mbits);
        if (mbits >= 0x7F80u) atomicOr(&g_error_flags[0], ERR_FLAG_NONFINITE);

        if (valid) {
            uint32_t out[4] = {0x77777777u, 0x77777777u, 0x77777777u, 0x77777777u};  // all-zero block: code 7
            if (m > 0.f && mbits < 0x7F80u) {
                // weights are coded in the order 6,7,4,5,2,3,0,1 of each group of 8 so that
                // word = 16 * word + code leaves weight 2j in the high nibble of byte j
                if ((m >= 7.8886091e-31f) && (m <= 1.2676506e30f)) {   // 2^-100 .. 2^100: Markstein division
                    const float y = __frcp_rn(m);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t word = 0;
#pragma unroll
                        for (int jj = 0; jj < 8; ++jj) {
                            const int i = (6 - 2 * (jj >> 1)) + (jj & 1);
                            const uint32_t pair = w[4 * q + (i >> 1)];
                            const float v = __uint_as_float((i & 1) ? (pair & 0xFFFF0000u) : (pair << 16));
                            word = word * 16u + nf4_code(div_markstein(v, m, y), lane_table);
                        }
                        out[q] = word;
                    }
                } else {                                                // extreme scales: IEEE division
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t word = 0;
#pragma unroll
                        for (int jj = 0; jj < 8; ++jj) {
                            const int i = (6 - 2 * (jj >> 1)) + (jj & 1);
                            const uint32_t pair = w[4 * q + (i >> 1)];
                            const float v = __uint_as_float((i & 1) ? (pair & 0xFFFF0000u) : (pair << 16));
                            word = word * 16u + nf4_code(__fdiv_rn(v, m), lane_table);
                        }
                        out[q] = word;
                    }
                }
            }
            codes[blk * 2 + sub] = make_uint4(out[0], out[1], out[2], out[3]);
            if (sub == 0) c1_out[blk] = m;
        }

        // fp64 pairwise tree over the warp's 16 blocks (even lanes, in order): xor-shuffles
        // by 2..16 pair neighbours level by level; one sum per warp
        double s = valid ? (double)m : 0.0;
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        s += __shfl_xor_sync(0xffffffffu, s, 4);
        s += __shfl_xor_sync(0xffffffffu, s, 8);
        s += __shfl_xor_sync(0xffffffffu, s, 16);
        if ((threadIdx.x & 31) == 0) warp_sums_out[chunk * (kQuantThreads / 32) + (threadIdx.x >> 5)] = s;
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
// every tree level (P1 = ceil(nb1/128), then ceil(P/1024) until 1).
size_t quantize_workspace_bytes(int64_t nb1) {
    size_t bytes = align_up((size_t)nb1 * sizeof(float), 256);
    int64_t p = (nb1 + kBlocksPerCta - 1) / kBlocksPerCta * (kQuantThreads / 32);   // one sum per warp (16 blocks)
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
    char* ws = static_cast<char*>(workspace);
    float* c1 = reinterpret_cast<float*>(ws);
    ws += align_up((size_t)nb1 * sizeof(float), 256);
    const int64_t n_chunks = (nb1 + kBlocksPerCta - 1) / kBlocksPerCta;
    int64_t p = n_chunks * (kQuantThreads / 32);                 // first tree level: one sum per 16 blocks
    double* level = reinterpret_cast<double*>(ws);
    ws += align_up((size_t)p * sizeof(double), 256);

    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t grid = std::min<int64_t>(n_chunks, (int64_t)sms * kCtasPerSm);
    nf4_quantize_blocks<<<(unsigned)grid, kQuantThreads, 0, stream>>>(
        static_cast<const uint4*>(W), nb1, reinterpret_cast<uint4*>(out->codes), c1, level, n_chunks,
        host_buckets());
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
