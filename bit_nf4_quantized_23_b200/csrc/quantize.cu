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
//                        repeated while more than 1024 partials are left
//                        (once from 2^20 to 2^30 weights, none below).
//   dq_blocks            the last tree level (at most 1024 partials) in
//                        each CTA, then per group of 256 blocks: mu from
//                        the total, d = c1 - mu, c2 = max|d|, E4M3 code
//                        of d / c2.
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
constexpr int kDqThreads = 256;                      // 8 warps, one group of 256 blocks per warp

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
// of a warp never meet in a shared-memory bank.  The shared address of entry k
// is table + 8*(32k + lane) = 256 * bits(y) + lane_off (mod 2^32) with
// lane_off = table + 8*lane - 256 * 0x4B400000, one multiply-add.
__device__ __forceinline__ uint32_t nf4_code_at(float x, float y, uint32_t lane_off) {
    const uint32_t addr = __float_as_uint(y) * 256u + lane_off;
    float thr, base;
    asm("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(thr), "=f"(base) : "r"(addr));
    return (uint32_t)__float_as_int(base) + (x > thr ? 1u : 0u);
}

__device__ __forceinline__ uint32_t nf4_code(float x, uint32_t lane_off) {
    return nf4_code_at(x, __fmaf_rn(x, 64.f, 12582976.f), lane_off);   // 1.5 * 2^23 + 64: bits 0x4B400000 + k
}

// One pass over W.  Persistent CTAs loop over chunks of 128 consecutive NF4
// blocks; two register buffers alternate so the next chunk's weights load
// while the current one is coded.  Two threads share a block (32 weights
// each).  Per chunk: packed codes, fp32 block absmax, and per warp the fp64
// pairwise-tree sum of its 16 blocks' c1 (aligned subtrees of the global
// tree, combined by tree_sum_pass).
__global__ void __launch_bounds__(kQuantThreads, kCtasPerSm)
nf4_quantize_blocks(const uint4* __restrict__ W, int64_t nb1, uint4* __restrict__ codes,
                    float* __restrict__ c1_out, double* __restrict__ warp_sums_out, int64_t n_chunks,
                    QuantBuckets qb) {
    allow_dependents();                                       // the tree pass (or the DQ kernel) may be scheduled now
    __shared__ float2 table[kTableWords];
    for (int i = threadIdx.x; i < kTableWords; i += kQuantThreads) table[i] = qb.e[i >> 5];
    __syncthreads();
    uint32_t table_addr;
    asm("{ .reg .u64 t; cvta.to.shared.u64 t, %1; cvt.u32.u64 %0, t; }" : "=r"(table_addr) : "l"(table));
    const uint32_t lane_off = table_addr + 8u * (threadIdx.x & 31) - 0x40000000u;   // 256 * 0x4B400000 mod 2^32
    const int sub = threadIdx.x & 1;

    auto load_chunk = [&](uint4 (&buf)[4], int64_t chunk) {
        const int64_t blk = chunk * kBlocksPerCta + (threadIdx.x >> 1);
#pragma unroll
        for (int j = 0; j < 4; ++j)
            buf[j] = (chunk < n_chunks && blk < nb1) ? W[blk * 8 + sub * 4 + j] : make_uint4(0, 0, 0, 0);
    };
    auto code_chunk = [&](const uint4 (&buf)[4], int64_t chunk) {
        const int64_t blk = chunk * kBlocksPerCta + (threadIdx.x >> 1);
        const bool valid = blk < nb1;
        const uint32_t w[16] = {buf[0].x, buf[0].y, buf[0].z, buf[0].w, buf[1].x, buf[1].y, buf[1].z, buf[1].w,
                                buf[2].x, buf[2].y, buf[2].z, buf[2].w, buf[3].x, buf[3].y, buf[3].z, buf[3].w};
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
                    // the two weights of each 32-bit word go through the division and the bucket
                    // FMA as one packed pair (the same per-element roundings as the scalar steps)
                    const float y = __frcp_rn(m);
                    const float2 y2 = make_float2(y, y), nm2 = make_float2(-m, -m);
                    const float2 k64 = make_float2(64.f, 64.f), kb = make_float2(12582976.f, 12582976.f);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t word = 0;
#pragma unroll
                        for (int pp = 3; pp >= 0; --pp) {              // elements (6,7), (4,5), (2,3), (0,1)
                            const uint32_t pair = w[4 * q + pp];
                            const float2 v = make_float2(__uint_as_float(pair << 16),
                                                         __uint_as_float(pair & 0xFFFF0000u));
                            const float2 q0 = mul2_rn(v, y2);
                            const float2 x = fma2_rn(fma2_rn(nm2, q0, v), y2, q0);   // Markstein, per element
                            const float2 b = fma2_rn(x, k64, kb);
                            word = word * 256u + nf4_code_at(x.x, b.x, lane_off) * 16u + nf4_code_at(x.y, b.y, lane_off);
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
                            word = word * 16u + nf4_code(__fdiv_rn(v, m), lane_off);
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
    };

    uint4 bufA[4], bufB[4];
    load_chunk(bufA, blockIdx.x);
    for (int64_t chunk = blockIdx.x; chunk < n_chunks; chunk += 2 * (int64_t)gridDim.x) {
        const int64_t next = chunk + gridDim.x;
        load_chunk(bufB, next);
        code_chunk(bufA, chunk);
        if (next >= n_chunks) break;
        load_chunk(bufA, next + gridDim.x);
        code_chunk(bufB, next);
    }
}

__global__ void __launch_bounds__(kTreeThreads)
tree_sum_pass(const double* __restrict__ in, int64_t n, double* __restrict__ out) {
    grid_dependency_wait();                                   // the previous level is complete
    allow_dependents();
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

// One warp per group of 256 first-level blocks (8 consecutive c1 per lane):
// mu from the tree sum, d = fp32(c1 - mu), c2 = max |d| over the group (warp
// shuffles), x2 = fp32(d / c2) correctly rounded (Markstein as above for c2 in
// [2^-100, 2^100], IEEE division outside), then its E4M3 code.
__global__ void __launch_bounds__(kDqThreads)
dq_blocks(const float* __restrict__ c1, int64_t nb1, const double* __restrict__ level, int np,
          uint8_t* __restrict__ c1_codes, float* __restrict__ c2_out, float* __restrict__ mu_out) {
    grid_dependency_wait();                                   // c1 and the tree's partial sums are complete
    const int lane = threadIdx.x & 31;
    // the last tree level, np <= 1024 partials, in warp 0 of every CTA: lane l sums partials
    // 32l .. 32l+31 pairwise, then the 32 lane sums pairwise by xor shuffles -- the same tree as a
    // tree_sum_pass over them (zero padding included)
    __shared__ double total;
    if (threadIdx.x < 32) {
        double v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 32 * lane + j < np ? level[32 * lane + j] : 0.0;
#pragma unroll
        for (int w = 1; w < 32; w <<= 1)
#pragma unroll
            for (int j = 0; j < 32; j += 2 * w) v[j] += v[j + w];
        double s = v[0];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) total = s;
    }
    __syncthreads();
    const int64_t g = (int64_t)blockIdx.x * (kDqThreads / 32) + (threadIdx.x >> 5);   // group
    const int64_t nb2 = (nb1 + 255) / 256;
    if (g >= nb2) return;
    const float mu = __double2float_rn(__ddiv_rn(total, (double)nb1));
    const int64_t i0 = g * 256 + lane * 8;
    float d[8];
    if (i0 + 8 <= nb1) {
        const float4 a = reinterpret_cast<const float4*>(c1 + i0)[0];
        const float4 b = reinterpret_cast<const float4*>(c1 + i0)[1];
        const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int k = 0; k < 8; ++k) d[k] = __fsub_rn(v[k], mu);
    } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) d[k] = i0 + k < nb1 ? __fsub_rn(c1[i0 + k], mu) : 0.f;
    }
    float c2 = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) c2 = fmaxf(c2, fabsf(d[k]));
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) c2 = fmaxf(c2, __shfl_xor_sync(0xffffffffu, c2, off));
    uint32_t code[8];
    if (c2 >= 7.8886091e-31f && c2 <= 1.2676506e30f) {
        const float y = __frcp_rn(c2);
#pragma unroll
        for (int k = 0; k < 8; ++k) code[k] = f32_to_e4m3_rn_sat(div_markstein(d[k], c2, y));
    } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) code[k] = f32_to_e4m3_rn_sat(c2 > 0.f ? __fdiv_rn(d[k], c2) : 0.f);
    }
    if (i0 + 8 <= nb1) {
        const uint2 packed = make_uint2(code[0] | code[1] << 8 | code[2] << 16 | code[3] << 24,
                                        code[4] | code[5] << 8 | code[6] << 16 | code[7] << 24);
        reinterpret_cast<uint2*>(c1_codes + i0)[0] = packed;
    } else {
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (i0 + k < nb1) c1_codes[i0 + k] = (uint8_t)code[k];
    }
    if (lane == 0) {
        c2_out[g] = c2;
        if (g == 0) *mu_out = mu;
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
    // with double quantization off the block constants are the output itself
    float* c1 = out->c1 ? out->c1 : reinterpret_cast<float*>(ws);
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
        host_buckets(out->codebook));
    QLORA_CHECK_LAUNCH();
    if (out->c1) return QLORA_OK;                             // single-level quantization: done
    while (p > kTreeThreads) {   // dq_blocks sums the last level (at most kTreeThreads partials) itself
        const int64_t np = (p + kTreeThreads - 1) / kTreeThreads;
        double* next = reinterpret_cast<double*>(ws);
        ws += align_up((size_t)np * sizeof(double), 256);
        (void)launch_dependent(tree_sum_pass, dim3((unsigned)np), dim3(kTreeThreads), 0, stream,
                               (const double*)level, p, next);
        QLORA_CHECK_LAUNCH();
        level = next;
        p = np;
    }
    const int64_t nb2 = (nb1 + 255) / 256;
    (void)launch_dependent(dq_blocks, dim3((unsigned)((nb2 + kDqThreads / 32 - 1) / (kDqThreads / 32))),
                           dim3(kDqThreads), 0, stream, (const float*)c1, nb1, (const double*)level, (int)p,
                           out->c1_codes, out->c2, out->mu);
    QLORA_CHECK_LAUNCH();
    return QLORA_OK;
}

}  // namespace qlora
