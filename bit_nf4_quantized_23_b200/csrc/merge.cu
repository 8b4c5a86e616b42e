// Merging the trained adapters into the frozen weight and requantizing.
//
// After fine-tuning, the adapter product is folded into the weight for
// inference ("Q103: What is QLoRA, and how does it differ from LoRA",
// follow-up 1: merge the LoRA weights after fine-tuning; "QLoRA 的原理是什么？
// 4-bit 量化权重真的参与训练吗？", section 5: merging and requantizing can add
// error again): W_merged = W_hat + (alpha / r) B A, here rounded once to
// the 16-bit compute type (bf16 or fp16):
//        W_merged[n,k] = bf16_rn(fp32(W_hat[n,k] + sum_j (s B[n,j]) A[j,k])),
// the rank-r sum accumulated in fp32 in ascending j.  Requantizing is the
// ordinary NF4 + double-quantization pass over W_merged.
//
// Tensor-core kernel (r % 8 == 0): one CTA per 128 x 128 output tile.  The
// whole rank reduction fits in shared memory at once (r <= 256: at most four
// 64-wide steps of a [128 x 64] B tile, K-major, and a [64 x 128] A tile,
// MN-major, all by TMA), tcgen05 accumulates B A in fp32 in TMEM, and the
// eight warps' epilogue dequantizes the matching W_hat row segment (one block
// per warp row) and writes bf16_rn(fp32(W_hat + s * acc)) -- s applied to the
// fp32 sum.  HBM traffic:
// 0.516 B/weight of packed weight in, 2 B/weight out.
//
// CUDA-core fallback (any r): one CTA writes a 64 x 64 tile (one first-level
// block per row): 256 threads, each 4 rows x 4 columns; s*B and A are staged
// through shared memory in chunks of 32 ranks; r FMAs per weight.
#include <cuda.h>

#include "qlora_internal.cuh"
#include "tc_ptx.cuh"
#include "gemm_tc.cuh"

namespace qlora {
namespace {

constexpr int kMergeThreads = 256;
constexpr int kTile = 64;
constexpr int kRChunk = 32;

__global__ void __launch_bounds__(kMergeThreads)
merge_lora(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ c1_codes, const float* __restrict__ c2,
           const float* __restrict__ mu_p, const float* __restrict__ c1f, int64_t N, int64_t K,
           const uint16_t* __restrict__ A, const uint16_t* __restrict__ B, int r, float s,
           uint16_t* __restrict__ out, NF4Tables tb, bool f16) {
    __shared__ float Bs[kTile][kRChunk + 1];         // s * B[n0 + i, j0 + j]
    __shared__ __align__(16) float As[kRChunk][kTile];   // A[j0 + j, k0 + c]
    __shared__ float q[16];
    if (threadIdx.x < 16) q[threadIdx.x] = tb.q[threadIdx.x];
    const int64_t k0 = (int64_t)blockIdx.x * kTile;
    const int64_t n0 = (int64_t)blockIdx.y * kTile;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc[4][4] = {};
    for (int j0 = 0; j0 < r; j0 += kRChunk) {
        __syncthreads();
        for (int e = threadIdx.x; e < kTile * kRChunk; e += kMergeThreads) {
            const int i = e / kRChunk, j = e % kRChunk;
            const int64_t n = n0 + i;
            Bs[i][j] = (n < N && j0 + j < r) ? __fmul_rn(s, from16(B[n * r + j0 + j], f16)) : 0.f;
            const int jj = e / kTile, c = e % kTile;
            As[jj][c] = (j0 + jj < r) ? from16(A[(int64_t)(j0 + jj) * K + k0 + c], f16) : 0.f;
        }
        __syncthreads();
        const int jn = min(kRChunk, r - j0);
        for (int j = 0; j < jn; ++j) {
            float b[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) b[u] = Bs[ty * 4 + u][j];
            const float4 a4 = reinterpret_cast<const float4*>(&As[j][tx * 4])[0];
            const float a[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 4; ++v) acc[u][v] = __fmaf_rn(b[u], a[v], acc[u][v]);
        }
    }
    // epilogue: W_hat of the 4 x 4 outputs (their block: row n, columns k0 .. k0 + 63), add, round
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int64_t n = n0 + ty * 4 + u;
        if (n >= N) continue;
        const int64_t blk = (n * K + k0) >> 6;
        const float c1p = c1f ? c1f[blk] : rebuild_c1(c1_codes[blk], c2[blk >> 8], *mu_p);
        const int64_t flat = n * K + k0 + tx * 4;                        // 4 weights = 2 code bytes
        const uint32_t two = (uint32_t)codes[flat >> 1] << 8 | codes[(flat >> 1) + 1];
        uint32_t o[4];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const uint32_t code = (two >> (12 - 4 * v)) & 0xFu;          // element order: high nibble first
            const float wh = from16(dequant_bits(q[code], c1p, f16), f16);
            o[v] = to16_rn(__fadd_rn(wh, acc[u][v]), f16);
        }
        reinterpret_cast<uint2*>(out + flat)[0] = make_uint2(o[0] | o[1] << 16, o[2] | o[3] << 16);
    }
}

constexpr int kMgThreads = 256;
constexpr int kMgN = 128;                           // output columns per CTA (TMEM columns)
constexpr uint32_t kMgAStep = 128 * 128;            // B tile [128 n x 64 ranks] bf16, K-major, swizzled
constexpr uint32_t kMgBStep = 2 * 8192;             // A tile [64 ranks x 128 k] bf16 as two MN-major chunks
// Layout for `steps` rank steps: A tiles, B tiles, then two barriers, the TMEM slot and the abort
// flag.  At least 48 KiB is requested so that at most four CTAs share an SM: their 128-column
// accumulators fill its 512 TMEM columns.
__host__ __device__ inline uint32_t mg_off_bar(int steps) { return (uint32_t)steps * (kMgAStep + kMgBStep); }
inline uint32_t mg_alloc(int steps) {
    const uint32_t need = mg_off_bar(steps) + 64 + 1024;
    return need < 48u * 1024u ? 48u * 1024u : need;
}

__global__ void __launch_bounds__(kMgThreads, 3)
merge_lora_tc(const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmA,
              const uint8_t* __restrict__ codes, const uint8_t* __restrict__ c1_codes, const float* __restrict__ c2,
              const float* __restrict__ mu_p, const float* __restrict__ c1f, int64_t N, int64_t K, int steps,
              float s, uint16_t* __restrict__ out, uint32_t* err, NF4Tables tb, bool f16) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base = (ptx::smem_addr(smem_raw) + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - ptx::smem_addr(smem_raw));
    const uint32_t off_bar = mg_off_bar(steps);
    const uint32_t sA = base, sB = base + (uint32_t)steps * kMgAStep;
    const uint32_t bar_full = base + off_bar, bar_acc = bar_full + 8;
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gbase + off_bar + 16);
    volatile int* abort = reinterpret_cast<volatile int*>(gbase + off_bar + 20);
    __shared__ float q[16];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t k0 = (int64_t)blockIdx.x * kMgN;
    const int64_t n0 = (int64_t)blockIdx.y * 128;
    if (threadIdx.x < 16) q[threadIdx.x] = tb.q[threadIdx.x];
    if (threadIdx.x == 0) {
        ptx::mbar_init(bar_full, 1);
        ptx::mbar_init(bar_acc, 1);
        *abort = 0;
        ptx::fence_barrier_init();
        ptx::fence_proxy_async_smem();
    }
    if (warp == 1) {
        ptx::tmem_alloc(base + off_bar + 16, kMgN);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 && ptx::elect_one_sync()) {
        ptx::mbar_arrive_expect_tx(bar_full, (uint32_t)steps * (kMgAStep + kMgBStep));
        for (int j = 0; j < steps; ++j) {
            ptx::tma_load_2d(sA + j * kMgAStep, &tmB, j * 64, (int32_t)n0, bar_full);
#pragma unroll
            for (int c = 0; c < 2; ++c)
                ptx::tma_load_2d(sB + j * kMgBStep + c * 8192, &tmA, (int32_t)(k0 + c * 64), j * 64, bar_full);
        }
    }
    __syncwarp();
    if (warp == 1) {
        const bool ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_full, 0, abort, err));
        if (ok) {
            ptx::tc_fence_after();
            if (ptx::elect_one_sync()) {
                const uint32_t idesc = ptx::idesc_set_f16(ptx::idesc_bf16_f32_ab(128, kMgN, 0, 1), f16);
                for (int j = 0; j < steps; ++j)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        ptx::mma_bf16_ss(tmem, ptx::smem_desc_sw128(sA + j * kMgAStep + kk * 32, 16, 1024),
                                         ptx::smem_desc_sw128(sB + j * kMgBStep + kk * 2048, 8192, 1024), idesc,
                                         (j | kk) != 0 ? 1u : 0u);
                ptx::mma_commit(bar_acc);
            }
        } else if (ptx::elect_one_sync()) {
            ptx::mma_commit(bar_acc);   // nothing issued: releases the epilogue's wait
        }
        __syncwarp();
    }
    // epilogue: warp w reads TMEM lanes 32 (w % 4).. = rows n0 + 32 (w % 4) + lane, columns
    // 64 (w / 4) .. + 63 (one first-level block); its codes and constant load before the wait
    const int quad = warp & 3, half = warp >> 2;
    const int64_t n = n0 + quad * 32 + lane;
    const int64_t flat = n * K + k0 + half * 64;
    uint4 cw[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
    float c1p = 0.f;
    if (n < N) {
        cw[0] = reinterpret_cast<const uint4*>(codes + (flat >> 1))[0];
        cw[1] = reinterpret_cast<const uint4*>(codes + (flat >> 1))[1];
        const int64_t blk = flat >> 6;
        c1p = c1f ? c1f[blk] : rebuild_c1(c1_codes[blk], c2[blk >> 8], *mu_p);
    }
    const bool acc_ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_acc, 0, abort, err));
    ptx::tc_fence_after();
    if (acc_ok && !*abort) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            uint32_t v[32];
            ptx::tmem_ld_32x32b_x32(tmem + ((uint32_t)(quad * 32) << 16) + half * 64 + c * 32, v);
            ptx::tmem_ld_wait();
            if (n >= N) continue;
            const uint32_t wds[4] = {cw[c].x, cw[c].y, cw[c].z, cw[c].w};
            uint32_t o[16];
#pragma unroll
            for (int b = 0; b < 16; ++b) {
                const uint32_t byte = (wds[b >> 2] >> (8 * (b & 3))) & 0xFFu;
                const float w0 = from16(dequant_bits(q[byte >> 4], c1p, f16), f16);     // element 2b
                const float w1 = from16(dequant_bits(q[byte & 0xFu], c1p, f16), f16);   // element 2b + 1
                const float y0 = __fadd_rn(w0, __fmul_rn(s, __uint_as_float(v[2 * b])));
                const float y1 = __fadd_rn(w1, __fmul_rn(s, __uint_as_float(v[2 * b + 1])));
                o[b] = pack16x2_rn(y0, y1, f16);
            }
            uint4* dst = reinterpret_cast<uint4*>(out + flat + c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (*abort && threadIdx.x == 0) ptx::mbar_wait_drain(bar_full, 0);   // copies in flight land first
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kMgN);
    }
}

}  // namespace

qlora_status launch_merge(const qlora_nf4_weight* w, const void* A, const void* B, int32_t r, float scale,
                          void* W_out, cudaStream_t stream) {
    const int64_t N = w->N, K = w->K;
    const bool tc = r % 8 == 0 && K % kMgN == 0 &&
                    (reinterpret_cast<uintptr_t>(A) & 15u) == 0 && (reinterpret_cast<uintptr_t>(B) & 15u) == 0;
    if (tc) {
        // B [N, r] (ranks contiguous; rows >= N and ranks >= r read as zero) and A [r, K]
        CUtensorMap tmB, tmA;
        if (!make_tmap_2d(&tmB, true, B, (uint64_t)r, (uint64_t)N, (uint64_t)r * 2, 64, 128, true))
            return QLORA_ERR_CUDA;
        if (!make_tmap_2d(&tmA, true, A, (uint64_t)K, (uint64_t)r, (uint64_t)K * 2, 64, 64, true))
            return QLORA_ERR_CUDA;
        static bool configured = false;
        if (!configured) {
            if (cudaFuncSetAttribute(merge_lora_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)mg_alloc(4)) !=
                cudaSuccess)
                return QLORA_ERR_CUDA;
            configured = true;
        }
        uint32_t* err = device_error_word();
        if (!err) return QLORA_ERR_CUDA;
        const dim3 grid((unsigned)(K / kMgN), (unsigned)((N + 127) / 128));
        const int steps = (r + 63) / 64;
        merge_lora_tc<<<grid, kMgThreads, mg_alloc(steps), stream>>>(
            tmB, tmA, w->codes, w->c1_codes, w->c2, w->mu, w->c1, N, K, steps, scale,
            static_cast<uint16_t*>(W_out), err, host_tables(w->codebook), w->compute_dtype == QLORA_DTYPE_F16);
        QLORA_CHECK_LAUNCH();
        return QLORA_OK;
    }
    const dim3 grid((unsigned)(K / kTile), (unsigned)((N + kTile - 1) / kTile));
    merge_lora<<<grid, kMergeThreads, 0, stream>>>(
        w->codes, w->c1_codes, w->c2, w->mu, w->c1, N, K, static_cast<const uint16_t*>(A),
        static_cast<const uint16_t*>(B), r, scale, static_cast<uint16_t*>(W_out), host_tables(w->codebook),
        w->compute_dtype == QLORA_DTYPE_F16);
    QLORA_CHECK_LAUNCH();
    return QLORA_OK;
}

}  // namespace qlora
