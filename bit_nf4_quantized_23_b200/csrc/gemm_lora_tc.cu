// LoRA-side GEMMs of the QLoRA linear layer on the tcgen05 tensor cores.
//
// The low-rank products ("QLoRA 的原理是什么？4-bit 量化权重真的参与训练吗？",
// section 7: only the LoRA parameters are trained; walkthrough of "QLoRA:
// Efficient Finetuning of Quantized LLMs", section 4.4: gradients flow through
// the frozen weight into the adapters) have one dimension of size r:
//     U  = X  A^T      [M, r]    reduction over K
//     dU = s dY B      [M, r]    reduction over N
//     dA = dU^T X      [r, K]    reduction over M   (computed as dA^T [K, r])
//     dB = s dY^T U    [N, r]    reduction over M
// Each is a [rows x R] output (R = r padded to a multiple of 64) with a long
// reduction, so the reduction is split over CTAs (deterministic: every split
// writes its own fp32 partial tile, a reduce kernel adds them in fixed order).
//
// Three operand modes:
//   K-major  A [rows, red] and B [R, red], both with the reduction contiguous
//            (X with A); one MMA per 16-wide step.
//   MN-major A from S [red, rows] (X or dY, rows contiguous) and B from the
//            bf16 hi/lo split V2 [red, 2R] of dU or s*U; two MMAs per step
//            (hi then lo) into the same fp32 accumulator, so the fp32 factor
//            keeps ~16 significant bits.
//   K-major A, MN-major B: A [rows, red] and B [red, r] itself (dY with B):
//            one MMA per step; columns r .. R-1 of B read as zero.
// Roles (192 threads): warp 0 lane 0 TMA, warp 1 TMEM owner + MMA issuer,
// warps 2-5 epilogue (TMEM -> fp32 partial tile).  No TMA multicast.
#include <cuda.h>

#include "qlora_internal.cuh"
#include "tc_ptx.cuh"
#include "gemm_tc.cuh"

namespace qlora {
namespace {

constexpr int kThreads = 192;
constexpr uint32_t kAStage = 128 * 128;           // 128 rows x 64 bf16
constexpr uint32_t kMaxSmem = 227 * 1024;

// Shared-memory layout for a given B stage size and stage count: A stages, B stages, then
// barriers full[S], empty[S], acc, the TMEM slot and the abort flag (1 KiB slack for alignment).
struct LoraLayout {
    uint32_t stages, b_stage, off_b, off_bars, off_slot, off_abort, alloc;
};
__host__ __device__ inline LoraLayout lora_layout(uint32_t stages, uint32_t b_stage) {
    LoraLayout l;
    l.stages = stages;
    l.b_stage = b_stage;
    l.off_b = stages * kAStage;
    l.off_bars = l.off_b + stages * b_stage;
    l.off_slot = l.off_bars + (2 * stages + 1) * 8;
    l.off_abort = l.off_slot + 4;
    l.alloc = l.off_abort + 4 + 1024;
    return l;
}

enum : int { kModeK = 0, kModeMN = 1, kModeKA_MNB = 2 };

template <int MODE>
__global__ void __launch_bounds__(kThreads, 2)
tc_lora_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, LoraGemmParams p) {
    grid_dependency_wait();                                   // operands written by the previous kernel
    allow_dependents();
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base = (ptx::smem_addr(smem_raw) + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - ptx::smem_addr(smem_raw));
    const LoraLayout lay = lora_layout(p.stages, p.b_stage);
    const int kStages = (int)lay.stages;
    const uint32_t kBStage = lay.b_stage;
    const uint32_t sA = base, sB = base + lay.off_b;
    const uint32_t bar_full = base + lay.off_bars;
    const uint32_t bar_empty = bar_full + 8 * kStages;
    const uint32_t bar_acc = bar_empty + 8 * kStages;
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gbase + lay.off_slot);
    volatile int* abort = reinterpret_cast<volatile int*>(gbase + lay.off_abort);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int R = p.R;
    const int64_t row0 = (int64_t)blockIdx.x * 128;
    const int k_begin = blockIdx.y * p.ksteps_per_split;
    const int k_end = min(p.ksteps_total, k_begin + p.ksteps_per_split);
    const int nk = k_end - k_begin;
    const uint32_t tmem_cols = p.tmem_cols;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(bar_full + 8 * s, 1);
            ptx::mbar_init(bar_empty + 8 * s, 1);
        }
        ptx::mbar_init(bar_acc, 1);
        *abort = 0;
        ptx::fence_barrier_init();
        ptx::fence_proxy_async_smem();
        ptx::tma_prefetch_map(&tmA);
        ptx::tma_prefetch_map(&tmB);
    }
    if (warp == 1) {
        ptx::tmem_alloc(base + lay.off_slot, tmem_cols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // TMA issuer: the whole warp runs the loop, one elected lane issues the copies
        constexpr bool MN = MODE == kModeMN;
        const uint32_t b_bytes = MN ? (uint32_t)R * 256u : (uint32_t)R * 128u;
        int issued = 0;
        for (int i = 0; i < nk; ++i) {
            const int s = i % kStages;
            const uint32_t ph = (uint32_t)(i / kStages) & 1u;
            if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar_empty + 8 * s, ph ^ 1u, abort, p.err))) break;
            issued = i + 1;
            if (ptx::elect_one_sync()) {
                const uint32_t fb = bar_full + 8 * s;
                const int ks = k_begin + i;
                const uint32_t a_dst = sA + s * kAStage, b_dst = sB + s * kBStage;
                ptx::mbar_arrive_expect_tx(fb, kAStage + b_bytes);
                if (MODE == kModeK) {
                    ptx::tma_load_2d(a_dst, &tmA, ks * 64, (int32_t)row0, fb);
                    ptx::tma_load_2d(b_dst, &tmB, ks * 64, 0, fb);
                } else if (MODE == kModeKA_MNB) {
                    ptx::tma_load_2d(a_dst, &tmA, ks * 64, (int32_t)row0, fb);
                    for (int c = 0; c < R / 64; ++c) ptx::tma_load_2d(b_dst + c * 8192, &tmB, c * 64, ks * 64, fb);
                } else {
                    ptx::tma_load_2d(a_dst, &tmA, (int32_t)row0, ks * 64, fb);
                    ptx::tma_load_2d(a_dst + 8192, &tmA, (int32_t)row0 + 64, ks * 64, fb);
                    const int chunks = R / 64;
                    for (int c = 0; c < chunks; ++c) {
                        ptx::tma_load_2d(b_dst + c * 8192, &tmB, c * 64, ks * 64, fb);
                        ptx::tma_load_2d(b_dst + (chunks + c) * 8192, &tmB, R + c * 64, ks * 64, fb);
                    }
                }
            }
            __syncwarp();
        }
        if (*abort) {   // drain this CTA's copies in flight before it exits
            for (int i = max(0, issued - kStages); i < issued; ++i)
                ptx::mbar_wait_drain(bar_full + 8 * (i % kStages), (uint32_t)(i / kStages) & 1u);
        }
    } else if (warp == 1) {
        // MMA issuer: the whole warp runs the loop, one elected lane issues the MMAs and commits
        const uint32_t idesc = ptx::idesc_set_f16(
            ptx::idesc_bf16_f32_ab(128, R, MODE == kModeMN ? 1 : 0, MODE != kModeK ? 1 : 0), p.f16 != 0);
        bool ok = true;
        for (int i = 0; i < nk && ok; ++i) {
            const int s = i % kStages;
            const uint32_t ph = (uint32_t)(i / kStages) & 1u;
            ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_full + 8 * s, ph, abort, p.err));
            if (!ok) break;
            ptx::tc_fence_after();
            if (ptx::elect_one_sync()) {
                const uint32_t a_base = sA + s * kAStage, b_base = sB + s * kBStage;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint32_t acc = (i | kk) != 0 ? 1u : 0u;
                    if (MODE == kModeK) {
                        ptx::mma_bf16_ss(tmem, ptx::smem_desc_sw128(a_base + kk * 32, 16, 1024),
                                         ptx::smem_desc_sw128(b_base + kk * 32, 16, 1024), idesc, acc);
                    } else if (MODE == kModeKA_MNB) {   // B: R/64 MN-major 64-column images, 8 KiB apart
                        ptx::mma_bf16_ss(tmem, ptx::smem_desc_sw128(a_base + kk * 32, 16, 1024),
                                         ptx::smem_desc_sw128(b_base + kk * 2048, 8192, 1024), idesc, acc);
                    } else {
                        const uint64_t ad = ptx::smem_desc_sw128(a_base + kk * 2048, 8192, 1024);
                        ptx::mma_bf16_ss(tmem, ad, ptx::smem_desc_sw128(b_base + kk * 2048, 8192, 1024), idesc,
                                         acc);
                        ptx::mma_bf16_ss(tmem, ad,
                                         ptx::smem_desc_sw128(b_base + (R / 64) * 8192 + kk * 2048, 8192, 1024),
                                         idesc, 1u);
                    }
                }
                ptx::mma_commit(bar_empty + 8 * s);
            }
            __syncwarp();
        }
        if (ptx::elect_one_sync()) {
            ptx::mma_commit(bar_acc);
            if (*abort) ptx::mbar_wait_drain(bar_acc, 0);   // issued MMAs finish before TMEM is freed
        }
        __syncwarp();
    } else {
        const bool acc_ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_acc, 0, abort, p.err));
        ptx::tc_fence_after();
        if (acc_ok) {
            const uint32_t quad = (uint32_t)(warp & 3);
            const int64_t row = row0 + quad * 32 + lane;
            float* dst = p.partial + ((int64_t)blockIdx.y * p.rows + row) * R;
#pragma unroll 1
            for (int c = 0; c < R / 32; ++c) {
                uint32_t v[32];
                ptx::tmem_ld_32x32b_x32(tmem + ((quad * 32u) << 16) + c * 32, v);
                ptx::tmem_ld_wait();
                if (row < p.rows) {
                    uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
                    for (int i = 0; i < 8; ++i) d4[i] = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                }
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, tmem_cols);
    }
}

template <int MODE>
qlora_status launch_lora(const CUtensorMap& tmA, const CUtensorMap& tmB, LoraGemmParams& p, int splits,
                         cudaStream_t stream) {
    constexpr bool MN = MODE == kModeMN;
    static bool configured = false;
    auto kern = tc_lora_gemm<MODE>;
    if (!configured) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMaxSmem) != cudaSuccess)
            return QLORA_ERR_CUDA;
        configured = true;
    }
    // B stage: K-major R rows x 128 B or R/64 MN-major chunks of 8 KiB (the same bytes), or the hi
    // and lo MN-major images (2 x R/64 chunks of 8 KiB).
    // Two CTAs per SM (one's epilogue overlaps the other's main loop) when three or more stages
    // fit in half of the shared memory, else one CTA with up to six stages.
    const uint32_t b_stage = MN ? (uint32_t)p.R * 256u : (uint32_t)p.R * 128u;
    const uint32_t stage = kAStage + b_stage;
    uint32_t stages = (kMaxSmem / 2 - 2048) / stage;
    if (stages < 3) stages = (kMaxSmem - 2048) / stage;
    if (stages > 6) stages = 6;
    if (stages < 2) return QLORA_ERR_UNSUPPORTED;
    p.stages = stages;
    p.b_stage = b_stage;
    const LoraLayout lay = lora_layout(stages, b_stage);
    const dim3 grid((unsigned)((p.rows + 127) / 128), (unsigned)splits);
    (void)launch_dependent(kern, grid, dim3(kThreads), lay.alloc, stream, tmA, tmB, p);
    QLORA_CHECK_LAUNCH();
    return QLORA_OK;
}

}  // namespace

// CTAs per SM the launch below uses: two when three or more stages fit in half of the
// shared memory, else one.
int lora_ctas_per_sm(int R, bool mn_major) {
    const uint32_t stage = kAStage + (mn_major ? (uint32_t)R * 256u : (uint32_t)R * 128u);
    return (kMaxSmem / 2 - 2048) / stage >= 3 ? 2 : 1;
}

// SMs assumed by the split rule: B200's 148.  The split count fixes the size of the partial
// buffer in the caller's workspace, so it must not depend on which device is current when the
// size is queried.
constexpr int64_t kSplitRuleSms = 148;

// Split count of the reduction: the one with the least waves x (a CTA's fixed cost, about two
// K-steps of streaming, + its K-steps), the smallest on ties (fewer partial tiles).  A launch a
// few CTAs past one wave would otherwise run a second, nearly empty wave.
int lora_splits(int64_t rows, int ksteps_total, int R, bool mn_major) {
    const int64_t tiles = (rows + 127) / 128;
    const int64_t slots = kSplitRuleSms * (int64_t)lora_ctas_per_sm(R, mn_major);
    int best = 1;
    int64_t best_cost = INT64_MAX;
    for (int s = 1; s <= ksteps_total && s <= 64; ++s) {
        const int64_t kps = (ksteps_total + s - 1) / s;
        const int64_t eff = (ksteps_total + kps - 1) / kps;          // splits after rounding kps up
        const int64_t cost = ((tiles * eff + slots - 1) / slots) * (2 + kps);
        if (cost < best_cost) { best_cost = cost; best = (int)eff; }
    }
    return best;
}

qlora_status launch_lora_gemm(const LoraGemmArgs& a, cudaStream_t stream) {
    LoraGemmParams p{};
    p.rows = a.rows;
    p.R = a.R;
    p.ksteps_total = (int)((a.red + 63) / 64);
    const int splits = lora_splits(a.rows, p.ksteps_total, a.R, a.mn_major);
    p.ksteps_per_split = (p.ksteps_total + splits - 1) / splits;
    p.partial = a.partial;
    p.f16 = a.f16;
    p.tmem_cols = a.R <= 64 ? 64u : (a.R <= 128 ? 128u : 256u);
    p.err = device_error_word();
    if (!p.err) return QLORA_ERR_CUDA;
    CUtensorMap tmA, tmB;
    if (!a.mn_major) {
        // A [rows, red] and B [R, red], reduction contiguous
        if (!make_tmap_2d(&tmA, true, a.A, a.red, a.rows, a.lda * 2, 64, 128, true)) return QLORA_ERR_CUDA;
        if (a.b_mn) {   // B [red, b_cols] with its columns contiguous; columns past b_cols read as zero
            if (!make_tmap_2d(&tmB, true, a.B, (uint64_t)a.b_cols, a.red, a.ldb * 2, 64, 64, true)) return QLORA_ERR_CUDA;
            return launch_lora<kModeKA_MNB>(tmA, tmB, p, splits, stream);
        }
        const uint64_t b_rows = a.b_rows > 0 ? (uint64_t)a.b_rows : (uint64_t)a.R;   // rows past it read as zero
        if (!make_tmap_2d(&tmB, true, a.B, a.red, b_rows, a.ldb * 2, 64, (uint32_t)a.R, true)) return QLORA_ERR_CUDA;
        return launch_lora<kModeK>(tmA, tmB, p, splits, stream);
    }
    // S [red, rows] with rows contiguous, V2 [red, 2R] (hi | lo)
    if (!make_tmap_2d(&tmA, true, a.A, a.rows, a.red, a.lda * 2, 64, 64, true)) return QLORA_ERR_CUDA;
    if (!make_tmap_2d(&tmB, true, a.B, 2 * (uint64_t)a.R, a.red, a.ldb * 2, 64, 64, true)) return QLORA_ERR_CUDA;
    return launch_lora<kModeMN>(tmA, tmB, p, splits, stream);
}

size_t lora_partial_bytes(int64_t rows, int64_t red, int R, bool mn_major) {
    const int ks = (int)((red + 63) / 64);
    return (size_t)lora_splits(rows, ks, R, mn_major) * (size_t)rows * (size_t)R * sizeof(float);
}

}  // namespace qlora
