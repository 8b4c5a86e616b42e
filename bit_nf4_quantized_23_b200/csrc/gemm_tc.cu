// Fused NF4-dequant GEMM on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Forward ("QLoRA 的原理是什么？4-bit 量化权重真的参与训练吗？", section 7: the 4-bit
// frozen weight is dequantized to BF16 for the matmul, the LoRA path is added
// to the output):
//     Y[M,N]  = X[M,K] W_hat[N,K]^T  +  U2[M,2R] B2[N,2R]^T
// Backward dX ("Science Depth M5-131", section 4 (1): on-the-fly dequantization
// in the backward pass too):
//     dX[M,K] = dY[M,N] W_hat[N,K]   +  dU2[M,2R] A2[2R,K]
// where U2 = [hi | lo] bf16 split of s*U (and dU2 of dU), B2 = [B | B] and
// A2 = [A ; A], each half zero-padded from r to R columns/rows, so that the
// low-rank term is computed by the tensor cores at ~fp32 accuracy as R extra
// reduction steps accumulated into the same fp32 TMEM accumulator.
//
// CTA tile: BM = 128*NUM_ACC rows of the output (tokens) x BN = 256 columns;
// one or two 128-row fp32 accumulators (256 TMEM columns each).  K-steps of 64
// reduction elements; STAGES-deep shared-memory ring:
//   A stage  [BM x 64] bf16, 128-byte swizzled rows, loaded by TMA;
//   B stage  [256 x 64] (forward: rows n, K-major) or four [64 x 64] images
//            (dX: rows = reduction n, MN-major with 64-wide MN chunks 8 KiB
//            apart), written either by the dequant warps from the NF4 codes
//            or by TMA for the LoRA segment: the two give identical images;
//   codes    the packed 4-bit codes of the B stage (8 KiB), loaded by TMA.
// Warp roles (192 threads): warp 0 lane 0 issues TMA; warp 1 owns TMEM and
// its lane 0 issues tcgen05.mma; warps 2-5 expand NF4 -> bf16 (one NF4 block
// of 64 weights per unit, through a 16-entry per-block lookup table held in
// byte-split registers and selected with byte permutes), then run the
// epilogue (TMEM -> registers -> global, bf16 or fp32).
// No TMA multicast is used anywhere.
#include <cuda.h>

#include "qlora_internal.cuh"
#include "tc_ptx.cuh"
#include "gemm_tc.cuh"

namespace qlora {
namespace {

constexpr int kBN = 256;
constexpr int kStages = 3;
constexpr int kThreads = 192;
constexpr uint32_t kBStageBytes = 256 * 128;
constexpr uint32_t kCodesStageBytes = 8192;

template <int NUM_ACC>
struct Layout {
    static constexpr uint32_t kBM = 128 * NUM_ACC;
    static constexpr uint32_t kAStageBytes = kBM * 128;
    static constexpr uint32_t kA = 0;
    static constexpr uint32_t kB = kA + kStages * kAStageBytes;
    static constexpr uint32_t kCodes = kB + kStages * kBStageBytes;
    static constexpr uint32_t kBars = kCodes + kStages * kCodesStageBytes;   // 8-byte aligned
    // barriers: full_a[S], full_b[S], empty[S], acc_full; then tmem slot and abort flag
    static constexpr uint32_t kTmemSlot = kBars + (3 * kStages + 1) * 8;
    static constexpr uint32_t kAbort = kTmemSlot + 4;
    static constexpr uint32_t kBytes = kAbort + 4;
    static constexpr uint32_t kAlloc = kBytes + 1024;      // slack for 1024-byte alignment
};

// prmt.b32 in its default mode: byte i of the result is source byte (s_i & 7)
// of {y, x}; when bit 3 of the selector nibble s_i is set, that byte's sign bit
// is replicated over all 8 bits.  (The __byte_perm intrinsic ignores bit 3, so
// the sign-replicating selectors below need the instruction itself.)
__device__ __forceinline__ uint32_t prmt(uint32_t x, uint32_t y, uint32_t s) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(x), "r"(y), "r"(s));
    return r;
}

struct Lut {
    uint32_t L[4], H[4];   // low / high bytes of the 16 bf16 entries, 4 entries per register
};

__device__ __forceinline__ void build_lut(Lut& t, float c1p, const NF4Tables& tb) {
    uint32_t P[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
        P[j] = pack_bf16x2_rn(__fmul_rn(tb.q[2 * j], c1p), __fmul_rn(tb.q[2 * j + 1], c1p));
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        t.L[j] = prmt(P[2 * j], P[2 * j + 1], 0x6420);
        t.H[j] = prmt(P[2 * j], P[2 * j + 1], 0x7531);
    }
}

// 8 codes (4 packed bytes, element 2j in the high nibble of byte j) -> 8 bf16.
__device__ __forceinline__ uint4 expand8(uint32_t w, const Lut& t) {
    const uint32_t s = ((w >> 4) & 0x0F0F0F0Fu) | ((w << 4) & 0xF0F0F0F0u);   // nibble i = element i
    uint32_t o[4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint32_t sh = s >> (16 * h);
        const uint32_t sel = sh & 0x7777u;
        const uint32_t mask = prmt(sh << 4, sh, 0xD9C8);    // 0xFF bytes where code >= 8 (sign replicate)
        const uint32_t la = prmt(t.L[0], t.L[1], sel);
        const uint32_t lb = prmt(t.L[2], t.L[3], sel);
        const uint32_t ha = prmt(t.H[0], t.H[1], sel);
        const uint32_t hb = prmt(t.H[2], t.H[3], sel);
        const uint32_t lo = (la & ~mask) | (lb & mask);
        const uint32_t hi = (ha & ~mask) | (hb & mask);
        o[2 * h] = prmt(lo, hi, 0x5140);
        o[2 * h + 1] = prmt(lo, hi, 0x7362);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
                 : "memory");
    return v;
}

// Expand one NF4 block (64 weights of one W row) into one 128-byte swizzled
// row of a B image.  code_lo/code_hi: the two 16-byte halves of its codes.
__device__ __forceinline__ void expand_block_row(uint32_t row_addr, uint32_t row_in_atom, uint4 c0, uint4 c1,
                                                 const Lut& t) {
    const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int c = 0; c < 8; ++c) st_shared_v4(row_addr + ((c ^ row_in_atom) << 4), expand8(w[c], t));
}

__device__ __forceinline__ void zero_row(uint32_t row_addr) {
#pragma unroll
    for (int c = 0; c < 8; ++c) st_shared_v4(row_addr + (c << 4), make_uint4(0, 0, 0, 0));
}

template <int NUM_ACC, bool DX>
__global__ void __launch_bounds__(kThreads, 1)
tc_gemm_nf4(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmCodes,
            const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1, TcGemmParams p) {
    using L = Layout<NUM_ACC>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base = (ptx::smem_addr(smem_raw) + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - ptx::smem_addr(smem_raw));
    const uint32_t sA = base + L::kA, sB = base + L::kB, sCodes = base + L::kCodes;
    const uint32_t bar_full_a = base + L::kBars;
    const uint32_t bar_full_b = bar_full_a + 8 * kStages;
    const uint32_t bar_empty = bar_full_b + 8 * kStages;
    const uint32_t bar_acc = bar_empty + 8 * kStages;
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gbase + L::kTmemSlot);
    volatile int* abort = reinterpret_cast<volatile int*>(gbase + L::kAbort);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n0 = (int64_t)blockIdx.x * kBN;        // output column tile
    const int64_t m0 = (int64_t)blockIdx.y * L::kBM;     // output row tile
    const int ks0 = p.ksteps0, ktotal = p.ksteps0 + p.ksteps1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(bar_full_a + 8 * s, 1);
            ptx::mbar_init(bar_full_b + 8 * s, 4);
            ptx::mbar_init(bar_empty + 8 * s, 1);
        }
        ptx::mbar_init(bar_acc, 1);
        *abort = 0;
        ptx::fence_barrier_init();
        ptx::fence_proxy_async_smem();
        ptx::tma_prefetch_map(&tmA0);
        ptx::tma_prefetch_map(&tmCodes);
        ptx::tma_prefetch_map(&tmA1);
        ptx::tma_prefetch_map(&tmB1);
    }
    if (warp == 1) {
        ptx::tmem_alloc(base + L::kTmemSlot, 256 * NUM_ACC);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            for (int it = 0; it < ktotal; ++it) {
                const int s = it % kStages;
                const uint32_t ph = (uint32_t)(it / kStages) & 1u;
                if (!ptx::mbar_wait(bar_empty + 8 * s, ph ^ 1u, abort, p.err)) break;
                const uint32_t fa = bar_full_a + 8 * s;
                const uint32_t a_dst = sA + s * L::kAStageBytes;
                const uint32_t b_dst = sB + s * kBStageBytes;
                if (it < ks0) {
                    ptx::mbar_arrive_expect_tx(fa, L::kAStageBytes + kCodesStageBytes);
                    ptx::tma_load_2d(a_dst, &tmA0, it * 64, (int32_t)m0, fa);
                    if (!DX) ptx::tma_load_2d(sCodes + s * kCodesStageBytes, &tmCodes, it * 32, (int32_t)n0, fa);
                    else ptx::tma_load_2d(sCodes + s * kCodesStageBytes, &tmCodes, (int32_t)(n0 / 2), it * 64, fa);
                } else {
                    const int j = it - ks0;
                    ptx::mbar_arrive_expect_tx(fa, L::kAStageBytes + kBStageBytes);
                    ptx::tma_load_2d(a_dst, &tmA1, j * 64, (int32_t)m0, fa);
                    if (!DX) {
                        ptx::tma_load_2d(b_dst, &tmB1, j * 64, (int32_t)n0, fa);
                    } else {
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            ptx::tma_load_2d(b_dst + c * 8192, &tmB1, (int32_t)(n0 + c * 64), j * 64, fa);
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_bf16_f32(128, kBN, DX ? 1 : 0);
            bool ok = true;
            for (int it = 0; it < ktotal && ok; ++it) {
                const int s = it % kStages;
                const uint32_t ph = (uint32_t)(it / kStages) & 1u;
                ok = ptx::mbar_wait(bar_full_a + 8 * s, ph, abort, p.err);
                if (ok && it < ks0) ok = ptx::mbar_wait(bar_full_b + 8 * s, ph, abort, p.err);
                if (!ok) break;
                ptx::tc_fence_after();
                const uint32_t a_base = sA + s * L::kAStageBytes;
                const uint32_t b_base = sB + s * kBStageBytes;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t bdesc = DX ? ptx::smem_desc_sw128(b_base + kk * 2048, 8192, 1024)
                                              : ptx::smem_desc_sw128(b_base + kk * 32, 16, 1024);
#pragma unroll
                    for (int h = 0; h < NUM_ACC; ++h) {
                        const uint64_t adesc = ptx::smem_desc_sw128(a_base + h * 16384 + kk * 32, 16, 1024);
                        ptx::mma_bf16_ss(tmem + h * 256, adesc, bdesc, idesc, (it | kk) != 0 ? 1u : 0u);
                    }
                }
                ptx::mma_commit(bar_empty + 8 * s);
            }
            ptx::mma_commit(bar_acc);   // arrives when every issued MMA has completed
        }
    } else {
        // ------------------------------------------------------------ dequant producers
        // Unit u of thread t: forward: B row (t + 128u), i.e. W row n0 + row, K-block it;
        // dX: W row it*64 + (t & 63), K-block (n0 + 64*kc)/64 with kc = (t >> 6) + 2u.
        // The block constants of step it+1 are loaded while step it is expanded.
        const int t = threadIdx.x - 64;        // 0..127
        const float mu = *p.mu;
        const int64_t blocks_per_row = p.WK / 64;
        uint32_t row_u[2], img_u[2], kc_u[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            if (!DX) {
                row_u[u] = (uint32_t)(t + 128 * u);
                img_u[u] = row_u[u] * 128u;
                kc_u[u] = 0;
            } else {
                row_u[u] = (uint32_t)(t & 63);
                kc_u[u] = (uint32_t)((t >> 6) + 2 * u);
                img_u[u] = kc_u[u] * 8192u + row_u[u] * 128u;
            }
        }
        // block index of unit u at step it, or -1 when the unit lies outside W
        auto unit_block = [&](int u, int it) -> int64_t {
            const int64_t n = DX ? (int64_t)it * 64 + row_u[u] : n0 + row_u[u];
            const int64_t k = DX ? n0 + (int64_t)kc_u[u] * 64 : (int64_t)it * 64;
            return (n < p.WN && k < p.WK) ? n * blocks_per_row + (k >> 6) : -1;
        };
        uint32_t code_nx[2] = {0, 0};
        float c2_nx[2] = {0.f, 0.f};
        int64_t blk_nx[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            blk_nx[u] = ks0 > 0 ? unit_block(u, 0) : -1;
            if (blk_nx[u] >= 0) {
                code_nx[u] = __ldg(p.c1_codes + blk_nx[u]);
                c2_nx[u] = __ldg(p.c2 + (blk_nx[u] >> 8));
            }
        }
        bool ok = true;
        for (int it = 0; it < ks0 && ok; ++it) {
            const int s = it % kStages;
            const uint32_t ph = (uint32_t)(it / kStages) & 1u;
            int64_t blk_cur[2];
            float c1p_u[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                blk_cur[u] = blk_nx[u];
                c1p_u[u] = blk_cur[u] >= 0 ? rebuild_c1(code_nx[u], c2_nx[u], mu) : 0.f;
                blk_nx[u] = (it + 1 < ks0) ? unit_block(u, it + 1) : -1;
                if (blk_nx[u] >= 0) {
                    code_nx[u] = __ldg(p.c1_codes + blk_nx[u]);
                    c2_nx[u] = __ldg(p.c2 + (blk_nx[u] >> 8));
                }
            }
            ok = ptx::mbar_wait(bar_full_a + 8 * s, ph, abort, p.err);
            ok = __all_sync(0xffffffffu, ok);          // leave the loop as a whole warp
            if (!ok) break;
            const uint32_t b_base = sB + s * kBStageBytes;
            const uint32_t c_base = sCodes + s * kCodesStageBytes;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const uint32_t row_addr = b_base + img_u[u];
                if (blk_cur[u] < 0) {
                    zero_row(row_addr);
                    continue;
                }
                uint4 c0, c1;
                if (!DX) {
                    // codes tile: 256 rows x 32 bytes, unswizzled; stagger the two halves to avoid bank conflicts
                    const uint32_t src = c_base + row_u[u] * 32u;
                    const uint32_t first = (row_u[u] >> 2) & 1u;
                    const uint4 x = ld_shared_v4(src + first * 16u);
                    const uint4 y = ld_shared_v4(src + (first ^ 1u) * 16u);
                    c0 = first ? y : x;
                    c1 = first ? x : y;
                } else {
                    // codes tile: 64 rows x 128 bytes, 128-byte swizzled; this unit's 32 bytes are chunks 2kc, 2kc+1
                    const uint32_t src = c_base + row_u[u] * 128u;
                    c0 = ld_shared_v4(src + (((2u * kc_u[u]) ^ (row_u[u] & 7u)) << 4));
                    c1 = ld_shared_v4(src + (((2u * kc_u[u] + 1u) ^ (row_u[u] & 7u)) << 4));
                }
                Lut lut;
                build_lut(lut, c1p_u[u], p.tb);
                expand_block_row(row_addr, row_u[u] & 7u, c0, c1, lut);
            }
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar_full_b + 8 * s);
        }

        // ------------------------------------------------------------ epilogue
        const bool acc_ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_acc, 0, abort, p.err));
        ptx::tc_fence_after();
        if (acc_ok) {
            const uint32_t quad = (uint32_t)(warp & 3);
#pragma unroll 1
            for (int h = 0; h < NUM_ACC; ++h) {
                const int64_t m = m0 + h * 128 + quad * 32 + lane;
#pragma unroll 1
                for (int c = 0; c < kBN / 32; ++c) {
                    const int64_t nb = n0 + c * 32;
                    if (nb >= p.Nout) break;
                    uint32_t v[32];
                    ptx::tmem_ld_32x32b_x32(tmem + ((quad * 32u) << 16) + h * 256 + c * 32, v);
                    ptx::tmem_ld_wait();
                    if (m >= p.M) continue;
                    const bool full = (nb + 32 <= p.Nout);
                    if (p.out_f32) {
                        float* dst = static_cast<float*>(p.out) + m * p.ldo + nb;
                        if (full && (p.ldo & 3) == 0) {
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                reinterpret_cast<uint4*>(dst)[i] =
                                    make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                        } else {
                            for (int i = 0; i < 32 && nb + i < p.Nout; ++i) dst[i] = __uint_as_float(v[i]);
                        }
                    } else {
                        uint16_t* dst = static_cast<uint16_t*>(p.out) + m * p.ldo + nb;
                        if (full && (p.ldo & 7) == 0) {
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                uint4 o;
                                o.x = pack_bf16x2_rn(__uint_as_float(v[8 * i + 0]), __uint_as_float(v[8 * i + 1]));
                                o.y = pack_bf16x2_rn(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3]));
                                o.z = pack_bf16x2_rn(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5]));
                                o.w = pack_bf16x2_rn(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7]));
                                reinterpret_cast<uint4*>(dst)[i] = o;
                            }
                        } else {
                            for (int i = 0; i < 32 && nb + i < p.Nout; ++i)
                                dst[i] = (uint16_t)f32_to_bf16_bits_rn(__uint_as_float(v[i]));
                        }
                    }
                }
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 256 * NUM_ACC);
    }
}

// ---------------------------------------------------------------------------- host

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return (EncodeTiledFn) nullptr;
        return reinterpret_cast<EncodeTiledFn>(f);
    }();
    return fn;
}

}  // namespace

bool make_tmap_2d(CUtensorMap* map, bool bf16, const void* base, uint64_t inner, uint64_t outer,
                  uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, bool swizzle128) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
              const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NUM_ACC, bool DX>
static qlora_status launch_one(const TcGemmArgs& a, cudaStream_t stream) {
    using L = Layout<NUM_ACC>;
    static bool configured = false;   // attribute set once per instantiation (idempotent, so races are benign)
    auto kern = tc_gemm_nf4<NUM_ACC, DX>;
    if (!configured) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kAlloc) != cudaSuccess)
            return QLORA_ERR_CUDA;
        configured = true;
    }
    const dim3 grid((unsigned)((a.p.Nout + kBN - 1) / kBN), (unsigned)((a.p.M + L::kBM - 1) / L::kBM));
    kern<<<grid, kThreads, L::kAlloc, stream>>>(a.tmA0, a.tmCodes, a.tmA1, a.tmB1, a.p);
    QLORA_CHECK_LAUNCH();
    return QLORA_OK;
}

qlora_status launch_tc_gemm_nf4(TcGemmArgs& a, bool dx, cudaStream_t stream) {
    const uint32_t bm = a.p.M > 128 ? 256 : 128;
    const qlora_nf4_weight* w = a.w;
    const int64_t N = w->N, K = w->K;
    // segment 0: A (X or dY) and the packed codes
    if (!dx) {
        if (!make_tmap_2d(&a.tmA0, true, a.A0, K, a.p.M, K * 2, 64, bm, true)) return QLORA_ERR_CUDA;
        if (!make_tmap_2d(&a.tmCodes, false, w->codes, K / 2, N, K / 2, 32, 256, false)) return QLORA_ERR_CUDA;
    } else {
        if (!make_tmap_2d(&a.tmA0, true, a.A0, N, a.p.M, N * 2, 64, bm, true)) return QLORA_ERR_CUDA;
        if (!make_tmap_2d(&a.tmCodes, false, w->codes, K / 2, N, K / 2, 128, 64, true)) return QLORA_ERR_CUDA;
    }
    // segment 1: LoRA operands, [M, 2R] and [N, 2R] (forward) or [2R, K] (dX)
    const int64_t R2 = 2 * (int64_t)a.Rpad;
    if (!make_tmap_2d(&a.tmA1, true, a.A1, R2, a.p.M, R2 * 2, 64, bm, true)) return QLORA_ERR_CUDA;
    if (!dx) {
        if (!make_tmap_2d(&a.tmB1, true, a.B1, R2, N, R2 * 2, 64, 256, true)) return QLORA_ERR_CUDA;
    } else {
        if (!make_tmap_2d(&a.tmB1, true, a.B1, K, R2, K * 2, 64, 64, true)) return QLORA_ERR_CUDA;
    }
    a.p.ksteps0 = (int)(((dx ? N : K) + 63) / 64);
    a.p.ksteps1 = (int)(R2 / 64);
    a.p.c1_codes = w->c1_codes;
    a.p.c2 = w->c2;
    a.p.mu = w->mu;
    a.p.WN = N;
    a.p.WK = K;
    a.p.tb = host_tables();
    a.p.err = device_error_word();
    if (!a.p.err) return QLORA_ERR_CUDA;
    if (bm == 256) return dx ? launch_one<2, true>(a, stream) : launch_one<2, false>(a, stream);
    return dx ? launch_one<1, true>(a, stream) : launch_one<1, false>(a, stream);
}

}  // namespace qlora
