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
// reduction steps accumulated into the same fp32 TMEM accumulator.  B2 and A2
// are not materialised when the tensor maps can read B and A themselves (the
// hi and lo steps load the same tile; ranks past r read as zero).
//
// CTA tile: BM = 128*NUM_ACC rows of the output (tokens) x BN = 256 columns;
// one or two 128-row fp32 accumulators (256 TMEM columns each).  K-steps of 64
// reduction elements; STAGES-deep shared-memory ring:
//   A stage  [BM x 64] bf16, 128-byte swizzled rows, loaded by TMA;
//   B stage  forward: [256 x 64] rows n, K-major: written by the dequant warps
//            as a non-swizzled image (8-row core matrices, chunk c of every row
//            at 4096 c), or loaded by TMA with 128-byte swizzle for the LoRA
//            steps (the MMA takes the matching descriptor per step);
//            dX: four [64 x 64] images (rows = reduction n, MN-major, 64-wide
//            MN chunks 8 KiB apart, 128-byte swizzled), written by the dequant
//            warps or by TMA for the LoRA steps, the two alike;
//   codes    the packed 4-bit codes of the B stage (8 KiB), loaded by TMA.
// Warp roles (320 threads): warp 0 issues TMA; warp 1 owns TMEM and issues
// tcgen05.mma (each loop runs on the whole warp, one elected lane issues);
// warps 2-9 expand NF4 -> bf16 (one NF4 block of 64 weights per thread and
// K-step, through a 16-entry per-block lookup table held in byte-split
// registers and selected with byte permutes), then run the epilogue (TMEM ->
// registers -> global, bf16 or fp32).  CTAs take output tiles in a grouped
// order (row tiles fastest within groups of 16) so concurrent CTAs share W.
// No TMA multicast is used anywhere.
#include <algorithm>
#include <climits>
#include <cstdlib>

#include <cuda.h>

#include "qlora_internal.cuh"
#include "tc_ptx.cuh"
#include "gemm_tc.cuh"

namespace qlora {
namespace {

constexpr int kBN = 256;
constexpr int kStages = 3;
constexpr int kProducerWarps = 8;             // fused GEMM: 8 producer/epilogue warps
constexpr int kGemmThreads = 64 + 32 * kProducerWarps;
constexpr int kGemmPrefetch = 2;              // block constants are loaded this many K-steps ahead
constexpr uint32_t kBStageBytes = 256 * 128;
constexpr uint32_t kCodesStageBytes = 8192;

template <int NUM_ACC>
struct Layout {
    static constexpr uint32_t kBM = 128 * NUM_ACC;
    static constexpr uint32_t kAStageBytes = kBM * 128;
    static constexpr uint32_t kA = 0;
    static constexpr uint32_t kB = kA + kStages * kAStageBytes;
    static constexpr uint32_t kCodes = kB + kStages * kBStageBytes;
    static constexpr uint32_t kE4 = kCodes + kStages * kCodesStageBytes;     // E4M3 values [256] fp32
    static constexpr uint32_t kBars = kE4 + 256 * 4;                         // 8-byte aligned
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

__device__ __forceinline__ void build_lut(Lut& t, float c1p, const NF4Tables& tb, bool f16) {
    uint32_t P[8];   // entries 2j, 2j+1 rounded to the compute dtype (bf16 or fp16), packed
    const float2 c2p = make_float2(c1p, c1p);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float2 e = mul2_rn(make_float2(tb.q[2 * j], tb.q[2 * j + 1]), c2p);   // fp32(q * c1'), per element
        P[j] = pack16x2_rn(e.x, e.y, f16);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        t.L[j] = prmt(P[2 * j], P[2 * j + 1], 0x6420);
        t.H[j] = prmt(P[2 * j], P[2 * j + 1], 0x7531);
    }
}

// 8 codes (4 packed bytes, element 2j in the high nibble of byte j) -> 8 bf16.
// The nibbles of w run e1, e0, e3, e2, ... from the least significant end; the
// table permutes keep that pair-swapped order and the final interleave undoes
// it.  Bytes whose code is >= 8 take entries 8-15 (sign-replicated bit 3).
__device__ __forceinline__ uint4 expand8(uint32_t w, const Lut& t) {
    const uint32_t u = w << 4;             // bit 3 of the low nibble of each byte -> that byte's bit 7
    const uint32_t wm = w & 0x77777777u;   // table index of every code; prmt reads selector bits 0-15
    uint32_t o[4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint32_t sel = h == 0 ? wm : (wm >> 16);
        const uint32_t mask = prmt(u, w, h == 0 ? 0xD9C8u : 0xFBEAu);
        const uint32_t la = prmt(t.L[0], t.L[1], sel);
        const uint32_t lb = prmt(t.L[2], t.L[3], sel);
        const uint32_t ha = prmt(t.H[0], t.H[1], sel);
        const uint32_t hb = prmt(t.H[2], t.H[3], sel);
        const uint32_t lo = (la & ~mask) | (lb & mask);
        const uint32_t hi = (ha & ~mask) | (hb & mask);
        o[2 * h] = prmt(lo, hi, 0x4051);
        o[2 * h + 1] = prmt(lo, hi, 0x6273);
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

// The same row in a non-swizzled K-major image (rows 16 bytes apart, chunk c of
// every row LBO bytes after chunk 0): the eight stores take immediate offsets from
// one address, and a warp's 32 rows fill 512 contiguous bytes per chunk.
template <uint32_t LBO>
__device__ __forceinline__ void expand_block_row_kn(uint32_t row_addr, uint4 c0, uint4 c1, const Lut& t) {
    const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int c = 0; c < 8; ++c) st_shared_v4(row_addr + c * LBO, expand8(w[c], t));
}

template <uint32_t LBO>
__device__ __forceinline__ void zero_row_kn(uint32_t row_addr) {
#pragma unroll
    for (int c = 0; c < 8; ++c) st_shared_v4(row_addr + c * LBO, make_uint4(0, 0, 0, 0));
}

// Output tile of CTA t: row tiles run fastest within groups of kRasterGroup of them, so the
// CTAs resident at one time share a W strip (read from HBM once, then from L2) and keep the
// group's activation panel resident in L2 across the column tiles.
constexpr int64_t kRasterGroup = 16;
__device__ __forceinline__ void raster_tile(int64_t t, int64_t mtiles, int64_t ntiles, int64_t& mt, int64_t& nt) {
    const int64_t per_group = kRasterGroup * ntiles;
    const int64_t first = (t / per_group) * kRasterGroup;
    const int64_t gm = min(mtiles - first, kRasterGroup);
    const int64_t local = t % per_group;
    mt = first + local % gm;
    nt = local / gm;
}

// Store 32 consecutive output columns nb .. nb+31 of row m (fp32, or rounded to the 16-bit
// compute dtype); columns at or past nlim (the end of the tile or of the row) are skipped.
__device__ __forceinline__ void store_row32(const TcGemmParams& p, int64_t m, int64_t nb, int64_t nlim,
                                            const uint32_t (&v)[32]) {
    const bool full = (nb + 32 <= nlim);
    if (p.out_f32) {
        float* dst = static_cast<float*>(p.out) + m * p.ldo + nb;
        if (full && (p.ldo & 3) == 0) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                reinterpret_cast<uint4*>(dst)[i] = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (nb + i < nlim) dst[i] = __uint_as_float(v[i]);
        }
    } else {
        uint16_t* dst = static_cast<uint16_t*>(p.out) + m * p.ldo + nb;
        const bool h = p.f16 != 0;
        if (full && (p.ldo & 7) == 0) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint4 o;
                o.x = pack16x2_rn(__uint_as_float(v[8 * i + 0]), __uint_as_float(v[8 * i + 1]), h);
                o.y = pack16x2_rn(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3]), h);
                o.z = pack16x2_rn(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5]), h);
                o.w = pack16x2_rn(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7]), h);
                reinterpret_cast<uint4*>(dst)[i] = o;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (nb + i < nlim) dst[i] = (uint16_t)to16_rn(__uint_as_float(v[i]), h);
        }
    }
}

template <int NUM_ACC, bool DX>
__global__ void __launch_bounds__(kGemmThreads, 1)
tc_gemm_nf4(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmCodes,
            const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1, TcGemmParams p) {
    grid_dependency_wait();                                   // operands written by the previous kernel
    allow_dependents();
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
    int64_t mt, nt;
    raster_tile(blockIdx.x, (p.M + L::kBM - 1) / L::kBM, (p.Nout + kBN - 1) / kBN, mt, nt);
    const int64_t n0 = nt * kBN;                          // output column tile
    const int64_t m0 = mt * L::kBM;                       // output row tile
    const int ks0 = p.ksteps0, ktotal = p.ksteps0 + p.ksteps1;
    float* e4tab = reinterpret_cast<float*>(gbase + L::kE4);
    if (threadIdx.x < 256) e4tab[threadIdx.x] = e4m3_to_f32(threadIdx.x);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(bar_full_a + 8 * s, 1);
            ptx::mbar_init(bar_full_b + 8 * s, kProducerWarps);
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
        // (the whole warp runs the loop; one elected lane issues the copies)
        int issued = 0;
        int s = 0;
        uint32_t ph = 0;
        for (int it = 0; it < ktotal; ++it) {
            if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar_empty + 8 * s, ph ^ 1u, abort, p.err))) break;
            issued = it + 1;
            if (ptx::elect_one_sync()) {
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
                    const int jb = p.b1_wrap ? j % p.b1_wrap : j;   // hi and lo steps share the B1 tile
                    ptx::mbar_arrive_expect_tx(fa, L::kAStageBytes + kBStageBytes);
                    ptx::tma_load_2d(a_dst, &tmA1, j * 64, (int32_t)m0, fa);
                    if (!DX) {
                        ptx::tma_load_2d(b_dst, &tmB1, jb * 64, (int32_t)n0, fa);
                    } else {
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            ptx::tma_load_2d(b_dst + c * 8192, &tmB1, (int32_t)(n0 + c * 64), jb * 64, fa);
                    }
                }
            }
            __syncwarp();
            if (++s == kStages) { s = 0; ph ^= 1u; }
        }
        if (*abort) {   // drain this CTA's copies in flight before it exits
            for (int it = max(0, issued - kStages); it < issued; ++it)
                ptx::mbar_wait_drain(bar_full_a + 8 * (it % kStages), (uint32_t)(it / kStages) & 1u);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // (the whole warp runs the loop; one elected lane issues the MMAs and their commits;
        // descriptors are built once and advanced by stage offsets: start address >> 4 in
        // the low 14 bits, every shared address is below 256 KiB, so no carry leaves them)
        const uint32_t idesc = ptx::idesc_set_f16(ptx::idesc_bf16_f32(128, kBN, DX ? 1 : 0), p.f16 != 0);
        const uint64_t adesc0 = ptx::smem_desc_sw128(sA, 16, 1024);
        const uint64_t bdesc0 = DX ? ptx::smem_desc_sw128(sB, 8192, 1024) : ptx::smem_desc_sw128(sB, 16, 1024);
        const uint64_t bdesc0_kn = ptx::smem_desc_kmajor_none(sB, kBN * 16, 128);   // forward W_hat steps
        bool ok = true;
        int s = 0;
        uint32_t ph = 0;
        for (int it = 0; it < ktotal && ok; ++it) {
            bool w = ptx::mbar_wait(bar_full_a + 8 * s, ph, abort, p.err);
            if (w && it < ks0) w = ptx::mbar_wait(bar_full_b + 8 * s, ph, abort, p.err);
            ok = __all_sync(0xffffffffu, w);
            if (!ok) break;
            ptx::tc_fence_after();
            if (ptx::elect_one_sync()) {
                const uint64_t ad = adesc0 + ((uint32_t)s * (L::kAStageBytes >> 4));
                const bool kn = !DX && it < ks0;
                const uint64_t bd = (kn ? bdesc0_kn : bdesc0) + ((uint32_t)s * (kBStageBytes >> 4));
                const uint32_t kstep = DX ? (2048 >> 4) : kn ? ((2 * kBN * 16) >> 4) : (32 >> 4);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t bdesc = bd + kk * kstep;
#pragma unroll
                    for (int h = 0; h < NUM_ACC; ++h)
                        ptx::mma_bf16_ss(tmem + h * 256, ad + h * (16384 >> 4) + kk * (32 >> 4), bdesc, idesc,
                                         (it | kk) != 0 ? 1u : 0u);
                }
                ptx::mma_commit(bar_empty + 8 * s);
            }
            __syncwarp();
            if (++s == kStages) { s = 0; ph ^= 1u; }
        }
        if (ptx::elect_one_sync()) {
            ptx::mma_commit(bar_acc);   // arrives when every issued MMA has completed
            if (*abort) ptx::mbar_wait_drain(bar_acc, 0);   // issued MMAs finish before TMEM is freed
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ dequant producers
        // Thread t (0..255) owns one unit per K-step: forward: B row t = W row n0 + t, K-block it;
        // dX: W row it*64 + (t & 63), K-block (n0 + 64*kc)/64 with kc = t >> 6.
        // The block constants are loaded kGemmPrefetch K-steps ahead (register queue).
        const int t = threadIdx.x - 64;
        const float mu = p.c1f ? 0.f : *p.mu;
        const int64_t blocks_per_row = p.WK / 64;
        const uint32_t row = DX ? (uint32_t)(t & 63) : (uint32_t)t;
        const uint32_t kc = DX ? (uint32_t)(t >> 6) : 0u;
        // forward: non-swizzled K-major image (row t at 16 t, chunk c at 4096 c);
        // dX: 128-byte-swizzled 64-row images, one per K-block, read as an MN-major operand
        const uint32_t img = DX ? kc * 8192u + row * 128u : row * 16u;
        // The unit of K-step `ahead` (the one whose constants load next): its first-level
        // block index moves by a fixed stride per step (forward: the next block of the same
        // W row; dX: the same K-block 64 W rows further), and it exists when the thread's
        // W row (forward) or K-block (dX) is in range, and in dX its row a_n < N.
        const bool lane_ok = DX ? (n0 + (int64_t)kc * 64 < p.WK) : (n0 + row < p.WN);
        const int64_t blk_step = DX ? 64 * blocks_per_row : 1;
        int64_t a_blk = DX ? (int64_t)row * blocks_per_row + (n0 >> 6) + kc : (n0 + row) * blocks_per_row;
        int64_t a_n = row;
        auto const_load = [&](int ahead, bool& v, uint32_t& code, float& c2) {
            v = lane_ok && ahead < ks0 && (!DX || a_n < p.WN);
            code = 0;
            c2 = 0.f;
            if (v) {
                if (p.c1f) {   // single-level constants: the queue's c2 slot carries c1
                    c2 = __ldg(p.c1f + a_blk);
                } else {
                    code = __ldg(p.c1_codes + a_blk);
                    c2 = __ldg(p.c2 + (a_blk >> 8));
                }
            }
            a_blk += blk_step;
            a_n += 64;
        };
        bool qv[kGemmPrefetch];
        uint32_t qcode[kGemmPrefetch];
        float qc2[kGemmPrefetch];
#pragma unroll
        for (int d = 0; d < kGemmPrefetch; ++d) const_load(d, qv[d], qcode[d], qc2[d]);
        bool ok = true;
        int s = 0;
        uint32_t ph = 0;
        for (int it = 0; it < ks0 && ok; ++it, s = (s + 1 == kStages) ? 0 : s + 1, ph ^= (s == 0) ? 1u : 0u) {
            const bool valid = qv[0];
            // c1' = fp32(fp32(v8 c2) + mu) with v8 from the shared E4M3 table, or the stored c1
            const float c1p = !valid ? 0.f : (p.c1f ? qc2[0] : __fadd_rn(__fmul_rn(e4tab[qcode[0]], qc2[0]), mu));
#pragma unroll
            for (int d = 0; d + 1 < kGemmPrefetch; ++d) {
                qv[d] = qv[d + 1];
                qcode[d] = qcode[d + 1];
                qc2[d] = qc2[d + 1];
            }
            const_load(it + kGemmPrefetch, qv[kGemmPrefetch - 1], qcode[kGemmPrefetch - 1], qc2[kGemmPrefetch - 1]);
            ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_full_a + 8 * s, ph, abort, p.err));
            if (!ok) break;
            const uint32_t row_addr = sB + s * kBStageBytes + img;
            if (!valid) {
                if (DX) zero_row(row_addr);
                else zero_row_kn<kBN * 16>(row_addr);
            } else {
                const uint32_t c_base = sCodes + s * kCodesStageBytes;
                uint4 c0, c1;
                if (!DX) {
                    // codes tile: 256 rows x 32 bytes, unswizzled (2-way bank conflicts on an idle pipe
                    // cost less than staggering the halves)
                    const uint32_t src = c_base + row * 32u;
                    c0 = ld_shared_v4(src);
                    c1 = ld_shared_v4(src + 16u);
                } else {
                    // codes tile: 64 rows x 128 bytes, 128-byte swizzled; this unit's 32 bytes are chunks 2kc, 2kc+1
                    const uint32_t src = c_base + row * 128u;
                    c0 = ld_shared_v4(src + (((2u * kc) ^ (row & 7u)) << 4));
                    c1 = ld_shared_v4(src + (((2u * kc + 1u) ^ (row & 7u)) << 4));
                }
                Lut lut;
                build_lut(lut, c1p, p.tb, p.f16 != 0);
                if (DX) expand_block_row(row_addr, row & 7u, c0, c1, lut);
                else expand_block_row_kn<kBN * 16>(row_addr, c0, c1, lut);
            }
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar_full_b + 8 * s);
        }

        // ------------------------------------------------------------ epilogue
        // Warp w reads TMEM lane quadrant (w & 3); the two warps of a quadrant split the columns.
        const bool acc_ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_acc, 0, abort, p.err));
        ptx::tc_fence_after();
        if (acc_ok) {
            const uint32_t quad = (uint32_t)(warp & 3);
            const int half = (warp - 2) >> 2;                 // 0 or 1
#pragma unroll 1
            for (int h = 0; h < NUM_ACC; ++h) {
                const int64_t m = m0 + h * 128 + quad * 32 + lane;
#pragma unroll 1
                for (int cc = 0; cc < kBN / 64; ++cc) {
                    const int c = half * (kBN / 64) + cc;
                    const int64_t nb = n0 + c * 32;
                    if (nb >= p.Nout) break;
                    uint32_t v[32];
                    ptx::tmem_ld_32x32b_x32(tmem + ((quad * 32u) << 16) + h * 256 + c * 32, v);
                    ptx::tmem_ld_wait();
                    if (m >= p.M) continue;
                    store_row32(p, m, nb, p.Nout, v);
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

// ---------------------------------------------------------------------------- fwd / dX on CTA pairs
//
// The same forward (Y = X W_hat^T + U2 B2^T) and dX (dX = dY W_hat + dU2 A2), computed by clusters
// of two CTAs that share each MMA (tcgen05 cta_group::2, M = 256 tokens x N = 256 output columns
// per instruction).  A pair's tile is 512 tokens x 256 output columns: CTA rank r holds tokens
// m0 + 256 r + [0, 256) (two 128-row halves, one per accumulator) and supplies output columns
// nr0 = n0 + 128 r + [0, 128) of operand B, so it expands only its half of the W tile (forward:
// W rows nr0 + [0, 128) of each K-step; dX: the two 64-weight blocks of columns nr0 + [0, 128) of
// each of the step's 64 W rows).  Each W tile is dequantized once per 512 tokens instead of once
// per 256, which halves the producers' work per MMA flop.
// Every CTA loads its own tiles (no load is shared between the two); the loads of the token
// tiles (and of the LoRA operands) count their bytes on the leader's (rank 0) barrier, because
// the leader issues the MMAs, which read both CTAs' shared memory.
// Warp roles as in the single-CTA kernel; the two producer groups of 4 warps take alternate
// K-steps (stage parity = group, 4 stages).
// Barriers, per CTA unless marked "leader":
//   full_a[s]  (leader) 1 arrival (the leader's expect-tx) + the token-tile bytes of both CTAs
//              (and, on LoRA steps, the B-operand bytes of both);
//   full_b[s]  (leader) 8 arrivals: the 4 producer warps of the stage's group in both CTAs;
//   codes[s]   1 arrival (this CTA's expect-tx) + this CTA's code-tile bytes;
//   empty[s]   1 arrival: the leader's commit after the MMAs that read stage s (it commits once
//              to its own barrier and once to the peer's, by cluster address);
//   acc        1 arrival: the leader's commit after the last MMA.
constexpr int kPairStages = 4;
constexpr uint32_t kPairAStage = 256 * 128;                  // 256 tokens x 64, 128-byte swizzled rows
constexpr uint32_t kPairBStage = 128 * 128;                  // 128 W rows x 64
constexpr uint32_t kPairCodesStage = 128 * 32;               // fwd: 128 W rows x 32 bytes; dX: 64 rows x 64 bytes
constexpr uint32_t kPairOffB = kPairStages * kPairAStage;
constexpr uint32_t kPairOffCodes = kPairOffB + kPairStages * kPairBStage;
constexpr uint32_t kPairOffE4 = kPairOffCodes + kPairStages * kPairCodesStage;
constexpr uint32_t kPairOffBars = kPairOffE4 + 256 * 4;
constexpr uint32_t kPairNumBars = 4 * kPairStages + 1;
constexpr uint32_t kPairOffSlot = kPairOffBars + kPairNumBars * 8;
constexpr uint32_t kPairOffAbort = kPairOffSlot + 4;
constexpr uint32_t kPairAlloc = kPairOffAbort + 4 + 1024;
static_assert(kPairAlloc <= 232448, "shared memory of one CTA");

template <bool DX>
__global__ void __launch_bounds__(kGemmThreads, 1)
tc_gemm_nf4_pair(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmCodes,
                 const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1, TcGemmParams p) {
    grid_dependency_wait();                                   // operands written by the previous kernel
    allow_dependents();
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base = (ptx::smem_addr(smem_raw) + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - ptx::smem_addr(smem_raw));
    const uint32_t sA = base, sB = base + kPairOffB, sCodes = base + kPairOffCodes;
    const uint32_t bar_full_a = base + kPairOffBars;
    const uint32_t bar_full_b = bar_full_a + 8 * kPairStages;
    const uint32_t bar_codes = bar_full_b + 8 * kPairStages;
    const uint32_t bar_empty = bar_codes + 8 * kPairStages;
    const uint32_t bar_acc = bar_empty + 8 * kPairStages;
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gbase + kPairOffSlot);
    volatile int* abort = reinterpret_cast<volatile int*>(gbase + kPairOffAbort);

    const uint32_t rank = ptx::cluster_ctarank();
    const bool leader = rank == 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int64_t mt, nt;
    const int bn = DX ? kBN : p.bn;                           // output columns of the pair tile
    const int hb = bn / 2;                                    // of which this CTA supplies
    raster_tile(blockIdx.x >> 1, (p.M + 511) / 512, (p.Nout + bn - 1) / bn, mt, nt);
    const int64_t m0 = mt * 512 + 256 * (int64_t)rank;       // this CTA's first token
    const int64_t n0 = nt * bn;                               // the pair's output column tile
    const int64_t nr0 = n0 + hb * (int64_t)rank;              // this CTA's output columns (forward: W rows)
    const int ks0 = p.ksteps0, ktotal = p.ksteps0 + p.ksteps1;
    float* e4tab = reinterpret_cast<float*>(gbase + kPairOffE4);
    if (threadIdx.x < 256) e4tab[threadIdx.x] = e4m3_to_f32(threadIdx.x);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPairStages; ++s) {
            ptx::mbar_init(bar_full_a + 8 * s, 1);
            ptx::mbar_init(bar_full_b + 8 * s, 8);
            ptx::mbar_init(bar_codes + 8 * s, 1);
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
        ptx::tmem_alloc_pair(base + kPairOffSlot, 512);
        ptx::tmem_relinquish_pair();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();                                      // both CTAs' barriers exist before any remote signal
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lead_full_a = ptx::mapa_shared(bar_full_a, 0);
    const uint32_t lead_full_b = ptx::mapa_shared(bar_full_b, 0);

    if (warp == 0) {
        // ------------------------------------------------------------ TMA (both CTAs)
        int issued = 0;
        int s = 0;
        uint32_t ph = 0;
        for (int it = 0; it < ktotal; ++it) {
            if (!__all_sync(0xffffffffu, ptx::mbar_wait(bar_empty + 8 * s, ph ^ 1u, abort, p.err))) break;
            issued = it + 1;
            if (ptx::elect_one_sync()) {
                const uint32_t a_dst = sA + s * kPairAStage;
                if (it < ks0) {
                    if (leader) ptx::mbar_arrive_expect_tx(bar_full_a + 8 * s, 2 * kPairAStage);
                    ptx::tma_load_2d_pair(a_dst, &tmA0, it * 64, (int32_t)m0, lead_full_a + 8 * s);
                    ptx::mbar_arrive_expect_tx(bar_codes + 8 * s, DX ? kPairCodesStage : 32u * (uint32_t)hb);
                    if (!DX)
                        ptx::tma_load_2d(sCodes + s * kPairCodesStage, &tmCodes, it * 32, (int32_t)nr0, bar_codes + 8 * s);
                    else
                        ptx::tma_load_2d(sCodes + s * kPairCodesStage, &tmCodes, (int32_t)(nr0 / 2), it * 64,
                                         bar_codes + 8 * s);
                } else {
                    const int j = it - ks0;
                    const int jb = p.b1_wrap ? j % p.b1_wrap : j;   // hi and lo steps share the B1 tile
                    if (leader)
                        ptx::mbar_arrive_expect_tx(bar_full_a + 8 * s,
                                                   2 * (kPairAStage + (DX ? kPairBStage : 128u * (uint32_t)hb)));
                    ptx::tma_load_2d_pair(a_dst, &tmA1, j * 64, (int32_t)m0, lead_full_a + 8 * s);
                    if (!DX) {
                        ptx::tma_load_2d_pair(sB + s * kPairBStage, &tmB1, jb * 64, (int32_t)nr0, lead_full_a + 8 * s);
                    } else {
#pragma unroll
                        for (int c = 0; c < 2; ++c)
                            ptx::tma_load_2d_pair(sB + s * kPairBStage + c * 8192, &tmB1, (int32_t)(nr0 + c * 64), jb * 64,
                                                  lead_full_a + 8 * s);
                    }
                }
            }
            __syncwarp();
            if (++s == kPairStages) { s = 0; ph ^= 1u; }
        }
        if (*abort) {   // drain what this CTA can observe: its code tiles, and (leader) the token tiles
            for (int it = max(0, issued - kPairStages); it < issued; ++it) {
                const uint32_t ph_i = (uint32_t)(it / kPairStages) & 1u;
                if (it < ks0) ptx::mbar_wait_drain(bar_codes + 8 * (it % kPairStages), ph_i);
                if (leader) ptx::mbar_wait_drain(bar_full_a + 8 * (it % kPairStages), ph_i);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader only)
        if (leader) {
            const uint32_t idesc = ptx::idesc_set_f16(ptx::idesc_bf16_f32(256, bn, DX ? 1 : 0), p.f16 != 0);
            const uint64_t adesc0 = ptx::smem_desc_sw128(sA, 16, 1024);
            // forward: LoRA steps read 128B-swizzled TMA tiles, W_hat steps the non-swizzled K-major image;
            // dX: both are two MN-major 64-column images 8 KiB apart
            const uint64_t bdesc0 = DX ? ptx::smem_desc_sw128(sB, 8192, 1024) : ptx::smem_desc_sw128(sB, 16, 1024);
            const uint64_t bdesc0_kn = ptx::smem_desc_kmajor_none(sB, 128 * 16, 128);
            const uint32_t peer_empty = ptx::mapa_shared(bar_empty, 1);
            const uint32_t peer_acc = ptx::mapa_shared(bar_acc, 1);
            bool ok = true;
            int s = 0;
            uint32_t ph = 0;
            for (int it = 0; it < ktotal && ok; ++it) {
                bool w = ptx::mbar_wait(bar_full_a + 8 * s, ph, abort, p.err);
                if (w && it < ks0) w = ptx::mbar_wait(bar_full_b + 8 * s, ph, abort, p.err);
                ok = __all_sync(0xffffffffu, w);
                if (!ok) break;
                ptx::tc_fence_after();
                if (ptx::elect_one_sync()) {
                    const uint64_t ad = adesc0 + ((uint32_t)s * (kPairAStage >> 4));
                    const bool kn = !DX && it < ks0;
                    const uint64_t bd = (kn ? bdesc0_kn : bdesc0) + ((uint32_t)s * (kPairBStage >> 4));
                    const uint32_t kstep = DX ? (2048 >> 4) : kn ? ((2 * 128 * 16) >> 4) : (32 >> 4);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
                        for (int h = 0; h < 2; ++h)
                            ptx::mma_bf16_ss_pair(tmem + h * 256, ad + h * (16384 >> 4) + kk * (32 >> 4),
                                                  bd + kk * kstep, idesc, (it | kk) != 0 ? 1u : 0u);
                    }
                    ptx::mma_commit_pair(bar_empty + 8 * s);          // this CTA's stage
                    ptx::mma_commit_pair(peer_empty + 8 * s);         // the peer's stage
                }
                __syncwarp();
                if (++s == kPairStages) { s = 0; ph ^= 1u; }
            }
            if (ptx::elect_one_sync()) {
                ptx::mma_commit_pair(bar_acc);
                ptx::mma_commit_pair(peer_acc);
                if (*abort) ptx::mbar_wait_drain(bar_acc, 0);   // issued MMAs finish before TMEM is freed
            }
            __syncwarp();
        }
    } else {
        // ------------------------------------------------------------ dequant producers (both CTAs)
        // group g expands the K-steps it = g, g + 2, ...; thread t of the group: forward: W row nr0 + t,
        // K-block it; dX: W row 64 it + (t & 63), K-block (nr0 >> 6) + kc with kc = t >> 6
        const int g = (warp - 2) >> 2;
        const int t = threadIdx.x - 64 - 128 * g;
        const float mu = p.c1f ? 0.f : *p.mu;
        const int64_t blocks_per_row = p.WK / 64;
        const uint32_t row = DX ? (uint32_t)(t & 63) : (uint32_t)t;
        const uint32_t kc = DX ? (uint32_t)(t >> 6) : 0u;
        const bool lane_ok = DX ? (nr0 + (int64_t)kc * 64 < p.WK) : (t < hb && nr0 + t < p.WN);
        const bool in_tile = DX || t < hb;                    // forward rows past a narrow tile are never read
        // block of the step whose constants load next, moving by a fixed stride per group step
        // (forward: 2 blocks along the row; dX: 128 W rows down)
        int64_t a_blk = DX ? ((int64_t)g * 64 + row) * blocks_per_row + (nr0 >> 6) + kc : (nr0 + t) * blocks_per_row + g;
        const int64_t blk_step = DX ? 128 * blocks_per_row : 2;
        int64_t a_n = (int64_t)g * 64 + row;                  // dX: the W row of that step
        auto const_load = [&](int step, bool& v, uint32_t& code, float& c2) {
            v = lane_ok && step < ks0 && (!DX || a_n < p.WN);
            code = 0;
            c2 = 0.f;
            if (v) {
                if (p.c1f) {
                    c2 = __ldg(p.c1f + a_blk);
                } else {
                    code = __ldg(p.c1_codes + a_blk);
                    c2 = __ldg(p.c2 + (a_blk >> 8));
                }
            }
            a_blk += blk_step;
            a_n += 128;
        };
        bool qv[kGemmPrefetch];
        uint32_t qcode[kGemmPrefetch];
        float qc2[kGemmPrefetch];
#pragma unroll
        for (int d = 0; d < kGemmPrefetch; ++d) const_load(g + 2 * d, qv[d], qcode[d], qc2[d]);
        bool ok = true;
        for (int it = g; it < ks0 && ok; it += 2) {
            const int s = it & (kPairStages - 1);
            const uint32_t ph = (uint32_t)(it / kPairStages) & 1u;
            const bool valid = qv[0];
            const float c1p = !valid ? 0.f : (p.c1f ? qc2[0] : __fadd_rn(__fmul_rn(e4tab[qcode[0]], qc2[0]), mu));
#pragma unroll
            for (int d = 0; d + 1 < kGemmPrefetch; ++d) {
                qv[d] = qv[d + 1];
                qcode[d] = qcode[d + 1];
                qc2[d] = qc2[d + 1];
            }
            const_load(it + 2 * kGemmPrefetch, qv[kGemmPrefetch - 1], qcode[kGemmPrefetch - 1], qc2[kGemmPrefetch - 1]);
            ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_codes + 8 * s, ph, abort, p.err));
            if (!ok) break;
            // forward: non-swizzled K-major image of 128 rows (row t at 16 t, chunk c at 2048 c);
            // dX: 128-byte-swizzled 64-row images, one per K-block, read as an MN-major operand
            const uint32_t row_addr = sB + s * kPairBStage + (DX ? kc * 8192u + row * 128u : row * 16u);
            if (!in_tile) {
                // nothing to write
            } else if (!valid) {
                if (DX) zero_row(row_addr);
                else zero_row_kn<128 * 16>(row_addr);
            } else {
                // codes: forward 128 rows x 32 bytes; dX 64 rows x 64 bytes (this CTA's two blocks)
                const uint32_t src = sCodes + s * kPairCodesStage + (DX ? row * 64u + kc * 32u : row * 32u);
                const uint4 c0 = ld_shared_v4(src);
                const uint4 c1 = ld_shared_v4(src + 16u);
                Lut lut;
                build_lut(lut, c1p, p.tb, p.f16 != 0);
                if (DX) expand_block_row(row_addr, row & 7u, c0, c1, lut);
                else expand_block_row_kn<128 * 16>(row_addr, c0, c1, lut);
            }
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive_cluster(lead_full_b + 8 * s);
        }

        // ------------------------------------------------------------ epilogue
        const bool acc_ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_acc, 0, abort, p.err));
        ptx::tc_fence_after();
        if (acc_ok) {
            const uint32_t quad = (uint32_t)(warp & 3);
            const int half = (warp - 2) >> 2;
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
                const int64_t m = m0 + h * 128 + quad * 32 + lane;
#pragma unroll 1
                for (int cc = 0; cc < kBN / 64; ++cc) {
                    const int c = half * (kBN / 64) + cc;
                    const int64_t nb = n0 + c * 32;
                    const int64_t nlim = min(p.Nout, n0 + bn);
                    if (nb >= nlim) break;
                    uint32_t v[32];
                    ptx::tmem_ld_32x32b_x32(tmem + ((quad * 32u) << 16) + h * 256 + c * 32, v);
                    ptx::tmem_ld_wait();
                    if (m >= p.M) continue;
                    store_row32(p, m, nb, nlim, v);
                }
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();                                      // no CTA leaves while its peer may still signal it
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_pair(tmem, 512);
    }
}

// ---------------------------------------------------------------------------- small-M forward
//
// Y[M,N] for M <= 16 tokens (decode), "swap-AB": D[n, m] = W_hat[n, :] X[m, :]^T
// with the dequantized weight as the 128-row MMA operand A (K-major image
// written by the producer warps) and the token tile as a 16-wide operand B.
// The work is the sequence of (tile of 128 W rows, K-step of 64) units, tile
// major; it is cut into G equal contiguous ranges, one per persistent CTA
// (stream-K), so every SM streams the same number of weight bytes whatever
// the shape.  A CTA's range crosses tiles: each (tile, CTA) piece is a
// segment, accumulated in one of two TMEM accumulators and written as an fp32
// partial tile to slot tile + CTA; decode_fixup then sums each tile's slots in
// CTA order (deterministic) and adds the LoRA term s U B^T in fp32.  U = X A^T
// itself is computed by the producer warps of the CTAs (one fp32 dot product per
// CTA and turn) while their first code tiles are on the way.
// Warp roles (320 threads): warp 0 lane 0 streams each unit's packed codes and
// token tile through a TMA ring (a ring slot is freed by the MMA that read it);
// warp 1 owns TMEM and issues tcgen05.mma; warps 2-9 are two producer groups of
// 4 warps that take alternate units (one W row of 64 weights per thread per
// unit), and each group runs the epilogue of the segments that use its
// accumulator.  The dequant is ALU-bound (byte-permute table lookups), so the
// producers do nothing else per unit.
constexpr int kDecThreads = 320;
constexpr int kDecCtasPerSm = 2;                // ~103 KB of shared memory per CTA
constexpr int kDecMaxCtas = 1024;
constexpr int kDecCodeStages = 6;               // codes + token ring (the HBM stream); even: stage parity = group
constexpr int kDecStages = 4;                   // dequantized-tile ring; stage parity = group
constexpr int kDecPrefetch = 2;                 // block constants are loaded this many units (of the group) ahead
constexpr uint32_t kDecAStage = 128 * 128;      // W_hat tile [128 rows x 64]
constexpr uint32_t kDecXStage = 16 * 128;       // X tile [16 tokens x 64], 128-byte swizzled rows (TMA)
constexpr uint32_t kDecCodesStage = 128 * 32;   // packed codes [128 rows x 32 bytes]
constexpr uint32_t kDecOffX = kDecStages * kDecAStage;
constexpr uint32_t kDecOffCodes = kDecOffX + kDecCodeStages * kDecXStage;
constexpr uint32_t kDecOffE4 = kDecOffCodes + kDecCodeStages * kDecCodesStage;   // E4M3 value table [256] fp32
constexpr uint32_t kDecOffBars = kDecOffE4 + 256 * 4;
// barriers: cfull[CS], cempty[CS], afull[S], aempty[S], accfull[2], accempty[2], drain
constexpr uint32_t kDecNumBars = 2 * kDecCodeStages + 2 * kDecStages + 5;
constexpr uint32_t kDecOffSlot = kDecOffBars + kDecNumBars * 8;
constexpr uint32_t kDecOffAbort = kDecOffSlot + 4;
constexpr uint32_t kDecOffRed = kDecOffAbort + 4;             // [8] fp32: per-warp sums of one U entry
constexpr uint32_t kDecAlloc = kDecOffRed + 32 + 1024;
constexpr uint32_t kDecSlotFloats = 16 * 128;   // one partial tile: [16 tokens][128 rows] fp32
static_assert(kDecCodeStages % 2 == 0 && kDecStages % 2 == 0, "ring stages alternate between the two groups");
static_assert(2 * (kDecAlloc + 1024) <= 233472, "two CTAs per SM");

// First unit of CTA b when U units are cut into G ranges.
__host__ __device__ __forceinline__ int64_t dec_range_begin(int64_t b, int64_t U, int64_t G) { return b * U / G; }

__global__ void __launch_bounds__(kDecThreads, kDecCtasPerSm)
tc_decode_nf4(const __grid_constant__ CUtensorMap tmCodes, const __grid_constant__ CUtensorMap tmX, DecodeParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base = (ptx::smem_addr(smem_raw) + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - ptx::smem_addr(smem_raw));
    const uint32_t sA = base, sX = base + kDecOffX, sCodes = base + kDecOffCodes;
    float* e4tab = reinterpret_cast<float*>(gbase + kDecOffE4);
    const uint32_t bar_cfull = base + kDecOffBars;
    const uint32_t bar_cempty = bar_cfull + 8 * kDecCodeStages;
    const uint32_t bar_afull = bar_cempty + 8 * kDecCodeStages;
    const uint32_t bar_aempty = bar_afull + 8 * kDecStages;
    const uint32_t bar_accfull = bar_aempty + 8 * kDecStages;
    const uint32_t bar_accempty = bar_accfull + 16;
    const uint32_t bar_drain = bar_accempty + 16;
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gbase + kDecOffSlot);
    volatile int* abort = reinterpret_cast<volatile int*>(gbase + kDecOffAbort);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = p.ksteps;                                   // units per tile
    const int64_t u0 = dec_range_begin(blockIdx.x, p.units, p.grid);
    const int n = (int)(dec_range_begin(blockIdx.x + 1, p.units, p.grid) - u0);   // units of this CTA
    const int64_t t0 = u0 / S;                                // tile of the first segment
    const int step0 = (int)(u0 - t0 * S);

    allow_dependents();                                       // the fixup may be scheduled now
    if (threadIdx.x < 256) e4tab[threadIdx.x] = e4m3_to_f32(threadIdx.x);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kDecCodeStages; ++s) {
            ptx::mbar_init(bar_cfull + 8 * s, 1);
            ptx::mbar_init(bar_cempty + 8 * s, 1);
        }
        for (int s = 0; s < kDecStages; ++s) {
            ptx::mbar_init(bar_afull + 8 * s, 4);
            ptx::mbar_init(bar_aempty + 8 * s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            ptx::mbar_init(bar_accfull + 8 * a, 1);
            ptx::mbar_init(bar_accempty + 8 * a, 4);
        }
        ptx::mbar_init(bar_drain, 1);
        *abort = 0;
        ptx::fence_barrier_init();
        ptx::fence_proxy_async_smem();
        ptx::tma_prefetch_map(&tmCodes);
        ptx::tma_prefetch_map(&tmX);
    }
    if (warp == 1) {
        ptx::tmem_alloc(base + kDecOffSlot, 32);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    grid_dependency_wait();                                   // inputs written by the previous kernel

    if (warp == 0) {
        // unit i: codes and token tile into ring slot i % kDecCodeStages, once the MMA that
        // read the slot's previous contents has completed (cempty, phase by phase); the whole
        // warp runs the loop and one elected lane issues the copies
        bool ok = true;
        int issued = 0;
        int64_t tile = t0;
        int step = step0;
        int cs = 0;
        uint32_t cph = 0;
        for (int i = 0; i < n && ok; ++i) {
            ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_cempty + 8 * cs, cph ^ 1u, abort, p.err));
            if (!ok) break;
            if (ptx::elect_one_sync()) {
                ptx::mbar_arrive_expect_tx(bar_cfull + 8 * cs, kDecCodesStage + kDecXStage);
                ptx::tma_load_2d(sCodes + cs * kDecCodesStage, &tmCodes, step * 32, (int32_t)(tile * 128),
                                 bar_cfull + 8 * cs);
                ptx::tma_load_2d(sX + cs * kDecXStage, &tmX, step * 64, 0, bar_cfull + 8 * cs);
            }
            __syncwarp();
            issued = i + 1;
            if (++step == S) { step = 0; ++tile; }
            if (++cs == kDecCodeStages) { cs = 0; cph ^= 1u; }
        }
        if (*abort) {   // drain this CTA's copies in flight before it exits
            for (int c = max(0, issued - kDecCodeStages); c < issued; ++c)
                ptx::mbar_wait_drain(bar_cfull + 8 * (c % kDecCodeStages), (uint32_t)(c / kDecCodeStages) & 1u);
        }
    } else if (warp == 1) {
        // MMA issuer: the whole warp runs the loop, one elected lane issues.  Descriptors are
        // built once and advanced by stage offsets (start address >> 4 in the low 14 bits;
        // every shared address here is below 256 KiB, so no carry leaves them).
        const uint32_t idesc = ptx::idesc_set_f16(ptx::idesc_bf16_f32_ab(128, 16, 0, 0), p.f16 != 0);
        const uint64_t adesc0 = ptx::smem_desc_kmajor_none(sA, 128 * 16, 128);   // W_hat rows, non-swizzled
        const uint64_t bdesc0 = ptx::smem_desc_sw128(sX, 16, 1024);
        bool ok = true;
        int step = step0, seg = 0;
        int s = 0, cs = 0;                                    // ring slots of unit i, and their phase bits
        uint32_t ph = 0, cph = 0;
        bool fresh = true;                                    // first unit of a segment: overwrite
        for (int i = 0; i < n && ok; ++i) {
            const int a = seg & 1;
            if (fresh && seg >= 2) {                          // accumulator a drained by segment seg-2's epilogue
                ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_accempty + 8 * a, (uint32_t)((seg - 2) >> 1) & 1u,
                                                             abort, p.err));
                if (!ok) { if (lane == 0) atomicMax(p.dbg, 0x61000000u | (uint32_t)i); break; }
            }
            ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_afull + 8 * s, ph, abort, p.err) &&
                                             ptx::mbar_wait(bar_cfull + 8 * cs, cph, abort, p.err));
            if (!ok) { if (lane == 0) atomicMax(p.dbg, 0x60000000u | (uint32_t)i); break; }
            ptx::tc_fence_after();
            const bool last = (step + 1 == S) || (i == n - 1);
            if (ptx::elect_one_sync()) {
                const uint64_t ad = adesc0 + ((uint32_t)s * (kDecAStage >> 4));
                const uint64_t bd = bdesc0 + ((uint32_t)cs * (kDecXStage >> 4));
                const uint32_t d = tmem + 16u * (uint32_t)a;
                constexpr uint32_t ak = (2 * 128 * 16) >> 4;       // one K step of 16: two core-matrix columns
                ptx::mma_bf16_ss(d, ad, bd, idesc, fresh ? 0u : 1u);
                ptx::mma_bf16_ss(d, ad + ak, bd + 2, idesc, 1u);
                ptx::mma_bf16_ss(d, ad + 2 * ak, bd + 4, idesc, 1u);
                ptx::mma_bf16_ss(d, ad + 3 * ak, bd + 6, idesc, 1u);
                ptx::mma_commit(bar_aempty + 8 * s);
                ptx::mma_commit(bar_cempty + 8 * cs);
                if (last) ptx::mma_commit(bar_accfull + 8 * a);   // segment ends: hand the accumulator over
            }
            __syncwarp();
            if (++s == kDecStages) { s = 0; ph ^= 1u; }
            if (++cs == kDecCodeStages) { cs = 0; cph ^= 1u; }
            fresh = last;
            if (++step == S) step = 0;
            if (last) ++seg;
        }
        if (ptx::elect_one_sync()) {
            ptx::mma_commit(bar_drain);
            if (*abort) ptx::mbar_wait_drain(bar_drain, 0);   // issued MMAs finish before TMEM is freed
        }
        __syncwarp();
    } else {
        // U = X A^T (fp32): dot products blockIdx.x, blockIdx.x + G, ... of the r*M, each over the 256
        // producer threads (16-byte chunks c = t, t + 256, ...; four in flight), then a fixed-order
        // reduction (xor shuffles, then the eight warp sums in order).  With per-token adapters token m
        // uses A[aidx[m]]; a token without one (-1) gets U = 0, an index >= n raises the BOUNDS flag.
        {
            const int tp = threadIdx.x - 64;
            float* red = reinterpret_cast<float*>(gbase + kDecOffRed);
            const int64_t n_dot = (int64_t)p.r * p.M;
            for (int64_t idx = blockIdx.x; idx < n_dot; idx += gridDim.x) {
                const int m = (int)(idx / p.r), j = (int)(idx % p.r);
                int64_t arow = j;
                bool have = true;
                if (p.aidx) {
                    const int a = p.aidx[m];
                    have = a >= 0 && a < p.n_adapters;
                    if (a >= p.n_adapters && tp == 0) atomicOr(p.err, ERR_FLAG_BOUNDS);
                    arow = (int64_t)a * p.r + j;
                }
                float acc = 0.f;
                if (have) {
                    const uint4* xr = p.X + (int64_t)m * p.K8;
                    const uint4* ar = p.A + arow * p.K8;
                    for (int64_t c0 = tp; c0 < p.K8; c0 += 4 * 256) {
                        uint4 xv[4], av[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int64_t c = c0 + q * 256;
                            xv[q] = c < p.K8 ? __ldg(xr + c) : make_uint4(0, 0, 0, 0);
                            av[q] = c < p.K8 ? __ldg(ar + c) : make_uint4(0, 0, 0, 0);
                        }
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const uint32_t xw[4] = {xv[q].x, xv[q].y, xv[q].z, xv[q].w};
                            const uint32_t aw[4] = {av[q].x, av[q].y, av[q].z, av[q].w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                acc = __fmaf_rn(from16(xw[e] & 0xFFFFu, p.f16), from16(aw[e] & 0xFFFFu, p.f16), acc);
                                acc = __fmaf_rn(from16(xw[e] >> 16, p.f16), from16(aw[e] >> 16, p.f16), acc);
                            }
                        }
                    }
                }
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, o));
                if (lane == 0) red[warp - 2] = acc;
                asm volatile("bar.sync 1, 256;" ::: "memory");   // the 8 producer warps
                if (tp == 0) {
                    float sum = 0.f;
                    for (int w = 0; w < 8; ++w) sum = __fadd_rn(sum, red[w]);
                    p.U[(int64_t)m * p.r + j] = have ? sum : 0.f;
                }
                asm volatile("bar.sync 1, 256;" ::: "memory");
            }
        }

        // producer group g takes units g, g + 2, ...; thread t expands W row tile*128 + t
        const int g = (warp - 2) >> 2;
        const int t = threadIdx.x - 64 - 128 * g;
        const int64_t nb1 = p.N * (p.K / 64);
        const int64_t kb = p.K / 64;
        const float mu = p.c1f ? 0.f : *p.mu;
        // a unit cursor: tile, K-step, the first-level block index of W row tile*128 + t at that
        // step, and whether that row exists (the last tile may be partial); advancing by `by`
        // units moves the block index by `by`, plus 128 rows less one tile of steps per tile crossed
        struct Cursor { int64_t tile, blk; int step; bool row_ok; };
        auto advance = [&](Cursor& c, int by) {
            c.step += by;
            c.blk += by;
            while (c.step >= S) {
                c.step -= S;
                ++c.tile;
                c.blk += 128 * kb - S;
                c.row_ok = c.tile * 128 + t < p.N;
            }
        };
        Cursor cur{t0, (t0 * 128 + t) * kb + step0, step0, t0 * 128 + t < p.N};
        advance(cur, g);
        auto const_load = [&](const Cursor& c, uint32_t& code, float& c2) {
            code = 0; c2 = 0.f;
            if (!c.row_ok) return;
            if (c.blk >= nb1) { atomicOr(p.err, ERR_FLAG_BOUNDS); atomicMax(p.dbg, 0x20000000u); return; }
            if (p.c1f) {   // single-level constants: the queue's c2 slot carries c1
                c2 = __ldg(p.c1f + c.blk);
            } else {
                code = __ldg(p.c1_codes + c.blk);
                c2 = __ldg(p.c2 + (c.blk >> 8));
            }
        };
        uint32_t qcode[kDecPrefetch];
        float qc2[kDecPrefetch];
        Cursor pf = cur;
#pragma unroll
        for (int d = 0; d < kDecPrefetch; ++d) {
            qcode[d] = 0; qc2[d] = 0.f;
            if (g + 2 * d < n) const_load(pf, qcode[d], qc2[d]);
            advance(pf, 2);
        }

        int epi_seg = g;                                      // next segment whose epilogue is ours
        const int last_seg = (int)((u0 + n - 1) / S - t0);
        auto epilogue = [&](int seg) -> bool {
            const int a = seg & 1;
            const bool ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_accfull + 8 * a, (uint32_t)(seg >> 1) & 1u,
                                                                    abort, p.err));
            if (!ok) { if (lane == 0) atomicMax(p.dbg, 0x70000000u | (uint32_t)seg); return false; }
            ptx::tc_fence_after();
            const uint32_t quad = (uint32_t)(warp & 3);
            uint32_t v[16];
            ptx::tmem_ld_32x32b_x16(tmem + ((quad * 32u) << 16) + 16u * (uint32_t)a, v);
            ptx::tmem_ld_wait();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar_accempty + 8 * a);
            float* dst = p.partial + (t0 + seg + (int64_t)blockIdx.x) * kDecSlotFloats + quad * 32 + lane;
#pragma unroll
            for (int m = 0; m < 16; ++m)
                if (m < p.M) dst[m * 128] = __uint_as_float(v[m]);
            return true;
        };

        bool ok = true;
        int cs = g, s = g;                                    // ring slots of unit i (parity g), phase bits
        uint32_t cph = 0, ph = 0;
        for (int i = g; i < n && ok; i += 2) {
            const int seg = (int)(cur.tile - t0);
            while (epi_seg < seg && ok) { ok = epilogue(epi_seg); epi_seg += 2; }
            if (!ok) break;
            const float c1p = p.c1f ? qc2[0]                                  // c1' = c1, or
                                    : __fadd_rn(__fmul_rn(e4tab[qcode[0]], qc2[0]), mu);   // fp32(fp32(v8 c2) + mu)
#pragma unroll
            for (int d = 0; d + 1 < kDecPrefetch; ++d) {
                qcode[d] = qcode[d + 1];
                qc2[d] = qc2[d + 1];
            }
            qcode[kDecPrefetch - 1] = 0; qc2[kDecPrefetch - 1] = 0.f;
            if (i + 2 * kDecPrefetch < n) const_load(pf, qcode[kDecPrefetch - 1], qc2[kDecPrefetch - 1]);
            bool w_ok = ptx::mbar_wait(bar_cfull + 8 * cs, cph, abort, p.err);
            if (!w_ok) atomicMax(p.dbg, 0x40000000u | (uint32_t)i);
            w_ok = w_ok && ptx::mbar_wait(bar_aempty + 8 * s, ph ^ 1u, abort, p.err);
            if (!w_ok) atomicMax(p.dbg, 0x50000000u | (uint32_t)i);
            ok = __all_sync(0xffffffffu, w_ok);
            if (!ok) break;
            const uint32_t row_addr = sA + s * kDecAStage + (uint32_t)t * 16u;   // non-swizzled K-major
            if (!cur.row_ok) {
                zero_row_kn<128 * 16>(row_addr);
            } else {
                const uint32_t src = sCodes + cs * kDecCodesStage + (uint32_t)t * 32u;
                const uint4 x = ld_shared_v4(src);
                const uint4 y = ld_shared_v4(src + 16u);
                Lut lut;
                build_lut(lut, c1p, p.tb, p.f16 != 0);
                expand_block_row_kn<128 * 16>(row_addr, x, y, lut);
            }
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar_afull + 8 * s);
            advance(cur, 2);
            advance(pf, 2);
            if ((cs += 2) >= kDecCodeStages) { cs -= kDecCodeStages; cph ^= 1u; }
            if ((s += 2) >= kDecStages) { s -= kDecStages; ph ^= 1u; }
        }
        while (ok && epi_seg <= last_seg) { ok = epilogue(epi_seg); epi_seg += 2; }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 32);
    }
}

// Y[m, n] = sum over the CTAs b covering tile n / 128 of partial[tile + b][m][n % 128] (in b
// order) + scale * sum_j U[m, j] B[n, j], converted to the output type.  CTA (tile, y) covers the
// tile's 128 rows for tokens 4y .. 4y+3; the slots' loads are issued eight slots at a time, so a
// tile split over a few CTAs costs one round trip to memory (the kernel is latency-bound).
constexpr int kFixTokens = 4;
constexpr int kFixSlotBatch = 8;

__global__ void __launch_bounds__(128)
decode_fixup(const float* __restrict__ partial, int64_t units, int64_t G, int S, int64_t M, int64_t N,
             const float* __restrict__ U, const uint16_t* __restrict__ B, int r, float scale, void* out, int out_f32,
             const int32_t* __restrict__ aidx, int n_adapters, bool f16) {
    extern __shared__ float us[];                             // us[j * 4 + q] = U[m0 + q, j]
    __shared__ int32_t tok_adapter[kFixTokens];
    const int m0 = (int)blockIdx.y * kFixTokens;
    grid_dependency_wait();                                   // partial tiles and U are complete
    for (int i = threadIdx.x; i < r * kFixTokens; i += 128) {
        const int j = i / kFixTokens, m = m0 + i % kFixTokens;
        us[i] = m < M ? U[(int64_t)m * r + j] : 0.f;
    }
    if (threadIdx.x < kFixTokens) {
        const int m = m0 + (int)threadIdx.x;
        const int a = (aidx && m < M) ? aidx[m] : 0;
        tok_adapter[threadIdx.x] = (a >= 0 && a < n_adapters) ? a : -1;
    }
    __syncthreads();
    const int64_t tile = blockIdx.x;
    const int64_t n = tile * 128 + threadIdx.x;
    if (n >= N) return;
    auto cta_of = [&](int64_t u) {                            // the CTA whose range holds unit u
        int64_t b = u * G / units;
        while (b + 1 < G && dec_range_begin(b + 1, units, G) <= u) ++b;
        while (b > 0 && dec_range_begin(b, units, G) > u) --b;
        return b;
    };
    const int64_t ba = cta_of(tile * S), bz = cta_of(tile * S + S - 1);
    const int nm = (int)(M - m0 < kFixTokens ? M - m0 : kFixTokens);
    float acc[kFixTokens];
#pragma unroll
    for (int q = 0; q < kFixTokens; ++q) acc[q] = 0.f;
    for (int64_t b0 = ba; b0 <= bz; b0 += kFixSlotBatch) {
        float v[kFixSlotBatch][kFixTokens];
#pragma unroll
        for (int s = 0; s < kFixSlotBatch; ++s) {
            const float* pp = partial + (tile + b0 + s) * kDecSlotFloats + (int64_t)m0 * 128 + threadIdx.x;
#pragma unroll
            for (int q = 0; q < kFixTokens; ++q) v[s][q] = (b0 + s <= bz && q < nm) ? pp[q * 128] : 0.f;
        }
#pragma unroll
        for (int s = 0; s < kFixSlotBatch; ++s)
#pragma unroll
            for (int q = 0; q < kFixTokens; ++q)
                if (b0 + s <= bz) acc[q] = __fadd_rn(acc[q], v[s][q]);
    }
    float lora[kFixTokens];
#pragma unroll
    for (int q = 0; q < kFixTokens; ++q) lora[q] = 0.f;
    if (aidx) {
        // per-token adapters: lora[q] = sum_j U[m, j] B[a(m)][n, j] (ascending j), 0 without one
#pragma unroll
        for (int q = 0; q < kFixTokens; ++q) {
            const int a = q < nm ? tok_adapter[q] : -1;
            if (a < 0) continue;
            const uint16_t* br = B + ((int64_t)a * N + n) * r;
            float d = 0.f;
            for (int j0 = 0; j0 < r; j0 += 8) {
                float bv[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) bv[k] = j0 + k < r ? from16(br[j0 + k], f16) : 0.f;
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    if (j0 + k < r) d = __fmaf_rn(us[(j0 + k) * kFixTokens + q], bv[k], d);
            }
            lora[q] = d;
        }
    } else {
        const uint16_t* brow = B + n * r;
        for (int j0 = 0; j0 < r; j0 += 8) {
            float bv[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) bv[k] = j0 + k < r ? from16(brow[j0 + k], f16) : 0.f;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                if (j0 + k >= r) continue;
                const float4 u4 = *reinterpret_cast<const float4*>(us + (j0 + k) * kFixTokens);
                lora[0] = __fmaf_rn(u4.x, bv[k], lora[0]);
                lora[1] = __fmaf_rn(u4.y, bv[k], lora[1]);
                lora[2] = __fmaf_rn(u4.z, bv[k], lora[2]);
                lora[3] = __fmaf_rn(u4.w, bv[k], lora[3]);
            }
        }
    }
#pragma unroll
    for (int q = 0; q < kFixTokens; ++q) {
        if (q < nm) {
            const int64_t m = m0 + q;
            const float y = __fmaf_rn(scale, lora[q], acc[q]);
            if (out_f32) static_cast<float*>(out)[m * N + n] = y;
            else static_cast<uint16_t*>(out)[m * N + n] = (uint16_t)to16_rn(y, f16);
        }
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
    const int64_t tiles = ((a.p.Nout + kBN - 1) / kBN) * ((a.p.M + L::kBM - 1) / L::kBM);
    if (tiles > INT32_MAX) return QLORA_ERR_SHAPE;
    const dim3 grid((unsigned)tiles);
    (void)launch_dependent(kern, grid, dim3(kGemmThreads), L::kAlloc, stream, a.tmA0, a.tmCodes, a.tmA1, a.tmB1,
                           a.p);
    QLORA_CHECK_LAUNCH();
    return QLORA_OK;
}

// The forward on CTA pairs: clusters of 2, one pair per 512 x 256 output tile.
template <bool DX>
static qlora_status launch_pair(const TcGemmArgs& a, cudaStream_t stream) {
    static bool configured = false;   // attribute set once per instantiation (idempotent, so races are benign)
    auto kern = tc_gemm_nf4_pair<DX>;
    if (!configured) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPairAlloc) != cudaSuccess)
            return QLORA_ERR_CUDA;
        configured = true;
    }
    const int bn = DX ? kBN : a.p.bn;
    const int64_t pairs = ((a.p.Nout + bn - 1) / bn) * ((a.p.M + 511) / 512);
    if (2 * pairs > INT32_MAX) return QLORA_ERR_SHAPE;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * pairs));
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = kPairAlloc;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    (void)cudaLaunchKernelEx(&cfg, kern, a.tmA0, a.tmCodes, a.tmA1, a.tmB1, a.p);
    QLORA_CHECK_LAUNCH();
    return QLORA_OK;
}

// Whether the forward and dX run on CTA pairs: more than 256 tokens (a pair's tile covers 512),
// unless the environment variable QLORA_PAIR_GEMM is set to 0 (the single-CTA kernels then run).
static bool use_pairs(int64_t M) {
    static const bool enabled = [] {
        const char* e = std::getenv("QLORA_PAIR_GEMM");
        return !(e && e[0] == '0');
    }();
    return enabled && M > 256;
}

// Forward pair-tile width: the multiple of 16 in {256, 240, 224} that minimises waves x width,
// the time of the launch when every pair runs one tile at a time (ties to the wider tile), with
// as many pairs in a wave as clusters of 2 fit on the GPU at once.  For example W[8192, *] at
// M = 2048: 256 gives 128 pair tiles (1.73 waves of 74 pairs, the second 73% full), 224 gives
// 148 (two full waves) of 7/8 the work each.  Now that the producers expand half a W tile per
// CTA the MMAs bound a tile, so its time follows its width.
static int pair_tile_width(int64_t M, int64_t N) {
    static int slots = 0;
    if (slots == 0) {
        int dev = 0, sms = 148;
        if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (unsigned)sms);
        cfg.blockDim = dim3(kGemmThreads);
        cfg.dynamicSmemBytes = kPairAlloc;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaFuncSetAttribute(tc_gemm_nf4_pair<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kPairAlloc) != cudaSuccess ||
            cudaOccupancyMaxActiveClusters(&n, tc_gemm_nf4_pair<false>, &cfg) != cudaSuccess || n < 1) {
            (void)cudaGetLastError();
            n = sms / 2;
        }
        slots = n;
    }
    static const int forced = [] {   // QLORA_PAIR_BN=256|240|224 forces the width (tuning override)
        const char* e = std::getenv("QLORA_PAIR_BN");
        const int v = e ? std::atoi(e) : 0;
        return (v == 256 || v == 240 || v == 224) ? v : 0;
    }();
    if (forced) return forced;
    const int64_t mtiles = (M + 511) / 512;
    int best = kBN;
    int64_t best_cost = INT64_MAX;
    for (int bn : {256, 240, 224}) {
        const int64_t tiles = mtiles * ((N + bn - 1) / bn);
        const int64_t cost = (tiles + slots - 1) / slots * bn;
        if (cost < best_cost) { best_cost = cost; best = bn; }
    }
    return best;
}

// Splits of the reduction so that tiles x splits fills one wave of CTAs.
static int64_t decode_grid(int64_t units, int sms) {
    return std::max<int64_t>(1, std::min<int64_t>({units, (int64_t)kDecCtasPerSm * sms, (int64_t)kDecMaxCtas}));
}

size_t decode_partial_bytes(int64_t N, int64_t K) {
    const int64_t tiles = (N + 127) / 128, units = tiles * (K / 64);
    const int64_t slots = tiles + std::min<int64_t>(units, kDecMaxCtas);
    return (size_t)slots * kDecSlotFloats * sizeof(float);
}

qlora_status launch_tc_decode(const DecodeArgs& a, cudaStream_t stream) {
    const qlora_nf4_weight* w = a.w;
    const int64_t N = w->N, K = w->K;
    static int sms = 0;
    if (sms == 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return QLORA_ERR_CUDA;
    }
    CUtensorMap tmCodes, tmX;
    if (!make_tmap_2d(&tmCodes, false, w->codes, K / 2, N, K / 2, 32, 128, false)) return QLORA_ERR_CUDA;
    if (!make_tmap_2d(&tmX, true, a.X, K, a.M, K * 2, 64, 16, true)) return QLORA_ERR_CUDA;
    DecodeParams p{};
    p.M = a.M; p.N = N; p.K = K;
    p.ksteps = (int32_t)(K / 64);
    const int64_t tiles = (N + 127) / 128;
    p.units = tiles * p.ksteps;
    p.grid = decode_grid(p.units, sms);
    p.c1_codes = w->c1_codes; p.c2 = w->c2; p.mu = w->mu; p.c1f = w->c1;
    p.f16 = w->compute_dtype == QLORA_DTYPE_F16;
    p.partial = a.partial;
    p.tb = host_tables(w->codebook);
    p.err = device_error_word();
    if (!p.err) return QLORA_ERR_CUDA;
    p.dbg = p.err + 1;
    static bool configured = false;
    if (!configured) {
        if (cudaFuncSetAttribute(tc_decode_nf4, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDecAlloc) !=
            cudaSuccess)
            return QLORA_ERR_CUDA;
        configured = true;
    }
    p.X = static_cast<const uint4*>(a.X);
    p.A = static_cast<const uint4*>(a.A);
    p.K8 = K / 8;
    p.r = a.r;
    p.U = a.U;
    p.aidx = a.aidx;
    p.n_adapters = a.n_adapters;
    // both kernels are launched with programmatic dependent launch: the dequant GEMM's prologue
    // (barriers, TMEM, tables) overlaps the previous kernel's tail and it waits for that kernel
    // before reading anything; the fixup waits for the GEMM's partial tiles and U
    (void)launch_dependent(tc_decode_nf4, dim3((unsigned)p.grid), dim3(kDecThreads), kDecAlloc, stream, tmCodes,
                           tmX, p);
    QLORA_CHECK_LAUNCH();
    const unsigned ty = (unsigned)((a.M + kFixTokens - 1) / kFixTokens);
    (void)launch_dependent(decode_fixup, dim3((unsigned)tiles, ty), dim3(128),
                           (size_t)a.r * kFixTokens * sizeof(float), stream,
                           (const float*)a.partial, p.units, p.grid, (int)p.ksteps, a.M, N, (const float*)a.U,
                           static_cast<const uint16_t*>(a.B), a.r, a.scale, a.out, (int)a.out_f32, a.aidx,
                           (int)a.n_adapters, p.f16 != 0);
    QLORA_CHECK_LAUNCH();
    return QLORA_OK;
}

qlora_status launch_tc_gemm_nf4(TcGemmArgs& a, bool dx, cudaStream_t stream) {
    const uint32_t bm = a.p.M > 128 ? 256 : 128;
    const qlora_nf4_weight* w = a.w;
    const int64_t N = w->N, K = w->K;
    const bool pair = use_pairs(a.p.M);
    a.p.bn = (pair && !dx) ? pair_tile_width(a.p.M, N) : kBN;
    const uint32_t wrows = pair ? (uint32_t)a.p.bn / 2 : 256;   // forward: W rows one CTA loads codes (and LoRA B rows) for
    // segment 0: A (X or dY) and the packed codes
    if (!dx) {
        if (!make_tmap_2d(&a.tmA0, true, a.A0, K, a.p.M, K * 2, 64, bm, true)) return QLORA_ERR_CUDA;
        if (!make_tmap_2d(&a.tmCodes, false, w->codes, K / 2, N, K / 2, 32, wrows, false)) return QLORA_ERR_CUDA;
    } else {
        if (!make_tmap_2d(&a.tmA0, true, a.A0, N, a.p.M, N * 2, 64, bm, true)) return QLORA_ERR_CUDA;
        if (pair) {   // this CTA's 64 bytes (two blocks) of each of the step's 64 W rows, unswizzled
            if (!make_tmap_2d(&a.tmCodes, false, w->codes, K / 2, N, K / 2, 64, 64, false)) return QLORA_ERR_CUDA;
        } else {
            if (!make_tmap_2d(&a.tmCodes, false, w->codes, K / 2, N, K / 2, 128, 64, true)) return QLORA_ERR_CUDA;
        }
    }
    // segment 1: LoRA operands, [M, 2R] and [N, 2R] (forward) or [2R, K] (dX)
    const int64_t R2 = 2 * (int64_t)a.Rpad;
    if (!make_tmap_2d(&a.tmA1, true, a.A1, R2, a.p.M, R2 * 2, 64, bm, true)) return QLORA_ERR_CUDA;
    if (a.b1_r > 0) {   // B [N, r] or A [r, K] directly
        const uint64_t r = (uint64_t)a.b1_r;
        if (!dx) {
            if (!make_tmap_2d(&a.tmB1, true, a.B1, r, N, r * 2, 64, wrows, true)) return QLORA_ERR_CUDA;
        } else {
            if (!make_tmap_2d(&a.tmB1, true, a.B1, K, r, K * 2, 64, 64, true)) return QLORA_ERR_CUDA;
        }
        a.p.b1_wrap = (int32_t)(R2 / 128);
    } else if (!dx) {
        if (!make_tmap_2d(&a.tmB1, true, a.B1, R2, N, R2 * 2, 64, wrows, true)) return QLORA_ERR_CUDA;
    } else {
        if (!make_tmap_2d(&a.tmB1, true, a.B1, K, R2, K * 2, 64, 64, true)) return QLORA_ERR_CUDA;
    }
    a.p.ksteps0 = (int)(((dx ? N : K) + 63) / 64);
    a.p.ksteps1 = (int)(R2 / 64);
    a.p.c1_codes = w->c1_codes;
    a.p.c1f = w->c1;
    a.p.f16 = w->compute_dtype == QLORA_DTYPE_F16;
    a.p.c2 = w->c2;
    a.p.mu = w->mu;
    a.p.WN = N;
    a.p.WK = K;
    a.p.tb = host_tables(w->codebook);
    a.p.err = device_error_word();
    if (!a.p.err) return QLORA_ERR_CUDA;
    if (pair) return dx ? launch_pair<true>(a, stream) : launch_pair<false>(a, stream);
    if (bm == 256) return dx ? launch_one<2, true>(a, stream) : launch_one<2, false>(a, stream);
    return dx ? launch_one<1, true>(a, stream) : launch_one<1, false>(a, stream);
}

}  // namespace qlora
