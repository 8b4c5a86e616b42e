// Host interface of the tcgen05 fused dequant-GEMM (gemm_tc.cu).
#pragma once

#include <cuda.h>

#include "qlora_internal.cuh"

namespace qlora {

struct TcGemmParams {
    int64_t M;              // output rows (tokens)
    int64_t Nout;           // output columns (N for the forward, K for dX)
    int32_t ksteps0;        // 64-wide reduction steps over the frozen weight
    int32_t ksteps1;        // 64-wide reduction steps over the LoRA operands
    const uint8_t* c1_codes;
    const float* c2;
    const float* mu;
    const float* c1f;       // double quantization off: fp32 block constants (c1_codes, c2, mu unused)
    int32_t f16;            // compute dtype fp16 (W_hat, activations and 16-bit outputs) instead of bf16
    int64_t WN, WK;         // shape of W
    void* out;
    int64_t ldo;
    int32_t out_f32;
    int32_t b1_wrap;        // 0, or R/64 when B1 is the undoubled B / A: LoRA step j reads its step j % b1_wrap
    int32_t bn;             // forward on CTA pairs: output columns per pair tile (256, 240 or 224; each CTA
                            // supplies bn / 2 of them); 256 everywhere else
    uint32_t* err;
    NF4Tables tb;
};

struct TcGemmArgs {
    const qlora_nf4_weight* w;
    const void* A0;         // X [M,K] (forward) or dY [M,N] (dX), bf16
    const void* A1;         // U2 or dU2 [M, 2*Rpad], bf16
    const void* B1;         // B2 [N, 2*Rpad] (forward) or A2 [2*Rpad, K] (dX), bf16; or, with b1_r > 0,
                            // B [N, b1_r] / A [b1_r, K] themselves (the hi and lo steps read the same tile,
                            // ranks past b1_r read as zero; B needs b1_r % 8 == 0)
    int32_t b1_r;
    int32_t Rpad;           // LoRA rank padded to a multiple of 64
    TcGemmParams p;
    CUtensorMap tmA0, tmCodes, tmA1, tmB1;
};

// Encodes the tensor maps and launches the forward (dx = false) or dX kernel.
qlora_status launch_tc_gemm_nf4(TcGemmArgs& a, bool dx, cudaStream_t stream);

// Small-M forward (M <= 16): swap-AB fused dequant-GEMM, stream-K over
// (tile, K-step) units with fp32 partial tiles and a fixup that adds the LoRA term.
struct DecodeParams {
    int64_t M, N, K;
    int32_t ksteps;         // K / 64: units per tile of 128 W rows
    int64_t units;          // tiles * ksteps
    int64_t grid;           // persistent CTAs; CTA b takes units [b*units/grid, (b+1)*units/grid)
    const uint8_t* c1_codes;
    const float* c2;
    const float* mu;
    const float* c1f;       // double quantization off: fp32 block constants (c1_codes, c2, mu unused)
    int32_t f16;            // compute dtype fp16 (W_hat, activations and 16-bit outputs) instead of bf16
    float* partial;         // [tiles + grid][16][128] fp32 partial tiles, slot = tile + CTA
    uint32_t* err;
    uint32_t* dbg;          // second device word: where a self-check or a wait gave up
    NF4Tables tb;
    // U = X A^T, computed by the producer warps before their first unit (written for the fixup)
    const uint4* X;         // [M, K] 16-bit, as 16-byte chunks
    const uint4* A;         // [r, K] (or [n_adapters, r, K] with aidx)
    int64_t K8;             // K / 8
    int32_t r;
    float* U;               // [M, r] fp32
    const int32_t* aidx;    // per-token adapter (-1: none) or NULL
    int32_t n_adapters;
};

struct DecodeArgs {
    const qlora_nf4_weight* w;
    const void* X;          // [M, K] bf16
    const void* A;          // [r, K] bf16
    const void* B;          // [N, r] bf16
    int32_t r;
    float scale;            // alpha / r
    int64_t M;
    void* out;
    int32_t out_f32;
    float* U;               // [M, r] fp32, written (X A^T)
    float* partial;         // decode_partial_bytes(N, K)
    const int32_t* aidx;    // multi-adapter: device [M] adapter of each token (-1: none); NULL: one adapter
    int32_t n_adapters;     // multi-adapter: A is [n_adapters, r, K], B is [n_adapters, N, r]
};

constexpr int64_t kDecodeMaxM = 16;
size_t decode_partial_bytes(int64_t N, int64_t K);
qlora_status launch_tc_decode(const DecodeArgs& a, cudaStream_t stream);

// LoRA-side GEMM (gemm_lora_tc.cu): partial[split][rows][R] = sum over the
// split's share of the reduction of A-operand rows times B-operand rows.
struct LoraGemmParams {
    int64_t rows;
    int32_t R;
    int32_t ksteps_total;
    int32_t ksteps_per_split;
    uint32_t tmem_cols;
    uint32_t stages, b_stage;   // pipeline depth and bytes of one B stage (set by the launcher)
    int32_t f16;                // operands in fp16 instead of bf16
    float* partial;
    uint32_t* err;
};

struct LoraGemmArgs {
    bool mn_major;     // false: A [rows, red] (lda), B [R, red] (ldb); true: A from S [red, rows], B from V2 [red, 2R]
    const void* A;
    int64_t lda;
    const void* B;
    int64_t ldb;
    int64_t rows, red;
    int32_t R;
    int64_t b_rows;    // K-major B: rows present in memory (B rows past it, up to R, read as zero); 0: R
    bool b_mn;         // with mn_major false: B is [red, b_cols] with its columns contiguous (ldb >= b_cols,
                       // ldb * 2 a multiple of 16); columns b_cols .. R-1 read as zero
    int64_t b_cols;
    float* partial;
    int32_t f16;       // operands in fp16 instead of bf16
};

qlora_status launch_lora_gemm(const LoraGemmArgs& a, cudaStream_t stream);
int lora_splits(int64_t rows, int ksteps_total, int R, bool mn_major);
size_t lora_partial_bytes(int64_t rows, int64_t red, int R, bool mn_major);

bool make_tmap_2d(CUtensorMap* map, bool bf16, const void* base, uint64_t inner, uint64_t outer,
                  uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, bool swizzle128);

}  // namespace qlora
