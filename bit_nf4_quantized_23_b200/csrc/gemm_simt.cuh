// Descriptors of the CUDA-core GEMM (gemm_simt.cu).
#pragma once

#include "qlora_internal.cuh"

namespace qlora {

enum SimtKind : int32_t {
    SIMT_BF16 = 0,   // element (row, k) = ((bf16*)ptr)[row*s_row + k*s_k]
    SIMT_F32 = 1,    // element (row, k) = ((float*)ptr)[row*s_row + k*s_k]
    SIMT_NF4 = 2,    // element (row, k) = W_hat[row][k]
    SIMT_NF4_T = 3,  // element (row, k) = W_hat[k][row]
    SIMT_F16 = 4     // element (row, k) = ((fp16*)ptr)[row*s_row + k*s_k]
};

struct SimtOperand {
    int32_t kind;
    const void* ptr;            // data, or the packed codes for the NF4 kinds
    int64_t s_row, s_k;
    const uint8_t* c1_codes;    // NF4 kinds only
    const float* c2;
    const float* mu;
    const float* c1f;           // NF4 kinds with double quantization off: fp32 block constants
    int64_t WK;                 // columns of W (NF4 kinds)
    int32_t codebook;           // NF4 kinds: qlora_codebook
    int32_t f16;                // NF4 kinds: W_hat rounded to fp16 (compute dtype) instead of bf16
};

struct SimtSegment {
    SimtOperand a, b;
    int64_t K;
    float scale;
};

struct SimtGemm {
    SimtSegment seg[2];
    int32_t nseg;
    int64_t M, N;
    void* C;                    // [M,N] row-major with leading dim ldc, or its transpose
    int32_t c_dtype;            // QLORA_DTYPE_BF16 / QLORA_DTYPE_F32 / QLORA_DTYPE_F16
    int64_t ldc;
    int32_t transpose_c;        // 1: element (m,n) stored at C[n*ldc + m]
};

inline SimtOperand simt_dense(int32_t kind, const void* p, int64_t s_row, int64_t s_k) {
    SimtOperand o{};
    o.kind = kind; o.ptr = p; o.s_row = s_row; o.s_k = s_k;
    return o;
}

inline SimtOperand simt_nf4(const qlora_nf4_weight* w, bool transposed) {
    SimtOperand o{};
    o.kind = transposed ? SIMT_NF4_T : SIMT_NF4;
    o.ptr = w->codes; o.c1_codes = w->c1_codes; o.c2 = w->c2; o.mu = w->mu; o.c1f = w->c1; o.WK = w->K;
    o.codebook = w->codebook;
    o.f16 = w->compute_dtype == QLORA_DTYPE_F16;
    return o;
}

qlora_status launch_simt_gemm(const SimtGemm& g, cudaStream_t stream);

}  // namespace qlora
