// LoRA operand preparation for the tensor-core GEMMs.
//
// The low-rank terms (alpha/r) U B^T and dU A of the QLoRA linear layer
// ("QLoRA 的原理是什么？4-bit 量化权重真的参与训练吗？", section 7: the LoRA path
// is added to the output) are accumulated by the tensor cores as extra
// reduction steps.  U and dU are fp32 and must not lose precision, so each is
// split into two bf16 parts hi = bf16(v), lo = bf16(v - hi) (together within
// 2^-17 relative of v), and the other operand is duplicated:
//     s U B^T = [hi | lo] [B | B]^T,      dU A = [hi | lo] [A ; A].
// Every half is zero-padded from r to R (a multiple of 64) columns or rows.
// The reduce kernels finish the split-reduction LoRA GEMMs of gemm_lora_tc.cu.
#include "qlora_internal.cuh"

namespace qlora {
namespace {

constexpr int kThreads = 256;

// V2[m, j] = hi(scale * V[m, j]), V2[m, R + j] = lo(scale * V[m, j]); zero for r <= j < R.
__global__ void split_hi_lo(const float* __restrict__ V, int64_t M, int r, int R, float scale,
                            uint16_t* __restrict__ V2) {
    const int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (i >= M * R) return;
    const int64_t m = i / R;
    const int j = (int)(i - m * R);
    const float v = j < r ? __fmul_rn(scale, V[m * r + j]) : 0.f;
    const uint32_t hi = f32_to_bf16_bits_rn(v);
    const uint32_t lo = f32_to_bf16_bits_rn(__fsub_rn(v, bf16_bits_to_f32(hi)));
    V2[m * 2 * R + j] = (uint16_t)hi;
    V2[m * 2 * R + R + j] = (uint16_t)lo;
}

// B2[n, j] = B2[n, R + j] = B[n, j]; zero for r <= j < R.
__global__ void dup_cols(const uint16_t* __restrict__ B, int64_t N, int r, int R, uint16_t* __restrict__ B2) {
    const int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (i >= N * R) return;
    const int64_t n = i / R;
    const int j = (int)(i - n * R);
    const uint16_t v = j < r ? B[n * r + j] : (uint16_t)0;
    B2[n * 2 * R + j] = v;
    B2[n * 2 * R + R + j] = v;
}

// A2[j, k] = A2[R + j, k] = A[j, k]; zero rows for r <= j < R.  Moves 8 bf16 per thread.
__global__ void dup_rows(const uint4* __restrict__ A, int r, int R, int64_t K8, uint4* __restrict__ A2) {
    const int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (i >= (int64_t)R * K8) return;
    const int64_t j = i / K8;
    const int64_t k = i - j * K8;
    const uint4 v = j < r ? A[j * K8 + k] : make_uint4(0, 0, 0, 0);
    A2[j * K8 + k] = v;
    A2[(R + j) * K8 + k] = v;
}

// Bt[j, n] = B[n, j] for j < r, zero rows for r <= j < R.
__global__ void transpose_pad(const uint16_t* __restrict__ B, int64_t N, int r, int R, uint16_t* __restrict__ Bt) {
    const int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (i >= (int64_t)R * N) return;
    const int64_t j = i / N;
    const int64_t n = i - j * N;
    Bt[i] = j < r ? B[n * r + j] : (uint16_t)0;
}

// Sum of the split partials partial[s][row][j] (fixed order s = 0, 1, ...).
__device__ __forceinline__ float sum_splits(const float* __restrict__ partial, int splits, int64_t rows, int R,
                                            int64_t row, int j) {
    float acc = 0.f;
    for (int s = 0; s < splits; ++s) acc = __fadd_rn(acc, partial[((int64_t)s * rows + row) * R + j]);
    return acc;
}

// out[row, j] = scale_out * S (j < r, when out is given) and the bf16 hi/lo split
// of scale_v2 * S into V2[row, j] and V2[row, R + j] (zero for r <= j < R).
__global__ void reduce_rows(const float* __restrict__ partial, int splits, int64_t rows, int r, int R,
                            float scale_out, float* __restrict__ out, float scale_v2, uint16_t* __restrict__ V2) {
    const int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (i >= rows * R) return;
    const int64_t row = i / R;
    const int j = (int)(i - row * R);
    const float S = sum_splits(partial, splits, rows, R, row, j);
    if (out && j < r) out[row * r + j] = __fmul_rn(scale_out, S);
    if (V2) {
        const float v = j < r ? __fmul_rn(scale_v2, S) : 0.f;
        const uint32_t hi = f32_to_bf16_bits_rn(v);
        const uint32_t lo = f32_to_bf16_bits_rn(__fsub_rn(v, bf16_bits_to_f32(hi)));
        V2[row * 2 * R + j] = (uint16_t)hi;
        V2[row * 2 * R + R + j] = (uint16_t)lo;
    }
}

// out[j, row] = S for j < r (the transposed [r, rows] result, e.g. dA from dA^T partials).
__global__ void reduce_transposed(const float* __restrict__ partial, int splits, int64_t rows, int r, int R,
                                  float* __restrict__ out) {
    const int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (i >= rows * (int64_t)r) return;
    const int64_t j = i / rows;
    const int64_t row = i - j * rows;
    out[j * rows + row] = sum_splits(partial, splits, rows, R, row, (int)j);
}

inline unsigned blocks(int64_t n) { return (unsigned)((n + kThreads - 1) / kThreads); }

}  // namespace

qlora_status launch_split_hi_lo(const float* V, int64_t M, int r, int R, float scale, void* V2,
                                cudaStream_t s) {
    split_hi_lo<<<blocks(M * R), kThreads, 0, s>>>(V, M, r, R, scale, static_cast<uint16_t*>(V2));
    QLORA_CHECK_LAUNCH();
    return QLORA_OK;
}

qlora_status launch_dup_cols(const void* B, int64_t N, int r, int R, void* B2, cudaStream_t s) {
    dup_cols<<<blocks(N * R), kThreads, 0, s>>>(static_cast<const uint16_t*>(B), N, r, R,
                                                static_cast<uint16_t*>(B2));
    QLORA_CHECK_LAUNCH();
    return QLORA_OK;
}

qlora_status launch_transpose_pad(const void* B, int64_t N, int r, int R, void* Bt, cudaStream_t s) {
    transpose_pad<<<blocks((int64_t)R * N), kThreads, 0, s>>>(static_cast<const uint16_t*>(B), N, r, R,
                                                              static_cast<uint16_t*>(Bt));
    QLORA_CHECK_LAUNCH();
    return QLORA_OK;
}

qlora_status launch_reduce_rows(const float* partial, int splits, int64_t rows, int r, int R, float scale_out,
                                float* out, float scale_v2, void* V2, cudaStream_t s) {
    reduce_rows<<<blocks(rows * R), kThreads, 0, s>>>(partial, splits, rows, r, R, scale_out, out, scale_v2,
                                                       static_cast<uint16_t*>(V2));
    QLORA_CHECK_LAUNCH();
    return QLORA_OK;
}

qlora_status launch_reduce_transposed(const float* partial, int splits, int64_t rows, int r, int R, float* out,
                                      cudaStream_t s) {
    reduce_transposed<<<blocks(rows * r), kThreads, 0, s>>>(partial, splits, rows, r, R, out);
    QLORA_CHECK_LAUNCH();
    return QLORA_OK;
}

qlora_status launch_dup_rows(const void* A, int r, int R, int64_t K, void* A2, cudaStream_t s) {
    const int64_t K8 = K / 8;
    dup_rows<<<blocks((int64_t)R * K8), kThreads, 0, s>>>(static_cast<const uint4*>(A), r, R, K8,
                                                          static_cast<uint4*>(A2));
    QLORA_CHECK_LAUNCH();
    return QLORA_OK;
}

}  // namespace qlora
