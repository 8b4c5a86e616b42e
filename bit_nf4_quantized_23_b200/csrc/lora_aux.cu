// LoRA operand preparation for the tensor-core GEMMs.
//
// The low-rank terms (alpha/r) U B^T and dU A of the QLoRA linear layer
// ("QLoRA 的原理是什么？4-bit 量化权重真的参与训练吗？", section 7: the LoRA path
// is added to the output) are accumulated by the tensor cores as extra
// reduction steps.  U and dU are fp32 and must not lose precision, so each is
// split into two parts of the 16-bit compute type, hi = t(v), lo = t(v - hi)
// (bf16: together within 2^-17 relative of v; fp16: 2^-23 while lo stays a
// normal fp16, i.e. |v| between ~2^-3 and 65504), and the other operand is
// read twice:
//     s U B^T = [hi | lo] [B | B]^T,      dU A = [hi | lo] [A ; A].
// The GEMMs read A and B themselves for the two halves (their tensor maps
// zero-fill ranks r .. R-1); only B with r % 8 != 0 (rows not 16-byte
// multiples) is copied into [B | B] here.
// Every half is zero-padded from r to R (a multiple of 64) columns or rows.
// The reduce kernels finish the split-reduction LoRA GEMMs of gemm_lora_tc.cu.
#include "qlora_internal.cuh"

namespace qlora {
namespace {

constexpr int kThreads = 256;

// V2[m, j] = hi(scale * V[m, j]), V2[m, R + j] = lo(scale * V[m, j]); zero for r <= j < R.
__global__ void split_hi_lo(const float* __restrict__ V, int64_t M, int r, int R, float scale,
                            uint16_t* __restrict__ V2, bool f16) {
    grid_dependency_wait();                                   // inputs of the previous kernel
    allow_dependents();
    const int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (i >= M * R) return;
    const int64_t m = i / R;
    const int j = (int)(i - m * R);
    const float v = j < r ? __fmul_rn(scale, V[m * r + j]) : 0.f;
    const uint32_t hi = to16_rn(v, f16);
    const uint32_t lo = to16_rn(__fsub_rn(v, from16(hi, f16)), f16);
    V2[m * 2 * R + j] = (uint16_t)hi;
    V2[m * 2 * R + R + j] = (uint16_t)lo;
}

// B2[n, j] = B2[n, R + j] = B[n, j]; zero for r <= j < R.
__global__ void dup_cols(const uint16_t* __restrict__ B, int64_t N, int r, int R, uint16_t* __restrict__ B2) {
    grid_dependency_wait();                                   // inputs of the previous kernel
    allow_dependents();
    const int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (i >= N * R) return;
    const int64_t n = i / R;
    const int j = (int)(i - n * R);
    const uint16_t v = j < r ? B[n * r + j] : (uint16_t)0;
    B2[n * 2 * R + j] = v;
    B2[n * 2 * R + R + j] = v;
}

// The same with 8 columns (16 bytes) per thread, for r % 8 == 0 (B rows are then 16-byte aligned).
__global__ void dup_cols8(const uint4* __restrict__ B, int64_t N, int r8, int R8, uint4* __restrict__ B2) {
    grid_dependency_wait();                                   // inputs of the previous kernel
    allow_dependents();
    const int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (i >= N * R8) return;
    const int64_t n = i / R8;
    const int c = (int)(i - n * R8);
    const uint4 v = c < r8 ? B[n * r8 + c] : make_uint4(0, 0, 0, 0);
    B2[n * 2 * R8 + c] = v;
    B2[n * 2 * R8 + R8 + c] = v;
}

// Bt[j, n] = B[n, j] for j < r, zero rows for r <= j < R.  A CTA moves a [64 n x 32 j] block
// through shared memory so that reads (along j) and writes (along n) are both coalesced.
__global__ void __launch_bounds__(256)
transpose_pad(const uint16_t* __restrict__ B, int64_t N, int r, int R, uint16_t* __restrict__ Bt) {
    grid_dependency_wait();                                   // inputs of the previous kernel
    allow_dependents();
    __shared__ uint16_t tile[32][64 + 2];
    const int64_t n0 = (int64_t)blockIdx.x * 64;
    const int j0 = blockIdx.y * 32;
    for (int e = threadIdx.x; e < 64 * 32; e += 256) {
        const int nn = e >> 5, jj = e & 31;
        const int64_t n = n0 + nn;
        tile[jj][nn] = (n < N && j0 + jj < r) ? B[n * r + j0 + jj] : (uint16_t)0;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < 64 * 32; e += 256) {
        const int jj = e >> 6, nn = e & 63;
        const int64_t n = n0 + nn;
        if (n < N && j0 + jj < R) Bt[(int64_t)(j0 + jj) * N + n] = tile[jj][nn];
    }
}

// Sum of the split partials partial[s][row][j] in the fixed order s = 0, 1, ...; the loads of
// eight splits are issued together (the kernels are latency-bound, not bandwidth-bound).
__device__ __forceinline__ float sum_splits(const float* __restrict__ partial, int splits, int64_t rows, int R,
                                            int64_t row, int j) {
    const int64_t stride = rows * R;
    const float* p = partial + row * R + j;
    float acc = 0.f;
    int s = 0;
    for (; s + 8 <= splits; s += 8) {
        float v[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) v[q] = p[(s + q) * stride];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc = __fadd_rn(acc, v[q]);
    }
    for (; s < splits; ++s) acc = __fadd_rn(acc, p[s * stride]);
    return acc;
}

// out[row, j] = scale_out * S (j < r, when out is given) and the bf16 hi/lo split
// of scale_v2 * S into V2[row, j] and V2[row, R + j] (zero for r <= j < R).
__global__ void reduce_rows(const float* __restrict__ partial, int splits, int64_t rows, int r, int R,
                            float scale_out, float* __restrict__ out, float scale_v2, uint16_t* __restrict__ V2,
                            bool f16) {
    grid_dependency_wait();                                   // inputs of the previous kernel
    allow_dependents();
    const int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (i >= rows * R) return;
    const int64_t row = i / R;
    const int j = (int)(i - row * R);
    const float S = sum_splits(partial, splits, rows, R, row, j);
    if (out && j < r) out[row * r + j] = __fmul_rn(scale_out, S);
    if (V2) {
        const float v = j < r ? __fmul_rn(scale_v2, S) : 0.f;
        const uint32_t hi = to16_rn(v, f16);
        const uint32_t lo = to16_rn(__fsub_rn(v, from16(hi, f16)), f16);
        V2[row * 2 * R + j] = (uint16_t)hi;
        V2[row * 2 * R + R + j] = (uint16_t)lo;
    }
}

// out[j, row] = S for j < r (the transposed [r, rows] result, e.g. dA from dA^T partials).
// A CTA sums a [16 rows x 64 j] block (reads along j, coalesced; each thread 4 elements with
// all their split loads issued before any add) into shared memory and writes it transposed
// (writes along rows, coalesced).
constexpr int kTrRows = 16;
__global__ void __launch_bounds__(256)
reduce_transposed(const float* __restrict__ partial, int splits, int64_t rows, int r, int R, float* __restrict__ out) {
    grid_dependency_wait();                                   // inputs of the previous kernel
    allow_dependents();
    __shared__ float tile[64][kTrRows + 1];
    const int64_t row0 = (int64_t)blockIdx.x * kTrRows;
    const int j0 = blockIdx.y * 64;
    const int64_t stride = rows * R;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    int64_t src[4];
    bool ok[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {                             // element e = tid + 256 u: row e / 64, j e % 64
        const int e = threadIdx.x + 256 * u;
        const int64_t row = row0 + (e >> 6);
        ok[u] = row < rows && j0 + (e & 63) < R;
        src[u] = row * R + j0 + (e & 63);
    }
    for (int s = 0; s < splits; s += 2) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            v[2 * u] = ok[u] ? partial[s * stride + src[u]] : 0.f;
            v[2 * u + 1] = (ok[u] && s + 1 < splits) ? partial[(s + 1) * stride + src[u]] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            acc[u] = __fadd_rn(acc[u], v[2 * u]);
            if (s + 1 < splits) acc[u] = __fadd_rn(acc[u], v[2 * u + 1]);
        }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int e = threadIdx.x + 256 * u;
        tile[e & 63][e >> 6] = acc[u];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < kTrRows * 64; e += 256) {
        const int jj = e / kTrRows, rr = e % kTrRows;
        const int64_t row = row0 + rr;
        if (row < rows && j0 + jj < r) out[(int64_t)(j0 + jj) * rows + row] = tile[jj][rr];
    }
}

inline unsigned blocks(int64_t n) { return (unsigned)((n + kThreads - 1) / kThreads); }

}  // namespace

qlora_status launch_split_hi_lo(const float* V, int64_t M, int r, int R, float scale, void* V2, bool f16,
                                cudaStream_t s) {
    (void)launch_dependent(split_hi_lo, dim3(blocks(M * R)), dim3(kThreads), 0, s, V, M, r, R, scale,
                           static_cast<uint16_t*>(V2), f16);
    QLORA_CHECK_LAUNCH();
    return QLORA_OK;
}

qlora_status launch_dup_cols(const void* B, int64_t N, int r, int R, void* B2, cudaStream_t s) {
    if (r % 8 == 0 && (reinterpret_cast<uintptr_t>(B) & 15u) == 0)
        (void)launch_dependent(dup_cols8, dim3(blocks(N * (R / 8))), dim3(kThreads), 0, s,
                               static_cast<const uint4*>(B), N, r / 8, R / 8, static_cast<uint4*>(B2));
    else
        (void)launch_dependent(dup_cols, dim3(blocks(N * R)), dim3(kThreads), 0, s,
                               static_cast<const uint16_t*>(B), N, r, R, static_cast<uint16_t*>(B2));
    QLORA_CHECK_LAUNCH();
    return QLORA_OK;
}

qlora_status launch_transpose_pad(const void* B, int64_t N, int r, int R, void* Bt, cudaStream_t s) {
    const dim3 grid((unsigned)((N + 63) / 64), (unsigned)((R + 31) / 32));
    (void)launch_dependent(transpose_pad, grid, dim3(256), 0, s, static_cast<const uint16_t*>(B), N, r, R,
                           static_cast<uint16_t*>(Bt));
    QLORA_CHECK_LAUNCH();
    return QLORA_OK;
}

qlora_status launch_reduce_rows(const float* partial, int splits, int64_t rows, int r, int R, float scale_out,
                                float* out, float scale_v2, void* V2, bool f16, cudaStream_t s) {
    (void)launch_dependent(reduce_rows, dim3(blocks(rows * R)), dim3(kThreads), 0, s, partial, splits, rows, r, R,
                           scale_out, out, scale_v2, static_cast<uint16_t*>(V2), f16);
    QLORA_CHECK_LAUNCH();
    return QLORA_OK;
}

qlora_status launch_reduce_transposed(const float* partial, int splits, int64_t rows, int r, int R, float* out,
                                      cudaStream_t s) {
    const dim3 grid((unsigned)((rows + kTrRows - 1) / kTrRows), (unsigned)((R + 63) / 64));
    (void)launch_dependent(reduce_transposed, grid, dim3(256), 0, s, partial, splits, rows, r, R, out);
    QLORA_CHECK_LAUNCH();
    return QLORA_OK;
}


}  // namespace qlora
