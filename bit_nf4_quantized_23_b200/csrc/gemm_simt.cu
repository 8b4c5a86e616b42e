// Plain CUDA-core GEMM with on-the-fly NF4 dequantization.
//
// C = sum over up to two segments s of  scale_s * sum_k A_s(m,k) * B_s(n,k),
// accumulated in fp32.  Each operand is a strided bf16, fp16 or fp32 matrix, or the
// dequantized frozen weight W_hat (as W_hat[n][k] or transposed, W_hat[k][n]),
// expanded element by element with the same arithmetic as the dequantize
// kernel.  This path is the correctness baseline of the library and the GEMM
// used for shapes the tensor-core kernel does not take; it is never a CPU path.
#include "qlora_internal.cuh"
#include "gemm_simt.cuh"

namespace qlora {
namespace {

constexpr int kTile = 64;
constexpr int kBK = 16;
constexpr int kThreads = 256;

__device__ __forceinline__ float load_operand(const SimtOperand& op, int64_t row, int64_t k,
                                              const float* q) {
    switch (op.kind) {
        case SIMT_BF16:
            return bf16_bits_to_f32(static_cast<const uint16_t*>(op.ptr)[row * op.s_row + k * op.s_k]);
        case SIMT_F32:
            return static_cast<const float*>(op.ptr)[row * op.s_row + k * op.s_k];
        case SIMT_F16:
            return f16_bits_to_f32(static_cast<const uint16_t*>(op.ptr)[row * op.s_row + k * op.s_k]);
        default: {
            const int64_t wr = (op.kind == SIMT_NF4) ? row : k;
            const int64_t wc = (op.kind == SIMT_NF4) ? k : row;
            const int64_t flat = wr * op.WK + wc;
            const uint32_t byte = static_cast<const uint8_t*>(op.ptr)[flat >> 1];
            const uint32_t code = (flat & 1) ? (byte & 0xFu) : (byte >> 4);
            const int64_t blk = flat >> 6;
            const float c1p = op.c1f ? op.c1f[blk] : rebuild_c1(op.c1_codes[blk], op.c2[blk >> 8], *op.mu);
            return from16(dequant_bits(q[code], c1p, op.f16 != 0), op.f16 != 0);
        }
    }
}

__global__ void __launch_bounds__(kThreads)
simt_gemm(SimtGemm g, NF4Tables tb) {
    __shared__ float q[16];
    __shared__ float As[kBK][kTile + 1];
    __shared__ float Bs[kBK][kTile + 1];
    if (threadIdx.x < 16) q[threadIdx.x] = tb.q[threadIdx.x];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const int64_t m0 = (int64_t)blockIdx.y * kTile, n0 = (int64_t)blockIdx.x * kTile;
    float total[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) total[i][j] = 0.f;

    for (int s = 0; s < g.nseg; ++s) {
        const SimtSegment& seg = g.seg[s];
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
        for (int64_t k0 = 0; k0 < seg.K; k0 += kBK) {
            __syncthreads();
            for (int e = threadIdx.x; e < kTile * kBK; e += kThreads) {
                const int r = e / kBK, kk = e % kBK;
                const int64_t gm = m0 + r, gn = n0 + r, gk = k0 + kk;
                As[kk][r] = (gm < g.M && gk < seg.K) ? load_operand(seg.a, gm, gk, q) : 0.f;
                Bs[kk][r] = (gn < g.N && gk < seg.K) ? load_operand(seg.b, gn, gk, q) : 0.f;
            }
            __syncthreads();
#pragma unroll
            for (int kk = 0; kk < kBK; ++kk) {
                float a[4], b[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
                for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) total[i][j] = fmaf(seg.scale, acc[i][j], total[i][j]);
    }

#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t m = m0 + ty * 4 + i;
        if (m >= g.M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t n = n0 + tx * 4 + j;
            if (n >= g.N) continue;
            const int64_t off = g.transpose_c ? n * g.ldc + m : m * g.ldc + n;
            if (g.c_dtype == QLORA_DTYPE_F32) {
                static_cast<float*>(g.C)[off] = total[i][j];
            } else {
                static_cast<uint16_t*>(g.C)[off] = (uint16_t)to16_rn(total[i][j], g.c_dtype == QLORA_DTYPE_F16);
            }
        }
    }
}

}  // namespace

qlora_status launch_simt_gemm(const SimtGemm& g, cudaStream_t stream) {
    if (g.M <= 0 || g.N <= 0) return QLORA_OK;
    const dim3 grid((unsigned)((g.N + kTile - 1) / kTile), (unsigned)((g.M + kTile - 1) / kTile));
    int codebook = QLORA_CODEBOOK_NF4;
    for (int i = 0; i < g.nseg; ++i)
        for (const SimtOperand* o : {&g.seg[i].a, &g.seg[i].b})
            if (o->kind == SIMT_NF4 || o->kind == SIMT_NF4_T) codebook = o->codebook;
    simt_gemm<<<grid, kThreads, 0, stream>>>(g, host_tables(codebook));
    QLORA_CHECK_LAUNCH();
    return QLORA_OK;
}

}  // namespace qlora
