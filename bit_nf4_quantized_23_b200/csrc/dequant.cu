// Dequantization of NF4 + Double Quantization to bf16 ("Science Depth M5-131:
// PEFT (LoRA / QLoRA / Prefix Tuning)", section 4 (1): W_hat = Dequant(W_NF4) * c1,
// performed on the fly in forward and backward).
//
// W_hat[n,k] = bf16_rn(fp32(q[code] * c1')) (fp16_rn for an fp16 compute dtype),
// c1' = fp32(fp32(e4m3(c1_code) * c2) + mu),
// or c1' = c1 when double quantization is off (fp32 constants stored).
// HBM-bound: 0.516 bytes read and 2 bytes written per weight.  The unit of work
// is one 32-bit word of packed codes (8 weights -> one 16-byte store).  A CTA
// covers kDeqUnroll x 256 consecutive words; thread t takes words t + 256 u, so
// every load and store instruction of a warp touches one contiguous span (128 B
// of codes, 512 B of output), and all of a thread's loads (codes and block
// constants) are issued before any arithmetic, which keeps 8 words per thread
// in flight against the HBM latency.
#include "qlora_internal.cuh"

namespace qlora {
namespace {

constexpr int kDeqThreads = 256;
constexpr int kDeqUnroll = 8;

__global__ void __launch_bounds__(kDeqThreads)
nf4_dequantize(const uint32_t* __restrict__ codes, const uint8_t* __restrict__ c1_codes,
               const float* __restrict__ c2, const float* __restrict__ mu_p, const float* __restrict__ c1f,
               int64_t n_words, uint4* __restrict__ out, NF4Tables tb, bool f16) {
    __shared__ float q[16];
    if (threadIdx.x < 16) q[threadIdx.x] = tb.q[threadIdx.x];
    const int64_t w0 = (int64_t)blockIdx.x * (kDeqThreads * kDeqUnroll) + threadIdx.x;
    uint32_t cw[kDeqUnroll], cc[kDeqUnroll];
    float cs[kDeqUnroll];
#pragma unroll
    for (int u = 0; u < kDeqUnroll; ++u) {
        const int64_t i = w0 + (int64_t)u * kDeqThreads;
        const bool v = i < n_words;
        const int64_t blk = i >> 3;                                // 8 words per block of 64
        cw[u] = v ? __ldcs(codes + i) : 0u;
        if (c1f) {
            cc[u] = 0u;
            cs[u] = v ? __ldg(c1f + blk) : 0.f;
        } else {
            cc[u] = v ? (uint32_t)__ldg(c1_codes + blk) : 0u;
            cs[u] = v ? __ldg(c2 + (blk >> 8)) : 0.f;
        }
    }
    const float mu = c1f ? 0.f : __ldg(mu_p);
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kDeqUnroll; ++u) {
        const int64_t i = w0 + (int64_t)u * kDeqThreads;
        if (i >= n_words) break;
        const float c1p = c1f ? cs[u] : rebuild_c1(cc[u], cs[u], mu);
        uint32_t o[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const uint32_t byte = (cw[u] >> (8 * b)) & 0xFFu;
            o[b] = pack16x2_rn(__fmul_rn(q[byte >> 4], c1p),       // element 2b (high nibble)
                               __fmul_rn(q[byte & 0xFu], c1p), f16);  // element 2b+1
        }
        __stcs(out + i, make_uint4(o[0], o[1], o[2], o[3]));
    }
}

}  // namespace

qlora_status launch_dequantize(const qlora_nf4_weight* w, void* W_out, cudaStream_t stream) {
    const int64_t n_words = w->N * w->K / 8;
    const int64_t per_cta = (int64_t)kDeqThreads * kDeqUnroll;
    const unsigned grid = (unsigned)((n_words + per_cta - 1) / per_cta);
    nf4_dequantize<<<grid, kDeqThreads, 0, stream>>>(
        reinterpret_cast<const uint32_t*>(w->codes), w->c1_codes, w->c2, w->mu, w->c1, n_words,
        static_cast<uint4*>(W_out), host_tables(w->codebook), w->compute_dtype == QLORA_DTYPE_F16);
    QLORA_CHECK_LAUNCH();
    return QLORA_OK;
}

}  // namespace qlora
