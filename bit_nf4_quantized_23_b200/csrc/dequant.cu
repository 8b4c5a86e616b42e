// Dequantization of NF4 + Double Quantization to bf16 ("Science Depth M5-131:
// PEFT (LoRA / QLoRA / Prefix Tuning)", section 4 (1): W_hat = Dequant(W_NF4) * c1,
// performed on the fly in forward and backward).
//
// W_hat[n,k] = bf16_rn(fp32(q[code] * c1')) (fp16_rn for an fp16 compute dtype),
// c1' = fp32(fp32(e4m3(c1_code) * c2) + mu),
// or c1' = c1 when double quantization is off (fp32 constants stored).
// HBM-bound: 0.516 bytes read and 2 bytes written per weight.  Each thread
// expands 16 weights (8 code bytes -> 32 output bytes, 16-byte stores).
#include "qlora_internal.cuh"

namespace qlora {
namespace {

constexpr int kDeqThreads = 256;

__global__ void __launch_bounds__(kDeqThreads)
nf4_dequantize(const uint2* __restrict__ codes, const uint8_t* __restrict__ c1_codes,
               const float* __restrict__ c2, const float* __restrict__ mu_p, const float* __restrict__ c1f,
               int64_t n16, uint4* __restrict__ out, NF4Tables tb, bool f16) {
    __shared__ float q[16];
    if (threadIdx.x < 16) q[threadIdx.x] = tb.q[threadIdx.x];
    __syncthreads();
    const int64_t i = (int64_t)blockIdx.x * kDeqThreads + threadIdx.x;   // group of 16 weights
    if (i >= n16) return;
    const int64_t blk = i >> 2;
    const float c1p = c1f ? c1f[blk] : rebuild_c1(c1_codes[blk], c2[blk >> 8], *mu_p);
    const uint2 c = codes[i];
    uint32_t o[8];
#pragma unroll
    for (int b = 0; b < 8; ++b) {
        const uint32_t byte = ((b < 4 ? c.x : c.y) >> (8 * (b & 3))) & 0xFFu;
        const float w0 = __fmul_rn(q[byte >> 4], c1p);      // element 2b (high nibble)
        const float w1 = __fmul_rn(q[byte & 0xFu], c1p);    // element 2b+1
        o[b] = pack16x2_rn(w0, w1, f16);
    }
    out[2 * i] = make_uint4(o[0], o[1], o[2], o[3]);
    out[2 * i + 1] = make_uint4(o[4], o[5], o[6], o[7]);
}

}  // namespace

qlora_status launch_dequantize(const qlora_nf4_weight* w, void* W_out, cudaStream_t stream) {
    const int64_t n16 = w->N * w->K / 16;
    const unsigned grid = (unsigned)((n16 + kDeqThreads - 1) / kDeqThreads);
    nf4_dequantize<<<grid, kDeqThreads, 0, stream>>>(
        reinterpret_cast<const uint2*>(w->codes), w->c1_codes, w->c2, w->mu, w->c1, n16,
        static_cast<uint4*>(W_out), host_tables(w->codebook), w->compute_dtype == QLORA_DTYPE_F16);
    QLORA_CHECK_LAUNCH();
    return QLORA_OK;
}

}  // namespace qlora
