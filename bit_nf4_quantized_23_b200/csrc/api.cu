// The C ABI of libqlora.so (declared in include/qlora.h): argument validation
// on the host, then the kernel launches of each operation.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <climits>
#include <cstring>
#include <mutex>

#include "qlora_internal.cuh"
#include "gemm_simt.cuh"
#include "gemm_tc.cuh"
#include "timing.cuh"

namespace qlora {

size_t quantize_workspace_bytes(int64_t nb1);
qlora_status launch_quantize(const void* W, int64_t N, int64_t K, const qlora_nf4_weight* out,
                             void* workspace, cudaStream_t stream);
qlora_status launch_dequantize(const qlora_nf4_weight* w, void* W_out, cudaStream_t stream);
qlora_status launch_int8_quantize(const void* W, int64_t n, int blocksize, int8_t* codes, float* alpha,
                                  cudaStream_t s);
qlora_status launch_int8_dequantize(const int8_t* codes, const float* alpha, int64_t n, int blocksize, void* out,
                                    int out_dtype, cudaStream_t s);
uint32_t* device_error_word();
qlora_status launch_bounded_wait_probe(uint64_t limit_ns, uint32_t* result, cudaStream_t s);
qlora_status launch_split_hi_lo(const float* V, int64_t M, int r, int R, float scale, void* V2, bool f16,
                                cudaStream_t s);
qlora_status launch_dup_cols(const void* B, int64_t N, int r, int R, void* B2, cudaStream_t s);
qlora_status launch_transpose_pad(const void* B, int64_t N, int r, int R, void* Bt, cudaStream_t s);
qlora_status launch_merge(const qlora_nf4_weight* w, const void* A, const void* B, int32_t r, float scale,
                          void* W_out, cudaStream_t stream);
qlora_status launch_reduce_rows(const float* partial, int splits, int64_t rows, int r, int R, float scale_out,
                                float* out, float scale_v2, void* V2, bool f16, cudaStream_t s);
qlora_status launch_reduce_transposed(const float* partial, int splits, int64_t rows, int r, int R, float* out,
                                      cudaStream_t s);

// Argument checks shared by the entry points (declared in qlora_internal.cuh).
qlora_status check_blocks(int32_t bs, int32_t bs2) {
    return (bs == 64 && bs2 == 256) ? QLORA_OK : QLORA_ERR_UNSUPPORTED;
}

qlora_status check_shape(int64_t N, int64_t K) {
    if (N < 1 || K < 1 || K % 64 != 0) return QLORA_ERR_SHAPE;
    if (N > (int64_t(1) << 40) / K) return QLORA_ERR_SHAPE;   // keeps every flat index in int64 range
    if (N > INT32_MAX || K > INT32_MAX) return QLORA_ERR_SHAPE;  // tensor-map coordinates are 32-bit
    return QLORA_OK;
}

qlora_status check_weight(const qlora_nf4_weight* w) {
    if (!w) return QLORA_ERR_INVALID_ARG;
    QLORA_TRY(check_blocks(w->blocksize, w->blocksize2));
    QLORA_TRY(check_shape(w->N, w->K));
    if (w->codebook != QLORA_CODEBOOK_NF4 && w->codebook != QLORA_CODEBOOK_UNIFORM4) return QLORA_ERR_INVALID_ARG;
    if (w->compute_dtype != QLORA_DTYPE_BF16 && w->compute_dtype != QLORA_DTYPE_F16) return QLORA_ERR_INVALID_ARG;
    if (!w->codes) return QLORA_ERR_INVALID_ARG;
    if (!aligned16(w->codes)) return QLORA_ERR_ALIGN;
    if (w->c1) {   // double quantization off: fp32 block constants only
        if (!aligned16(w->c1)) return QLORA_ERR_ALIGN;
        return QLORA_OK;
    }
    if (!w->c1_codes || !w->c2 || !w->mu) return QLORA_ERR_INVALID_ARG;
    if (!aligned16(w->c1_codes) || !aligned16(w->c2) || !aligned16(w->mu)) return QLORA_ERR_ALIGN;
    return QLORA_OK;
}

qlora_status check_dev(const void* p) {
    if (!p) return QLORA_ERR_INVALID_ARG;
    return aligned16(p) ? QLORA_OK : QLORA_ERR_ALIGN;
}

namespace {

std::atomic<uint64_t> g_launches{0};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

qlora_status check_lora(int64_t M, int32_t r, float alpha) {
    if (M < 1 || M > (int64_t(1) << 31)) return QLORA_ERR_SHAPE;
    if (r < 1 || r > 256) return QLORA_ERR_INVALID_ARG;
    if (!std::isfinite(alpha)) return QLORA_ERR_INVALID_ARG;
    return QLORA_OK;
}

// LoRA rank padded to a multiple of 64 (each hi/lo half fills whole 64-wide reduction steps).
inline int32_t rank_pad(int32_t r) { return (r + 63) / 64 * 64; }

// Workspace of the linear layer (every piece 256-byte aligned):
//   U   fp32 [M,r]        (when the caller keeps none)
//   dU  fp32 [M,r]
//   U2  bf16 [M,2R]       hi/lo split of s*U
//   dU2 bf16 [M,2R]       hi/lo split of dU
//   B2  bf16 [N,2R]       [B | B] (only when r % 8 != 0; otherwise the GEMM reads B itself)
//   Bt  bf16 [R,N]        B^T, zero-padded (the dU GEMM reads it only when r % 8 != 0)
//   partial fp32          split-reduction partial sums of the LoRA GEMMs
struct LinearWs {
    size_t u_off, du_off, u2_off, du2_off, b2_off, bt_off, part_off, total;
};

LinearWs linear_ws(int64_t M, int64_t N, int64_t K, int32_t r) {
    const size_t R = (size_t)rank_pad(r);
    LinearWs l;
    size_t o = 0;
    l.u_off = o;   o += align_up((size_t)M * r * sizeof(float), 256);
    l.du_off = o;  o += align_up((size_t)M * r * sizeof(float), 256);
    l.u2_off = o;  o += align_up((size_t)M * 2 * R * 2, 256);
    l.du2_off = o; o += align_up((size_t)M * 2 * R * 2, 256);
    l.b2_off = o;  o += align_up((size_t)N * 2 * R * 2, 256);
    l.bt_off = o;  o += align_up(R * (size_t)N * 2, 256);
    size_t part = lora_partial_bytes(M, K, (int)R, false);          // U
    part = std::max(part, lora_partial_bytes(M, N, (int)R, false));  // dU
    part = std::max(part, lora_partial_bytes(K, M, (int)R, true));   // dA
    part = std::max(part, lora_partial_bytes(N, M, (int)R, true));   // dB
    if (M <= kDecodeMaxM) part = std::max(part, decode_partial_bytes(N, K));   // decode partial tiles
    l.part_off = o; o += align_up(part, 256);
    l.total = o;
    return l;
}

// U = X A^T on the tensor cores, reduced into U (fp32, may be null) and U2 = hi/lo(s U).
// A [r, K] is read directly (ranks r .. R-1 read as zero).
qlora_status lora_U(const void* X, const void* A, int64_t M, int64_t K, int32_t r, int32_t R, float s_lora,
                    float* U, void* U2, float* partial, bool f16, cudaStream_t s) {
    TimerScope t(QLORA_TIMER_LORA, s);
    LoraGemmArgs g{};
    g.mn_major = false; g.A = X; g.lda = K; g.B = A; g.ldb = K; g.rows = M; g.red = K; g.R = R; g.partial = partial;
    g.b_rows = r;
    g.f16 = f16;
    QLORA_TRY(launch_lora_gemm(g, s));
    const int splits = lora_splits(M, (int)((K + 63) / 64), R, false);
    return launch_reduce_rows(partial, splits, M, r, R, 1.f, U, s_lora, U2, f16, s);
}

// The backward's adapter-gradient work (dA, dB and their reductions) runs on a second stream of
// the lowest priority, forked from the caller's stream after dU is ready and joined back before
// the call returns: it reads only dU, X, dY and U, none of which the dX GEMM writes, so it can
// fill the SMs that the dX GEMM's last wave of tiles leaves idle.  One side stream per device,
// created on first use; calls from several host threads share it (their adapter work is then
// serialised on it, which is correct but not concurrent).
cudaStream_t side_stream() {
    static std::mutex mu;
    static cudaStream_t streams[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!streams[dev]) {
        int least = 0, greatest = 0;
        if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess) return nullptr;
        cudaStream_t st = nullptr;
        if (cudaStreamCreateWithPriority(&st, cudaStreamNonBlocking, least) != cudaSuccess) return nullptr;
        streams[dev] = st;
    }
    return streams[dev];
}

// dA = dU^T X (computed as dA^T [K, R] = X^T dU) and dB = s dY^T U = dY^T (s U) from the hi/lo
// operands dU2 and U2, on stream g; both use the split-partial region in turn.
qlora_status lora_gradients_tc(const void* X, const void* dY, int64_t M, int64_t N, int64_t K, int32_t r,
                               int32_t R, bool f16, float* dA, float* dB, const void* U2, const void* dU2,
                               float* partial, cudaStream_t g) {
    {
        TimerScope t(QLORA_TIMER_LORA, g);
        LoraGemmArgs a{};
        a.mn_major = true; a.A = X; a.lda = K; a.B = dU2; a.ldb = 2 * R; a.rows = K; a.red = M; a.R = R;
        a.partial = partial;
        a.f16 = f16;
        QLORA_TRY(launch_lora_gemm(a, g));
        QLORA_TRY(launch_reduce_transposed(partial, lora_splits(K, (int)((M + 63) / 64), R, true), K, r, R, dA, g));
    }
    {
        TimerScope t(QLORA_TIMER_LORA, g);
        LoraGemmArgs a{};
        a.mn_major = true; a.A = dY; a.lda = N; a.B = U2; a.ldb = 2 * R; a.rows = N; a.red = M; a.R = R;
        a.partial = partial;
        a.f16 = f16;
        QLORA_TRY(launch_lora_gemm(a, g));
        QLORA_TRY(launch_reduce_rows(partial, lora_splits(N, (int)((M + 63) / 64), R, true), N, r, R, 1.f, dB, 0.f,
                                     nullptr, f16, g));
    }
    return QLORA_OK;
}

// Output dtypes a layer may write: fp32, or its 16-bit compute dtype.
qlora_status check_out_dtype(int32_t dt, const qlora_nf4_weight* w) {
    return (dt == QLORA_DTYPE_F32 || dt == w->compute_dtype) ? QLORA_OK : QLORA_ERR_INVALID_ARG;
}

}  // namespace

void note_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

bool sync_check_enabled() {
    static const bool on = std::getenv("QLORA_SYNC_CHECK") != nullptr;
    return on;
}

bool sync_check(const char* where) {
    const cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        std::fprintf(stderr, "[qlora] kernel launched from %s failed: %s\n", where, cudaGetErrorString(e));
        return false;
    }
    return true;
}

}  // namespace qlora

using namespace qlora;

extern "C" {

const char* qlora_status_string(qlora_status s) {
    switch (s) {
        case QLORA_OK: return "QLORA_OK";
        case QLORA_ERR_INVALID_ARG: return "QLORA_ERR_INVALID_ARG: null pointer or argument out of range";
        case QLORA_ERR_SHAPE: return "QLORA_ERR_SHAPE: need N, K, M >= 1 and K % 64 == 0";
        case QLORA_ERR_ALIGN: return "QLORA_ERR_ALIGN: device pointers must be 16-byte aligned";
        case QLORA_ERR_UNSUPPORTED: return "QLORA_ERR_UNSUPPORTED: only blocksize 64 and blocksize2 256";
        case QLORA_ERR_NONFINITE: return "QLORA_ERR_NONFINITE: the weight held Inf or NaN";
        case QLORA_ERR_TIMEOUT: return "QLORA_ERR_TIMEOUT: a bounded device wait ran out";
        case QLORA_ERR_CUDA: return "QLORA_ERR_CUDA: a CUDA call or kernel launch failed";
        case QLORA_ERR_WORKSPACE: return "QLORA_ERR_WORKSPACE: workspace missing or too small";
        case QLORA_ERR_TOO_LARGE:
            return "QLORA_ERR_TOO_LARGE: more than 67108864 weights for the static scratch of "
                   "qlora_quantize_nf4_dq_noalloc";
    }
    return "QLORA_ERR_UNKNOWN";
}

qlora_status qlora_nf4_sizes(int64_t N, int64_t K, int32_t blocksize, int32_t blocksize2,
                             size_t* codes_bytes, size_t* c1_codes_bytes, size_t* c2_bytes,
                             size_t* quant_workspace_bytes) {
    QLORA_TRY(check_blocks(blocksize, blocksize2));
    QLORA_TRY(check_shape(N, K));
    const int64_t nb1 = N * K / 64;
    const int64_t nb2 = (nb1 + 255) / 256;
    if (codes_bytes) *codes_bytes = (size_t)(N * K / 2);
    if (c1_codes_bytes) *c1_codes_bytes = (size_t)nb1;
    if (c2_bytes) *c2_bytes = (size_t)nb2 * sizeof(float);
    if (quant_workspace_bytes) *quant_workspace_bytes = quantize_workspace_bytes(nb1);
    return QLORA_OK;
}

qlora_status qlora_codebook_values(int32_t codebook, float values[16], float thresholds[15]) {
    if (codebook != QLORA_CODEBOOK_NF4 && codebook != QLORA_CODEBOOK_UNIFORM4) return QLORA_ERR_INVALID_ARG;
    const NF4Tables& tb = host_tables(codebook);
    if (values) std::memcpy(values, tb.q, sizeof(tb.q));
    if (thresholds) std::memcpy(thresholds, tb.t, sizeof(tb.t));
    return QLORA_OK;
}

qlora_status qlora_nf4_codebook(float values[16], float thresholds[15]) {
    return qlora_codebook_values(QLORA_CODEBOOK_NF4, values, thresholds);
}

qlora_status qlora_quantize_nf4_dq(const void* W, int64_t N, int64_t K, int32_t blocksize,
                                   int32_t blocksize2, const qlora_nf4_weight* out,
                                   void* workspace, size_t workspace_bytes, void* stream) {
    QLORA_TRY(check_blocks(blocksize, blocksize2));
    QLORA_TRY(check_shape(N, K));
    QLORA_TRY(check_dev(W));
    QLORA_TRY(check_weight(out));
    if (out->N != N || out->K != K) return QLORA_ERR_SHAPE;
    if (!workspace || workspace_bytes < quantize_workspace_bytes(N * K / 64)) return QLORA_ERR_WORKSPACE;
    if (!aligned16(workspace)) return QLORA_ERR_ALIGN;
    TimerScope t(QLORA_TIMER_QUANTIZE, static_cast<cudaStream_t>(stream));
    return launch_quantize(W, N, K, out, workspace, static_cast<cudaStream_t>(stream));
}

qlora_status qlora_merge_lora(const qlora_nf4_weight* w, const void* A, const void* B, int32_t r, float alpha,
                              void* W_out, void* stream) {
    QLORA_TRY(check_weight(w));
    QLORA_TRY(check_lora(1, r, alpha));
    QLORA_TRY(check_dev(A));
    QLORA_TRY(check_dev(B));
    QLORA_TRY(check_dev(W_out));
    return launch_merge(w, A, B, r, alpha / (float)r, W_out, static_cast<cudaStream_t>(stream));
}

static qlora_status check_int8(int64_t n, int32_t blocksize) {
    if (blocksize != 64 && blocksize != 128 && blocksize != 256) return QLORA_ERR_UNSUPPORTED;
    if (n < 1 || n % blocksize != 0) return QLORA_ERR_SHAPE;
    if (n / 8 > (int64_t)INT32_MAX * 256) return QLORA_ERR_SHAPE;
    return QLORA_OK;
}

qlora_status qlora_quantize_int8_absmax(const void* W, int64_t n, int32_t blocksize, int8_t* codes, float* alpha,
                                        void* stream) {
    QLORA_TRY(check_dev(W));
    QLORA_TRY(check_dev(codes));
    QLORA_TRY(check_dev(alpha));
    QLORA_TRY(check_int8(n, blocksize));
    return launch_int8_quantize(W, n, blocksize, codes, alpha, static_cast<cudaStream_t>(stream));
}

qlora_status qlora_dequantize_int8_absmax(const int8_t* codes, const float* alpha, int64_t n, int32_t blocksize,
                                          void* out, int32_t out_dtype, void* stream) {
    QLORA_TRY(check_dev(codes));
    QLORA_TRY(check_dev(alpha));
    QLORA_TRY(check_dev(out));
    QLORA_TRY(check_int8(n, blocksize));
    if (out_dtype != QLORA_DTYPE_BF16 && out_dtype != QLORA_DTYPE_F16 && out_dtype != QLORA_DTYPE_F32)
        return QLORA_ERR_INVALID_ARG;
    return launch_int8_dequantize(codes, alpha, n, blocksize, out, out_dtype, static_cast<cudaStream_t>(stream));
}

qlora_status qlora_dequantize(const qlora_nf4_weight* w, void* W_out, void* stream) {
    QLORA_TRY(check_weight(w));
    QLORA_TRY(check_dev(W_out));
    TimerScope t(QLORA_TIMER_DEQUANTIZE, static_cast<cudaStream_t>(stream));
    return launch_dequantize(w, W_out, static_cast<cudaStream_t>(stream));
}

qlora_status qlora_linear_workspace_size(int64_t M, int64_t N, int64_t K, int32_t r, size_t* bytes) {
    QLORA_TRY(check_shape(N, K));
    QLORA_TRY(check_lora(M, r, 1.0f));
    if (!bytes) return QLORA_ERR_INVALID_ARG;
    *bytes = linear_ws(M, N, K, r).total;
    return QLORA_OK;
}

qlora_status qlora_linear_fwd(const qlora_nf4_weight* w, const void* X, int64_t M,
                              const void* A, const void* B, int32_t r, float alpha,
                              void* Y, int32_t y_dtype, float* U_save,
                              void* workspace, size_t workspace_bytes, void* stream) {
    QLORA_TRY(check_weight(w));
    QLORA_TRY(check_lora(M, r, alpha));
    QLORA_TRY(check_dev(X));
    QLORA_TRY(check_dev(A));
    QLORA_TRY(check_dev(B));
    QLORA_TRY(check_dev(Y));
    QLORA_TRY(check_out_dtype(y_dtype, w));
    if (U_save && !aligned16(U_save)) return QLORA_ERR_ALIGN;
    const LinearWs lw = linear_ws(M, w->N, w->K, r);
    if (!workspace || workspace_bytes < lw.total) return QLORA_ERR_WORKSPACE;
    if (!aligned16(workspace)) return QLORA_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t N = w->N, K = w->K;
    const bool f16 = w->compute_dtype == QLORA_DTYPE_F16;
    char* ws = static_cast<char*>(workspace);
    float* U = U_save ? U_save : reinterpret_cast<float*>(ws + lw.u_off);
    const float scale = alpha / (float)r;
    const int32_t R = rank_pad(r);
    void* U2 = ws + lw.u2_off;
    void* B2 = ws + lw.b2_off;
    float* partial = reinterpret_cast<float*>(ws + lw.part_off);
    if (M <= kDecodeMaxM) {
        // decode: U = X A^T and the LoRA term are computed in fp32 around the dequant GEMM
        DecodeArgs d{};
        d.w = w; d.X = X; d.A = A; d.B = B; d.r = r; d.scale = scale; d.M = M; d.out = Y;
        d.out_f32 = (y_dtype == QLORA_DTYPE_F32); d.U = U; d.partial = partial;
        TimerScope t(QLORA_TIMER_DECODE, s);
        return launch_tc_decode(d, s);
    }
    const bool b_direct = (r % 8 == 0);   // B rows are 16-byte multiples: the GEMM reads B itself
    if (!b_direct) {
        TimerScope t(QLORA_TIMER_LORA, s);
        QLORA_TRY(launch_dup_cols(B, N, r, R, B2, s));
    }
    QLORA_TRY(lora_U(X, A, M, K, r, R, scale, U, U2, partial, f16, s));
    TcGemmArgs a{};
    a.w = w; a.A0 = X; a.A1 = U2; a.Rpad = R;
    a.B1 = b_direct ? B : B2;
    a.b1_r = b_direct ? r : 0;
    a.p.M = M; a.p.Nout = N; a.p.out = Y; a.p.ldo = N; a.p.out_f32 = (y_dtype == QLORA_DTYPE_F32);
    TimerScope t(QLORA_TIMER_FWD_MAIN, s);
    return launch_tc_gemm_nf4(a, false, s);
}

qlora_status qlora_linear_fwd_multi(const qlora_nf4_weight* w, const void* X, int64_t M, const void* A_all,
                                    const void* B_all, int32_t n_adapters, const int32_t* adapter_idx, int32_t r,
                                    float alpha, void* Y, int32_t y_dtype, float* U_save, void* workspace,
                                    size_t workspace_bytes, void* stream) {
    QLORA_TRY(check_weight(w));
    QLORA_TRY(check_lora(M, r, alpha));
    if (M > kDecodeMaxM) return QLORA_ERR_SHAPE;
    if (n_adapters < 1) return QLORA_ERR_INVALID_ARG;
    QLORA_TRY(check_dev(X));
    QLORA_TRY(check_dev(A_all));
    QLORA_TRY(check_dev(B_all));
    QLORA_TRY(check_dev(Y));
    if (!adapter_idx) return QLORA_ERR_INVALID_ARG;
    QLORA_TRY(check_out_dtype(y_dtype, w));
    if (U_save && !aligned16(U_save)) return QLORA_ERR_ALIGN;
    const LinearWs lw = linear_ws(M, w->N, w->K, r);
    if (!workspace || workspace_bytes < lw.total) return QLORA_ERR_WORKSPACE;
    if (!aligned16(workspace)) return QLORA_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    DecodeArgs d{};
    d.w = w; d.X = X; d.A = A_all; d.B = B_all; d.r = r; d.scale = alpha / (float)r; d.M = M; d.out = Y;
    d.out_f32 = (y_dtype == QLORA_DTYPE_F32);
    d.U = U_save ? U_save : reinterpret_cast<float*>(ws + lw.u_off);
    d.partial = reinterpret_cast<float*>(ws + lw.part_off);
    d.aidx = adapter_idx; d.n_adapters = n_adapters;
    TimerScope t(QLORA_TIMER_DECODE, s);
    return launch_tc_decode(d, s);
}

qlora_status qlora_linear_bwd(const qlora_nf4_weight* w, const void* X, const void* dY, int64_t M,
                              const void* A, const void* B, int32_t r, float alpha,
                              const float* U_saved, void* dX, int32_t dx_dtype,
                              float* dA, float* dB,
                              void* workspace, size_t workspace_bytes, void* stream) {
    QLORA_TRY(check_weight(w));
    QLORA_TRY(check_lora(M, r, alpha));
    QLORA_TRY(check_dev(X));
    QLORA_TRY(check_dev(dY));
    QLORA_TRY(check_dev(A));
    QLORA_TRY(check_dev(B));
    QLORA_TRY(check_dev(dA));
    QLORA_TRY(check_dev(dB));
    if (dX) {
        QLORA_TRY(check_dev(dX));
        QLORA_TRY(check_out_dtype(dx_dtype, w));
    }
    if (U_saved && !aligned16(U_saved)) return QLORA_ERR_ALIGN;
    const LinearWs lw = linear_ws(M, w->N, w->K, r);
    if (!workspace || workspace_bytes < lw.total) return QLORA_ERR_WORKSPACE;
    if (!aligned16(workspace)) return QLORA_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t N = w->N, K = w->K;
    char* ws = static_cast<char*>(workspace);
    const float scale = alpha / (float)r;
    const int32_t R = rank_pad(r);
    const bool f16 = w->compute_dtype == QLORA_DTYPE_F16;
    const int32_t act = f16 ? SIMT_F16 : SIMT_BF16;   // activation / adapter operand kind (CUDA-core path)

    if (N % 8 == 0) {
        // Tensor-core path (dY rows are 16-byte strided, so dY can be a TMA source).
        void* U2 = ws + lw.u2_off;
        void* dU2 = ws + lw.du2_off;
        void* Bt = ws + lw.bt_off;
        float* dUf = reinterpret_cast<float*>(ws + lw.du_off);
        float* partial = reinterpret_cast<float*>(ws + lw.part_off);
        // the dU GEMM reads B [N, r] itself as an MN-major operand when its rows are 16-byte strided
        // (r % 8 == 0); otherwise from B^T, zero-padded to R rows
        const bool b_direct = r % 8 == 0;
        if (!b_direct) {
            TimerScope t(QLORA_TIMER_LORA, s);
            QLORA_TRY(launch_transpose_pad(B, N, r, R, Bt, s));
        }
        {   // dU = s dY B  ->  dU (fp32) and its hi/lo split
            TimerScope t(QLORA_TIMER_LORA, s);
            LoraGemmArgs g{};
            g.mn_major = false; g.A = dY; g.lda = N; g.rows = M; g.red = N; g.R = R;
            if (b_direct) {
                g.B = B; g.ldb = r; g.b_mn = true; g.b_cols = r;
            } else {
                g.B = Bt; g.ldb = N;
            }
            g.partial = partial;
            g.f16 = f16;
            QLORA_TRY(launch_lora_gemm(g, s));
            QLORA_TRY(launch_reduce_rows(partial, lora_splits(M, (int)((N + 63) / 64), R, false), M, r, R, scale, dUf, scale,
                                         dU2, f16, s));
        }
        // fork: the adapter gradients go to the side stream once dU is written; U2 (hi/lo of s U),
        // which only the dB GEMM reads, is prepared there too
        // (the caller's stream may be the null stream, so the fork is flagged, not inferred from g)
        const bool forked = dX != nullptr;
        cudaStream_t g = forked ? side_stream() : s;
        cudaEvent_t fork = nullptr, join = nullptr;
        if (forked && !g) return QLORA_ERR_CUDA;
        if (forked) {
            if (cudaEventCreateWithFlags(&fork, cudaEventDisableTiming) != cudaSuccess) return QLORA_ERR_CUDA;
            if (cudaEventCreateWithFlags(&join, cudaEventDisableTiming) != cudaSuccess) {
                cudaEventDestroy(fork);
                return QLORA_ERR_CUDA;
            }
            const bool ok = cudaEventRecord(fork, s) == cudaSuccess && cudaStreamWaitEvent(g, fork, 0) == cudaSuccess;
            cudaEventDestroy(fork);
            if (!ok) { cudaEventDestroy(join); return QLORA_ERR_CUDA; }
        }
        qlora_status st = QLORA_OK;
        if (dX) {   // dX = dY W_hat + dU A
            TcGemmArgs a{};
            a.w = w; a.A0 = dY; a.A1 = dU2; a.B1 = A; a.b1_r = r; a.Rpad = R;   // A [r, K] read directly
            a.p.M = M; a.p.Nout = K; a.p.out = dX; a.p.ldo = K; a.p.out_f32 = (dx_dtype == QLORA_DTYPE_F32);
            TimerScope t(QLORA_TIMER_DX_MAIN, s);
            st = launch_tc_gemm_nf4(a, true, s);
        }
        if (st == QLORA_OK) {
            if (U_saved) {
                TimerScope t(QLORA_TIMER_LORA, g);
                st = launch_split_hi_lo(U_saved, M, r, R, scale, U2, f16, g);
            } else {
                st = lora_U(X, A, M, K, r, R, scale, nullptr, U2, partial, f16, g);
            }
        }
        if (st == QLORA_OK) st = lora_gradients_tc(X, dY, M, N, K, r, R, f16, dA, dB, U2, dU2, partial, g);
        if (forked) {   // join: the caller's stream resumes after the adapter gradients too
            const bool ok = cudaEventRecord(join, g) == cudaSuccess && cudaStreamWaitEvent(s, join, 0) == cudaSuccess;
            cudaEventDestroy(join);
            if (!ok && st == QLORA_OK) st = QLORA_ERR_CUDA;
        }
        return st;
    }


    // CUDA-core path for N % 8 != 0.
    const float* U = U_saved;
    if (!U) {
        float* Uw = reinterpret_cast<float*>(ws + lw.u_off);
        SimtGemm g{};
        g.nseg = 1;
        g.seg[0].a = simt_dense(act, X, K, 1);
        g.seg[0].b = simt_dense(act, A, K, 1);
        g.seg[0].K = K; g.seg[0].scale = 1.f;
        g.M = M; g.N = r; g.C = Uw; g.c_dtype = QLORA_DTYPE_F32; g.ldc = r;
        TimerScope t(QLORA_TIMER_LORA, s);
        QLORA_TRY(launch_simt_gemm(g, s));
        U = Uw;
    }
    float* dU = reinterpret_cast<float*>(ws + lw.du_off);
    {   // dU = s dY B
        SimtGemm g{};
        g.nseg = 1;
        g.seg[0].a = simt_dense(act, dY, N, 1);
        g.seg[0].b = simt_dense(act, B, 1, r);
        g.seg[0].K = N; g.seg[0].scale = scale;
        g.M = M; g.N = r; g.C = dU; g.c_dtype = QLORA_DTYPE_F32; g.ldc = r;
        TimerScope t(QLORA_TIMER_LORA, s);
        QLORA_TRY(launch_simt_gemm(g, s));
    }
    if (dX) {   // dX = dY W_hat + dU A on the CUDA cores
        SimtGemm g{};
        g.nseg = 2;
        g.seg[0].a = simt_dense(act, dY, N, 1);
        g.seg[0].b = simt_nf4(w, true);
        g.seg[0].K = N; g.seg[0].scale = 1.f;
        g.seg[1].a = simt_dense(SIMT_F32, dU, r, 1);
        g.seg[1].b = simt_dense(act, A, 1, K);
        g.seg[1].K = r; g.seg[1].scale = 1.f;
        g.M = M; g.N = K; g.C = dX; g.c_dtype = dx_dtype; g.ldc = K;
        TimerScope t(QLORA_TIMER_DX_MAIN, s);
        QLORA_TRY(launch_simt_gemm(g, s));
    }
    {   // dA = dU^T X   ([r,K])
        SimtGemm g{};
        g.nseg = 1;
        g.seg[0].a = simt_dense(SIMT_F32, dU, 1, r);
        g.seg[0].b = simt_dense(act, X, 1, K);
        g.seg[0].K = M; g.seg[0].scale = 1.f;
        g.M = r; g.N = K; g.C = dA; g.c_dtype = QLORA_DTYPE_F32; g.ldc = K;
        TimerScope t(QLORA_TIMER_LORA, s);
        QLORA_TRY(launch_simt_gemm(g, s));
    }
    {   // dB = s dY^T U   ([N,r])
        SimtGemm g{};
        g.nseg = 1;
        g.seg[0].a = simt_dense(act, dY, 1, N);
        g.seg[0].b = simt_dense(SIMT_F32, U, 1, r);
        g.seg[0].K = M; g.seg[0].scale = scale;
        g.M = N; g.N = r; g.C = dB; g.c_dtype = QLORA_DTYPE_F32; g.ldc = r;
        TimerScope t(QLORA_TIMER_LORA, s);
        QLORA_TRY(launch_simt_gemm(g, s));
    }
    return QLORA_OK;
}

qlora_status qlora_read_device_errors(void* stream, int32_t clear, uint32_t* flags) {
    uint32_t* word = device_error_word();
    if (!word) return QLORA_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t h[2] = {0, 0};
    if (cudaMemcpyAsync(h, word, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess) return QLORA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return QLORA_ERR_CUDA;
    if (h[1] && sync_check_enabled()) std::fprintf(stderr, "[qlora] device location code 0x%08x\n", h[1]);
    if (clear && (h[0] || h[1])) {
        if (cudaMemsetAsync(word, 0, sizeof(h), s) != cudaSuccess) return QLORA_ERR_CUDA;
        if (cudaStreamSynchronize(s) != cudaSuccess) return QLORA_ERR_CUDA;
    }
    if (flags) *flags = h[0];
    if (h[0] & ERR_FLAG_TIMEOUT) return QLORA_ERR_TIMEOUT;
    if (h[0] & ERR_FLAG_NONFINITE) return QLORA_ERR_NONFINITE;
    return QLORA_OK;
}

qlora_status qlora_selftest_bounded_wait(uint32_t limit_us, uint32_t* result, void* stream) {
    if (limit_us < 1 || limit_us > 1000000) return QLORA_ERR_INVALID_ARG;
    QLORA_TRY(check_dev(result));
    return launch_bounded_wait_probe((uint64_t)limit_us * 1000ull, result, static_cast<cudaStream_t>(stream));
}

uint64_t qlora_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
