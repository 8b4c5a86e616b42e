/*
 * qlora.h - C ABI of libqlora.so, the B200 (sm_100a) QLoRA quantized linear layer.
 *
 * The library quantizes a frozen bf16 weight W[N,K] to 4-bit NormalFloat (NF4)
 * codes with Double Quantization of the block constants, dequantizes it, and
 * runs the LoRA-augmented linear layer forward and backward through the
 * dequantized weight.  The operations follow these web pages on QLoRA:
 *
 *   [SD]  airsota.com, "Science Depth M5-131: PEFT (LoRA / QLoRA / Prefix Tuning)",
 *         section 3 "Mathematical Principles & Derivation" (NF4 quantile grid,
 *         absmax blocks of B = 64, nearest-code rule, Double Quantization to 8-bit
 *         floats with second-level block 256) and section 4 "Industrial
 *         Trade-offs" (1) (on-the-fly dequantization in forward and backward).
 *   [QP]  offer.aigcbaba.com, "QLoRA 的原理是什么？4-bit 量化权重真的参与训练吗？",
 *         section 7: 4-bit frozen weight -> dequantize to BF16 -> matmul with the
 *         BF16 activation, LoRA path added to the output; gradients update only
 *         the LoRA parameters.
 *   [QR]  ainexis.cn, walkthrough of "QLoRA: Efficient Finetuning of Quantized
 *         LLMs", section 4.4: backpropagation passes through the frozen 4-bit
 *         weight into the adapters.
 *   [CH9] mdooai.com, "Ch.09 QLoRA 与量化：缩得更小再微调", section "2. INT8
 *         量化" (the absmax INT8 worked example: scale so that the block's largest
 *         magnitude maps to 127, store rounded integers, divide by the scale to
 *         recover) and section "3. 一个底座，多个适配器": one shared compressed
 *         base, one thin adapter per task.
 *   [Q103] agentalpha.top, "Q103: What is QLoRA, and how does it differ from
 *         LoRA", follow-up 1: after fine-tuning, merge the LoRA weights and
 *         dequantize for fast inference.
 *
 * Conventions for every entry point
 * ---------------------------------
 *  - Every array is row-major and contiguous.  W is [N,K] (nn.Linear layout,
 *    Y = X W^T); X is [M,K]; A is [r,K]; B is [N,r]; Y and dY are [M,N].
 *  - bf16 arrays are passed as `const void*` / `void*` holding IEEE bfloat16.
 *  - Pointers marked "device" must point to memory of the current CUDA device
 *    and be 16-byte aligned.  The caller allocates and frees all of it; the
 *    library allocates nothing on the device and keeps no pointer after a call.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  All device
 *    work is enqueued on it and the call returns without synchronizing.
 *  - Argument errors are detected on the host before anything is launched and
 *    are returned as a status; nothing is written in that case.  A launch
 *    failure returns QLORA_ERR_CUDA.  No C++ exception crosses this ABI.
 *  - Every kernel wait on the device is bounded; a wait that runs out sets a
 *    device flag, read with qlora_read_device_errors().
 */
#ifndef QLORA_H_
#define QLORA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QLORA_OK = 0,
    QLORA_ERR_INVALID_ARG = 1,   /* null pointer, bad dtype code, r or alpha out of range */
    QLORA_ERR_SHAPE = 2,         /* N, K or M < 1, or K % 64 != 0 */
    QLORA_ERR_ALIGN = 3,         /* a device pointer is not 16-byte aligned */
    QLORA_ERR_UNSUPPORTED = 4,   /* blocksize != 64 or blocksize2 != 256 */
    QLORA_ERR_NONFINITE = 5,     /* the weight held Inf or NaN (reported by qlora_read_device_errors) */
    QLORA_ERR_TIMEOUT = 6,       /* a bounded device wait ran out (reported by qlora_read_device_errors) */
    QLORA_ERR_CUDA = 7,          /* a CUDA runtime call or kernel launch failed */
    QLORA_ERR_WORKSPACE = 8,     /* workspace pointer null or smaller than the size query returned */
    QLORA_ERR_TOO_LARGE = 9      /* tensor larger than qlora_quantize_nf4_dq_noalloc's static scratch */
} qlora_status;

typedef enum { QLORA_DTYPE_BF16 = 0, QLORA_DTYPE_F32 = 1, QLORA_DTYPE_F16 = 2 } qlora_dtype;

/* Code-value sets (the 16 values a 4-bit code indexes). */
typedef enum {
    QLORA_CODEBOOK_NF4 = 0,       /* NormalFloat: normal quantiles with an exact zero ([SD] section 3 part 1) */
    QLORA_CODEBOOK_UNIFORM4 = 1   /* 16 evenly spaced values on [-1, 1] (the uniform 4-bit grid NF4 is
                                     compared with, [SD] section 4 (2)); no exact zero */
} qlora_codebook;

/*
 * A quantized frozen weight: the stored buffers of NF4 + Double Quantization
 * ([SD] section 3, parts 1 and 2).  All pointers are device memory owned by
 * the caller; sizes come from qlora_nf4_sizes().
 *
 *   codes    uint8 [N*K/2]  two 4-bit code indices per byte, element 2j of the
 *                           row-major flattening in the HIGH nibble of byte j,
 *                           element 2j+1 in the low nibble.  Index i stands for
 *                           the i-th value of the codebook in ascending order
 *                           (NF4: 0 = -1, 7 = 0, 15 = +1).
 *   c1_codes uint8 [nb1]    one FP8 E4M3 code per block of 64 weights
 *                           (nb1 = N*K/64): the block's absmax, centred by mu
 *                           and scaled by its group's c2.
 *   c2       fp32  [nb2]    absmax of the centred constants per group of 256
 *                           blocks (nb2 = ceil(nb1/256)).
 *   mu       fp32  [1]      mean of all block absmax values.
 *   codebook qlora_codebook the value set the codes index (0 = NF4).
 *   c1       fp32  [nb1]    NULL for double quantization (the default).  When
 *                           set, double quantization is off: the fp32 block
 *                           absmax values are stored here and c1_codes, c2,
 *                           mu are neither written nor read (they may be NULL)
 *                           -- the single-level variant that trades 0.37 bits
 *                           per weight for one fewer lookup per block.
 *
 *   compute_dtype          the 16-bit type the layer computes in ([QP] section 4:
 *                          bf16 is the usual compute type, fp16 where bf16 is not
 *                          well supported).  The dequantized weight is rounded to
 *                          it, and X, A, B, dY (and 16-bit Y, dX, W_out) of the
 *                          linear, decode and merge entry points are in it.  The
 *                          weight to quantize is always bf16.
 *
 * With double quantization the rebuilt block constant is
 * c1' = fp32(fp32(e4m3(c1_code) * c2) + mu); without it c1' = c1.  The
 * dequantized weight is round_nearest_even(fp32(q[code] * c1')) in the compute
 * dtype.  A zero-initialised codebook, compute_dtype and c1 give NF4 with
 * double quantization computing in bf16.
 */
typedef struct {
    uint8_t* codes;
    uint8_t* c1_codes;
    float*   c2;
    float*   mu;
    int64_t  N;
    int64_t  K;
    int32_t  blocksize;   /* must be 64 */
    int32_t  blocksize2;  /* must be 256 */
    int32_t  codebook;    /* qlora_codebook */
    int32_t  compute_dtype; /* QLORA_DTYPE_BF16 (0) or QLORA_DTYPE_F16: see below */
    float*   c1;          /* NULL: double quantization; else fp32 block constants [N*K/64] */
} qlora_nf4_weight;

/* Human-readable name of a status code (static storage; never NULL). */
const char* qlora_status_string(qlora_status s);

/*
 * Sizes in bytes of the stored buffers of W[N,K] and of the scratch that
 * qlora_quantize_nf4_dq needs.  Host only; launches nothing.
 * Footprint ([SD] section 3 part 2): 8 bits per 64 weights for c1_codes plus
 * 32 bits per 64*256 weights for c2, i.e. 0.126953125 bits per weight, plus 4
 * bytes for mu.  Any output pointer may be NULL.
 * Errors: QLORA_ERR_SHAPE (N < 1, K < 1, K % 64 != 0), QLORA_ERR_UNSUPPORTED.
 */
qlora_status qlora_nf4_sizes(int64_t N, int64_t K, int32_t blocksize, int32_t blocksize2,
                             size_t* codes_bytes, size_t* c1_codes_bytes, size_t* c2_bytes,
                             size_t* quant_workspace_bytes);

/*
 * The library's own NF4 code values (16 fp32, ascending) and the 15 decision
 * thresholds its quantize kernel uses, computed on the host at first use.
 * The values are the normal quantiles of [SD] section 3 part 1, read as the
 * asymmetric construction with an exact zero and end points -1 and +1:
 * 8 positive quantiles Phi^-1(p) for p evenly spaced from
 * delta = ((1 - 1/30) + (1 - 1/32))/2 towards 1/2 (1/2 excluded), 7 negative
 * ones likewise, and 0; divided by the largest; computed in double, rounded to
 * float.  threshold[j] is the largest float not above (q[j] + q[j+1]) / 2, so
 * "x > threshold[j]" counts the codes x is nearer to than q[j] (ties go to
 * the lower index).  Either pointer may be NULL.  Host only.
 */
qlora_status qlora_nf4_codebook(float values[16], float thresholds[15]);

/*
 * The same for any codebook: QLORA_CODEBOOK_NF4 gives qlora_nf4_codebook's
 * values; QLORA_CODEBOOK_UNIFORM4 gives -1 + 2i/15 (i = 0..15) computed in
 * double and rounded to float, with thresholds by the same rule.
 * Errors: QLORA_ERR_INVALID_ARG for an unknown codebook.  Host only.
 */
qlora_status qlora_codebook_values(int32_t codebook, float values[16], float thresholds[15]);

/*
 * NF4 + Double Quantization of a frozen bf16 weight ([SD] section 3, parts 1-2).
 *   W          device bf16 [N,K], read only; must be finite.
 *   out        host struct whose four device buffers are written; out->N, K,
 *              blocksize, blocksize2 must equal the arguments.
 *   workspace  device scratch of at least quant_workspace_bytes from
 *              qlora_nf4_sizes (fp32 block absmax values and fp64 partial sums).
 * Per block of 64: c1 = max|w|; x = fp32(w / c1) (0 when c1 == 0); code =
 * nearest NF4 value, ties to the lower index.  Then mu = mean of all c1 (fp64
 * sum over a fixed pairwise tree, rounded to fp32); per group of 256 blocks
 * c2 = max|fp32(c1 - mu)|; c1_code = E4M3 round-to-nearest-even of
 * fp32((c1 - mu) / c2) (0 when c2 == 0).  Deterministic and bit-exact.
 * out->codebook selects the code values (the nearest-value rule is the same);
 * with out->c1 set, the fp32 c1 values are written there and the second level
 * is skipped.  A non-finite weight sets the device NONFINITE flag.
 */
qlora_status qlora_quantize_nf4_dq(const void* W, int64_t N, int64_t K,
                                   int32_t blocksize, int32_t blocksize2,
                                   const qlora_nf4_weight* out,
                                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * qlora_quantize_nf4_dq without a workspace argument, for callers that cannot
 * allocate device memory when they quantize (for example a plugin whose host
 * framework owns every device allocation and passes only input and output
 * pointers, or a latency-critical path that must not call cudaMalloc/cudaFree,
 * which may synchronize the device).  The pages have no counterpart: this is a
 * deployment variant of the same operation with the same bit-exact results.
 *   Scratch: a static array of 4.75 MiB in the library's device image, held by
 *   every GPU that loads the library until the process exits.  Tensors of more
 *   than 67,108,864 weights (e.g. larger than W[8192,8192]) return
 *   QLORA_ERR_TOO_LARGE before anything is launched.
 *   The call allocates nothing.  All calls on a device share the one array and
 *   it keeps the last call's contents (nothing in it needs to start at zero);
 *   calls that overlap on the GPU race and give wrong results.  The first call
 *   on a device looks up the array's device address (once, with that device
 *   current): make that first call before any stream capture.
 *   Other arguments and errors as qlora_quantize_nf4_dq.
 */
qlora_status qlora_quantize_nf4_dq_noalloc(const void* W, int64_t N, int64_t K,
                                           int32_t blocksize, int32_t blocksize2,
                                           const qlora_nf4_weight* out, void* stream);

/*
 * Dequantize to bf16 ([SD] section 4 (1): W_hat = Dequant(W_NF4) * c1):
 * W_out[n,k] = bf16_rn(fp32(q[code] * c1')), bit-exact.
 *   W_out  device bf16 [N,K], written.
 */
qlora_status qlora_dequantize(const qlora_nf4_weight* w, void* W_out, void* stream);

/*
 * Workspace bytes needed by qlora_linear_fwd / qlora_linear_bwd for the given
 * shape (LoRA operand copies, split-reduction partial sums).  Host only.
 */
qlora_status qlora_linear_workspace_size(int64_t M, int64_t N, int64_t K, int32_t r, size_t* bytes);

/*
 * Forward of the QLoRA linear layer ([QP] section 7 diagram; LoRA scale
 * s = alpha / r):
 *     U = X A^T                      (fp32, never rounded to bf16 before use)
 *     Y = X W_hat^T + s U B^T        (fp32 accumulation, then y_dtype)
 *   w        quantized weight (device buffers), not written.
 *   X        device bf16 [M,K];  A device bf16 [r,K];  B device bf16 [N,r].
 *   Y        device [M,N] of y_dtype (QLORA_DTYPE_BF16 or QLORA_DTYPE_F32).
 *   U_save   device fp32 [M,r] or NULL; when given, U is stored for the backward.
 *   1 <= r <= 256; alpha finite.
 */
qlora_status qlora_linear_fwd(const qlora_nf4_weight* w, const void* X, int64_t M,
                              const void* A, const void* B, int32_t r, float alpha,
                              void* Y, int32_t y_dtype, float* U_save,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * Forward for a batch of at most 16 tokens that each use their own adapter
 * over one shared quantized base weight ([CH9] section "3. 一个底座，多个适配器":
 * one shared compressed base, each task swaps only a thin LoRA adapter):
 *     Y[m] = X[m] W_hat^T + s (X[m] A_a^T) B_a^T,  a = adapter_idx[m], s = alpha / r,
 * and Y[m] = X[m] W_hat^T for a token with adapter_idx[m] == -1.
 *   A_all       device bf16 [n_adapters, r, K]
 *   B_all       device bf16 [n_adapters, N, r]
 *   adapter_idx device int32 [M]; an index >= n_adapters is treated as -1 and
 *               raises the device BOUNDS flag (bit 2 of qlora_read_device_errors).
 *   U_save      optional device fp32 [M, r]: U[m] = X[m] A_a^T (0 without adapter).
 *   workspace   at least qlora_linear_workspace_size(M, N, K, r) bytes.
 * The base product uses the same small-M kernel as qlora_linear_fwd.
 * Errors: QLORA_ERR_SHAPE for M > 16, QLORA_ERR_INVALID_ARG for n_adapters < 1
 * or a null adapter_idx, and those of qlora_linear_fwd.
 */
qlora_status qlora_linear_fwd_multi(const qlora_nf4_weight* w, const void* X, int64_t M,
                                    const void* A_all, const void* B_all, int32_t n_adapters,
                                    const int32_t* adapter_idx, int32_t r, float alpha,
                                    void* Y, int32_t y_dtype, float* U_save,
                                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward of the QLoRA linear layer through the frozen dequantized weight
 * ([QR] section 4.4; [QP] section 7: no gradient reaches the 4-bit codes):
 *     dU = s dY B                    (fp32)
 *     dX = dY W_hat + dU A           (dX_dtype; skipped when dX is NULL)
 *     dA = dU^T X                    (fp32 [r,K], overwritten)
 *     dB = s dY^T U, U = X A^T       (fp32 [N,r], overwritten)
 *   U_saved  device fp32 [M,r] from the forward, or NULL to recompute it.
 *   The weight buffers are never written.
 */
qlora_status qlora_linear_bwd(const qlora_nf4_weight* w, const void* X, const void* dY, int64_t M,
                              const void* A, const void* B, int32_t r, float alpha,
                              const float* U_saved, void* dX, int32_t dx_dtype,
                              float* dA, float* dB,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * Merge trained adapters into the frozen weight for inference ([Q103]
 * follow-up 1; [QP] section 5: merging and requantizing can add error): with
 * s = alpha / r,
 *   W_out[n,k] = bf16_rn(fp32(W_hat[n,k] + sum_j fp32(s * B[n,j]) * A[j,k])),
 * the rank-r sum taken in ascending j with fp32 fused multiply-adds and W_hat
 * the dequantized weight (any codebook, with or without double quantization).
 * Requantize W_out with qlora_quantize_nf4_dq to serve the merged model in 4 bits.
 *   w      quantized weight (read only);
 *   A      device bf16 [r,K];  B  device bf16 [N,r];
 *   W_out  device bf16 [N,K], written.
 * Errors: QLORA_ERR_INVALID_ARG (null pointer, r outside 1..256, alpha not
 * finite), QLORA_ERR_ALIGN, and the weight checks of qlora_dequantize.
 */
qlora_status qlora_merge_lora(const qlora_nf4_weight* w, const void* A, const void* B, int32_t r, float alpha,
                              void* W_out, void* stream);

/*
 * Blockwise absmax INT8 quantization, the 8-bit comparison quantizer of [CH9]
 * section "2. INT8 量化" (steps 1-3).  For each block b of `blocksize`
 * consecutive elements of the flat tensor, in fp32 with round-to-nearest-even:
 *   alpha[b] = 127 / max|x| (IEEE division); 0 for an all-zero block, +inf
 *              when max|x| < 127 / FLT_MAX;
 *   codes[i] = round half away from zero of (x[i] * alpha[b]), clamped to
 *              [-127, 127]; 0 for x[i] = 0.
 *   W          device bf16 [n], read;  n >= 1 and n % blocksize == 0.
 *   blocksize  64, 128 or 256.
 *   codes      device int8 [n], written;  alpha  device fp32 [n / blocksize], written.
 * Errors: QLORA_ERR_INVALID_ARG (null pointer), QLORA_ERR_SHAPE (n < 1 or
 * n % blocksize != 0), QLORA_ERR_UNSUPPORTED (another blocksize),
 * QLORA_ERR_ALIGN.  A block holding Inf or NaN gets alpha 0 and zero codes and
 * raises the non-finite device flag (qlora_read_device_errors).
 */
qlora_status qlora_quantize_int8_absmax(const void* W, int64_t n, int32_t blocksize, int8_t* codes, float* alpha,
                                        void* stream);

/*
 * Dequantize blockwise absmax INT8 ([CH9] section "2. INT8 量化", step 4:
 * divide by the scale):
 *   out[i] = fp32(codes[i] / alpha[b]) (IEEE division; 0 when alpha[b] = 0),
 *            rounded to nearest even into out_dtype.
 *   out        device [n] of out_dtype (QLORA_DTYPE_BF16, _F16 or _F32), written.
 * Other arguments and errors as qlora_quantize_int8_absmax; a bad out_dtype
 * returns QLORA_ERR_INVALID_ARG.
 */
qlora_status qlora_dequantize_int8_absmax(const int8_t* codes, const float* alpha, int64_t n, int32_t blocksize,
                                          void* out, int32_t out_dtype, void* stream);

/*
 * Device error flags raised since the last clear (bit 0: a bounded wait timed
 * out; bit 1: a non-finite weight was seen).  Synchronizes the stream, reads
 * the flags of the current device and clears them when `clear` is nonzero.
 * Returns QLORA_ERR_TIMEOUT or QLORA_ERR_NONFINITE when a flag is set.
 */
qlora_status qlora_read_device_errors(void* stream, int32_t clear, uint32_t* flags);

/*
 * Failure-detection self-test of the bounded device waits (no page counterpart).
 * Launches one thread that waits, through the same bounded mbarrier wait every
 * kernel of the library uses, on a barrier that nothing completes, with a limit
 * of `limit_us` microseconds.  The wait gives up, raises the timeout device flag
 * (read it with qlora_read_device_errors, which then returns QLORA_ERR_TIMEOUT)
 * and the kernel returns: the context stays usable.  Nothing faults or hangs.
 *   limit_us  1 .. 1,000,000.
 *   result    device uint32 [2], written: [0] = 1 if the wait completed (never
 *             expected), [1] = 1 if the wait set the CTA's abort flag.
 * Errors: QLORA_ERR_INVALID_ARG (limit out of range, null result),
 * QLORA_ERR_ALIGN.
 */
qlora_status qlora_selftest_bounded_wait(uint32_t limit_us, uint32_t* result, void* stream);

/* Number of kernels this library has launched in this process (host counter). */
uint64_t qlora_launch_count(void);

/*
 * Kernel timing for benchmarks.  While enabled, the library records a CUDA
 * event pair on the launch stream around each timed unit of work, grouped by
 * kind.  qlora_timing_read synchronizes on the recorded events and returns the
 * number of timed units and their total device time in milliseconds for one
 * kind; `reset` nonzero clears all kinds afterwards.  Off by default.
 */
typedef enum {
    QLORA_TIMER_QUANTIZE = 0,     /* a whole qlora_quantize_nf4_dq (all its kernels) */
    QLORA_TIMER_DEQUANTIZE = 1,   /* a whole qlora_dequantize */
    QLORA_TIMER_FWD_MAIN = 2,     /* the fused dequant-GEMM kernel producing Y */
    QLORA_TIMER_DX_MAIN = 3,      /* the fused dequant-GEMM kernel producing dX */
    QLORA_TIMER_LORA = 4,         /* each LoRA-side kernel (U, dU, dA, dB and their operand prep) */
    QLORA_TIMER_DECODE = 5,       /* the small-M forward kernel */
    QLORA_TIMER_KINDS = 6
} qlora_timer_kind;

qlora_status qlora_timing_enable(int32_t on);
qlora_status qlora_timing_read(int32_t kind, uint64_t* launches, double* total_ms, int32_t reset);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_H_ */
