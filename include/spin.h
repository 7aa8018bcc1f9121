/*
 * spin.h -- C ABI of libspin.so: SpinQuant's online Hadamard rotations (R3 and
 * R4) fused with the low-bit quantisers that follow them, for NVIDIA B200
 * (sm_100a).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  * Pointers are device pointers the caller owns (allocated by any means).
 *    The library allocates, frees and synchronises nothing, and no entry
 *    point blocks, with one exception: spin_device_status() reads the
 *    device status word synchronously (see there).
 *  * Each call validates its arguments on the host, then enqueues its kernels
 *    on `stream` (a cudaStream_t; NULL is the legacy default stream) and
 *    returns. A non-SPIN_OK status means nothing was enqueued, except
 *    SPIN_ERR_CUDA, which reports a failed launch (spin_last_cuda_error()
 *    returns the cudaError_t value). Faults inside a kernel surface later, at
 *    the caller's next synchronisation, as with any CUDA launch.
 *  * tokens/rows == 0 is a successful no-op.
 *  * bfloat16 and float16 buffers are passed as `void*` holding the 16-bit
 *    patterns, so this header needs no CUDA header.
 *  * Input and output buffers must not overlap unless a parameter says so.
 *  * Calls on the same stream are ordered; calls that run concurrently on
 *    different streams may share inputs but not outputs.
 *
 * Quantised layout
 * ----------------
 *  Two 4-bit codes per byte: element 2j in the low nibble of byte j,
 *  element 2j+1 in the high nibble. Symmetric codes are 4-bit two's
 *  complement in [-8, 7]; asymmetric codes are unsigned in [0, 15].
 *  spin_hadamard_quant_int8 instead writes one 8-bit two's-complement code
 *  per element, element j at byte j, in [-128, 127].
 *
 * Sources are cited by page title and section:
 *  "SpinQuant, when rotations are worth learning" -- section "Four rotation
 *    sites, two of them free" (R3 on Q and K after RoPE, R4 on the
 *    down-projection input), section "Paper vs. code" (K-cache quantisation
 *    needs a power-of-two head dim because R3 uses the fast transform).
 *  "Rotations: QuaRot, SpinQuant and incoherence" -- section "Hadamard
 *    matrices" (Sylvester H_n; (1/sqrt n) H_n orthogonal; randomised
 *    (1/sqrt n) H_n diag(+-1); Kronecker products), section "Why it's free"
 *    (O(d log d) transform), widget "Try it" (rotate, quantize, rotate back).
 *  "SpinQuant Guide: Learned Rotations for 4-Bit LLMs" -- section "The Outlier
 *    Curse" (INT4 range [-8, 7], step = max|x| / 7), section "End-to-End
 *    Implementation" (step clamped below at 1e-8; dequant = code * step),
 *    section "RoPE Compatibility with 4-Bit KV Caching" (RoPE rotates 2-D
 *    pairs; KV cache stored as 4-bit).
 */
#ifndef SPIN_H_
#define SPIN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st *spin_stream_t;

typedef enum spin_status_t {
  SPIN_OK = 0,
  SPIN_ERR_INVALID_ARG = 1,      /* null pointer, bad count, clip outside (0, 1], ... */
  SPIN_ERR_UNSUPPORTED_SIZE = 2, /* n or head_dim not a supported power of two */
  SPIN_ERR_MISALIGNED = 3,       /* a pointer is not 16-byte aligned */
  SPIN_ERR_CUDA = 4,             /* a CUDA call or launch failed: see spin_last_cuda_error() */
  SPIN_ERR_DEVICE = 5,           /* the current device is not compute capability 10.0 */
  SPIN_ERR_SCRATCH_LIMIT = 6     /* the call needs more scratch than the library's built-in array */
} spin_status_t;

/* flags */
#define SPIN_NO_ROTATE 1u       /* skip the diagonal and the transform (direct quantisation / identity) */
#define SPIN_CUDA_CORES_ONLY 2u /* R4: use the CUDA-core kernel even where the tensor-core kernel applies */
#define SPIN_TENSOR_CORES 4u    /* R4: use the tensor-core kernel wherever n allows it, at any batch size */

/* spin_dequant_hadamard_inverse modes */
#define SPIN_SYM_INT4_F32SCALE 0 /* signed codes, fp32 scale per row: value = code * scale */
#define SPIN_ASYM_INT4_F16SZ 1   /* unsigned codes, fp16 scale and zero per row: (code - zero) * scale */

/* output dtypes */
#define SPIN_BF16 0
#define SPIN_F32 1

/*
 * R4: rotate the down-projection input and quantise it per token
 * ("SpinQuant, when rotations are worth learning", "Four rotation sites":
 * R4 is a fixed Hadamard on the down-projection input; "SpinQuant Guide",
 * "The Outlier Curse": symmetric INT4 with step max|x| / 7).
 *
 * For each of `tokens` rows x (n bfloat16 values, row-major, contiguous):
 *   y = H_n D x / sqrt(n)     (H_n Sylvester order, D = diag(+-1), D = I if sign_bits == NULL)
 *   m = max_j |y_j|,  scale = max(clip * m / 7, 1e-8)
 *   code_j = clamp(round_half_even(y_j / scale), -8, 7)
 * Arithmetic is fp32 on the device (the transform is exact reassociation of
 * the same sums; only rounding order differs from an fp64 evaluation).
 *
 *  x_bf16      [tokens, n] bf16, 16-byte aligned, read only
 *  tokens      >= 0
 *  n           power of two, 128 <= n <= 32768
 *  clip        0 < clip <= 1 (scale multiplier; codes saturate beyond it)
 *  q_packed_u8 [tokens, n/2] bytes, 16-byte aligned, written
 *  scales_f32  [tokens] fp32, 4-byte aligned, written (the step, in y units)
 *  stream      cudaStream_t
 * Errors: SPIN_ERR_INVALID_ARG (null pointer with tokens > 0, tokens < 0,
 * clip outside (0, 1] or NaN), SPIN_ERR_UNSUPPORTED_SIZE (n),
 * SPIN_ERR_MISALIGNED, SPIN_ERR_DEVICE, SPIN_ERR_CUDA.
 */
spin_status_t spin_hadamard_quant_int4(const void *x_bf16, int64_t tokens, int32_t n, float clip,
                                       uint8_t *q_packed_u8, float *scales_f32,
                                       spin_stream_t stream);

/*
 * Superset of spin_hadamard_quant_int4 ("Rotations: QuaRot, SpinQuant and
 * incoherence", "Hadamard matrices": the randomised transform
 * (1/sqrt n) H_n diag(+-1)).
 *  sign_bits  nullable; [n/32] uint32 words, bit j of the mask set means
 *             d_j = -1. 4-byte aligned.
 *  flags      bitwise OR of
 *             SPIN_NO_ROTATE: quantise x directly (no D, no H), used to
 *               measure the direct-quantisation error;
 *             SPIN_CUDA_CORES_ONLY: at n = 128 and 256 the transform, and at
 *               n = 512 .. 16384, and at n = 32768 without sign_bits,
 *               the first Kronecker factor (H_128; two of them at n = 32768;
 *               H_64 at n = 512) normally runs on the tensor cores (exact
 *               +-1 x bf16 products, fp32 accumulation; at n = 128 and 256 the
 *               diagonal rides in the +-1 operand); this bit selects the kernel
 *               that runs every butterfly on the CUDA cores instead.
 *               Both give the same codes up to the rounding-tie band and the
 *               same steps to fp32 accumulation order. By default the
 *               tensor-core kernel runs only when the batch has at least 128 MMA
 *               groups (128 x max(1, 256 / (n/128)) tokens), since it pays a
 *               per-block setup that small (decode) batches do not amortise;
 *             SPIN_TENSOR_CORES: use the tensor-core kernel wherever n allows,
 *               whatever the batch size (not with SPIN_CUDA_CORES_ONLY).
 * spin_hadamard_quant_int4(...) == spin_hadamard_quant_int4_ex(..., NULL, 0, ...).
 */
spin_status_t spin_hadamard_quant_int4_ex(const void *x_bf16, int64_t tokens, int32_t n,
                                          float clip, const uint32_t *sign_bits, uint32_t flags,
                                          uint8_t *q_packed_u8, float *scales_f32,
                                          spin_stream_t stream);

/*
 * R4 with per-token INT8 codes ("SpinQuant Guide: Learned Rotations for 4-Bit
 * LLMs", section "The Outlier Curse": the symmetric b-bit rule, range
 * [-2^(b-1), 2^(b-1) - 1] and step max / (2^(b-1) - 1), here at b = 8 -- the
 * 8-bit activations of the W4A8 decoding figure in "SpinQuant, when rotations
 * are worth learning", section "Measured effects").
 * For each of `tokens` rows x:
 *   y = H_n D x / sqrt(n),  m = max_j |y_j|,  scale = max(clip * m / 127, 1e-8)
 *   code_j = clamp(round_half_even(y_j / scale), -128, 127)
 *
 *  x_bf16, tokens, n, clip, sign_bits, flags, scales_f32, stream: as in
 *             spin_hadamard_quant_int4_ex (same kernels and dispatch, the same
 *             SPIN_NO_ROTATE / SPIN_CUDA_CORES_ONLY / SPIN_TENSOR_CORES bits)
 *  q_i8       [tokens, n] int8 codes (one two's-complement byte per element,
 *             element j at byte j), 16-byte aligned, written
 * Errors: as spin_hadamard_quant_int4_ex.
 */
spin_status_t spin_hadamard_quant_int8(const void *x_bf16, int64_t tokens, int32_t n, float clip,
                                       const uint32_t *sign_bits, uint32_t flags, int8_t *q_i8,
                                       float *scales_f32, spin_stream_t stream);

/*
 * R4 for a row length that is not a power of two, n = m b with b = 2^k
 * ("Rotations: QuaRot, SpinQuant and incoherence", section "Hadamard matrices":
 * other sizes use a Kronecker product of a Sylvester matrix with a small known
 * Hadamard matrix). The pages name no small matrix; H_m here is Paley's
 * construction from the quadratic character chi mod a prime q, with the core
 * matrix C of order q + 1: C[0][0] = 0, C[0][j] = 1, C[i][j] = chi(j - i) for
 * i, j > 0, and C[i][0] = -1 (type I) or +1 (type II).
 *   type I  (q = m - 1 prime, q = 3 mod 4):        H_m = C + I
 *   type II (q = m/2 - 1 prime, q = 1 mod 4, and m - 1 not a type I prime):
 *           H_m = C (x) [[1, -1], [-1, -1]] + I (x) [[1, 1], [1, -1]]
 * For each of `tokens` rows x (element e = b i + j: i < m indexes H_m, j < b the
 * Sylvester H_b; the diagonal D comes first, as for powers of two):
 *   y = (H_m (x) H_b) D x / sqrt(n), then the per-token rule of
 *   spin_hadamard_quant_int4 (bits = 4) or spin_hadamard_quant_int8 (bits = 8).
 *
 *  x_bf16     [tokens, n] bf16, 16-byte aligned
 *  m          order of H_m: one with a Paley form (12, 20, 24, 28, 44, 48, ...)
 *  n          m b with b a power of two >= 128 and n / 128 a multiple of 16, at most
 *             128 (n = 6144, 10240, 12288 or 14336 for m = 12, 20, 12 or 28, ...);
 *             tokens * n / 128 < 2^31
 *  sign_bits  nullable, [ceil(n/32)] words, bit e set => d_e = -1, 4-byte aligned
 *  flags      0 or SPIN_TENSOR_CORES (one kernel, on the tensor cores, for every batch)
 *  bits       4: q is [tokens, n/2] packed INT4 bytes; 8: q is [tokens, n] int8 codes
 *  q          16-byte aligned, written; scales_f32 [tokens] fp32, 4-byte aligned, written
 * Errors: SPIN_ERR_UNSUPPORTED_SIZE ((m, n) outside the above), SPIN_ERR_INVALID_ARG
 * (null pointer with tokens > 0, tokens < 0, clip outside (0, 1], bits not 4 or 8,
 * other flag bits), SPIN_ERR_MISALIGNED, SPIN_ERR_DEVICE, SPIN_ERR_CUDA.
 */
spin_status_t spin_hadamard_quant_kron(const void *x_bf16, int64_t tokens, int32_t m, int32_t n, float clip,
                                       const uint32_t *sign_bits, uint32_t flags, int32_t bits, void *q,
                                       float *scales_f32, spin_stream_t stream);

/*
 * R3 + INT4 KV cache ("SpinQuant, when rotations are worth learning", "Four
 * rotation sites": R3 is a fixed Hadamard on queries and keys after RoPE,
 * there only to make the KV cache quantisable; "SpinQuant Guide", "RoPE
 * Compatibility with 4-Bit KV Caching": RoPE rotates 2-D coordinate pairs).
 *
 * For every token (b, s) and head:
 *   RoPE (rotate-half pairing): for p < d/2, a = pos[b,s] * theta^(-2p/d),
 *     (x_p, x_{p+d/2}) <- (x_p cos a - x_{p+d/2} sin a, x_{p+d/2} cos a + x_p sin a)
 *   Q heads: q_out = bf16(H_d RoPE(q) / sqrt(d))
 *   K heads: k' = H_d RoPE(k) / sqrt(d), quantised asymmetrically
 *   V heads: v, quantised asymmetrically (no RoPE, no rotation)
 * Asymmetric INT4 per (token, kv head) group of d values x:
 *   lo = min(clip * min x, 0), hi = max(clip * max x, 0)
 *   scale = fp16((hi - lo) / 15) (round to nearest even); if it is 0: scale = 1, zero = 0
 *   zero  = clamp(round_half_even(-lo / scale), 0, 15)        (stored as fp16, exact)
 *   code  = clamp(round_half_even(x / scale) + zero, 0, 15)
 * The cache slot of token (b, s) is cache_offset + s; `pos` only sets the
 * RoPE angle.
 *
 *  q, k, v      [batch, seq, n_q_heads | n_kv_heads, head_dim] bf16, 16-byte aligned
 *  pos          [batch, seq] int32 RoPE positions (>= 0)
 *  theta        RoPE base (> 0), e.g. 10000
 *  head_dim     128 (power of two; other sizes return SPIN_ERR_UNSUPPORTED_SIZE)
 *  batch, seq   > 0 (0 is a no-op); n_q_heads, n_kv_heads > 0, n_q_heads % n_kv_heads == 0;
 *               n_q_heads <= 256, n_q_heads + 2 n_kv_heads <= 384 and
 *               batch * seq * n_q_heads < 2^31, else SPIN_ERR_UNSUPPORTED_SIZE
 *  clip         0 < clip <= 1
 *  q_out        [batch, seq, n_q_heads, head_dim] bf16, 16-byte aligned; may equal q
 *  k_cache, v_cache  [batch, n_kv_heads, cache_len, head_dim/2] bytes, 16-byte aligned
 *  k_scale, k_zero, v_scale, v_zero  [batch, n_kv_heads, cache_len] fp16
 *  cache_len    >= cache_offset + seq;  cache_offset >= 0
 */
spin_status_t spin_rope_hadamard_kvquant(const void *q, const void *k, const void *v,
                                         const int32_t *pos, float theta, int32_t head_dim,
                                         int32_t batch, int32_t seq, int32_t n_q_heads,
                                         int32_t n_kv_heads, float clip, void *q_out,
                                         uint8_t *k_cache, uint8_t *v_cache, void *k_scale,
                                         void *k_zero, void *v_scale, void *v_zero,
                                         int32_t cache_len, int32_t cache_offset,
                                         spin_stream_t stream);

/*
 * Dequantise and rotate back ("Rotations: QuaRot, SpinQuant and
 * incoherence", widget "Try it": rotate, quantize, rotate back; "Hadamard
 * matrices": H_n / sqrt(n) is orthogonal and symmetric, so the inverse of
 * H_n D / sqrt(n) is D H_n / sqrt(n); "SpinQuant Guide", "End-to-End
 * Implementation": dequant = code * scale).
 *
 * For each of `rows` rows of n codes:
 *   mode SPIN_SYM_INT4_F32SCALE: v_j = code_j * scale            (scale: fp32 [rows])
 *   mode SPIN_ASYM_INT4_F16SZ:   v_j = (code_j - zero) * scale   (scale, zero: fp16 [rows])
 *   out = D H_n v / sqrt(n)   unless flags has SPIN_NO_ROTATE (then out = v)
 * A KV cache [batch, n_kv_heads, cache_len, head_dim/2] is rows = batch *
 * n_kv_heads * cache_len rows of n = head_dim (use SPIN_NO_ROTATE for V: R3
 * rotates K only; RoPE is not undone).
 *
 *  codes      [rows, n/2] bytes, 16-byte aligned
 *  n          power of two, 128 <= n <= 32768
 *  scale      [rows] fp32 or fp16 by mode; zero [rows] fp16 (asym) or NULL (sym)
 *  sign_bits  nullable, as in spin_hadamard_quant_int4_ex
 *  flags      bitwise OR of SPIN_NO_ROTATE and at most one of
 *             SPIN_CUDA_CORES_ONLY: at n = 128 and 256 the transform, and at
 *               n = 512 .. 32768 its first Kronecker factor (H_128; H_64 at
 *               n = 512), normally run on the tensor cores (the codes minus the
 *               zero point are exact fp16 integers and so is every sum, so both
 *               kernels give the same bits); this bit selects the kernel that
 *               runs every butterfly on the CUDA cores instead. By default the
 *               tensor-core kernel runs only from 128 MMA groups up (128 rows per
 *               group at n = 128 and 256, 64 at n = 512, 128 x max(1, 256 /
 *               (n/128)) rows from 1024);
 *             SPIN_TENSOR_CORES: use the tensor-core kernel at any row count
 *               (not with SPIN_NO_ROTATE).
 *             Other bits: SPIN_ERR_INVALID_ARG.
 *  out        [rows, n] bf16 or fp32 (out_dtype), 16-byte aligned
 */
spin_status_t spin_dequant_hadamard_inverse(const uint8_t *codes, int64_t rows, int32_t n,
                                            int32_t mode, const void *scale, const void *zero,
                                            const uint32_t *sign_bits, uint32_t flags, void *out,
                                            int32_t out_dtype, spin_stream_t stream);

/*
 * Decode attention over the INT4 KV cache that spin_rope_hadamard_kvquant writes
 * ("SpinQuant Guide: Learned Rotations for 4-Bit LLMs", the KV4 serving diagram:
 * rotated keys stored in the cache as INT4 meet the rotated queries in a fused INT4
 * dot product; "SpinQuant: rotate before you round", section "Deployment
 * implications": the rotation pays only with KV4 kernels). One step: for batch row
 * b, query head h and its kv head g = h / (n_q_heads / n_kv_heads), over the cache
 * slots j < lens[b] of row (b, g):
 *   khat_j = (code_j - zero_j) * scale_j      (K and V alike, fp16 scale and zero)
 *   score_j = (q_h . khat_j) * softmax_scale
 *   out_h = sum_j softmax(score)_j * vhat_j
 * R3 rotated q and k by the same orthogonal matrix, so the scores need no inverse
 * rotation; V was not rotated, so out is in the value basis. Arithmetic is fp32.
 *
 *  q          [batch, n_q_heads, head_dim] bf16 (the rotated queries, as q_out of
 *             spin_rope_hadamard_kvquant), 16-byte aligned
 *  k_cache, v_cache  [batch, n_kv_heads, cache_len, head_dim/2] bytes, 16-byte aligned
 *  k_scale, k_zero, v_scale, v_zero  [batch, n_kv_heads, cache_len] fp16, 2-byte aligned
 *  lens       [batch] int32 in device memory: slots attended in each row; a value
 *             outside [0, cache_len] is clamped to it, and a row with 0 slots gives 0
 *  head_dim   128; n_q_heads / n_kv_heads in {1, 2, 4, 8}; batch, n_q_heads and
 *             n_kv_heads at most 65535 (else SPIN_ERR_UNSUPPORTED_SIZE)
 *  softmax_scale  > 0 and finite, usually 1 / sqrt(head_dim)
 *  out        [batch, n_q_heads, head_dim] bf16 or fp32 (out_dtype), 16-byte aligned
 *  workspace  caller-owned device scratch of at least
 *             spin_decode_attention_workspace_bytes(batch, n_q_heads, cache_len) bytes,
 *             16-byte aligned; its contents on entry do not matter and are
 *             overwritten (the per-chunk partials); calls that may run at the same
 *             time need separate workspaces
 * Two kernels on `stream`: per 256-slot chunk partials, then their merge.
 * Errors: SPIN_ERR_INVALID_ARG (null pointer with batch > 0, cache_len < 1, sizes
 * < 0, softmax_scale, out_dtype, workspace too small), SPIN_ERR_UNSUPPORTED_SIZE,
 * SPIN_ERR_MISALIGNED, SPIN_ERR_DEVICE, SPIN_ERR_CUDA.
 */
spin_status_t spin_decode_attention_int4kv(const void *q, const uint8_t *k_cache, const uint8_t *v_cache,
                                           const void *k_scale, const void *k_zero, const void *v_scale,
                                           const void *v_zero, const int32_t *lens, int32_t batch,
                                           int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                           int32_t cache_len, float softmax_scale, void *out, int32_t out_dtype,
                                           void *workspace, size_t workspace_bytes, spin_stream_t stream);

/* Workspace bytes spin_decode_attention_int4kv needs (batch x n_q_heads x
 * ceil(cache_len / 256) partials of head_dim + 2 fp32 values); 0 for sizes <= 0. */
size_t spin_decode_attention_workspace_bytes(int32_t batch, int32_t n_q_heads, int32_t cache_len);

/*
 * W4A4 GEMM on packed INT4 codes ("SpinQuant Guide: Learned Rotations for 4-Bit
 * LLMs", section "End-to-End Implementation": the quantised layer output is the
 * product of the quantised activations and the quantised weights, each dequantised as
 * code x scale; section "Production Engineering and Cluster Deployment Best
 * Practices": the rotated weights W R^T are baked offline into packed INT4 nibbles and
 * multiplied on INT4 tensor cores):
 *   out[t][o] = x_scales[t] w_scales[o] sum_k q_x[t][k] q_w[o][k]
 * The activations are what spin_hadamard_quant_int4_ex / _kron write (per-token codes
 * and fp32 steps); the weights are packed the same way, one row and one fp32 step per
 * output channel (rows of W R^T quantised by the same symmetric INT4 rule: run the
 * weight rows through spin_hadamard_quant_int4_ex with the activations' diagonal at
 * clip 1.0). The integer sum is exact (int32 accumulation on the tensor cores); the
 * product of the two steps and the sum are rounded once each to fp32, then to bf16
 * when out_dtype is SPIN_BF16.
 *  x_codes   [tokens, k/2] packed 4-bit two's-complement codes, element 2j in the low
 *            nibble of byte j, 16-byte aligned
 *  x_scales  [tokens] fp32, 4-byte aligned
 *  w_codes   [n_out, k/2] packed codes of the weight rows, 16-byte aligned
 *  w_scales  [n_out] fp32, 16-byte aligned
 *  n_out     a multiple of 256; k a multiple of 128, 128 .. 65536
 *  out       [tokens, n_out] fp32 or bf16 (out_dtype), 16-byte aligned
 * One kernel on `stream`; tokens == 0 is a no-op.
 * Errors: SPIN_ERR_INVALID_ARG (tokens < 0, a NULL pointer, out_dtype),
 * SPIN_ERR_UNSUPPORTED_SIZE (n_out, k or tokens outside the ranges above),
 * SPIN_ERR_MISALIGNED, SPIN_ERR_DEVICE, SPIN_ERR_CUDA.
 */
spin_status_t spin_w4a4_gemm(const uint8_t *x_codes, const float *x_scales, int64_t tokens, const uint8_t *w_codes,
                             const float *w_scales, int32_t n_out, int32_t k, void *out, int32_t out_dtype,
                             spin_stream_t stream);

/* Bytes of the scratch array built into the library for
 * spin_decode_attention_int4kv_noalloc (held by every GPU that loads the library). */
#define SPIN_NOALLOC_SCRATCH_BYTES (4u << 20)

/*
 * spin_decode_attention_int4kv for callers that cannot allocate device memory
 * (no counterpart on the pages). Some callers have no way to provide the workspace:
 * a plugin inside an inference engine that owns all device memory and gives the plugin
 * no scratch, or a latency-critical serving loop that must not call cudaMalloc
 * because it can synchronise the device. This entry point takes the same arguments
 * except the workspace and allocates nothing: the per-chunk partials go to a scratch
 * array compiled into the library, SPIN_NOALLOC_SCRATCH_BYTES (4 MiB) on every GPU
 * that loads the library, kept until the process exits.
 *  * Limit: batch x n_q_heads x ceil(cache_len / 256) x 520 bytes (the value of
 *    spin_decode_attention_workspace_bytes) must not exceed SPIN_NOALLOC_SCRATCH_BYTES,
 *    e.g. 4 rows x 32 heads of a 4096-slot cache use 1.06 MB; larger calls return
 *    SPIN_ERR_SCRATCH_LIMIT and enqueue nothing.
 *  * The first call on a device looks up the array's device address on the host
 *    (cudaGetSymbolAddress, with that device current) and keeps it; make that first
 *    call on each device before any stream capture.
 *  * Every call on a device shares the one array, and nothing in it needs to start at
 *    zero (each call writes every partial it reads). Calls whose kernels can overlap
 *    on the GPU -- on different streams or from different host threads without an
 *    ordering between them -- race on the array and give wrong results; order them
 *    (one stream, or events).
 * Errors: those of spin_decode_attention_int4kv (other than a small workspace),
 * SPIN_ERR_SCRATCH_LIMIT, and SPIN_ERR_CUDA if the address lookup fails.
 */
spin_status_t spin_decode_attention_int4kv_noalloc(const void *q, const uint8_t *k_cache, const uint8_t *v_cache,
                                                   const void *k_scale, const void *k_zero, const void *v_scale,
                                                   const void *v_zero, const int32_t *lens, int32_t batch,
                                                   int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                                   int32_t cache_len, float softmax_scale, void *out,
                                                   int32_t out_dtype, spin_stream_t stream);

/*
 * Device status word of the current device: nonzero once a kernel of this
 * library gave up on an internal wait (a pipeline barrier that did not
 * complete within about two seconds); that kernel then stopped early and its
 * outputs are incomplete. Copies the word to *status and, if reset != 0,
 * clears it. Synchronous, the one entry point that blocks: it waits for work
 * on the legacy default stream (and so for every launch of this library that
 * the caller has enqueued on a blocking stream) before it reads the word.
 * Errors: SPIN_ERR_INVALID_ARG (status NULL), SPIN_ERR_CUDA.
 */
spin_status_t spin_device_status(uint32_t *status, int reset);

/*
 * Test hook for failure detection (no counterpart on the pages). While
 * enabled (nonzero), every tensor-core R4 launch withholds the completion
 * signal of its first MMA group and shortens its wait budget to about a
 * millisecond, so the bounded waits run out, each block takes its abort path
 * (drains its copies and MMAs, frees TMEM, returns) and the device status word
 * becomes nonzero; those launches' outputs are incomplete. Process-wide; call
 * it with 0 to restore normal operation. Never needed outside tests.
 */
void spin_test_stall_tensor_core_waits(int enable);

/* Operations for spin_uses_tensor_cores. */
#define SPIN_OP_HADAMARD_QUANT 0 /* spin_hadamard_quant_int4[_ex] and spin_hadamard_quant_int8 */
#define SPIN_OP_DEQUANT_INVERSE 1 /* spin_dequant_hadamard_inverse */

/*
 * Host-only query (no device access, no launch): 1 if a call of operation `op`
 * with these arguments would run a tensor-core kernel, 0 if it would run the
 * CUDA-core kernel, -1 if the arguments are invalid for `op` (n not a supported
 * power of two, rows < 0 or above the entry point's limit -- 2^47 - 1 tokens for
 * SPIN_OP_HADAMARD_QUANT, 2^46 - 1 rows for SPIN_OP_DEQUANT_INVERSE --, unknown op
 * or flag bits). has_signs != 0 means a sign_bits mask would be passed. The
 * answer follows the same rules as the entry points' own dispatch.
 */
int spin_uses_tensor_cores(int32_t op, int64_t rows, int32_t n, uint32_t flags, int32_t has_signs);

/* Human-readable name of a status code (static storage). */
const char *spin_status_string(spin_status_t status);

/* cudaError_t value of the last failed CUDA call made by this library in the
 * calling thread (0 if none). */
int spin_last_cuda_error(void);

/* Library version as major * 10000 + minor * 100 + patch. */
int spin_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SPIN_H_ */
