// spin_launch.h -- host-side launchers behind the C ABI (internal header).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace spin {

constexpr uint32_t kNoRotate = 1u;        // same value as SPIN_NO_ROTATE
constexpr uint32_t kCudaCoresOnly = 2u;   // same value as SPIN_CUDA_CORES_ONLY
constexpr uint32_t kTensorCores = 4u;     // same value as SPIN_TENSOR_CORES

// SPIN_OK for cudaSuccess; otherwise records `e` for spin_last_cuda_error() and
// returns SPIN_ERR_CUDA (as every entry point reports a failed CUDA call).
int report_cuda_error(cudaError_t e);

// Number of blocks of `kernel` that are resident on the current device at once
// (SM count x blocks per SM), with the dynamic shared-memory opt-in applied.
// Cached per kernel and device after the first call.
cudaError_t resident_slots(const void *kernel, int threads, int dyn_smem, int *slots);

// cuTensorMapEncodeTiled from the driver (null if unavailable), looked up once.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// R4 with per-token codes of `bits` = 4 (two per byte) or 8 (one signed byte each).
cudaError_t launch_rotate_quant(const void *x, int64_t tokens, int log_n, float clip, const uint32_t *signs,
                                uint32_t flags, int bits, uint8_t *q, float *scales, cudaStream_t stream);

// Tensor-core R4 kernels (n = 128, 256 and 2048 to 32768; n = 32768 without a
// sign diagonal): availability and launcher.
bool tc_rotate_quant_supported(int log_n, int64_t tokens, uint32_t flags, bool has_signs);
// n = m 2^k that is not a power of two: Paley's type for m (1, 2, or 0 for none), whether
// the tensor-core kernel covers (m, n) (2^k >= 128, n / 128 a multiple of 16 up to 128),
// and its launch (k1_tc.cu).
int paley_type(int m);
bool kron_supported(int m, int64_t n);
cudaError_t launch_rotate_quant_kron(int m, int n, int bits, const void *x, int64_t tokens, float clip,
                                     const uint32_t *signs, uint8_t *q, float *scales, cudaStream_t stream);
// Decode attention over the INT4 KV cache (k4_decode_attn.cu): workspace bytes for
// the split partials, supported query heads per kv head, and the two launches.
size_t decode_attention_workspace_bytes(int batch, int n_q_heads, int cache_len);
bool decode_attention_group_supported(int group);
cudaError_t launch_decode_attention(const void *q, const uint8_t *k_cache, const uint8_t *v_cache,
                                    const void *k_scale, const void *k_zero, const void *v_scale,
                                    const void *v_zero, const int32_t *lens, int batch, int n_q_heads,
                                    int n_kv_heads, int cache_len, float softmax_scale, void *out, bool out_f32,
                                    float *workspace, cudaStream_t stream);
// W4A4 GEMM on packed INT4 codes (k5_w4a4_gemm.cu): shapes it takes (n_out a multiple
// of 256, k a multiple of 128 up to 65536), the launch, and its status word.
bool w4a4_shape_supported(int64_t tokens, int n_out, int k);
cudaError_t launch_w4a4_gemm(const uint8_t *xq, const float *xs, int64_t tokens, const uint8_t *wq, const float *ws,
                             int n_out, int k, void *out, bool out_f32, cudaStream_t stream);
cudaError_t read_gemm_status(unsigned int *status, bool reset);
cudaError_t launch_rotate_quant_tc(int log_n, int bits, const void *x, int64_t tokens, float clip,
                                   const uint32_t *signs, uint8_t *q, float *scales, cudaStream_t stream);

// Test hook: make the tensor-core R4 kernel withhold one internal signal.
void set_stall_test(int enable);

// Device status words set by kernels whose bounded waits ran out (the tensor-core
// R4 kernel, the R3 kernel and the tensor-core dequantise kernel each keep one).
cudaError_t read_device_status(unsigned int *status, bool reset);
cudaError_t read_rope_status(unsigned int *status, bool reset);

// Tensor-core dequantise + inverse kernels (n = 128, 256 and 4096 to 32768): availability
// and launcher.
bool tc_dequant_supported(int log_n, int64_t rows, uint32_t flags);
cudaError_t launch_dequant_inverse_tc(int log_n, const uint8_t *codes, int64_t rows, int mode, const void *scale,
                                      const void *zero, const uint32_t *signs, void *out, int out_dtype,
                                      cudaStream_t stream);
cudaError_t read_dequant_status(unsigned int *status, bool reset);

cudaError_t launch_dequant_inverse(const uint8_t *codes, int64_t rows, int log_n, int mode,
                                   const void *scale, const void *zero, const uint32_t *signs,
                                   uint32_t flags, void *out, int out_dtype, cudaStream_t stream);

// Head counts and token counts the R3 kernel takes: n_q_heads <= 256,
// n_q_heads + 2 n_kv_heads <= 384, batch * seq * n_q_heads < 2^31.
bool rope_shape_supported(int n_q_heads, int n_kv_heads, int64_t tokens);
cudaError_t launch_rope_hadamard_kvquant(const void *q, const void *k, const void *v,
                                         const int32_t *pos, float theta, int batch, int seq,
                                         int n_q_heads, int n_kv_heads, float clip, void *q_out,
                                         uint8_t *k_cache, uint8_t *v_cache, void *k_scale,
                                         void *k_zero, void *v_scale, void *v_zero, int cache_len,
                                         int cache_offset, cudaStream_t stream);

}  // namespace spin
