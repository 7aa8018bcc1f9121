// api.cu -- the extern "C" entry points declared in include/spin.h: argument
// validation on the host, then one kernel launch on the caller's stream.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <map>
#include <mutex>
#include <tuple>

#include "spin.h"
#include "spin_launch.h"

namespace spin {

namespace {
thread_local int g_last_cuda_error = 0;

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int log2_pow2(int64_t n) {
  if (n <= 0 || (n & (n - 1)) != 0) return -1;
  int l = 0;
  while ((int64_t(1) << l) < n) ++l;
  return l;
}

spin_status_t cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SPIN_OK;
  g_last_cuda_error = static_cast<int>(e);
  return SPIN_ERR_CUDA;
}

// The kernels are built for sm_100a only: require compute capability 10.0.
spin_status_t check_device() {
  static std::mutex mu;
  static std::map<int, bool> ok;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e);
  std::lock_guard<std::mutex> lock(mu);
  auto it = ok.find(dev);
  if (it == ok.end()) {
    int major = 0, minor = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
      return cuda_status(e);
    if ((e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
      return cuda_status(e);
    it = ok.emplace(dev, major == 10 && minor == 0).first;
  }
  return it->second ? SPIN_OK : SPIN_ERR_DEVICE;
}

bool valid_clip(float clip) { return clip > 0.0f && clip <= 1.0f; }  // false for NaN
}  // namespace

int report_cuda_error(cudaError_t e) { return static_cast<int>(cuda_status(e)); }

cudaError_t resident_slots(const void *kernel, int threads, int dyn_smem, int *slots) {
  static std::mutex mu;
  static std::map<std::tuple<const void *, int, int, int>, int> cache;
  static std::map<std::pair<const void *, int>, bool> opted_in;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const auto key = std::make_tuple(kernel, dev, threads, dyn_smem);
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(key);
  if (it != cache.end()) {
    *slots = it->second;
    return cudaSuccess;
  }
  // Opt in once to the device's full per-block shared memory, so that no
  // later call with a smaller request can lower the limit an earlier,
  // larger launch configuration relies on.
  if (!opted_in[std::make_pair(kernel, dev)]) {
    int optin = 0;
    if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, kernel)) != cudaSuccess) return e;
    const int dyn_max = optin - (int)fa.sharedSizeBytes;  // static + dynamic must fit the opt-in limit
    if (dyn_smem > dyn_max) return cudaErrorInvalidConfiguration;
    if ((e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_max)) != cudaSuccess)
      return e;
    // All of the unified L1/shared storage as shared memory, so the blocks per SM
    // found below are the blocks that become resident at launch (none of these
    // kernels relies on L1 caching).
    if ((e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                  (int)cudaSharedmemCarveoutMaxShared)) != cudaSuccess)
      return e;
    opted_in[std::make_pair(kernel, dev)] = true;
  }
  int sms = 0, per_sm = 0;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, dyn_smem)) != cudaSuccess)
    return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  cache.emplace(key, sms * per_sm);
  *slots = sms * per_sm;
  return cudaSuccess;
}

}  // namespace spin

using namespace spin;

// R4 with `bits` = 4 or 8: host-side checks, then the launch.
static spin_status_t hadamard_quant(const void *x_bf16, int64_t tokens, int32_t n, float clip,
                                    const uint32_t *sign_bits, uint32_t flags, int bits, uint8_t *q,
                                    float *scales_f32, spin_stream_t stream) {
  const int log_n = log2_pow2(n);
  if (log_n < 7 || log_n > 15) return SPIN_ERR_UNSUPPORTED_SIZE;
  if (tokens < 0 || !valid_clip(clip) || (flags & ~(SPIN_NO_ROTATE | SPIN_CUDA_CORES_ONLY | SPIN_TENSOR_CORES)) != 0 ||
      (flags & SPIN_CUDA_CORES_ONLY && flags & SPIN_TENSOR_CORES))
    return SPIN_ERR_INVALID_ARG;
  if (tokens == 0) return SPIN_OK;
  if (!x_bf16 || !q || !scales_f32) return SPIN_ERR_INVALID_ARG;
  if (tokens > (INT64_MAX >> 16)) return SPIN_ERR_INVALID_ARG;
  if (!aligned(x_bf16, 16) || !aligned(q, 16) || !aligned(scales_f32, 4) || (sign_bits && !aligned(sign_bits, 4)))
    return SPIN_ERR_MISALIGNED;
  spin_status_t st = check_device();
  if (st != SPIN_OK) return st;
  return cuda_status(launch_rotate_quant(x_bf16, tokens, log_n, clip, sign_bits, flags, bits, q, scales_f32,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

extern "C" {

spin_status_t spin_hadamard_quant_int4_ex(const void *x_bf16, int64_t tokens, int32_t n, float clip,
                                          const uint32_t *sign_bits, uint32_t flags,
                                          uint8_t *q_packed_u8, float *scales_f32,
                                          spin_stream_t stream) {
  return hadamard_quant(x_bf16, tokens, n, clip, sign_bits, flags, 4, q_packed_u8, scales_f32, stream);
}

spin_status_t spin_hadamard_quant_int8(const void *x_bf16, int64_t tokens, int32_t n, float clip,
                                       const uint32_t *sign_bits, uint32_t flags, int8_t *q_i8,
                                       float *scales_f32, spin_stream_t stream) {
  return hadamard_quant(x_bf16, tokens, n, clip, sign_bits, flags, 8, reinterpret_cast<uint8_t *>(q_i8),
                        scales_f32, stream);
}

spin_status_t spin_hadamard_quant_int4(const void *x_bf16, int64_t tokens, int32_t n, float clip,
                                       uint8_t *q_packed_u8, float *scales_f32, spin_stream_t stream) {
  return spin_hadamard_quant_int4_ex(x_bf16, tokens, n, clip, nullptr, 0u, q_packed_u8, scales_f32, stream);
}

spin_status_t spin_hadamard_quant_kron(const void *x_bf16, int64_t tokens, int32_t m, int32_t n, float clip,
                                       const uint32_t *sign_bits, uint32_t flags, int32_t bits, void *q,
                                       float *scales_f32, spin_stream_t stream) {
  if (!kron_supported(m, n)) return SPIN_ERR_UNSUPPORTED_SIZE;
  if (tokens < 0 || !valid_clip(clip) || (flags & ~SPIN_TENSOR_CORES) != 0 || (bits != 4 && bits != 8))
    return SPIN_ERR_INVALID_ARG;
  if (tokens == 0) return SPIN_OK;
  if (!x_bf16 || !q || !scales_f32) return SPIN_ERR_INVALID_ARG;
  if (tokens >= ((int64_t(1) << 31) / (n / 128))) return SPIN_ERR_UNSUPPORTED_SIZE;  // 32-bit TMA row coordinates
  if (!aligned(x_bf16, 16) || !aligned(q, 16) || !aligned(scales_f32, 4) || (sign_bits && !aligned(sign_bits, 4)))
    return SPIN_ERR_MISALIGNED;
  spin_status_t st = check_device();
  if (st != SPIN_OK) return st;
  return cuda_status(launch_rotate_quant_kron(m, n, bits, x_bf16, tokens, clip, sign_bits, static_cast<uint8_t *>(q),
                                              scales_f32, reinterpret_cast<cudaStream_t>(stream)));
}

spin_status_t spin_w4a4_gemm(const uint8_t *x_codes, const float *x_scales, int64_t tokens, const uint8_t *w_codes,
                             const float *w_scales, int32_t n_out, int32_t k, void *out, int32_t out_dtype,
                             spin_stream_t stream) {
  if (tokens < 0 || (out_dtype != SPIN_BF16 && out_dtype != SPIN_F32)) return SPIN_ERR_INVALID_ARG;
  if (!w4a4_shape_supported(tokens, n_out, k)) return SPIN_ERR_UNSUPPORTED_SIZE;
  if (tokens == 0) return SPIN_OK;
  if (!x_codes || !x_scales || !w_codes || !w_scales || !out) return SPIN_ERR_INVALID_ARG;
  if (!aligned(x_codes, 16) || !aligned(w_codes, 16) || !aligned(out, 16) || !aligned(w_scales, 16) ||
      !aligned(x_scales, 4))
    return SPIN_ERR_MISALIGNED;
  spin_status_t st = check_device();
  if (st != SPIN_OK) return st;
  return cuda_status(launch_w4a4_gemm(x_codes, x_scales, tokens, w_codes, w_scales, n_out, k, out,
                                      out_dtype == SPIN_F32, reinterpret_cast<cudaStream_t>(stream)));
}

spin_status_t spin_rope_hadamard_kvquant(const void *q, const void *k, const void *v, const int32_t *pos,
                                         float theta, int32_t head_dim, int32_t batch, int32_t seq,
                                         int32_t n_q_heads, int32_t n_kv_heads, float clip, void *q_out,
                                         uint8_t *k_cache, uint8_t *v_cache, void *k_scale, void *k_zero,
                                         void *v_scale, void *v_zero, int32_t cache_len,
                                         int32_t cache_offset, spin_stream_t stream) {
  if (head_dim != 128) return SPIN_ERR_UNSUPPORTED_SIZE;
  if (batch < 0 || seq < 0 || n_q_heads <= 0 || n_kv_heads <= 0 || n_q_heads % n_kv_heads != 0 ||
      !valid_clip(clip) || !(theta > 0.0f) || !std::isfinite(theta) || cache_offset < 0 ||
      (int64_t)cache_len < (int64_t)cache_offset + seq)
    return SPIN_ERR_INVALID_ARG;
  if (!rope_shape_supported(n_q_heads, n_kv_heads, (int64_t)batch * seq)) return SPIN_ERR_UNSUPPORTED_SIZE;
  if (batch == 0 || seq == 0) return SPIN_OK;
  if (!q || !k || !v || !pos || !q_out || !k_cache || !v_cache || !k_scale || !k_zero || !v_scale || !v_zero)
    return SPIN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(q_out, 16) || !aligned(k_cache, 16) ||
      !aligned(v_cache, 16) || !aligned(pos, 4) || !aligned(k_scale, 2) || !aligned(k_zero, 2) ||
      !aligned(v_scale, 2) || !aligned(v_zero, 2))
    return SPIN_ERR_MISALIGNED;
  spin_status_t st = check_device();
  if (st != SPIN_OK) return st;
  return cuda_status(launch_rope_hadamard_kvquant(q, k, v, pos, theta, batch, seq, n_q_heads, n_kv_heads, clip,
                                                  q_out, k_cache, v_cache, k_scale, k_zero, v_scale, v_zero,
                                                  cache_len, cache_offset,
                                                  reinterpret_cast<cudaStream_t>(stream)));
}

size_t spin_decode_attention_workspace_bytes(int32_t batch, int32_t n_q_heads, int32_t cache_len) {
  if (batch <= 0 || n_q_heads <= 0 || cache_len <= 0) return 0;
  return decode_attention_workspace_bytes(batch, n_q_heads, cache_len);
}

spin_status_t spin_decode_attention_int4kv(const void *q, const uint8_t *k_cache, const uint8_t *v_cache,
                                           const void *k_scale, const void *k_zero, const void *v_scale,
                                           const void *v_zero, const int32_t *lens, int32_t batch,
                                           int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                           int32_t cache_len, float softmax_scale, void *out, int32_t out_dtype,
                                           void *workspace, size_t workspace_bytes, spin_stream_t stream) {
  if (batch < 0 || n_q_heads <= 0 || n_kv_heads <= 0 || cache_len < 1 || n_q_heads % n_kv_heads != 0 ||
      !(softmax_scale > 0.0f) || !std::isfinite(softmax_scale) || (out_dtype != SPIN_BF16 && out_dtype != SPIN_F32))
    return SPIN_ERR_INVALID_ARG;
  if (head_dim != 128 || !decode_attention_group_supported(n_q_heads / n_kv_heads) || batch > 65535 ||
      n_q_heads > 65535 || n_kv_heads > 65535)
    return SPIN_ERR_UNSUPPORTED_SIZE;
  if (batch == 0) return SPIN_OK;
  if (!q || !k_cache || !v_cache || !k_scale || !k_zero || !v_scale || !v_zero || !lens || !out || !workspace)
    return SPIN_ERR_INVALID_ARG;
  if (workspace_bytes < decode_attention_workspace_bytes(batch, n_q_heads, cache_len)) return SPIN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
      !aligned(workspace, 16) || !aligned(lens, 4) || !aligned(k_scale, 2) || !aligned(k_zero, 2) ||
      !aligned(v_scale, 2) || !aligned(v_zero, 2))
    return SPIN_ERR_MISALIGNED;
  spin_status_t st = check_device();
  if (st != SPIN_OK) return st;
  return cuda_status(launch_decode_attention(q, k_cache, v_cache, k_scale, k_zero, v_scale, v_zero, lens, batch,
                                             n_q_heads, n_kv_heads, cache_len, softmax_scale, out,
                                             out_dtype == SPIN_F32, static_cast<float *>(workspace),
                                             reinterpret_cast<cudaStream_t>(stream)));
}

spin_status_t spin_dequant_hadamard_inverse(const uint8_t *codes, int64_t rows, int32_t n, int32_t mode,
                                            const void *scale, const void *zero, const uint32_t *sign_bits,
                                            uint32_t flags, void *out, int32_t out_dtype,
                                            spin_stream_t stream) {
  const int log_n = log2_pow2(n);
  if (log_n < 7 || log_n > 15) return SPIN_ERR_UNSUPPORTED_SIZE;
  if (rows < 0 || (mode != SPIN_SYM_INT4_F32SCALE && mode != SPIN_ASYM_INT4_F16SZ) ||
      (out_dtype != SPIN_BF16 && out_dtype != SPIN_F32) ||
      (flags & ~(SPIN_NO_ROTATE | SPIN_CUDA_CORES_ONLY | SPIN_TENSOR_CORES)) != 0 ||
      (flags & (SPIN_CUDA_CORES_ONLY | SPIN_TENSOR_CORES)) == (SPIN_CUDA_CORES_ONLY | SPIN_TENSOR_CORES))
    return SPIN_ERR_INVALID_ARG;
  if (rows == 0) return SPIN_OK;
  if (!codes || !scale || !out || (mode == SPIN_ASYM_INT4_F16SZ && !zero)) return SPIN_ERR_INVALID_ARG;
  if (rows > (INT64_MAX >> 17)) return SPIN_ERR_INVALID_ARG;
  if (!aligned(codes, 16) || !aligned(out, 16) || !aligned(scale, mode == SPIN_SYM_INT4_F32SCALE ? 4 : 2) ||
      (zero && !aligned(zero, 2)) || (sign_bits && !aligned(sign_bits, 4)))
    return SPIN_ERR_MISALIGNED;
  spin_status_t st = check_device();
  if (st != SPIN_OK) return st;
  return cuda_status(launch_dequant_inverse(codes, rows, log_n, mode, scale, zero, sign_bits, flags, out,
                                            out_dtype, reinterpret_cast<cudaStream_t>(stream)));
}

void spin_test_stall_tensor_core_waits(int enable) { set_stall_test(enable); }

const char *spin_status_string(spin_status_t status) {
  switch (status) {
    case SPIN_OK: return "SPIN_OK";
    case SPIN_ERR_INVALID_ARG: return "SPIN_ERR_INVALID_ARG";
    case SPIN_ERR_UNSUPPORTED_SIZE: return "SPIN_ERR_UNSUPPORTED_SIZE";
    case SPIN_ERR_MISALIGNED: return "SPIN_ERR_MISALIGNED";
    case SPIN_ERR_CUDA: return "SPIN_ERR_CUDA";
    case SPIN_ERR_DEVICE: return "SPIN_ERR_DEVICE";
    case SPIN_ERR_SCRATCH_LIMIT: return "SPIN_ERR_SCRATCH_LIMIT";
  }
  return "SPIN_ERR_UNKNOWN";
}

int spin_last_cuda_error(void) { return g_last_cuda_error; }

spin_status_t spin_device_status(uint32_t *status, int reset) {
  if (!status) return SPIN_ERR_INVALID_ARG;
  unsigned int v = 0, w = 0, u = 0, g = 0;
  spin_status_t st = cuda_status(read_device_status(&v, reset != 0));
  if (st == SPIN_OK) st = cuda_status(read_rope_status(&w, reset != 0));
  if (st == SPIN_OK) st = cuda_status(read_dequant_status(&u, reset != 0));
  if (st == SPIN_OK) st = cuda_status(read_gemm_status(&g, reset != 0));
  *status = v | w | u | g;
  return st;
}

int spin_uses_tensor_cores(int32_t op, int64_t rows, int32_t n, uint32_t flags, int32_t has_signs) {
  const int log_n = log2_pow2(n);
  if (log_n < 7 || log_n > 15 || rows < 0) return -1;
  if ((flags & ~(SPIN_NO_ROTATE | SPIN_CUDA_CORES_ONLY | SPIN_TENSOR_CORES)) != 0 ||
      (flags & (SPIN_CUDA_CORES_ONLY | SPIN_TENSOR_CORES)) == (SPIN_CUDA_CORES_ONLY | SPIN_TENSOR_CORES))
    return -1;
  // the entry points' own upper bounds on the row count
  if (op == SPIN_OP_HADAMARD_QUANT) {
    if (rows > (INT64_MAX >> 16)) return -1;
  } else if (op == SPIN_OP_DEQUANT_INVERSE) {
    if (rows > (INT64_MAX >> 17)) return -1;
  } else {
    return -1;
  }
  if (flags & SPIN_CUDA_CORES_ONLY) return 0;
  if (op == SPIN_OP_HADAMARD_QUANT) return tc_rotate_quant_supported(log_n, rows, flags, has_signs != 0) ? 1 : 0;
  return tc_dequant_supported(log_n, rows, flags) ? 1 : 0;
}

int spin_version(void) { return 100; }

}  // extern "C"
