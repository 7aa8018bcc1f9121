// k4_decode_attn_noalloc.cu -- decode attention over the INT4 KV cache for callers that
// cannot allocate device memory.
//
// spin_decode_attention_int4kv writes its per-chunk partials to a workspace the caller
// allocates. Some callers cannot do that at the point of the call: a plugin inside an
// inference engine that owns every byte of device memory and hands the plugin no
// scratch, or a real-time serving loop that must not call cudaMalloc because it can
// synchronise the device and stall every stream. This entry point needs nothing from
// them: the partials go to a fixed scratch array compiled into the library.
//
// The array is a file-scope __device__ variable. In host code its name is only a
// host-side stand-in, not a device address, so the host asks the runtime for the
// device address (cudaGetSymbolAddress) once per device, with that device current,
// and passes that address to the kernels. Every GPU that loads the library holds the
// array until the process exits.
#include <cuda_runtime.h>

#include <cstdint>
#include <map>
#include <mutex>

#include "spin.h"
#include "spin_launch.h"

namespace spin {
namespace {

// 4 MiB: batch x n_q_heads x ceil(cache_len / 256) partials of 130 fp32 values each
// (e.g. 4 rows x 32 heads x 16 chunks of a 4096-slot cache use 1.06 MB).
constexpr size_t kScratchBytes = SPIN_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) float g_attn_scratch[kScratchBytes / sizeof(float)];

// Device address of g_attn_scratch on the current device, looked up on the first call
// on each device and kept.
cudaError_t scratch_address(void **ptr) {
  static std::mutex mu;
  static std::map<int, void *> addr;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  auto it = addr.find(dev);
  if (it == addr.end()) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_attn_scratch);
    if (e != cudaSuccess) return e;
    it = addr.emplace(dev, p).first;
  }
  *ptr = it->second;
  return cudaSuccess;
}

}  // namespace
}  // namespace spin

extern "C" spin_status_t spin_decode_attention_int4kv_noalloc(
    const void *q, const uint8_t *k_cache, const uint8_t *v_cache, const void *k_scale, const void *k_zero,
    const void *v_scale, const void *v_zero, const int32_t *lens, int32_t batch, int32_t n_q_heads,
    int32_t n_kv_heads, int32_t head_dim, int32_t cache_len, float softmax_scale, void *out, int32_t out_dtype,
    spin_stream_t stream) {
  // Arguments the workspace entry point rejects before it looks at the workspace go to it
  // unchanged (batch = 0 is its no-op); otherwise the partials must fit the array.
  if (batch <= 0 || n_q_heads <= 0 || n_kv_heads <= 0 || cache_len < 1)
    return spin_decode_attention_int4kv(q, k_cache, v_cache, k_scale, k_zero, v_scale, v_zero, lens, batch,
                                        n_q_heads, n_kv_heads, head_dim, cache_len, softmax_scale, out, out_dtype,
                                        nullptr, 0, stream);
  if (spin_decode_attention_workspace_bytes(batch, n_q_heads, cache_len) > spin::kScratchBytes)
    return SPIN_ERR_SCRATCH_LIMIT;
  void *scratch = nullptr;
  const cudaError_t e = spin::scratch_address(&scratch);
  if (e != cudaSuccess) return static_cast<spin_status_t>(spin::report_cuda_error(e));
  return spin_decode_attention_int4kv(q, k_cache, v_cache, k_scale, k_zero, v_scale, v_zero, lens, batch,
                                      n_q_heads, n_kv_heads, head_dim, cache_len, softmax_scale, out, out_dtype,
                                      scratch, spin::kScratchBytes, stream);
}
