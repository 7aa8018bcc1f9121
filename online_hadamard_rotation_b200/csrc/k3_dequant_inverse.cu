// k3_dequant_inverse.cu -- dequantise packed INT4 rows and rotate them back:
// out = D H_n v / sqrt(n) with v_j = code_j * scale (symmetric) or
// (code_j - zero) * scale (asymmetric), or out = v with no rotation.
//
// "Rotations: QuaRot, SpinQuant and incoherence", widget "Try it": rotate,
// quantize, rotate back; section "Hadamard matrices": H_n / sqrt(n) is
// orthogonal and symmetric, so D H_n / sqrt(n) inverts H_n D / sqrt(n).
// "SpinQuant Guide: Learned Rotations for 4-Bit LLMs", section "End-to-End
// Implementation": dequantised value = code * scale.
//
// The codes (minus the zero point) are small integers, so the transform runs
// on them exactly in fp32 (|sum| <= 15 * 2^15 < 2^24) and the row's
// scale / sqrt(n) is applied once at the end.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <type_traits>

#include "spin_launch.h"
#include "spin_tile.cuh"

namespace spin {
namespace {

template <int TB, int LOGN, bool ROTATE, bool SIGNS>
__global__ void __launch_bounds__(1 << (TB - 7))
    k3_dequant_inverse(const uint32_t *__restrict__ codes, int64_t rows, float inv_sqrt_n,
                       const void *__restrict__ scale, const __half *__restrict__ zero,
                       const uint32_t *__restrict__ signs, void *__restrict__ out, bool asym,
                       bool out_f32) {
  constexpr int ROWS = 1 << (TB - LOGN);
  constexpr uint32_t NMASK = (1u << LOGN) - 1u;
  using LI = L1<TB>;
  using LO = std::conditional_t<ROTATE, OutLayout<TB>, L1<TB>>;

  extern __shared__ float4 smem_raw[];
  float *sm = reinterpret_cast<float *>(smem_raw);
  const uint32_t t = threadIdx.x;
  const int64_t ntiles = (rows + ROWS - 1) / ROWS;

  for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    float v[kRegs];
    const uint32_t *ct = codes + tile * (int64_t)(1 << (TB - 3));
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t E = LI::thr(t) | LI::reg(8 * j);
      const int64_t row = tile * ROWS + (E >> LOGN);
      uint32_t w = 0u;
      float z = 0.f;
      if (row < rows) {
        w = __ldcs(ct + (E >> 3));
        if (asym) z = __half2float(zero[row]);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t nib = (w >> (4 * i)) & 0xFu;
        v[8 * j + i] = asym ? (float)nib - z : (float)((int)(nib ^ 8u) - 8);
      }
    }
    if constexpr (ROTATE) tile_fwht<TB, LOGN>(v, sm, t);

#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t E = LO::thr(t) | LO::reg(8 * j);
      const int64_t row = tile * ROWS + (E >> LOGN);
      if (row >= rows) continue;
      const float s = asym ? __half2float(static_cast<const __half *>(scale)[row])
                           : static_cast<const float *>(scale)[row];
      const float m = ROTATE ? s * inv_sqrt_n : s;
      float o[8];
      uint32_t sb = 0u;
      if constexpr (SIGNS) {
        const uint32_t e = E & NMASK;
        sb = (__ldg(signs + (e >> 5)) >> (e & 31u)) & 0xFFu;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float r = v[8 * j + i] * m;
        if constexpr (SIGNS) r = __uint_as_float(__float_as_uint(r) ^ (((sb >> i) & 1u) << 31));
        o[i] = r;
      }
      const int64_t off = tile * (int64_t)(1 << TB) + E;
      if (out_f32) {
        float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(out) + off);
        __stcs(dst, make_float4(o[0], o[1], o[2], o[3]));
        __stcs(dst + 1, make_float4(o[4], o[5], o[6], o[7]));
      } else {
        uint4 p = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                             pack_bf16x2(o[6], o[7]));
        __stcs(reinterpret_cast<uint4 *>(static_cast<uint16_t *>(out) + off), p);
      }
    }
  }
}

template <int TB, int LOGN, bool ROTATE, bool SIGNS>
cudaError_t launch_one(const uint8_t *codes, int64_t rows, const void *scale, const void *zero,
                       const uint32_t *signs, void *out, bool asym, bool out_f32, cudaStream_t stream) {
  auto kern = k3_dequant_inverse<TB, LOGN, ROTATE, SIGNS>;
  constexpr int kThreads = 1 << (TB - 7);
  constexpr int kSmem = ROTATE ? (1 << TB) * (int)sizeof(float) : 0;
  int slots = 0;
  cudaError_t err = resident_slots(reinterpret_cast<const void *>(kern), kThreads, kSmem, &slots);
  if (err != cudaSuccess) return err;
  constexpr int ROWS = 1 << (TB - LOGN);
  const int64_t ntiles = (rows + ROWS - 1) / ROWS;
  const int64_t grid = ntiles < (int64_t)slots ? ntiles : (int64_t)slots;
  const float inv_sqrt_n = (float)(1.0 / std::sqrt((double)(1 << LOGN)));
  kern<<<(unsigned)grid, kThreads, kSmem, stream>>>(reinterpret_cast<const uint32_t *>(codes), rows,
                                                    inv_sqrt_n, scale, static_cast<const __half *>(zero),
                                                    signs, out, asym, out_f32);
  return cudaGetLastError();
}

template <int LOGN>
cudaError_t launch_n(const uint8_t *codes, int64_t rows, int mode, const void *scale, const void *zero,
                     const uint32_t *signs, uint32_t flags, void *out, int out_dtype, cudaStream_t stream) {
  constexpr int TB = LOGN <= 14 ? 14 : 15;
  const bool asym = mode == 1, f32 = out_dtype == 1;
  if (flags & kNoRotate)
    return launch_one<TB, LOGN, false, false>(codes, rows, scale, zero, nullptr, out, asym, f32, stream);
  if (signs) return launch_one<TB, LOGN, true, true>(codes, rows, scale, zero, signs, out, asym, f32, stream);
  return launch_one<TB, LOGN, true, false>(codes, rows, scale, zero, nullptr, out, asym, f32, stream);
}

}  // namespace

cudaError_t launch_dequant_inverse(const uint8_t *codes, int64_t rows, int log_n, int mode,
                                   const void *scale, const void *zero, const uint32_t *signs,
                                   uint32_t flags, void *out, int out_dtype, cudaStream_t stream) {
  if (!(flags & kCudaCoresOnly) && tc_dequant_supported(log_n, rows, flags))
    return launch_dequant_inverse_tc(log_n, codes, rows, mode, scale, zero, signs, out, out_dtype, stream);
  flags &= ~(kCudaCoresOnly | kTensorCores);
  switch (log_n) {
    case 7: return launch_n<7>(codes, rows, mode, scale, zero, signs, flags, out, out_dtype, stream);
    case 8: return launch_n<8>(codes, rows, mode, scale, zero, signs, flags, out, out_dtype, stream);
    case 9: return launch_n<9>(codes, rows, mode, scale, zero, signs, flags, out, out_dtype, stream);
    case 10: return launch_n<10>(codes, rows, mode, scale, zero, signs, flags, out, out_dtype, stream);
    case 11: return launch_n<11>(codes, rows, mode, scale, zero, signs, flags, out, out_dtype, stream);
    case 12: return launch_n<12>(codes, rows, mode, scale, zero, signs, flags, out, out_dtype, stream);
    case 13: return launch_n<13>(codes, rows, mode, scale, zero, signs, flags, out, out_dtype, stream);
    case 14: return launch_n<14>(codes, rows, mode, scale, zero, signs, flags, out, out_dtype, stream);
    case 15: return launch_n<15>(codes, rows, mode, scale, zero, signs, flags, out, out_dtype, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace spin
