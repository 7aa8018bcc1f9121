// k1_rotate_quant.cu -- R4 on CUDA cores: bf16 rows -> optional +-1 diagonal
// -> Walsh-Hadamard transform -> per-row max|y| -> symmetric INT4 codes packed
// two per byte (or INT8 codes, one per byte), plus an fp32 step per row, in one
// pass over memory.
//
// "SpinQuant, when rotations are worth learning", section "Four rotation
// sites": R4 is a fixed Hadamard on the down-projection input.
// "Rotations: QuaRot, SpinQuant and incoherence", section "Hadamard
// matrices": (1/sqrt n) H_n diag(+-1); example "a hidden state with an
// outlier channel": per-token 4-bit step max/7.
// "SpinQuant Guide: Learned Rotations for 4-Bit LLMs", section "The Outlier
// Curse": INT4 range [-8, 7]; section "End-to-End Implementation": the step is
// clamped below at 1e-8. The same rule at b = 8 bits gives the per-token INT8
// codes (range [-128, 127], step max / 127).
//
// The transform is computed unnormalised (u = H_n D x); the 1/sqrt(n) factor
// is folded into the step, since the codes do not depend on it (Q = 7 or 127):
//   step = max(clip * max|u| / sqrt(n) / Q, 1e-8),   code = clamp(rne(u / (sqrt(n) * step)), -Q-1, Q).
// Codes come out of two FMAs: v = sat(u * c/(2Q+1) + (Q+1)/(2Q+1)) clamps to the
// code range, and fma(v, 2Q+1, 1.5 * 2^23) rounds (2Q+1) v to the nearest
// integer (ties to even) in the low mantissa bits, where byte permutes pick
// them up.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <type_traits>

#include "spin_launch.h"
#include "spin_tile.cuh"

namespace spin {
namespace {

constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23: adding it rounds to an integer in the low bits

__device__ __forceinline__ float fma_sat(float a, float b, float c) {
  float r;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 8 biased codes (0..15, in the low byte of each word) -> one word of 8 nibbles,
// code k in nibble k, converted to 4-bit two's complement.
__device__ __forceinline__ uint32_t pack8(const uint32_t (&b)[8]) {
  const uint32_t e = __byte_perm(__byte_perm(b[0], b[2], 0x0040), __byte_perm(b[4], b[6], 0x0040), 0x5410);
  const uint32_t o = __byte_perm(__byte_perm(b[1], b[3], 0x0040), __byte_perm(b[5], b[7], 0x0040), 0x5410);
  return (e | (o << 4)) ^ 0x88888888u;
}

// 4 biased codes (0..255, in the low byte of each word) -> one word of 4 bytes,
// code k in byte k, converted to 8-bit two's complement.
__device__ __forceinline__ uint32_t pack4(uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
  return __byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410) ^ 0x80808080u;
}

template <int BITS, int TB, int LOGN, bool ROTATE, bool SIGNS>
__device__ __forceinline__ void rotate_quant_body(const uint4 *__restrict__ x, int64_t tokens, float clip,
                                                  float inv_sqrt_n, const uint32_t *__restrict__ signs,
                                                  uint32_t *__restrict__ q, float *__restrict__ scales) {
  constexpr float QMAX = BITS == 4 ? 7.0f : 127.0f;   // largest code
  constexpr float LEVELS = 2.0f * QMAX + 1.0f;        // 15 or 255 steps across the range
  constexpr int ROWS = 1 << (TB - LOGN);  // rows per tile
  constexpr uint32_t NMASK = (1u << LOGN) - 1u;
  using LI = L1<TB>;
  using LO = std::conditional_t<ROTATE, OutLayout<TB>, L1<TB>>;
  constexpr int HB = LO::kHi;                           // element bit of output register bit 3
  constexpr int SH = LOGN > HB ? LOGN - HB : 0;         // register-octet index -> row slot
  constexpr int NR = (LOGN >= HB + 4) ? 1 : (16 >> SH); // distinct rows among a thread's registers

  extern __shared__ float4 smem_raw[];
  float *sm = reinterpret_cast<float *>(smem_raw);
  __shared__ uint32_t rowmax[ROWS];
  __shared__ float rowc15[ROWS];

  const uint32_t t = threadIdx.x;
  const uint32_t lane = t & 31u;
  const int64_t ntiles = (tokens + ROWS - 1) / ROWS;

  // Sign bytes of this thread's 16 octets: the element positions inside a row
  // that a thread loads are the same for every tile.
  uint32_t sgn[4] = {0u, 0u, 0u, 0u};
  if constexpr (SIGNS) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t e = (LI::thr(t) | LI::reg(8 * j)) & NMASK;
      const uint32_t byte = (__ldg(signs + (e >> 5)) >> (e & 31u)) & 0xFFu;
      sgn[j >> 2] |= byte << ((j & 3) * 8);
    }
  }

  uint4 nx[16];
  auto load_tile = [&](int64_t tile) {
    const uint4 *base = x + tile * (int64_t)(1 << (TB - 3));
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t E = LI::thr(t) | LI::reg(8 * j);
      const int64_t row = tile * ROWS + (E >> LOGN);
      nx[j] = row < tokens ? __ldcs(base + (E >> 3)) : make_uint4(0u, 0u, 0u, 0u);
    }
  };

  int64_t tile = blockIdx.x;
  if (tile < ntiles) load_tile(tile);
  for (; tile < ntiles; tile += gridDim.x) {
    float v[kRegs];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t w[4] = {nx[j].x, nx[j].y, nx[j].z, nx[j].w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        uint32_t lo = w[h] << 16, hi = w[h] & 0xFFFF0000u;
        if constexpr (SIGNS) {
          const uint32_t sb = sgn[j >> 2] >> ((j & 3) * 8 + 2 * h);
          lo ^= (sb << 31);
          hi ^= ((sb >> 1) << 31);
        }
        v[8 * j + 2 * h] = __uint_as_float(lo);
        v[8 * j + 2 * h + 1] = __uint_as_float(hi);
      }
    }
    if (t < (uint32_t)ROWS) rowmax[t] = 0u;
    const int64_t next = tile + gridDim.x;
    if (next < ntiles) load_tile(next);  // prefetch while this tile is transformed

    if constexpr (ROTATE) {
      tile_fwht<TB, LOGN>(v, sm, t);
    } else {
      __syncthreads();
    }

    // ---- per-row max |u|
    const uint32_t thr_row = LO::thr(t) >> LOGN;
    float pm[NR];
#pragma unroll
    for (int k = 0; k < NR; ++k) pm[k] = 0.f;
#pragma unroll
    for (int r = 0; r < kRegs; ++r) {
      const int k = (r >> 3) >> SH;
      pm[k] = fmaxf(pm[k], fabsf(v[r]));
    }
    constexpr uint32_t kRed = (3 + 0 < LOGN ? 1u : 0u) | (3 + 1 < LOGN ? 2u : 0u) |
                              (3 + 2 < LOGN ? 4u : 0u) | (3 + 3 < LOGN ? 8u : 0u) |
                              (3 + 4 < LOGN ? 16u : 0u);
#pragma unroll
    for (int k = 0; k < NR; ++k) {
#pragma unroll
      for (int b = 0; b < 5; ++b)
        if (kRed & (1u << b)) pm[k] = fmaxf(pm[k], __shfl_xor_sync(0xFFFFFFFFu, pm[k], 1 << b));
    }
    if ((lane & kRed) == 0u) {
#pragma unroll
      for (int k = 0; k < NR; ++k) {
        const uint32_t row = thr_row | ((((uint32_t)(k << SH)) << HB) >> LOGN);
        atomicMax(&rowmax[row], __float_as_uint(pm[k]));
      }
    }
    __syncthreads();
    if (t < (uint32_t)ROWS) {
      const float m = __uint_as_float(rowmax[t]) * inv_sqrt_n;
      const float s = fmaxf(clip * m / QMAX, 1e-8f);
      rowc15[t] = (inv_sqrt_n / s) / LEVELS;
      const int64_t row = tile * ROWS + t;
      if (row < tokens) scales[row] = s;
    }
    __syncthreads();

    // ---- quantise, pack, store
    constexpr float k815 = (QMAX + 1.0f) / LEVELS;  // code 0 sits at (Q + 1) / (2Q + 1)
    uint32_t *qt = q + tile * (int64_t)(1 << (TB - 3)) * (BITS / 4);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t rr = ((((uint32_t)(j >> SH) << SH)) << HB) >> LOGN;
      const float c15 = rowc15[thr_row | rr];
      uint32_t b[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float vv = fma_sat(v[8 * j + i], c15, k815);
        b[i] = __float_as_uint(fmaf(vv, LEVELS, kMagic));
      }
      const uint32_t E = LO::thr(t) | LO::reg(8 * j);
      if (tile * ROWS + (E >> LOGN) < tokens) {
        if constexpr (BITS == 4)
          __stcs(qt + (E >> 3), pack8(b));
        else
          __stcs(reinterpret_cast<uint2 *>(qt) + (E >> 3),
                 make_uint2(pack4(b[0], b[1], b[2], b[3]), pack4(b[4], b[5], b[6], b[7])));
      }
    }
  }
}

template <int TB, int LOGN, bool ROTATE, bool SIGNS>
__global__ void __launch_bounds__(1 << (TB - 7))
    k1_rotate_quant_int4(const uint4 *__restrict__ x, int64_t tokens, float clip, float inv_sqrt_n,
                         const uint32_t *__restrict__ signs, uint32_t *__restrict__ q,
                         float *__restrict__ scales) {
  rotate_quant_body<4, TB, LOGN, ROTATE, SIGNS>(x, tokens, clip, inv_sqrt_n, signs, q, scales);
}

template <int TB, int LOGN, bool ROTATE, bool SIGNS>
__global__ void __launch_bounds__(1 << (TB - 7))
    k1_rotate_quant_int8(const uint4 *__restrict__ x, int64_t tokens, float clip, float inv_sqrt_n,
                         const uint32_t *__restrict__ signs, uint32_t *__restrict__ q,
                         float *__restrict__ scales) {
  rotate_quant_body<8, TB, LOGN, ROTATE, SIGNS>(x, tokens, clip, inv_sqrt_n, signs, q, scales);
}

template <int BITS, int TB, int LOGN, bool ROTATE, bool SIGNS>
cudaError_t launch_one(const void *x, int64_t tokens, float clip, const uint32_t *signs, uint8_t *q,
                       float *scales, cudaStream_t stream) {
  auto kern = BITS == 4 ? k1_rotate_quant_int4<TB, LOGN, ROTATE, SIGNS> : k1_rotate_quant_int8<TB, LOGN, ROTATE, SIGNS>;
  constexpr int kThreads = 1 << (TB - 7);
  constexpr int kSmem = (1 << TB) * (int)sizeof(float);
  int slots = 0;
  cudaError_t err = resident_slots(reinterpret_cast<const void *>(kern), kThreads, kSmem, &slots);
  if (err != cudaSuccess) return err;
  constexpr int ROWS = 1 << (TB - LOGN);
  const int64_t ntiles = (tokens + ROWS - 1) / ROWS;
  const int64_t grid = ntiles < (int64_t)slots ? ntiles : (int64_t)slots;
  const float inv_sqrt_n = ROTATE ? (float)(1.0 / std::sqrt((double)(1 << LOGN))) : 1.0f;
  kern<<<(unsigned)grid, kThreads, kSmem, stream>>>(static_cast<const uint4 *>(x), tokens, clip,
                                                    inv_sqrt_n, signs, reinterpret_cast<uint32_t *>(q),
                                                    scales);
  return cudaGetLastError();
}

template <int BITS, int LOGN>
cudaError_t launch_n(const void *x, int64_t tokens, float clip, const uint32_t *signs, uint32_t flags,
                     uint8_t *q, float *scales, cudaStream_t stream) {
  constexpr int TB = LOGN <= 14 ? 14 : 15;
  if (flags & kNoRotate)
    return launch_one<BITS, TB, LOGN, false, false>(x, tokens, clip, nullptr, q, scales, stream);
  if (signs) return launch_one<BITS, TB, LOGN, true, true>(x, tokens, clip, signs, q, scales, stream);
  return launch_one<BITS, TB, LOGN, true, false>(x, tokens, clip, nullptr, q, scales, stream);
}

template <int BITS>
cudaError_t launch_bits(const void *x, int64_t tokens, int log_n, float clip, const uint32_t *signs,
                        uint32_t flags, uint8_t *q, float *scales, cudaStream_t stream) {
  switch (log_n) {
    case 7: return launch_n<BITS, 7>(x, tokens, clip, signs, flags, q, scales, stream);
    case 8: return launch_n<BITS, 8>(x, tokens, clip, signs, flags, q, scales, stream);
    case 9: return launch_n<BITS, 9>(x, tokens, clip, signs, flags, q, scales, stream);
    case 10: return launch_n<BITS, 10>(x, tokens, clip, signs, flags, q, scales, stream);
    case 11: return launch_n<BITS, 11>(x, tokens, clip, signs, flags, q, scales, stream);
    case 12: return launch_n<BITS, 12>(x, tokens, clip, signs, flags, q, scales, stream);
    case 13: return launch_n<BITS, 13>(x, tokens, clip, signs, flags, q, scales, stream);
    case 14: return launch_n<BITS, 14>(x, tokens, clip, signs, flags, q, scales, stream);
    case 15: return launch_n<BITS, 15>(x, tokens, clip, signs, flags, q, scales, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_rotate_quant(const void *x, int64_t tokens, int log_n, float clip, const uint32_t *signs,
                                uint32_t flags, int bits, uint8_t *q, float *scales, cudaStream_t stream) {
  if (bits != 4 && bits != 8) return cudaErrorInvalidValue;
  if (!(flags & kCudaCoresOnly) && tc_rotate_quant_supported(log_n, tokens, flags, signs != nullptr))
    return launch_rotate_quant_tc(log_n, bits, x, tokens, clip, signs, q, scales, stream);
  flags &= ~(kCudaCoresOnly | kTensorCores);
  return bits == 4 ? launch_bits<4>(x, tokens, log_n, clip, signs, flags, q, scales, stream)
                   : launch_bits<8>(x, tokens, log_n, clip, signs, flags, q, scales, stream);
}

}  // namespace spin
