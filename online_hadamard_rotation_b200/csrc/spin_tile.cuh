// spin_tile.cuh -- register-resident fast Walsh-Hadamard transform over
// tiles of 2^14 (or 2^15) elements, for sm_100a.
//
// The transform is the Sylvester-order H_n ("Rotations: QuaRot, SpinQuant and
// incoherence", section "Hadamard matrices"). It factors over the bits of the
// element index: H_n = product over index bits b of (butterfly on bit b),
// and these factors commute, so the stages may run in any order and any
// grouping ("Hadamard matrices": Kronecker products of smaller Hadamards).
//
// A tile holds 2^TB consecutive elements of the input (one row for n >= 2^14,
// 2^(14-log n) whole rows for smaller n). Each thread owns 128 of them in
// registers, so a tile is 128 threads (TB = 14) or 256 threads (TB = 15).
// Three register layouts are used; each maps (thread, register) to the
// element index E inside the tile:
//   L1  E = t << 3 | (r & 7) | (r >> 3) << (TB - 4)        global loads/stores
//   L2  E = (t & 7) | (t >> 3) << 10 | r << 3               after the transpose
//   L3  (TB = 15 only) E = (t & 127) << 3 | (t >> 7) << 14 | (r & 7) | (r >> 3) << 10
// In L1 every warp touches 512 contiguous bytes per 16-byte access; the
// butterflies whose index bit lives in the register index run in registers;
// one pass through shared memory (fp32, 64 KiB or 128 KiB) moves to L2 and
// a second one moves to the output layout, whose 8 consecutive elements per
// register octet are what the packers and the stores need.
//
// The shared-memory word address of element E is XOR-swizzled so that both
// the 16-byte accesses of L1/L3 and the 4-byte accesses of L2 are free of
// bank conflicts:
//   A(E) = E[1:0] | (E2^E3) << 2 | (E10^E4) << 3 | (E11^E5) << 4 | E[9:3] << 5 | E[..:12] << 12
#pragma once

#include <cstdint>

namespace spin {

constexpr int kRegs = 128;  // elements per thread

__host__ __device__ constexpr uint32_t swz(uint32_t E) {
  return (E & 3u) | ((((E >> 2) ^ (E >> 3)) & 1u) << 2) | ((((E >> 10) ^ (E >> 4)) & 1u) << 3) |
         ((((E >> 11) ^ (E >> 5)) & 1u) << 4) | (((E >> 3) & 127u) << 5) | ((E >> 12) << 12);
}

// ---------------------------------------------------------------- layouts
template <int TB>
struct L1 {
  static constexpr int kHi = TB - 4;  // register bits 3..6 -> E bits kHi..kHi+3
  __device__ static uint32_t thr(uint32_t t) { return t << 3; }
  __host__ __device__ static constexpr uint32_t reg(int r) {
    return (uint32_t)(r & 7) | ((uint32_t)(r >> 3) << kHi);
  }
};
struct L2 {
  __device__ static uint32_t thr(uint32_t t) { return (t & 7u) | ((t >> 3) << 10); }
  __host__ __device__ static constexpr uint32_t reg(int r) { return (uint32_t)r << 3; }
};
struct L3 {  // TB = 15 output layout
  static constexpr int kHi = 10;
  __device__ static uint32_t thr(uint32_t t) { return ((t & 127u) << 3) | ((t >> 7) << 14); }
  __host__ __device__ static constexpr uint32_t reg(int r) {
    return (uint32_t)(r & 7) | ((uint32_t)(r >> 3) << 10);
  }
};

// The output layout of a tile: L1 for TB = 14, L3 for TB = 15.
template <int TB>
struct OutLayout;
template <>
struct OutLayout<14> : L1<14> {};
template <>
struct OutLayout<15> : L3 {};

// ---------------------------------------------------------------- butterflies
// Two butterflies (a0, b0) and (a1, b1) with one packed f32x2 add and sub.
__device__ __forceinline__ void bfly2(float &a0, float &a1, float &b0, float &b1) {
  uint64_t A, B, S, D;
  asm("mov.b64 %0, {%1, %2};" : "=l"(A) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(B) : "f"(b0), "f"(b1));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(S) : "l"(A), "l"(B));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(D) : "l"(A), "l"(B));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(S));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(b0), "=f"(b1) : "l"(D));
}

// Butterfly stage over register-index bit P: (v[i], v[i | 2^P]) -> (sum, difference).
template <int P>
__device__ __forceinline__ void stage(float (&v)[kRegs]) {
  if constexpr (P == 0) {
#pragma unroll
    for (int i = 0; i < kRegs; i += 2) {
      float a = v[i], b = v[i + 1];
      v[i] = a + b;
      v[i + 1] = a - b;
    }
  } else {
#pragma unroll
    for (int i = 0; i < kRegs; i += 2) {
      if ((i >> P) & 1) continue;
      bfly2(v[i], v[i + 1], v[i + (1 << P)], v[i + 1 + (1 << P)]);
    }
  }
}

// Run the stage for register bit P iff the element-index bit it carries is
// below LOGN (i.e. it is a bit of the position inside a row, not a row bit).
template <int P, int EBIT, int LOGN>
__device__ __forceinline__ void stage_if(float (&v)[kRegs]) {
  if constexpr (EBIT < LOGN) stage<P>(v);
}

// ---------------------------------------------------------------- transposes
// Store registers of layout LA and load them back in layout LB through the
// swizzled fp32 buffer `sm`. The caller places the barrier between the two.
template <class LA>
__device__ __forceinline__ void store_v4(const float (&v)[kRegs], float *sm, uint32_t t) {
  const uint32_t a0 = swz(LA::thr(t));
#pragma unroll
  for (int r = 0; r < kRegs; r += 4) {
    const uint32_t c = swz(LA::reg(r));
    const uint32_t addr = (a0 ^ (c & 0x1Cu)) + (c & ~0x1Cu);
    *reinterpret_cast<float4 *>(sm + addr) = make_float4(v[r], v[r + 1], v[r + 2], v[r + 3]);
  }
}

template <class LA>
__device__ __forceinline__ void load_v4(float (&v)[kRegs], const float *sm, uint32_t t) {
  const uint32_t a0 = swz(LA::thr(t));
#pragma unroll
  for (int r = 0; r < kRegs; r += 4) {
    const uint32_t c = swz(LA::reg(r));
    const uint32_t addr = (a0 ^ (c & 0x1Cu)) + (c & ~0x1Cu);
    const float4 f = *reinterpret_cast<const float4 *>(sm + addr);
    v[r] = f.x;
    v[r + 1] = f.y;
    v[r + 2] = f.z;
    v[r + 3] = f.w;
  }
}

__device__ __forceinline__ void store_l2(const float (&v)[kRegs], float *sm, uint32_t t) {
  const uint32_t a0 = swz(L2::thr(t));
#pragma unroll
  for (int r = 0; r < kRegs; ++r) {
    const uint32_t c = swz(L2::reg(r));
    sm[(a0 ^ (c & 0x1Cu)) + (c & ~0x1Cu)] = v[r];
  }
}

__device__ __forceinline__ void load_l2(float (&v)[kRegs], const float *sm, uint32_t t) {
  const uint32_t a0 = swz(L2::thr(t));
#pragma unroll
  for (int r = 0; r < kRegs; ++r) {
    const uint32_t c = swz(L2::reg(r));
    v[r] = sm[(a0 ^ (c & 0x1Cu)) + (c & ~0x1Cu)];
  }
}

// ---------------------------------------------------------------- the transform
// Input: v in layout L1<TB>. Output: v in OutLayout<TB> holding the
// unnormalised Walsh-Hadamard transform of every row of the tile (rows of
// 2^LOGN elements). `sm` is the tile's fp32 shared buffer (2^TB floats).
// Contains __syncthreads(); every thread of the block must call it.
template <int TB, int LOGN>
__device__ __forceinline__ void tile_fwht(float (&v)[kRegs], float *sm, uint32_t t) {
  static_assert(TB == 14 || TB == 15, "tile bits");
  static_assert(LOGN >= 7 && LOGN <= TB, "row size");
  constexpr int H = L1<TB>::kHi;
  // round 1 (L1): element bits 0, 1, 2 and H..H+3
  stage_if<0, 0, LOGN>(v);
  stage_if<1, 1, LOGN>(v);
  stage_if<2, 2, LOGN>(v);
  stage_if<3, H + 0, LOGN>(v);
  stage_if<4, H + 1, LOGN>(v);
  stage_if<5, H + 2, LOGN>(v);
  stage_if<6, H + 3, LOGN>(v);
  __syncthreads();  // the previous user of `sm` is done
  store_v4<L1<TB>>(v, sm, t);
  __syncthreads();
  load_l2(v, sm, t);
  // round 2 (L2): element bits 3..9
  stage_if<0, 3, LOGN>(v);
  stage_if<1, 4, LOGN>(v);
  stage_if<2, 5, LOGN>(v);
  stage_if<3, 6, LOGN>(v);
  stage_if<4, 7, LOGN>(v);
  stage_if<5, 8, LOGN>(v);
  stage_if<6, 9, LOGN>(v);
  __syncthreads();
  store_l2(v, sm, t);
  __syncthreads();
  load_v4<OutLayout<TB>>(v, sm, t);
  if constexpr (TB == 15) stage_if<3, 10, LOGN>(v);  // element bit 10 lives at L3 register bit 3
}

// ---------------------------------------------------------------- conversions
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

}  // namespace spin
