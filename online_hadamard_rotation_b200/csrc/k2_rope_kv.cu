// k2_rope_kv.cu -- R3 and the INT4 KV cache on CUDA cores.
//
// "SpinQuant, when rotations are worth learning", section "Four rotation
// sites": R3 is a fixed Hadamard applied to queries and keys after RoPE, there
// to make the KV cache quantisable; section "Paper vs. code": the K cache path
// needs a power-of-two head dim, since R3 is the fast transform.
// "SpinQuant Guide: Learned Rotations for 4-Bit LLMs", section "RoPE
// Compatibility with 4-Bit KV Caching": RoPE rotates 2-D coordinate pairs and
// the KV cache is stored as 4-bit integers.
//
// Two neighbouring threads own one head vector (d = 128 values): thread h of
// the pair holds elements (p + 32 h, p + 32 h + 64) for p < 32, so RoPE's pair
// partners (p, p + 64) and six of the seven butterfly stages stay in its
// registers, and the stage over element bit 5 is one shuffle with the partner
// lane; the group min/max combine with one more. Head vectors reach shared memory through 16-byte
// cp.async copies that are coalesced in global memory; inside a 256-byte smem
// row the 16-byte chunk c sits at c ^ (row & 7), so eight threads reading
// chunk c of eight consecutive rows hit eight different bank groups. The
// copies for the next group of tokens are in flight while the current group
// is computed (two buffers).
//
// Q: out = bf16(H RoPE(q) / sqrt(d)), stored from registers (each thread writes
// four 16-byte pieces of its head row). K: H RoPE(k) / sqrt(d), V: v, each
// quantised asymmetrically per (token, kv head) group and written straight to
// its cache row (64 bytes) with fp16 scale and zero.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "spin_launch.h"
#include "spin_tile.cuh"

namespace spin {
namespace {

constexpr int kD = 128;          // head dim handled by this kernel
constexpr int kRowBytes = kD * 2;
constexpr float kInvSqrtDf = 0.0883883476f;         // 1/sqrt(128)
constexpr int kTabStride = kD / 2 + 2;               // float2 entries per token in the RoPE table
constexpr double kInv2Pi = 0.15915494309189535;     // 1 / (2 pi)
constexpr double k2PiHi = 6.283185307179586;        // 2 pi rounded to double
constexpr double k2PiLo = 2.4492935982947064e-16;   // 2 pi - k2PiHi

__device__ __forceinline__ float fma_sat(float a, float b, float c) {
  float r;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// byte offset of 16-byte chunk c of smem row r
__device__ __forceinline__ uint32_t chunk_off(uint32_t r, uint32_t c) {
  return r * kRowBytes + ((c ^ (r & 7u)) << 4);
}

constexpr int kHalf = 64;  // values per thread

// H_128 on a head vector split over a lane pair. Register j of half h holds
// element (j & 31) + 32 h + 64 (j >> 5): register bits 0-4 are element bits
// 0-4, register bit 5 is element bit 6, and element bit 5 is the lane pair.
__device__ __forceinline__ void fwht128_pair(float (&x)[kHalf], uint32_t h, unsigned pair_mask) {
#pragma unroll
  for (int i = 0; i < kHalf; i += 2) {
    const float a = x[i], b = x[i + 1];
    x[i] = a + b;
    x[i + 1] = a - b;
  }
#pragma unroll
  for (int st = 2; st < kHalf; st <<= 1) {
#pragma unroll
    for (int i = 0; i < kHalf; i += 2) {
      if (i & st) continue;
      bfly2(x[i], x[i + 1], x[i + st], x[i + st + 1]);
    }
  }
  // element bit 5: (a, b) -> (a + b, a - b) with a on half 0 and b on half 1
  const float sgn = h ? -1.0f : 1.0f;
#pragma unroll
  for (int i = 0; i < kHalf; ++i) {
    const float w = __shfl_xor_sync(pair_mask, x[i], 1);
    x[i] = fmaf(x[i], sgn, w);
  }
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// (r0, r1) = bit patterns of fma(a, 15, 1.5 * 2^23) for a pair: one packed FMA rounds two
// scaled codes to integers (ties to even) in their low mantissa bits.
__device__ __forceinline__ void round15_x2(float a0, float a1, uint32_t &r0, uint32_t &r1) {
  uint64_t A, R;
  asm("mov.b64 %0, {%1, %2};" : "=l"(A) : "f"(a0), "f"(a1));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(R) : "l"(A), "l"(0x4170000041700000ull), "l"(0x4B4000004B400000ull));
  asm("mov.b64 {%0, %1}, %2;" : "=r"(r0), "=r"(r1) : "l"(R));
}

// Asymmetric INT4 of one group of 128 values held by a lane pair (64 each, in
// the split of fwht128_pair); each thread writes its 32 code bytes, half 0 the
// fp16 scale and zero.
__device__ __forceinline__ void quant_asym_store_pair(const float (&x)[kHalf], float clip, uint32_t h,
                                                      unsigned pair_mask, uint8_t *codes_row, __half *scale_dst,
                                                      __half *zero_dst) {
  float mn[4], mx[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    mn[k] = fmin3(x[16 * k], x[16 * k + 1], x[16 * k + 2]);
    mx[k] = fmax3(x[16 * k], x[16 * k + 1], x[16 * k + 2]);
#pragma unroll
    for (int j = 3; j < 15; j += 2) {
      mn[k] = fmin3(mn[k], x[16 * k + j], x[16 * k + j + 1]);
      mx[k] = fmax3(mx[k], x[16 * k + j], x[16 * k + j + 1]);
    }
    mn[k] = fminf(mn[k], x[16 * k + 15]);
    mx[k] = fmaxf(mx[k], x[16 * k + 15]);
  }
  float vmn = fminf(fminf(mn[0], mn[1]), fminf(mn[2], mn[3]));
  float vmx = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
  vmn = fminf(vmn, __shfl_xor_sync(pair_mask, vmn, 1));
  vmx = fmaxf(vmx, __shfl_xor_sync(pair_mask, vmx, 1));
  const float lo = fminf(clip * vmn, 0.f), hi = fmaxf(clip * vmx, 0.f);
  __half s16 = __float2half_rn((hi - lo) / 15.0f);
  float s = __half2float(s16), z = 0.f;
  if (s == 0.f) {
    s16 = __float2half_rn(1.0f);
    s = 1.0f;
  } else {
    z = fminf(fmaxf(rintf(-lo / s), 0.f), 15.f);
  }
  const float c15 = (1.0f / s) / 15.0f, z15 = z / 15.0f;
#pragma unroll
  for (int q = 0; q < 2; ++q) {  // registers 32 q .. 32 q + 31 -> code bytes 32 q + 16 h .. + 15
    uint32_t words[4];
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
      const int w = 4 * q + wi;
      uint32_t b[8];
      float t[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) t[i] = fma_sat(x[8 * w + i], c15, z15);
#pragma unroll
      for (int i = 0; i < 8; i += 2) round15_x2(t[i], t[i + 1], b[i], b[i + 1]);
      const uint32_t e = __byte_perm(__byte_perm(b[0], b[2], 0x0040), __byte_perm(b[4], b[6], 0x0040), 0x5410);
      const uint32_t o = __byte_perm(__byte_perm(b[1], b[3], 0x0040), __byte_perm(b[5], b[7], 0x0040), 0x5410);
      words[wi] = e | (o << 4);
    }
    __stcs(reinterpret_cast<uint4 *>(codes_row + 32 * q + 16 * h), make_uint4(words[0], words[1], words[2], words[3]));
  }
  if (h == 0) {
    *scale_dst = s16;
    *zero_dst = __float2half_rn(z);
  }
}

struct K2Args {
  const uint16_t *q, *k, *v;
  const int32_t *pos;
  uint16_t *q_out;
  uint8_t *k_cache, *v_cache;
  __half *k_scale, *k_zero, *v_scale, *v_zero;
  int64_t ntok;  // batch * seq
  int seq, hq, hkv, tok_per_group, cache_len, cache_offset;
  float clip, inv_sqrt_d;
  double theta;
};

__global__ void __launch_bounds__(192, 3) k2_rope_hadamard_kvquant(K2Args a) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int rows_tok = a.hq + 2 * a.hkv;
  const int G = a.tok_per_group;
  const int rows = G * rows_tok;
  uint8_t *stage[2] = {smem, smem + (size_t)rows * kRowBytes};
  float2 *table[2];
  table[0] = reinterpret_cast<float2 *>(smem + 2 * (size_t)rows * kRowBytes);
  table[1] = table[0] + G * kTabStride;
  double *inv_freq = reinterpret_cast<double *>(table[1] + G * kTabStride);

  const int t = threadIdx.x, nt = blockDim.x;
  const int64_t ngroups = (a.ntok + G - 1) / G;

  for (int p = t; p < kD / 2; p += nt) inv_freq[p] = pow(a.theta, -2.0 * p / (double)kD);
  __syncthreads();

  // Issue the copies of group g into buffer b and fill its RoPE table.
  auto prefetch = [&](int64_t g, int b) {
    const int64_t tok0 = g * G;
    const int ntk = (int)((a.ntok - tok0) < G ? (a.ntok - tok0) : G);
    // Q rows [0, ntk*hq), then K rows, then V rows (token-major inside each)
    const int nq = ntk * a.hq, nk = ntk * a.hkv;
    const int chunks = (nq + 2 * nk) * (kRowBytes / 16);
    for (int i = t; i < chunks; i += nt) {
      const int r = i >> 4, c = i & 15;
      const uint16_t *src;
      int sr;
      if (r < nq) {
        src = a.q + (tok0 * a.hq + r) * kD;
        sr = r;
      } else if (r < nq + nk) {
        src = a.k + (tok0 * a.hkv + (r - nq)) * kD;
        sr = G * a.hq + (r - nq);
      } else {
        src = a.v + (tok0 * a.hkv + (r - nq - nk)) * kD;
        sr = G * (a.hq + a.hkv) + (r - nq - nk);
      }
      cp_async16(stage[b] + chunk_off(sr, c), src + c * 8);
    }
    cp_async_commit();
    for (int i = t; i < ntk * (kD / 2); i += nt) {
      const int tk = i / (kD / 2), p = i % (kD / 2);
      // angle pos * theta^(-2p/d) in fp64, reduced to [-pi, pi] by Cody-Waite
      // (2 pi split into a head and a tail, each multiple subtracted with an FMA),
      // then the fp32 sine and cosine of the reduced angle
      const double ang = (double)a.pos[tok0 + tk] * inv_freq[p];
      const double k = rint(ang * kInv2Pi);
      const double red = fma(-k, k2PiLo, fma(-k, k2PiHi, ang));
      float sn, cs;
      sincosf((float)red, &sn, &cs);
      // 1/sqrt(d) of the rotation is folded into the angle's cosine and sine. Layout
      // [token][j][half] (p = 32 half + j) with a padded token stride, so the two
      // threads of a pair and neighbouring tokens read different banks.
      table[b][tk * kTabStride + 2 * (p & 31) + (p >> 5)] = make_float2(cs * kInvSqrtDf, sn * kInvSqrtDf);
    }
  };

  int64_t g = blockIdx.x;
  int buf = 0;
  if (g < ngroups) prefetch(g, 0);
  for (; g < ngroups; g += gridDim.x, buf ^= 1) {
    __syncthreads();  // every thread is done with the buffer the next copies overwrite
    const int64_t gn = g + gridDim.x;
    if (gn < ngroups) prefetch(gn, buf ^ 1);
    else cp_async_commit();  // keep the group count uniform
    cp_async_wait_1();
    __syncthreads();

    const int64_t tok0 = g * G;
    const int ntk = (int)((a.ntok - tok0) < G ? (a.ntok - tok0) : G);
    uint8_t *sb = stage[buf];
    const float2 *tb = table[buf];

    for (int rh = t; rh < 2 * rows; rh += nt) {
      const int r = rh >> 1;
      const uint32_t hf = (uint32_t)rh & 1u;               // which half of the head vector
      const unsigned pm = 3u << ((threadIdx.x & 31u) & ~1u);  // this lane pair
      int kind, tk, h;
      if (r < G * a.hq) {
        kind = 0; tk = r / a.hq; h = r % a.hq;
      } else if (r < G * (a.hq + a.hkv)) {
        // row order (head, token) so neighbouring rows write neighbouring cache slots
        const int i = r - G * a.hq;
        kind = 1; h = i / G; tk = i % G;
      } else {
        const int i = r - G * (a.hq + a.hkv);
        kind = 2; h = i / G; tk = i % G;
      }
      if (tk >= ntk) continue;
      const int sr = kind == 0 ? tk * a.hq + h : G * a.hq + (kind == 2 ? G * a.hkv : 0) + tk * a.hkv + h;
      float x[kHalf];
#pragma unroll
      for (int c = 0; c < 8; ++c) {  // chunks 4 hf .. 4 hf + 3 and 8 + 4 hf .. 8 + 4 hf + 3
        const uint32_t chunk = (c & 3u) + 4u * hf + 8u * (c >> 2);
        const uint4 w = *reinterpret_cast<const uint4 *>(sb + chunk_off(sr, chunk));
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          x[8 * c + 2 * k] = bf16lo(ww[k]);
          x[8 * c + 2 * k + 1] = bf16hi(ww[k]);
        }
      }
      const int64_t tok = tok0 + tk;
      if (kind != 2) {
        const float2 *cs = tb + tk * kTabStride + hf;
#pragma unroll
        for (int j = 0; j < 32; ++j) {  // pair (p, p + 64) with p = 32 hf + j
          const float2 e = cs[2 * j];
          const float x0 = x[j], x1 = x[j + 32];
          x[j] = fmaf(x0, e.x, -x1 * e.y);
          x[j + 32] = fmaf(x1, e.x, x0 * e.y);
        }
        fwht128_pair(x, hf, pm);
      }
      if (kind == 0) {
        // rotated Q straight to global memory: registers 0-31 are bytes 64 hf .. 64 hf + 63
        // of the head row, registers 32-63 bytes 128 + 64 hf .. 128 + 64 hf + 63
        uint4 *qrow = reinterpret_cast<uint4 *>(a.q_out + (tok * a.hq + h) * kD);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t chunk = (c & 3u) + 4u * hf + 8u * (c >> 2);
          __stcs(qrow + chunk, make_uint4(pack_bf16x2(x[8 * c], x[8 * c + 1]), pack_bf16x2(x[8 * c + 2], x[8 * c + 3]),
                                          pack_bf16x2(x[8 * c + 4], x[8 * c + 5]),
                                          pack_bf16x2(x[8 * c + 6], x[8 * c + 7])));
        }
      } else {
        const int64_t b = tok / a.seq, s = tok % a.seq;
        const int64_t crow = (b * a.hkv + h) * (int64_t)a.cache_len + a.cache_offset + s;
        if (kind == 1)
          quant_asym_store_pair(x, a.clip, hf, pm, a.k_cache + crow * (kD / 2), a.k_scale + crow, a.k_zero + crow);
        else
          quant_asym_store_pair(x, a.clip, hf, pm, a.v_cache + crow * (kD / 2), a.v_scale + crow, a.v_zero + crow);
      }
    }
  }
  cp_async_wait_1();
  asm volatile("cp.async.wait_all;" ::: "memory");
}

}  // namespace

cudaError_t launch_rope_hadamard_kvquant(const void *q, const void *k, const void *v,
                                         const int32_t *pos, float theta, int batch, int seq,
                                         int n_q_heads, int n_kv_heads, float clip, void *q_out,
                                         uint8_t *k_cache, uint8_t *v_cache, void *k_scale,
                                         void *k_zero, void *v_scale, void *v_zero, int cache_len,
                                         int cache_offset, cudaStream_t stream) {
  const int rows_tok = n_q_heads + 2 * n_kv_heads;
  int G = 1;
  while (G < 8 && 2 * G * rows_tok <= 96) G *= 2;  // tokens per group: at most 96 head vectors
  const int rows = G * rows_tok;
  int threads = 2 * rows < 192 ? ((2 * rows + 31) / 32) * 32 : 192;  // two threads per head vector
  const size_t smem = 2 * (size_t)rows * kRowBytes + 2 * (size_t)G * kTabStride * sizeof(float2) +
                      (kD / 2) * sizeof(double);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  int slots = 0;
  cudaError_t err =
      resident_slots(reinterpret_cast<const void *>(k2_rope_hadamard_kvquant), threads, (int)smem, &slots);
  if (err != cudaSuccess) return err;
  K2Args a;
  a.q = static_cast<const uint16_t *>(q);
  a.k = static_cast<const uint16_t *>(k);
  a.v = static_cast<const uint16_t *>(v);
  a.pos = pos;
  a.q_out = static_cast<uint16_t *>(q_out);
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.k_scale = static_cast<__half *>(k_scale);
  a.k_zero = static_cast<__half *>(k_zero);
  a.v_scale = static_cast<__half *>(v_scale);
  a.v_zero = static_cast<__half *>(v_zero);
  a.ntok = (int64_t)batch * seq;
  a.seq = seq;
  a.hq = n_q_heads;
  a.hkv = n_kv_heads;
  a.tok_per_group = G;
  a.cache_len = cache_len;
  a.cache_offset = cache_offset;
  a.clip = clip;
  a.inv_sqrt_d = (float)(1.0 / std::sqrt((double)kD));
  a.theta = (double)theta;
  const int64_t ngroups = (a.ntok + G - 1) / G;
  const int64_t grid = ngroups < slots ? ngroups : slots;
  k2_rope_hadamard_kvquant<<<(unsigned)grid, threads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace spin
