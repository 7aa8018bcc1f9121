// k2_rope_kv.cu -- R3 and the INT4 KV cache on CUDA cores, fed by TMA.
//
// "SpinQuant, when rotations are worth learning", section "Four rotation
// sites": R3 is a fixed Hadamard applied to queries and keys after RoPE, there
// to make the KV cache quantisable; section "Paper vs. code": the K cache path
// needs a power-of-two head dim, since R3 is the fast transform.
// "SpinQuant Guide: Learned Rotations for 4-Bit LLMs", section "RoPE
// Compatibility with 4-Bit KV Caching": RoPE rotates 2-D coordinate pairs and
// the KV cache is stored as 4-bit integers.
//
// Q: out = bf16(H RoPE(q) / sqrt(d)). K: H RoPE(k) / sqrt(d), V: v, each
// quantised asymmetrically per (token, kv head) group and written to its cache
// row (64 code bytes) with fp16 scale and zero.
//
// Work unit: a group of G consecutive tokens (G <= 8, at most 96 head vectors).
// A persistent CTA walks groups blockIdx.x, + gridDim.x, ... through two
// shared-memory buffers:
//   * A buffer holds the group's Q, K and V rows as two tiles (head elements
//     0-63 and 64-127), 128 bytes per row with the 128-byte swizzle (16-byte
//     chunk c of row r sits at c ^ (r & 7)), filled by six TMA box loads that
//     complete one mbarrier. Rows of tokens past the end read as zero.
//   * Two lanes own one head vector. Lane h of the pair holds, in register j,
//     element (j & 31) + 32 h + 64 (j >> 5): RoPE's partners (p, p + 64) and the
//     butterflies over element bits 0-4 and 6 stay in its registers, and the
//     butterfly over bit 5 is one shuffle with the partner lane.
//   * RoPE followed by the bit-6 butterfly is one 2 x 2 map per pair,
//     (a, b) -> (a (c + s) + b (c - s), a (c - s) - b (c + s)) with c, s the
//     cosine and sine of the pair's angle; the buffer's table holds
//     ((c + s) / sqrt(d), (c - s) / sqrt(d)) per token and pair, so 1/sqrt(d)
//     costs nothing either.
//   * Warps never meet at a block-wide barrier: a warp that is done with a
//     buffer adds one to its counter in shared memory, and the warp that
//     completes the count refills the buffer with the group two steps ahead
//     (TMA loads first, then the RoPE table and cache row bases, then its
//     arrival on the buffer's mbarrier).
//   * The group's head vectors form warp-sized chunks (Q rows, then K, then V,
//     token-major); warp w takes chunk (w - i) mod W at the CTA's i-th group, so
//     Q (RoPE + H), K (RoPE + H + INT4) and V (INT4) work rotates over warps.
// Every mbarrier wait is bounded by a clock budget; on expiry the CTA records a
// status (read by spin_device_status), stops issuing loads, drains the loads it
// issued and returns.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>

#include "spin_launch.h"
#include "spin_tile.cuh"
#include "tc_ptx.cuh"

namespace spin {

// Nonzero once an R3 launch gave up on a wait (see spin_device_status).
__device__ unsigned int g_rope_status = 0u;

namespace {

constexpr int kD = 128;                              // head dim handled by this kernel
constexpr int kMaxThreads = 128;
constexpr int kMaxGroupRows = 96;                    // head vectors per group (at most)
constexpr int kTabHalf = 34;                         // float2 entries per half table (32 + 2 pad)
constexpr int kTabTok = 72;                          // float2 entries per token (two halves + pad)
constexpr float kInvSqrtDf = 0.0883883476f;          // 1/sqrt(128)
constexpr double kInv2Pi = 0.15915494309189535;      // 1 / (2 pi)
constexpr double k2PiHi = 6.283185307179586;         // 2 pi rounded to double
constexpr double k2PiLo = 2.4492935982947064e-16;    // 2 pi - k2PiHi
constexpr long long kTimeoutCycles = 4000000000LL;   // about two seconds

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

// Eight consecutive values -> one word of unsigned INT4 codes, value k in nibble k:
// u = clamp(rne(v c + z), 0, 15) (c = 1 / step, z the integer zero point). One packed
// FMA forms v c + z, a packed multiply by 2^-149 (the smallest subnormal) rounds it to
// nearest even onto the subnormal grid, so the bit pattern is the integer (negative
// values keep the sign bit), and cvt.pack.sat clamps two of them to [0, 15] and packs
// them (second operand in the low nibble).
__device__ __forceinline__ uint32_t codes8_asym(const float *v, uint64_t c2, uint64_t z2) {
  uint32_t r[8], d = 0u;
#pragma unroll
  for (int k = 0; k < 8; k += 2) {
    uint64_t A, T, R;
    asm("mov.b64 %0, {%1, %2};" : "=l"(A) : "f"(v[k]), "f"(v[k + 1]));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(T) : "l"(A), "l"(c2), "l"(z2));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(R) : "l"(T), "l"(0x0000000100000001ull));
    asm("mov.b64 {%0, %1}, %2;" : "=r"(r[k]), "=r"(r[k + 1]) : "l"(R));
  }
#pragma unroll
  for (int k = 6; k >= 0; k -= 2)  // d = (d << 8) | sat(r[k + 1]) << 4 | sat(r[k])
    asm("cvt.pack.sat.u4.s32.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(r[k + 1]), "r"(r[k]), "r"(d));
  return d;
}

__device__ __forceinline__ uint64_t pair(float x) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ void fma_pair(float &a0, float &a1, float s, float w0, float w1) {
  uint64_t A, S, Wv, R;
  asm("mov.b64 %0, {%1, %2};" : "=l"(A) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %1};" : "=l"(S) : "f"(s));
  asm("mov.b64 %0, {%1, %2};" : "=l"(Wv) : "f"(w0), "f"(w1));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(R) : "l"(A), "l"(S), "l"(Wv));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(R));
}

__device__ __forceinline__ void st_v8_cs(void *p, const uint32_t *w) {
  asm volatile("st.global.cs.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]), "r"(w[1]),
               "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

__device__ __forceinline__ void unpack8(const uint4 w, float *x) {
  x[0] = bf16lo(w.x);
  x[1] = bf16hi(w.x);
  x[2] = bf16lo(w.y);
  x[3] = bf16hi(w.y);
  x[4] = bf16lo(w.z);
  x[5] = bf16hi(w.z);
  x[6] = bf16lo(w.w);
  x[7] = bf16hi(w.w);
}

// Butterflies over element bits 0-4 (register bits 0-4), two pairs per packed op:
// registers j and j + 32 travel together.
__device__ __forceinline__ void fwht_low5(float (&x)[64]) {
#pragma unroll
  for (int st = 1; st < 32; st <<= 1) {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if (j & st) continue;
      bfly2(x[j], x[j + 32], x[j + st], x[j + st + 32]);
    }
  }
}

// Butterfly over element bit 5, which is the lane within the pair: lane 0 keeps
// a + b, lane 1 keeps a - b (a on lane 0, b on lane 1).
__device__ __forceinline__ void fwht_pair_bit(float (&x)[64], uint32_t h, unsigned pair_mask) {
  const float sgn = h ? -1.0f : 1.0f;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float w0 = __shfl_xor_sync(pair_mask, x[j], 1);
    const float w1 = __shfl_xor_sync(pair_mask, x[j + 32], 1);
    fma_pair(x[j], x[j + 32], sgn, w0, w1);
  }
}

struct K2Args {
  uint16_t *q_out;
  uint8_t *k_cache, *v_cache;
  __half *k_scale, *k_zero, *v_scale, *v_zero;
  const int32_t *pos;
  int ntok;  // batch * seq
  int seq, hq, hkv, G, cache_len, cache_offset;
  int rq, rk;    // tile rows of the Q region and of the K (= V) region, multiples of 8
  int nslots;    // 2 * G * (hq + 2 hkv): one per half head vector
  int q32;       // q_out is 32-byte aligned
  float clip;
  double theta;
};

// Shared-memory carve-up (offsets from a 1024-byte aligned base).
struct K2Layout {
  uint32_t tile_bytes, buf_bytes, off_tab, off_cbase, off_freq, off_desc, off_bar, total;
};
__host__ __device__ __forceinline__ K2Layout k2_layout(int G, int rq, int rk, int nslots) {
  K2Layout L;
  L.tile_bytes = (uint32_t)(rq + 2 * rk) * 128u;
  L.buf_bytes = 2u * L.tile_bytes;
  L.off_tab = 2u * L.buf_bytes;
  L.off_cbase = L.off_tab + 2u * (uint32_t)G * kTabTok * 8u;
  L.off_freq = L.off_cbase + 2u * (uint32_t)G * 8u;
  L.off_desc = L.off_freq + (kD / 2) * 8u;
  L.off_bar = (L.off_desc + (uint32_t)nslots * 4u + 15u) & ~15u;
  L.total = L.off_bar + 64u;
  return L;
}

// Slot descriptor: tile row (10 bits), head (9), token in group (3), kind (2), half (1).
__device__ __forceinline__ uint32_t make_desc(const K2Args &a, int s) {
  const int r = s >> 1, hf = s & 1, G = a.G;
  int kind, tk, h, srow;
  if (r < G * a.hq) {
    kind = 0; tk = r / a.hq; h = r - tk * a.hq; srow = r;
  } else if (r < G * (a.hq + a.hkv)) {
    const int i = r - G * a.hq;
    kind = 1; tk = i / a.hkv; h = i - tk * a.hkv; srow = a.rq + i;
  } else {
    const int i = r - G * (a.hq + a.hkv);
    kind = 2; tk = i / a.hkv; h = i - tk * a.hkv; srow = a.rq + a.rk + i;
  }
  return (uint32_t)srow | ((uint32_t)h << 10) | ((uint32_t)tk << 19) | ((uint32_t)kind << 22) | ((uint32_t)hf << 24);
}

struct K2Shared {
  uint8_t *base;
  float2 *tab;      // [2][G][kTabTok]
  int64_t *cbase;   // [2][G]
  double *inv_freq; // [64]
  uint64_t *full;   // [2]
  uint32_t *cnt;    // [2] warps done with the buffer
  uint32_t *issued; // [2] loads issued into the buffer
  volatile uint32_t *abort_flag;
};

// Refill buffer b with group g (executed by one whole warp).
__device__ __forceinline__ void load_group(const K2Args &a, const K2Shared &S, const K2Layout &L,
                                           const CUtensorMap *mq, const CUtensorMap *mk, const CUtensorMap *mv,
                                           int64_t g, int b, int lane) {
  const int G = a.G;
  const int tok0 = (int)(g * G);
  const int ntk = min(G, a.ntok - tok0);
  uint64_t *bar = &S.full[b];
  if (lane == 0) {
    const uint32_t bytes = (uint32_t)(2 * 128 * G * (a.hq + 2 * a.hkv));
    tc::mbar_expect_tx(bar, bytes);
    tc::fence_proxy_async_smem();  // earlier generic accesses to the buffer come before the copies
    uint8_t *tl = S.base + (uint32_t)b * L.buf_bytes;
    uint8_t *tr = tl + L.tile_bytes;
    tc::tma_load_2d(tl, mq, bar, 0, tok0 * a.hq);
    tc::tma_load_2d(tr, mq, bar, 64, tok0 * a.hq);
    tc::tma_load_2d(tl + a.rq * 128, mk, bar, 0, tok0 * a.hkv);
    tc::tma_load_2d(tr + a.rq * 128, mk, bar, 64, tok0 * a.hkv);
    tc::tma_load_2d(tl + (a.rq + a.rk) * 128, mv, bar, 0, tok0 * a.hkv);
    tc::tma_load_2d(tr + (a.rq + a.rk) * 128, mv, bar, 64, tok0 * a.hkv);
    S.issued[b] += 1u;
  }
  float2 *tb = S.tab + b * G * kTabTok;
  for (int i = lane; i < ntk * (kD / 2); i += 32) {
    const int tk = i >> 6, p = i & 63;
    // angle pos * theta^(-2p/d) in fp64, reduced to [-pi, pi] by Cody-Waite
    // (2 pi split into a head and a tail, each multiple subtracted with an FMA),
    // then the fp32 sine and cosine of the reduced angle
    const double ang = (double)a.pos[tok0 + tk] * S.inv_freq[p];
    const double k = rint(ang * kInv2Pi);
    const double red = fma(-k, k2PiLo, fma(-k, k2PiHi, ang));
    float sn, cs;
    sincosf((float)red, &sn, &cs);
    tb[tk * kTabTok + (p >> 5) * kTabHalf + (p & 31)] = make_float2((cs + sn) * kInvSqrtDf, (cs - sn) * kInvSqrtDf);
  }
  if (lane < ntk) {
    const int tok = tok0 + lane;
    const int bb = tok / a.seq, s = tok - bb * a.seq;
    S.cbase[b * G + lane] = (int64_t)bb * a.hkv * a.cache_len + a.cache_offset + s;
  }
  __syncwarp();
  if (lane == 0) tc::mbar_arrive(bar);  // publishes the table with the loaded rows
}

// Asymmetric INT4 of one group of 128 values held by a lane pair (64 each, register j
// = element (j & 31) + 32 h + 64 (j >> 5)); the thread writes its 32 code bytes
// (16 at byte 16 h, 16 at byte 32 + 16 h), lane 0 of the pair the scale, lane 1 the zero.
__device__ __forceinline__ void quant_asym_store(const float (&x)[64], float clip, uint32_t h, unsigned pair_mask,
                                                 uint8_t *codes_row, __half *scale_dst, __half *zero_dst) {
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
  const uint64_t c2 = pair(1.0f / s), z2 = pair(z);
  uint32_t words[2][4];
#pragma unroll
  for (int wi = 0; wi < 4; ++wi) {  // registers 8 wi .. 8 wi + 7 and 32 + 8 wi .. 32 + 8 wi + 7
    words[0][wi] = codes8_asym(x + 8 * wi, c2, z2);
    words[1][wi] = codes8_asym(x + 32 + 8 * wi, c2, z2);
  }
  // registers 32 q .. 32 q + 31 -> code bytes 32 q + 16 h .. + 15
  __stcs(reinterpret_cast<uint4 *>(codes_row + 16 * h), make_uint4(words[0][0], words[0][1], words[0][2], words[0][3]));
  __stcs(reinterpret_cast<uint4 *>(codes_row + 32 + 16 * h),
         make_uint4(words[1][0], words[1][1], words[1][2], words[1][3]));
  if (h == 0) *scale_dst = s16;
  else *zero_dst = __float2half_rn(z);
}

__device__ __forceinline__ bool wait_full(uint64_t *bar, uint32_t parity, volatile uint32_t *abort_flag) {
  if (tc::mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!tc::mbar_try_wait(bar, parity)) {
    if (*abort_flag || clock64() - t0 > kTimeoutCycles) return false;
  }
  return true;
}

__global__ void __launch_bounds__(kMaxThreads, 4)
    k2_rope_hadamard_kvquant(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                             const __grid_constant__ CUtensorMap mv, const K2Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  const K2Layout L = k2_layout(a.G, a.rq, a.rk, a.nslots);
  K2Shared S;
  S.base = sm;
  S.tab = reinterpret_cast<float2 *>(sm + L.off_tab);
  S.cbase = reinterpret_cast<int64_t *>(sm + L.off_cbase);
  S.inv_freq = reinterpret_cast<double *>(sm + L.off_freq);
  uint32_t *desc = reinterpret_cast<uint32_t *>(sm + L.off_desc);
  S.full = reinterpret_cast<uint64_t *>(sm + L.off_bar);
  S.cnt = reinterpret_cast<uint32_t *>(sm + L.off_bar + 16);
  S.issued = S.cnt + 2;
  S.abort_flag = S.cnt + 4;

  const int t = threadIdx.x, lane = t & 31, warp = t >> 5, W = blockDim.x >> 5;
  const int G = a.G;
  const int64_t ngroups = ((int64_t)a.ntok + G - 1) / G;
  const int64_t grid = gridDim.x;

  if (t == 0) {
    tc::mbar_init(&S.full[0], 1);
    tc::mbar_init(&S.full[1], 1);
    S.cnt[0] = S.cnt[1] = 0u;
    S.issued[0] = S.issued[1] = 0u;
    *S.abort_flag = 0u;
    tc::fence_barrier_init();
    tc::prefetch_tensormap(&mq);
    tc::prefetch_tensormap(&mk);
    tc::prefetch_tensormap(&mv);
  }
  for (int p = t; p < kD / 2; p += blockDim.x) S.inv_freq[p] = pow(a.theta, -2.0 * p / (double)kD);
  for (int s = t; s < a.nslots; s += blockDim.x) desc[s] = make_desc(a, s);
  __syncthreads();
  if (warp == 0) {
    if ((int64_t)blockIdx.x < ngroups) load_group(a, S, L, &mq, &mk, &mv, blockIdx.x, 0, lane);
    if ((int64_t)blockIdx.x + grid < ngroups) load_group(a, S, L, &mq, &mk, &mv, blockIdx.x + grid, 1, lane);
  }

  const unsigned pm = 3u << (lane & 30);  // this lane pair
  int it = 0;
  for (int64_t g = blockIdx.x; g < ngroups; g += grid, ++it) {
    const int b = it & 1;
    const bool ok = wait_full(&S.full[b], (uint32_t)(it >> 1) & 1u, S.abort_flag);
    if (!__all_sync(0xffffffffu, ok)) {
      if (lane == 0 && !*S.abort_flag) {
        *S.abort_flag = 1u;
        atomicOr(&g_rope_status, 2u);
      }
      break;
    }
    const int tok0 = (int)(g * G);
    const int ntk = min(G, a.ntok - tok0);
    const uint8_t *tl = S.base + (uint32_t)b * L.buf_bytes;
    const float4 *tb = reinterpret_cast<const float4 *>(S.tab + b * G * kTabTok);
    const int64_t *cb = S.cbase + b * G;
    int c = (warp - it) % W;
    if (c < 0) c += W;
    for (; c * 32 < a.nslots; c += W) {
      const int s = c * 32 + lane;
      if (s >= a.nslots) continue;
      const uint32_t d = desc[s];
      const uint32_t srow = d & 1023u, h = (d >> 10) & 511u, tk = (d >> 19) & 7u, kind = (d >> 22) & 3u,
                     hf = d >> 24;
      if ((int)tk >= ntk) continue;
      // registers 0-31: elements 32 hf + j from the left tile; 32-63: 64 + 32 hf + j from the right
      const uint8_t *rl = tl + srow * 128u;
      const uint8_t *rr = rl + L.tile_bytes;
      const uint32_t sw = (4u * hf) ^ (srow & 7u);
      float x[64];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        unpack8(*reinterpret_cast<const uint4 *>(rl + ((sw ^ k) << 4)), x + 8 * k);
        unpack8(*reinterpret_cast<const uint4 *>(rr + ((sw ^ k) << 4)), x + 32 + 8 * k);
      }
      const int tok = tok0 + (int)tk;
      if (kind != 2) {
        // RoPE and the butterfly over element bit 6, scaled by 1/sqrt(d)
        const float4 *tp = tb + tk * (kTabTok / 2) + hf * (kTabHalf / 2);
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float4 e = tp[j >> 1];  // (P_j, M_j, P_j+1, M_j+1)
          float a0 = x[j], b0 = x[j + 32], a1 = x[j + 1], b1 = x[j + 33];
          x[j] = fmaf(a0, e.x, b0 * e.y);
          x[j + 32] = fmaf(a0, e.y, -(b0 * e.x));
          x[j + 1] = fmaf(a1, e.z, b1 * e.w);
          x[j + 33] = fmaf(a1, e.w, -(b1 * e.z));
        }
        fwht_low5(x);
        fwht_pair_bit(x, hf, pm);
      }
      if (kind == 0) {
        uint8_t *qrow = reinterpret_cast<uint8_t *>(a.q_out + ((int64_t)tok * a.hq + h) * kD);
#pragma unroll
        for (int part = 0; part < 4; ++part) {  // registers 16 part .. + 15
          uint32_t w[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) w[i] = pack_bf16x2(x[16 * part + 2 * i], x[16 * part + 2 * i + 1]);
          // registers 0-15 -> bytes 64 hf .., 16-31 -> 64 hf + 32, 32-47 -> 128 + 64 hf, 48-63 -> 160 + 64 hf
          uint8_t *dst = qrow + 128 * (part >> 1) + 64 * hf + 32 * (part & 1);
          if (a.q32) {
            st_v8_cs(dst, w);
          } else {
            __stcs(reinterpret_cast<uint4 *>(dst), make_uint4(w[0], w[1], w[2], w[3]));
            __stcs(reinterpret_cast<uint4 *>(dst + 16), make_uint4(w[4], w[5], w[6], w[7]));
          }
        }
      } else {
        const int64_t crow = cb[tk] + (int64_t)h * a.cache_len;
        if (kind == 1)
          quant_asym_store(x, a.clip, hf, pm, a.k_cache + crow * (kD / 2), a.k_scale + crow, a.k_zero + crow);
        else
          quant_asym_store(x, a.clip, hf, pm, a.v_cache + crow * (kD / 2), a.v_scale + crow, a.v_zero + crow);
      }
    }
    // count this warp out of buffer b; the last one refills it
    __syncwarp();
    uint32_t last = 0u;
    if (lane == 0) {
      __threadfence_block();
      last = atomicAdd(&S.cnt[b], 1u) == (uint32_t)(W - 1) ? 1u : 0u;
      __threadfence_block();
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    if (last) {
      if (lane == 0) S.cnt[b] = 0u;
      const int64_t gn = g + 2 * grid;
      if (gn < ngroups && !*S.abort_flag) load_group(a, S, L, &mq, &mk, &mv, gn, b, lane);
    }
  }
  __syncthreads();
  if (t == 0 && *S.abort_flag) {
    // let the loads this CTA issued land before its shared memory goes away
    for (int b = 0; b < 2; ++b) {
      if (S.issued[b] == 0u) continue;
      const uint32_t par = (S.issued[b] - 1u) & 1u;
      const long long t0 = clock64();
      while (!tc::mbar_try_wait(&S.full[b], par) && clock64() - t0 < kTimeoutCycles) {
      }
    }
  }
}

bool make_map(CUtensorMap *map, const void *base, int64_t rows, int box_rows) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool rope_shape_supported(int n_q_heads, int n_kv_heads, int64_t tokens) {
  return n_q_heads >= 1 && n_q_heads <= 256 && n_kv_heads >= 1 && n_q_heads + 2 * n_kv_heads <= 384 &&
         tokens >= 0 && tokens * n_q_heads < (int64_t(1) << 31);
}

cudaError_t launch_rope_hadamard_kvquant(const void *q, const void *k, const void *v,
                                         const int32_t *pos, float theta, int batch, int seq,
                                         int n_q_heads, int n_kv_heads, float clip, void *q_out,
                                         uint8_t *k_cache, uint8_t *v_cache, void *k_scale,
                                         void *k_zero, void *v_scale, void *v_zero, int cache_len,
                                         int cache_offset, cudaStream_t stream) {
  const int64_t ntok = (int64_t)batch * seq;
  if (!rope_shape_supported(n_q_heads, n_kv_heads, ntok)) return cudaErrorInvalidValue;
  if (ntok == 0) return cudaSuccess;
  const int rows_tok = n_q_heads + 2 * n_kv_heads;
  int G = 1;
  while (G < 8 && 2 * G * rows_tok <= kMaxGroupRows) G *= 2;  // tokens per group
  K2Args a;
  a.q_out = static_cast<uint16_t *>(q_out);
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.k_scale = static_cast<__half *>(k_scale);
  a.k_zero = static_cast<__half *>(k_zero);
  a.v_scale = static_cast<__half *>(v_scale);
  a.v_zero = static_cast<__half *>(v_zero);
  a.pos = pos;
  a.ntok = (int)ntok;
  a.seq = seq;
  a.hq = n_q_heads;
  a.hkv = n_kv_heads;
  a.G = G;
  a.cache_len = cache_len;
  a.cache_offset = cache_offset;
  a.rq = (G * n_q_heads + 7) / 8 * 8;
  a.rk = (G * n_kv_heads + 7) / 8 * 8;
  a.nslots = 2 * G * rows_tok;
  a.q32 = (reinterpret_cast<uintptr_t>(q_out) & 31u) == 0;
  a.clip = clip;
  a.theta = (double)theta;
  const K2Layout L = k2_layout(G, a.rq, a.rk, a.nslots);
  const size_t smem = (size_t)L.total + 1024;  // + alignment slack
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  const int threads = a.nslots < kMaxThreads ? (a.nslots + 31) / 32 * 32 : kMaxThreads;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, ntok * n_q_heads, G * n_q_heads) || !make_map(&mk, k, ntok * n_kv_heads, G * n_kv_heads) ||
      !make_map(&mv, v, ntok * n_kv_heads, G * n_kv_heads))
    return cudaErrorInvalidValue;
  int slots = 0;
  cudaError_t err =
      resident_slots(reinterpret_cast<const void *>(k2_rope_hadamard_kvquant), threads, (int)smem, &slots);
  if (err != cudaSuccess) return err;
  const int64_t ngroups = (ntok + G - 1) / G;
  const int64_t grid = ngroups < slots ? ngroups : slots;
  k2_rope_hadamard_kvquant<<<(unsigned)grid, threads, smem, stream>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

cudaError_t read_rope_status(unsigned int *status, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(status, g_rope_status, sizeof(unsigned int));
  if (e != cudaSuccess || !reset) return e;
  const unsigned int zero = 0u;
  return cudaMemcpyToSymbol(g_rope_status, &zero, sizeof(unsigned int));
}

}  // namespace spin
