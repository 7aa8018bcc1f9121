// k4_decode_attn.cu -- one decode step of attention over the 4-bit KV cache that the
// R3 kernel writes.
//
// "SpinQuant Guide: Learned Rotations for 4-Bit LLMs", the KV4 serving diagram: the
// rotated keys are stored in the KV cache as INT4 and meet the rotated queries in a
// fused INT4 dot product; section "RoPE Compatibility with 4-Bit KV Caching": the KV
// cache is kept at 4 bits. "SpinQuant: rotate before you round", section "Deployment
// implications": a rotation pays only once the runtime has KV4 kernels. R3 rotates q
// and k by the same orthogonal H / sqrt(d), so q . k needs no inverse rotation; V is
// not rotated.
//
// For batch row b and query head h (kv head g = h / (hq / hkv)), over the slots
// j < len[b] of the cache row (b, g):
//   khat_j = (c_j - z_j) s_j,  score_j = (q_h . khat_j) * softmax_scale,
//   p = softmax(score),  out_h = sum_j p_j vhat_j,  vhat_j = (c'_j - z'_j) s'_j.
// Split over the cache: block (chunk, g, b) takes 256 slots for all G = hq / hkv query
// heads of kv head g and writes, per head, the chunk's max score m, sum of
// exp(score - m) l and sum of exp(score - m) vhat (d values) to the caller's
// workspace; a second kernel merges the chunks of each (b, h). The dot products use
// q . khat = s (q . c - z sum(q)), the value sum sum_j w_j (c'_j - z'_j) with
// w_j = p_j s'_j = sum_j w_j c'_j - sum_j w_j z'_j, so every inner product runs on
// the small integer codes: each nibble becomes an exact float through one byte
// permute into the pattern 0x4B0000uu (2^23 + u) and a packed subtraction of 2^23.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "spin_launch.h"

namespace spin {
namespace {

constexpr int kD = 128;       // head_dim
constexpr int kChunk = 256;   // cache slots per block
constexpr int kThreads = 256;
constexpr int kPart = kD + 2;  // floats per (b, h, chunk) partial: m, l, d sums

// {a0, a1} + {b0, b1} * {c0, c1}, one packed FMA
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  uint64_t A, B, C, R;
  asm("mov.b64 %0, {%1, %2};" : "=l"(A) : "f"(a.x), "f"(a.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(B) : "f"(b.x), "f"(b.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(C) : "f"(c.x), "f"(c.y));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(R) : "l"(B), "l"(C), "l"(A));
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(R));
  return r;
}

// Eight nibbles of a code word (element k in bits 4k .. 4k + 3) as exact floats, in
// pairs (element 2k, element 2k + 1).
__device__ __forceinline__ void nibbles8(uint32_t w, float2 (&f)[4]) {
  const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;  // even, odd elements
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    // byte k of lo / hi under the exponent of 2^23: the float 2^23 + u
    const float e = __uint_as_float(__byte_perm(lo, 0x4B000000u, 0x7440u + k));
    const float o = __uint_as_float(__byte_perm(hi, 0x4B000000u, 0x7440u + k));
    f[k] = ffma2(make_float2(-8388608.0f, -8388608.0f), make_float2(e, o), make_float2(1.0f, 1.0f));
  }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

template <int G>
struct AttnSmem {
  float q[G][kD];            // queries as fp32
  float qsum[G];             // sum_i q_i per head
  float w[kChunk][G];        // scores, then p_j s'_j
  float red[kThreads / 32][G];
  float m[G], l[G], z[G];    // chunk max, sum of exp, sum_j w_j z'_j
  float acc[kThreads / 32][G][kD];  // per-warp partial value sums
};

template <int G>
__global__ void __launch_bounds__(kThreads)
    k4_attn_partial(const __nv_bfloat16 *__restrict__ q, const uint8_t *__restrict__ kc,
                    const uint8_t *__restrict__ vc, const __half *__restrict__ ks, const __half *__restrict__ kz,
                    const __half *__restrict__ vs, const __half *__restrict__ vz, const int32_t *__restrict__ lens,
                    int hq, int hkv, int cache_len, int nsplit, float softmax_scale, float *__restrict__ ws) {
  extern __shared__ float4 smem_raw[];
  AttnSmem<G> &S = *reinterpret_cast<AttnSmem<G> *>(smem_raw);
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  int len = lens[b];
  len = len < 0 ? 0 : (len > cache_len ? cache_len : len);  // out-of-range lengths are clamped
  const int start = split * kChunk;
  const int cnt = min(kChunk, len - start);
  // partial of head h = g G + hh: ws[((b hq + h) nsplit + split) kPart ..]
  auto part = [&](int hh) { return ws + (((int64_t)b * hq + g * G + hh) * nsplit + split) * kPart; };
  if (cnt <= 0) {  // nothing of this row's cache in the chunk: an empty partial
    if (t < G) {
      part(t)[0] = -INFINITY;
      part(t)[1] = 0.0f;
    }
    return;
  }
  const int64_t row0 = ((int64_t)b * hkv + g) * cache_len + start;  // first cache row of the chunk
  const int dg = t & 15, sg = t >> 4;  // value phase: dims 8 dg .. 8 dg + 7 of slots sg, sg + 16, ...

  // every global load of the block is issued here, before any barrier, so their
  // latencies overlap: thread t's key row (slot t), and its 16 words of value codes
  uint4 krow[4] = {};
  float ksc = 0.0f, kzr = 0.0f, vsc = 0.0f, vzr = 0.0f;
  if (t < cnt) {
    const uint4 *kr = reinterpret_cast<const uint4 *>(kc + (row0 + t) * (kD / 2));
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) krow[c4] = __ldg(kr + c4);
    ksc = __half2float(ks[row0 + t]);
    kzr = __half2float(kz[row0 + t]);
    vsc = __half2float(vs[row0 + t]);
    vzr = __half2float(vz[row0 + t]);
  }
  uint32_t vw[kChunk / 16];
#pragma unroll
  for (int u = 0; u < kChunk / 16; ++u) {
    const int j = sg + 16 * u;
    vw[u] = j < cnt ? __ldg(reinterpret_cast<const uint32_t *>(vc + (row0 + j) * (kD / 2)) + dg) : 0u;
  }

  // queries of the G heads as fp32, and their sums
  for (int i = t; i < G * kD; i += kThreads)
    S.q[i / kD][i % kD] = __bfloat162float(q[((int64_t)b * hq + g * G) * kD + i]);
  __syncthreads();
  if (t < G * 32) {  // warp h sums head h's query
    const int hh = t >> 5;
    float v = S.q[hh][lane] + S.q[hh][lane + 32] + S.q[hh][lane + 64] + S.q[hh][lane + 96];
    v = warp_sum(v);
    if (lane == 0) S.qsum[hh] = v;
  }
  __syncthreads();

  // scores: thread t takes slot start + t
  float sc[G];
  if (t < cnt) {
    float2 acc[G];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) acc[hh] = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {
      const uint32_t words[4] = {krow[c4].x, krow[c4].y, krow[c4].z, krow[c4].w};
#pragma unroll
      for (int wi = 0; wi < 4; ++wi) {
        float2 f[4];
        nibbles8(words[wi], f);
        const int e0 = 32 * c4 + 8 * wi;  // first element of this word
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
          const float4 qa = *reinterpret_cast<const float4 *>(&S.q[hh][e0]);
          const float4 qb = *reinterpret_cast<const float4 *>(&S.q[hh][e0 + 4]);
          acc[hh] = ffma2(acc[hh], make_float2(qa.x, qa.y), f[0]);
          acc[hh] = ffma2(acc[hh], make_float2(qa.z, qa.w), f[1]);
          acc[hh] = ffma2(acc[hh], make_float2(qb.x, qb.y), f[2]);
          acc[hh] = ffma2(acc[hh], make_float2(qb.z, qb.w), f[3]);
        }
      }
    }
#pragma unroll
    for (int hh = 0; hh < G; ++hh) sc[hh] = ksc * ((acc[hh].x + acc[hh].y) - kzr * S.qsum[hh]) * softmax_scale;
  } else {
#pragma unroll
    for (int hh = 0; hh < G; ++hh) sc[hh] = -INFINITY;
  }
  // chunk max per head
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    const float v = warp_max(sc[hh]);
    if (lane == 0) S.red[warp][hh] = v;
  }
  __syncthreads();
  if (t < G) {
    float v = S.red[0][t];
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) v = fmaxf(v, S.red[w][t]);
    S.m[t] = v;
  }
  __syncthreads();
  // p_j = exp(score_j - m), l = sum p_j; w_j = p_j s'_j and sum_j w_j z'_j
  float p[G], wz[G];
  {
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      p[hh] = t < cnt ? __expf(sc[hh] - S.m[hh]) : 0.0f;
      S.w[t][hh] = p[hh] * vsc;
      wz[hh] = p[hh] * vsc * vzr;
    }
  }
  __syncthreads();  // S.red is reused below
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    const float a = warp_sum(p[hh]);
    if (lane == 0) S.red[warp][hh] = a;
  }
  __syncthreads();
  if (t < G) {
    float v = 0.0f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) v += S.red[w][t];
    S.l[t] = v;
  }
  __syncthreads();
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    const float a = warp_sum(wz[hh]);
    if (lane == 0) S.red[warp][hh] = a;
  }
  __syncthreads();
  if (t < G) {
    float v = 0.0f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) v += S.red[w][t];
    S.z[t] = v;
  }

  // value sums: thread t takes dims 8 dg .. 8 dg + 7 of every 16th slot from sg (the
  // code words loaded at the start)
  {
    float2 acc[G][4];
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[hh][k] = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int u = 0; u < kChunk / 16; ++u) {
      const int j = sg + 16 * u;
      if (j >= cnt) break;
      float2 f[4];
      nibbles8(vw[u], f);
      float wj[G];
#pragma unroll
      for (int hh = 0; hh < G; ++hh) wj[hh] = S.w[j][hh];
#pragma unroll
      for (int hh = 0; hh < G; ++hh)
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[hh][k] = ffma2(acc[hh][k], make_float2(wj[hh], wj[hh]), f[k]);
    }
    // combine the two slot groups of a warp (lanes l and l ^ 16), then the warps
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        acc[hh][k].x += __shfl_xor_sync(0xFFFFFFFFu, acc[hh][k].x, 16);
        acc[hh][k].y += __shfl_xor_sync(0xFFFFFFFFu, acc[hh][k].y, 16);
      }
    if (lane < 16) {
#pragma unroll
      for (int hh = 0; hh < G; ++hh)
#pragma unroll
        for (int k = 0; k < 4; ++k) {  // pair k holds elements 2k and 2k + 1 of the 8
          S.acc[warp][hh][8 * dg + 2 * k] = acc[hh][k].x;
          S.acc[warp][hh][8 * dg + 2 * k + 1] = acc[hh][k].y;
        }
    }
  }
  __syncthreads();
  for (int o = t; o < G * kD; o += kThreads) {
    const int hh = o / kD, i = o % kD;
    float v = 0.0f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) v += S.acc[w][hh][i];
    part(hh)[2 + i] = v - S.z[hh];
  }
  if (t < G) {
    part(t)[0] = S.m[t];
    part(t)[1] = S.l[t];
  }
}

// Merge the chunks of (b, h): out = sum_c e^(m_c - M) a_c / sum_c e^(m_c - M) l_c.
template <bool F32>
__global__ void __launch_bounds__(kD)
    k4_attn_combine(const float *__restrict__ ws, const int32_t *__restrict__ lens, int hq, int cache_len,
                    int nsplit, void *__restrict__ out) {
  const int h = blockIdx.x, b = blockIdx.y, i = threadIdx.x;
  int len = lens[b];
  len = len < 0 ? 0 : (len > cache_len ? cache_len : len);
  const int used = (len + kChunk - 1) / kChunk;  // chunks that hold slots of this row
  const float *pp = ws + ((int64_t)b * hq + h) * nsplit * kPart;
  // chunks in batches of 8 whose loads are all issued before any is used; a running
  // maximum rescales the sums when it grows
  float M = -INFINITY, num = 0.0f, den = 0.0f;
  for (int c0 = 0; c0 < used; c0 += 8) {
    float m[8], l[8], a[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const bool in = c0 + u < used;
      m[u] = in ? pp[(c0 + u) * kPart] : -INFINITY;
      l[u] = in ? pp[(c0 + u) * kPart + 1] : 0.0f;
      a[u] = in ? pp[(c0 + u) * kPart + 2 + i] : 0.0f;
    }
    float Mn = M;
#pragma unroll
    for (int u = 0; u < 8; ++u) Mn = fmaxf(Mn, m[u]);
    const float r = M == -INFINITY ? 0.0f : __expf(M - Mn);
    num *= r;
    den *= r;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float e = m[u] == -INFINITY ? 0.0f : __expf(m[u] - Mn);
      den += e * l[u];
      num += e * a[u];
    }
    M = Mn;
  }
  const float r = used > 0 ? num / den : 0.0f;
  const int64_t o = ((int64_t)b * hq + h) * kD + i;
  if constexpr (F32) static_cast<float *>(out)[o] = r;
  else static_cast<__nv_bfloat16 *>(out)[o] = __float2bfloat16_rn(r);
}

template <int G>
cudaError_t launch_g(const void *q, const uint8_t *kc, const uint8_t *vc, const void *ks, const void *kz,
                     const void *vs, const void *vz, const int32_t *lens, int batch, int hq, int hkv, int cache_len,
                     float softmax_scale, void *out, bool f32, float *ws, cudaStream_t stream) {
  const int nsplit = (cache_len + kChunk - 1) / kChunk;
  constexpr int smem = (int)sizeof(AttnSmem<G>);
  static_assert(smem <= 48 * 1024, "fits the default dynamic shared memory of a block");
  k4_attn_partial<G><<<dim3(nsplit, hkv, batch), kThreads, smem, stream>>>(
      static_cast<const __nv_bfloat16 *>(q), kc, vc, static_cast<const __half *>(ks),
      static_cast<const __half *>(kz), static_cast<const __half *>(vs), static_cast<const __half *>(vz), lens, hq,
      hkv, cache_len, nsplit, softmax_scale, ws);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (f32)
    k4_attn_combine<true><<<dim3(hq, batch), kD, 0, stream>>>(ws, lens, hq, cache_len, nsplit, out);
  else
    k4_attn_combine<false><<<dim3(hq, batch), kD, 0, stream>>>(ws, lens, hq, cache_len, nsplit, out);
  return cudaGetLastError();
}

}  // namespace

size_t decode_attention_workspace_bytes(int batch, int n_q_heads, int cache_len) {
  const int64_t nsplit = (cache_len + kChunk - 1) / kChunk;
  return (size_t)((int64_t)batch * n_q_heads * nsplit * kPart * (int64_t)sizeof(float));
}

bool decode_attention_group_supported(int group) { return group == 1 || group == 2 || group == 4 || group == 8; }

cudaError_t launch_decode_attention(const void *q, const uint8_t *k_cache, const uint8_t *v_cache,
                                    const void *k_scale, const void *k_zero, const void *v_scale,
                                    const void *v_zero, const int32_t *lens, int batch, int n_q_heads,
                                    int n_kv_heads, int cache_len, float softmax_scale, void *out, bool out_f32,
                                    float *workspace, cudaStream_t stream) {
  switch (n_q_heads / n_kv_heads) {
    case 1: return launch_g<1>(q, k_cache, v_cache, k_scale, k_zero, v_scale, v_zero, lens, batch, n_q_heads,
                               n_kv_heads, cache_len, softmax_scale, out, out_f32, workspace, stream);
    case 2: return launch_g<2>(q, k_cache, v_cache, k_scale, k_zero, v_scale, v_zero, lens, batch, n_q_heads,
                               n_kv_heads, cache_len, softmax_scale, out, out_f32, workspace, stream);
    case 4: return launch_g<4>(q, k_cache, v_cache, k_scale, k_zero, v_scale, v_zero, lens, batch, n_q_heads,
                               n_kv_heads, cache_len, softmax_scale, out, out_f32, workspace, stream);
    case 8: return launch_g<8>(q, k_cache, v_cache, k_scale, k_zero, v_scale, v_zero, lens, batch, n_q_heads,
                               n_kv_heads, cache_len, softmax_scale, out, out_f32, workspace, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace spin
