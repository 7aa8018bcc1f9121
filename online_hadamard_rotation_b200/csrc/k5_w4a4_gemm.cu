// k5_w4a4_gemm.cu -- W4A4 GEMM on packed INT4 codes, on the tensor cores.
//
// "SpinQuant Guide: Learned Rotations for 4-Bit LLMs", section "End-to-End
// Implementation": the quantised layer output is the product of the quantised
// activations and the quantised weights, each dequantised as code x scale; section
// "Production Engineering and Cluster Deployment Best Practices": the rotated weights
// W R^T are baked offline into packed INT4 nibbles and the product runs on INT4 tensor
// cores. Here the activations are the R4 kernel's output as it stands (per-token codes
// and fp32 steps) and the weights are packed the same way, one step per output channel:
//   y[t][o] = s_x[t] s_w[o] sum_k q_x[t][k] q_w[o][k].
//
// The sum runs exactly on the tensor cores (tcgen05.mma kind::i8, int32 accumulation in
// TMEM). sm_100 has no 4-bit integer MMA, so converter warps widen each chunk's nibbles
// to int8 in shared memory: the byte holding codes 2j and 2j + 1 gives 16 q_{2j} as
// (b << 4) & 0xF0 and 16 q_{2j+1} as b & 0xF0, one shift and two masks per eight codes.
// A word's eight codes come out in the order 0, 2, 4, 6, 1, 3, 5, 7; both operands use
// the same order, so the contraction is unchanged, and the accumulator holds exactly
// 256 sum q_x q_w (|sum| <= 64 k, so k <= 65536 keeps it inside int32).
//
// Tile: 128 tokens (MMA M) x 256 output channels (N), the contraction in chunks of 128
// codes. Roles (256 threads, one CTA per output tile):
//   warp 0      TMA loads of each chunk's packed tiles (64-byte rows: 8 KiB of x, 16 KiB
//               of w) into a four-stage ring; rows past the last token read as zero
//   warp 1      TMEM owner and MMA issuer: four K = 32 MMAs per chunk, M = 128, N = 256
//   warps 2-7   converters: packed codes -> int8 operands (K-major, 128-byte swizzle)
//               in a two-stage ring; warps 4-7 then read the accumulator (TMEM lane =
//               token) and write y = (s_x s_w) (acc / 256) as fp32 or bf16
// Every mbarrier wait is bounded by a clock budget; on expiry the CTA records a status
// (read by spin_device_status), stops, waits for its copies and MMAs and frees TMEM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "spin_launch.h"
#include "spin_tile.cuh"
#include "tc_ptx.cuh"

namespace spin {

// Nonzero once a W4A4 GEMM launch gave up on a wait (see spin_device_status).
__device__ unsigned int g_gemm_status = 0u;

namespace {

constexpr int kThreads = 256;
constexpr int kConv = 192;                      // converter threads (warps 2-7)
constexpr int BM = 128, BN = 256, BK = 128;     // tokens x output channels x codes per chunk
constexpr int kPS = 3, kOS = 3;                 // packed and operand ring stages
constexpr uint32_t kPackA = BM * BK / 2;        // 8 KiB of packed x codes per chunk
constexpr uint32_t kPackStage = kPackA + BN * BK / 2;  // + 16 KiB of packed w codes
constexpr uint32_t kOpA = BM * BK;              // 16 KiB of int8 x operand
constexpr uint32_t kOpStage = kOpA + BN * BK;   // + 32 KiB of int8 w operand
constexpr uint32_t kOffP = 0;                   // packed ring
constexpr uint32_t kOffO = kOffP + kPS * kPackStage;  // operand ring (1024-byte aligned)
constexpr uint32_t kOffBar = kOffO + kOS * kOpStage;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;  // + alignment slack
constexpr uint32_t kTmemCols = 256;
constexpr int kQPT = (BM + BN) * 4 / kConv;     // packed quads per converter thread and chunk
constexpr long long kTimeoutCycles = 4000000000LL;     // about two seconds
static_assert(kOffO % 1024 == 0 && kOpStage % 1024 == 0 && kOpA % 1024 == 0, "swizzled operand alignment");
static_assert(kSmemBytes <= 232448, "shared memory per block");
static_assert(kQPT * kConv == (BM + BN) * 4, "the quads of a chunk divide evenly among the converters");

struct Shared {
  uint64_t pfull[kPS], pempty[kPS], ofull[kOS], oempty[kOS], tfull, drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Shared) <= 256, "barrier area");

// kind::i8 instruction descriptor: s32 accumulator, signed 8-bit A and B, both K-major,
// M = 128, N = 256.
constexpr uint32_t kIdesc = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

// D[tmem] (+)= A[smem desc] * B[smem desc], kind::i8 (int8 inputs, int32 accumulate)
__device__ __forceinline__ void umma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ bool wait_bounded(uint64_t *bar, uint32_t parity, Shared &S, bool honor_abort) {
  if (tc::mbar_try_wait_suspend(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (tc::mbar_try_wait_suspend(bar, parity)) return true;
    if (honor_abort && *reinterpret_cast<volatile int *>(&S.abort)) return false;
    if (clock64() - t0 > kTimeoutCycles) {
      *reinterpret_cast<volatile int *>(&S.abort) = 1;
      atomicOr(&g_gemm_status, 1u);
      return false;
    }
  }
}

// 16 packed codes (8 bytes) -> 16 int8 values 16 q, the even codes of each 4-byte word
// first: one 16-byte chunk of an operand row from two words.
__device__ __forceinline__ uint4 widen2(uint32_t w0, uint32_t w1) {
  return make_uint4((w0 << 4) & 0xF0F0F0F0u, w0 & 0xF0F0F0F0u, (w1 << 4) & 0xF0F0F0F0u, w1 & 0xF0F0F0F0u);
}

template <bool F32>
__global__ void __launch_bounds__(kThreads, 1)
    k5_w4a4_gemm(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap wmap,
                 const float *__restrict__ xs, const float *__restrict__ ws, int64_t tokens, int n_out, int k,
                 void *__restrict__ out) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, derived from the shared array itself so that accesses
  // through it stay shared-memory accesses
  uint8_t *smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  Shared &S = *reinterpret_cast<Shared *>(smem + kOffBar);
  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31u;
  const int tile_m = (int)blockIdx.x, tile_n = (int)blockIdx.y;
  const int nchunks = k / BK;

  // ------------------------------------------------------------ setup
  if (threadIdx.x == 0) {
    for (int s = 0; s < kPS; ++s) {
      tc::mbar_init(&S.pfull[s], 1);
      tc::mbar_init(&S.pempty[s], 1);
    }
    for (int s = 0; s < kOS; ++s) {
      tc::mbar_init(&S.ofull[s], 1);
      tc::mbar_init(&S.oempty[s], 1);
    }
    tc::mbar_init(&S.tfull, 1);
    tc::mbar_init(&S.drain, 1);
    S.abort = 0;
    tc::fence_barrier_init();
    tc::prefetch_tensormap(&xmap);
    tc::prefetch_tensormap(&wmap);
  }
  if (warp == 1) {
    tc::tmem_alloc(&S.tmem_base, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  // ------------------------------------------------------------ roles
  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int c = 0; c < nchunks; ++c) {
        const int ps = c % kPS;
        // the stage's previous chunk (c - kPS) has been converted
        if (c >= kPS && !wait_bounded(&S.pempty[ps], (uint32_t)((c / kPS - 1) & 1), S, true)) break;
        uint8_t *dst = smem + kOffP + ps * kPackStage;
        tc::mbar_arrive_expect_tx(&S.pfull[ps], kPackStage);
        tc::tma_load_2d(dst, &xmap, &S.pfull[ps], c * (BK / 2), tile_m * BM);
        tc::tma_load_2d(dst + kPackA, &wmap, &S.pfull[ps], c * (BK / 2), tile_n * BN);
        issued = c + 1;
      }
      // every issued copy has landed before the CTA can leave
      for (int s = 0; s < kPS && s < issued; ++s) {
        const int last = s + ((issued - 1 - s) / kPS) * kPS;
        wait_bounded(&S.pfull[s], (uint32_t)((last / kPS) & 1), S, false);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t sO = tc::smem_u32(smem + kOffO);
      bool ok = true;
      for (int c = 0; c < nchunks; ++c) {
        const int os = c % kOS;
        if (!wait_bounded(&S.ofull[os], (uint32_t)((c / kOS) & 1), S, true)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        const uint32_t a = sO + os * kOpStage, b = a + kOpA;
#pragma unroll
        for (int s = 0; s < BK / 32; ++s)  // K = 32 codes (32 bytes) per MMA
          umma_i8(tmem, tc::smem_desc(a + s * 32, 16, 1024), tc::smem_desc(b + s * 32, 16, 1024),
                  (c > 0 || s > 0) ? 1u : 0u);
        tc::umma_commit(&S.oempty[os]);
      }
      if (ok) tc::umma_commit(&S.tfull);
    }
  } else {
    // converters: chunk c's packed rows (x rows 0-127, then w rows 128-383, 64 bytes
    // each) -> int8 operand rows of 128 bytes, 16-byte chunk j of row r at j ^ (r & 7)
    const uint32_t cid = threadIdx.x - 64;
    for (int c = 0; c < nchunks; ++c) {
      const int ps = c % kPS, os = c % kOS;
      if (!wait_bounded(&S.pfull[ps], (uint32_t)((c / kPS) & 1), S, true)) break;
      if (c >= kOS && !wait_bounded(&S.oempty[os], (uint32_t)((c / kOS - 1) & 1), S, true)) break;
      const uint8_t *pk = smem + kOffP + ps * kPackStage;
      uint8_t *op = smem + kOffO + os * kOpStage;
      // all of a thread's loads first, then its stores (four 16-byte quads per packed row)
      uint4 wv[kQPT];
#pragma unroll
      for (int j = 0; j < kQPT; ++j) {
        const uint32_t qd = cid + (uint32_t)j * kConv;
        wv[j] = *reinterpret_cast<const uint4 *>(pk + (qd >> 2) * 64u + (qd & 3u) * 16u);
      }
#pragma unroll
      for (int j = 0; j < kQPT; ++j) {
        const uint32_t qd = cid + (uint32_t)j * kConv;
        const uint32_t row = qd >> 2, qi = qd & 3u, sw = row & 7u;
        uint8_t *orow = op + row * 128u;
        *reinterpret_cast<uint4 *>(orow + (((2u * qi) ^ sw) << 4)) = widen2(wv[j].x, wv[j].y);
        *reinterpret_cast<uint4 *>(orow + (((2u * qi + 1u) ^ sw) << 4)) = widen2(wv[j].z, wv[j].w);
      }
      tc::fence_proxy_async_smem();
      tc::named_sync(1, kConv);
      if (cid == 0) {
        tc::mbar_arrive(&S.ofull[os]);
        tc::mbar_arrive(&S.pempty[ps]);
      }
    }
    if (warp >= 4 && warp < 8 && wait_bounded(&S.tfull, 0, S, true)) {
      // epilogue: TMEM lane = token row of the tile, columns = output channels
      tc::tc_fence_after();
      const uint32_t q4 = warp & 3u;
      const int64_t t = (int64_t)tile_m * BM + q4 * 32 + lane;
      const float sx = t < tokens ? __ldg(xs + t) : 0.0f;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t r[32];
        tc::tmem_ld32(tmem + ((q4 * 32u) << 16) + (uint32_t)c0, r);
        tc::tmem_wait_ld();
        if (t >= tokens) continue;
        const int o0 = tile_n * BN + c0;
        float y[32];
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const float4 s4 = __ldg(reinterpret_cast<const float4 *>(ws + o0 + j));
          // acc = 256 sum q_x q_w exactly; the sum (|sum| < 2^24) converts exactly
          y[j] = (sx * s4.x) * (float)((int32_t)r[j] >> 8);
          y[j + 1] = (sx * s4.y) * (float)((int32_t)r[j + 1] >> 8);
          y[j + 2] = (sx * s4.z) * (float)((int32_t)r[j + 2] >> 8);
          y[j + 3] = (sx * s4.w) * (float)((int32_t)r[j + 3] >> 8);
        }
        if constexpr (F32) {
          float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(out) + t * (int64_t)n_out + o0);
#pragma unroll
          for (int j = 0; j < 8; ++j) dst[j] = make_float4(y[4 * j], y[4 * j + 1], y[4 * j + 2], y[4 * j + 3]);
        } else {
          uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(out) + t * (int64_t)n_out + o0);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            dst[j] = make_uint4(pack_bf16x2(y[8 * j], y[8 * j + 1]), pack_bf16x2(y[8 * j + 2], y[8 * j + 3]),
                                pack_bf16x2(y[8 * j + 4], y[8 * j + 5]), pack_bf16x2(y[8 * j + 6], y[8 * j + 7]));
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) {
      tc::umma_commit(&S.drain);  // arrives once every MMA this thread issued is complete
      wait_bounded(&S.drain, 0, S, false);
    }
    __syncwarp();
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// 2-D map over packed codes [rows][k / 2 bytes], boxes of 64 bytes x box_rows rows.
bool make_codes_map(CUtensorMap *map, const uint8_t *base, int64_t rows, int k, int box_rows) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)(k / 2), (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(k / 2)};
  const cuuint32_t box[2] = {(cuuint32_t)(BK / 2), (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool F32>
cudaError_t launch(const uint8_t *xq, const float *xs, int64_t tokens, const uint8_t *wq, const float *ws, int n_out,
                   int k, void *out, cudaStream_t stream) {
  CUtensorMap xmap, wmap;
  std::memset(&xmap, 0, sizeof(xmap));
  std::memset(&wmap, 0, sizeof(wmap));
  if (!make_codes_map(&xmap, xq, tokens, k, BM) || !make_codes_map(&wmap, wq, n_out, k, BN))
    return cudaErrorInvalidValue;
  auto kern = k5_w4a4_gemm<F32>;
  int slots = 0;
  cudaError_t e = resident_slots(reinterpret_cast<const void *>(kern), kThreads, (int)kSmemBytes, &slots);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((tokens + BM - 1) / BM), (unsigned)(n_out / BN));
  kern<<<grid, kThreads, kSmemBytes, stream>>>(xmap, wmap, xs, ws, tokens, n_out, k, out);
  return cudaGetLastError();
}

}  // namespace

bool w4a4_shape_supported(int64_t tokens, int n_out, int k) {
  return tokens >= 0 && (tokens + BM - 1) / BM <= 0x7FFFFFFF && tokens <= 0x7FFFFFFF - BM && n_out >= BN &&
         n_out % BN == 0 && n_out / BN <= 65535 && k >= BK && k % BK == 0 && k <= 65536;
}

cudaError_t launch_w4a4_gemm(const uint8_t *xq, const float *xs, int64_t tokens, const uint8_t *wq, const float *ws,
                             int n_out, int k, void *out, bool out_f32, cudaStream_t stream) {
  if (tokens == 0) return cudaSuccess;
  return out_f32 ? launch<true>(xq, xs, tokens, wq, ws, n_out, k, out, stream)
                 : launch<false>(xq, xs, tokens, wq, ws, n_out, k, out, stream);
}

cudaError_t read_gemm_status(unsigned int *status, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(status, g_gemm_status, sizeof(unsigned int));
  if (e != cudaSuccess || !reset) return e;
  const unsigned int zero = 0u;
  return cudaMemcpyToSymbol(g_gemm_status, &zero, sizeof(unsigned int));
}

}  // namespace spin
