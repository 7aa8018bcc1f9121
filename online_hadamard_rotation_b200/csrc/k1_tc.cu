// k1_tc.cu -- R4 on the tensor cores: for n = 2048 to 32768 the first Kronecker
// factor runs on tcgen05 (below); for n = 128 and 256 the whole transform does
// (tokens as the MMA's M, further down).
//
// "Rotations: QuaRot, SpinQuant and incoherence", section "Hadamard matrices":
// the Sylvester H_n is a Kronecker product of smaller Sylvester matrices, and
// the randomised transform is (1/sqrt n) H_n diag(+-1). "SpinQuant, when
// rotations are worth learning", section "Four rotation sites": R4 is the fixed
// Hadamard on the down-projection input. "SpinQuant Guide", section "The
// Outlier Curse": symmetric INT4, step max|y| / 7.
//
// A token row x of n = 128 B bf16 values is the 128 x B matrix X[a][b], with
// element index e = B a + b (B = 8, 16, 32, 64, 128; n = 32768 is two such blocks,
// n = 512 two 64-row tokens per 128-row block,
// see Shape). Then H_n x = vec(H_128 X H_B):
//   1. tcgen05.mma computes Y = H_128 X (contraction over a) for 256 / B tokens
//      at once (M = 128, N = 256, K = 128, bf16 in, fp32 accumulate in TMEM).
//      H is exactly +-1 and X is exactly bf16, so every product is exact and
//      only the fp32 accumulation rounds.
//   2. Each epilogue thread owns one row a' of Y (one TMEM lane) over 128
//      columns, i.e. 128 / B token segments of B values; it runs the log2(B)
//      butterfly stages of the second factor in registers, then each token's
//      max, step, INT4 codes and nibble packing. Row a' of a token is B / 2
//      contiguous code bytes.
//
// Work: one CTA per group of 256 / B tokens is launched; one CTA fits an SM, and each
// resident CTA, after its own group, takes over groups of CTAs that have not started
// yet (cluster launch control `try_cancel`), so the work spreads dynamically over the
// SMs and the last groups land wherever an SM is free.
// Roles (384 threads, one CTA per SM, persistent over groups):
//   warp 0      TMA producer: 64 KiB per group (boxes of [128 rows][min(B, 64)]
//               bf16 with 32-, 64- or 128-byte swizzle) into a three-stage ring
//   warp 1      TMEM owner and MMA issuer (8 MMAs of K = 16 per group)
//   warps 2-3   +-1 diagonal: XOR of the bf16 sign bits in shared memory, with
//               each thread's sign words held in registers
//   warps 4-7   epilogue for TMEM columns 0-127 of each group
//   warps 8-11  epilogue for columns 128-255
// TMEM holds two 256-column accumulators, so the MMA of group i + 1 overlaps
// the epilogue of group i. Each epilogue thread stores its code bytes straight
// to global memory. The launch allows programmatic dependent launch: the
// prologue may overlap the tail of the previous kernel in the stream, and no
// global memory is read or written before griddepcontrol.wait returns. Every
// mbarrier wait is bounded by a clock budget; on expiry the CTA records a
// status, drains its copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "spin_launch.h"
#include "spin_tile.cuh"
#include "tc_ptx.cuh"

namespace spin {

// Nonzero once a tensor-core kernel gave up on a wait (see spin_device_status).
__device__ unsigned int g_device_status = 0u;

namespace {

constexpr int kThreads = 384;
constexpr int kStages = 3;
constexpr uint32_t kGroupBytes = 65536;            // one MMA group: 128 rows x 256 columns of bf16
constexpr uint32_t kOffH = 0;                      // A operand: H_128, K-major, 2 x 16 KiB
constexpr uint32_t kOffX = 32768;                  // ring of kStages x 64 KiB
constexpr uint32_t kOffBar = kOffX + kStages * kGroupBytes;
constexpr uint32_t kSmemBytes = kOffBar + 2048 + 1024;  // barrier area + alignment slack (227 KiB in all)
constexpr long long kTimeoutCycles = 4000000000LL;     // about two seconds
constexpr long long kStallTestCycles = 2000000LL;      // about a millisecond, for the stall test hook

// Shape constants for n = 2^LOGN. For n = 32768 (SPLIT) a token is 256 rows of
// B = 128 columns: H_n = H_2 (x) H_128 (x) H_128, and the top factor H_2 pairs the row
// blocks X_0 (rows 0-127) and X_1 (rows 128-255). The group is that one token: the
// MMA accumulates H_128 X_0 + H_128 X_1 into TMEM columns 0-127 and H_128 X_0 -
// H_128 X_1 (negated A) into columns 128-255, so epilogue warpgroup g holds output
// rows 128 g + a' and the token's max spans both warpgroups.
//
// KR > 0 (KRON) is a row of n = m 2^k = 128 KR values that is not a power of two
// ("Rotations: QuaRot, SpinQuant and incoherence", "Hadamard matrices": sizes that
// are not powers of two use a Kronecker product with a small known Hadamard matrix):
// element e = b i + j (i < m the index of Paley's H_m, j < b = 2^k the Sylvester
// index) is row r = (b / 128) i + (j >> 7), column j & 127 of a KR x 128 tile, and
// H_m (x) H_b = (H_m (x) H_{b/128}) (x) H_128. The MMA's A operand is the KR x KR
// matrix H_m (x) H_{b/128} (zero-padded to 128 x 128) instead of H_128; everything
// after it is the n = 16384 shape with KR rows per token.
template <int LOGN, int KR = 0>
struct Shape {
  static constexpr bool KRON = KR > 0;
  static constexpr bool SPLIT = !KRON && LOGN == 15;
  // n = 512 (PAIR): a token is 64 rows of B = 8 columns (H_512 = H_64 (x) H_8) and each
  // 128-row TMA box holds two consecutive tokens, rows 0-63 and 64-127. The MMA's A
  // operand is H_64 (+) H_64 (block diagonal), so the two tokens stay apart; TMEM lanes
  // 0-63 hold the first token's rows, 64-127 the second's, and a token's max spans two
  // of an epilogue warpgroup's warps.
  static constexpr bool PAIR = !KRON && LOGN == 9;
  static constexpr int B = (SPLIT || KRON) ? 128 : PAIR ? 8 : 1 << (LOGN - 7);  // columns per row
  static constexpr int LOGB = (SPLIT || KRON) ? 7 : PAIR ? 3 : LOGN - 7;
  static constexpr int BOXH = KRON ? KR : 128;     // rows per TMA box and per MMA contraction
  static constexpr int ROWS = SPLIT ? 256 : PAIR ? 64 : BOXH;  // rows per token
  static constexpr int TPB = PAIR ? 2 : 1;         // tokens per 128-row box
  static constexpr int TOK = SPLIT ? 1 : TPB * 256 / B;  // tokens per MMA group
  static constexpr int SEG = SPLIT ? 1 : 128 / B;  // column segments per epilogue thread
  static constexpr int BOXW = B < 64 ? B : 64;     // TMA box width (columns)
  static constexpr int ROWB = BOXW * 2;            // bytes per smem tile row (16, 32, 64 or 128)
  static constexpr int CBOX = B / BOXW;            // column boxes per row block
  static constexpr int BPT = PAIR ? 1 : CBOX * ROWS / BOXH;  // boxes per token (PAIR: per token pair)
  static constexpr uint32_t BOXBYTES = (uint32_t)BOXH * ROWB;  // bytes per box
  static constexpr int CPR = ROWB / 16;            // 16-byte chunks per tile row
  static constexpr uint32_t LAYOUT = ROWB == 128 ? 2u : ROWB == 64 ? 4u : ROWB == 32 ? 6u : 0u;  // UMMA swizzle: 128, 64, 32 B, none
  // MN-major B operand strides: swizzled tiles step by box along N and by 8 rows along
  // K; the no-swizzle layout (16-byte rows, one 8 x 16 B core matrix per 8 rows) swaps
  // the roles of the two offsets, its leading offset stepping along K.
  static constexpr uint32_t LBO = LAYOUT == 0 ? 8u * ROWB : BOXBYTES;
  static constexpr uint32_t SBO = LAYOUT == 0 ? BOXBYTES : 8u * ROWB;
  static constexpr uint32_t TOKBYTES = (uint32_t)ROWS * B * 2;  // input bytes of one token
  static constexpr int NPOS = (int)(TOKBYTES / 16 / 64);  // sign positions per sign thread
  static constexpr int SIGN_ITERS = (int)(TOK * TOKBYTES / 16 / 64);  // chunks per sign thread per group
  static constexpr int KSTEPS = BOXH / 16;         // MMA steps of K = 16 per row block
  static constexpr int64_t OUTB = (int64_t)ROWS * B / 2;  // code bytes per token (INT4)
  static_assert(KRON ? (KR % 16 == 0 && KR >= 16 && KR <= 128) : (LOGN >= 9 && LOGN <= 15),
                "this tensor-core R4 kernel covers n = 512 .. 32768 and n = 128 KR, KR = 16 .. 128");
  static_assert(TOK * TOKBYTES <= kGroupBytes && SIGN_ITERS % 4 == 0 && NPOS >= 1, "stage layout");
};

// Paley's Hadamard matrix of order m, as a kernel argument: type I (q = m - 1, prime,
// q = 3 mod 4) or type II (q = m/2 - 1, prime, q = 1 mod 4); qr bit a is set when a
// (0 < a < q) is a square mod q. bq = b / 128 = KR / m, a power of two 2^lbq.
struct KronParams {
  int m, type, q, bq, lbq;
  uint32_t qr[4];
};

// Quadratic character of a mod q from the residue mask, for -q < a < q: 0, +1 or -1.
__device__ __forceinline__ int chi(int a, const KronParams &kp) {
  if (a < 0) a += kp.q;
  if (a == 0) return 0;
  return ((kp.qr[a >> 5] >> (a & 31)) & 1u) ? 1 : -1;
}

// Entry (i, j) of Paley's H_m. With the core matrix C of order q + 1 -- C[0][0] = 0,
// C[0][j] = 1, C[i][0] = -1 (type I) or +1 (type II), C[i][j] = chi(j - i) otherwise
// (1 <= i, j <= q, so -q < j - i < q) --
// type I is C + I and type II replaces each entry c of C by c [[1, -1], [-1, -1]]
// plus [[1, 1], [1, -1]] on the diagonal.
__device__ __forceinline__ int paley_entry(int i, int j, const KronParams &kp) {
  auto core = [&](int a, int b) {
    if (a == 0 && b == 0) return 0;
    if (a == 0) return 1;
    if (b == 0) return kp.type == 1 ? -1 : 1;
    return chi(b - a, kp);
  };
  if (kp.type == 1) return core(i, j) + (i == j ? 1 : 0);
  const int u = i & 1, v = j & 1, c = core(i >> 1, j >> 1);
  const int am = (u == 0 && v == 0) ? 1 : -1;   // [[1, -1], [-1, -1]]
  const int bm = (u == 1 && v == 1) ? -1 : 1;   // [[1, 1], [1, -1]]
  return c * am + ((i >> 1) == (j >> 1) ? bm : 0);
}

constexpr int kRing = 8;  // group ids in flight between the producer and the epilogue

struct Shared {
  uint4 clc_resp;          // response of the pending work-stealing request
  uint64_t full[kStages], sgn[kStages], empty[kStages], tfull[2], tempty[2], drain, clc;
  uint64_t gfull[kRing];   // group id i & 7 written
  int64_t gid[kRing];      // group of the CTA's i-th step (i & 7), -1 once there is none
  int64_t egid[2];         // epilogue warpgroup g's current group
  uint32_t tmem_base;
  int abort;
  int dec[3];
  long long budget;        // clock cycles a wait may take before the CTA gives up
  float wmax[2][2][4][16];  // [warpgroup][group parity][warp][token segment]
};
static_assert(sizeof(Shared) <= 2048, "barrier area");

// Work stealing by cluster launch control: ask the hardware to cancel a CTA of this
// grid that has not started yet; its 16-byte response lands in `resp` and completes
// `bar`. Issued by one thread, never again after a response that cancelled nothing.
__device__ __forceinline__ void clc_request(uint4 *resp, uint64_t *bar) {
  tc::mbar_arrive_expect_tx(bar, 16);
  asm volatile(
      "clusterlaunchcontrol.try_cancel.async.shared::cta.mbarrier::complete_tx::bytes.b128 [%0], [%1];" ::"r"(
          tc::smem_u32(resp)),
      "r"(tc::smem_u32(bar))
      : "memory");
}
// The cancelled CTA's x index, or -1 if the request cancelled nothing.
__device__ __forceinline__ int64_t clc_result(const uint4 *resp) {
  uint32_t ok, x;
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b128 q;\n\t"
      "ld.shared.b128 q, [%2];\n\t"
      "clusterlaunchcontrol.query_cancel.is_canceled.pred.b128 p, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t"
      "clusterlaunchcontrol.query_cancel.get_first_ctaid::x.b32.b128 %1, q;\n\t}"
      : "=r"(ok), "=r"(x)
      : "r"(tc::smem_u32(resp))
      : "memory");
  return ok ? (int64_t)x : -1;
}

template <class SS>
__device__ __forceinline__ bool wait_bounded(uint64_t *bar, uint32_t parity, SS &S, bool honor_abort) {
  if (tc::mbar_try_wait_suspend(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (tc::mbar_try_wait_suspend(bar, parity)) return true;
    if (honor_abort && *reinterpret_cast<volatile int *>(&S.abort)) return false;
    if (clock64() - t0 > S.budget) {
      *reinterpret_cast<volatile int *>(&S.abort) = 1;
      atomicOr(&g_device_status, 1u);
      return false;
    }
  }
}


// Codes on the subnormal grid. For 0 <= t < 2^23 the bit pattern of t * 2^-149 (a
// multiply by the smallest subnormal, rounded to nearest even) is rne(t), because the
// grid's spacing is 2^-149; for t < 0 the sign bit is set, so the pattern read as a
// signed integer is negative. cvt.pack.sat then clamps two such integers to the code
// range and packs them: biased codes u = code + 2^(b-1) need no clamp of their own.
// (r0, r1) = rne(v0 cq + bias), rne(v1 cq + bias) as such patterns: one packed FMA and
// one packed multiply (c2 = {cq, cq}, b2 = {bias, bias}).
__device__ __forceinline__ void biased_codes_x2(float v0, float v1, uint64_t c2, uint64_t b2, uint32_t &r0,
                                                uint32_t &r1) {
  uint64_t A, T, R;
  asm("mov.b64 %0, {%1, %2};" : "=l"(A) : "f"(v0), "f"(v1));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(T) : "l"(A), "l"(c2), "l"(b2));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(R) : "l"(T), "l"(0x0000000100000001ull));
  asm("mov.b64 {%0, %1}, %2;" : "=r"(r0), "=r"(r1) : "l"(R));
}

// 1 / x from the hardware reciprocal (within an ulp or so, for the normal x used here).
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ uint64_t pair(float x) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(x));
  return r;
}

// 8 consecutive values -> one word of INT4 codes, value k in nibble k (two's
// complement): u = clamp(rne(v cq) + 8, 0, 15), code = u - 8 (cq = 1 / step, in the
// values' scale).
__device__ __forceinline__ uint32_t codes8(const float *v, uint64_t c2) {
  constexpr uint64_t kBias = 0x4100000041000000ull;  // {8, 8}
  uint32_t r[8], d = 0u;
#pragma unroll
  for (int k = 0; k < 8; k += 2) biased_codes_x2(v[k], v[k + 1], c2, kBias, r[k], r[k + 1]);
#pragma unroll
  for (int k = 6; k >= 0; k -= 2)  // d = (d << 8) | sat(r[k + 1]) << 4 | sat(r[k])
    asm("cvt.pack.sat.u4.s32.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(r[k + 1]), "r"(r[k]), "r"(d));
  return d ^ 0x88888888u;
}

// 8 consecutive values -> two words of INT8 codes, value k in byte k (two's
// complement): u = clamp(rne(v cq) + 128, 0, 255), code = u - 128.
__device__ __forceinline__ void codes8_int8(const float *v, uint64_t c2, uint32_t &w0, uint32_t &w1) {
  constexpr uint64_t kBias = 0x4300000043000000ull;  // {128, 128}
  uint32_t r[8];
#pragma unroll
  for (int k = 0; k < 8; k += 2) biased_codes_x2(v[k], v[k + 1], c2, kBias, r[k], r[k + 1]);
  uint32_t d0 = 0u, d1 = 0u;
  asm("cvt.pack.sat.u8.s32.b32 %0, %1, %2, %3;" : "=r"(d0) : "r"(r[3]), "r"(r[2]), "r"(d0));
  asm("cvt.pack.sat.u8.s32.b32 %0, %1, %2, %3;" : "=r"(d0) : "r"(r[1]), "r"(r[0]), "r"(d0));
  asm("cvt.pack.sat.u8.s32.b32 %0, %1, %2, %3;" : "=r"(d1) : "r"(r[7]), "r"(r[6]), "r"(d1));
  asm("cvt.pack.sat.u8.s32.b32 %0, %1, %2, %3;" : "=r"(d1) : "r"(r[5]), "r"(r[4]), "r"(d1));
  w0 = d0 ^ 0x80808080u;
  w1 = d1 ^ 0x80808080u;
}

__device__ __forceinline__ void st_v8_cs(void *p, const uint32_t *w) {
  asm volatile("st.global.cs.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]), "r"(w[1]),
               "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}


// Named barrier that also ANDs a predicate over the participating threads: every
// thread leaves with the same answer, so a decision taken on it stays uniform.
// Not .aligned: threads of a warp may reach it on different paths.
__device__ __forceinline__ bool bar_red_and(uint32_t id, uint32_t threads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.cta.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}

// byte offset of 16-byte chunk `ch` (0..7) of row `r` in a 128-byte-swizzled [rows][128 B] tile
__device__ __forceinline__ uint32_t sw128(uint32_t r, uint32_t ch) { return r * 128u + ((ch ^ (r & 7u)) << 4); }

// One bulk copy global -> shared that completes `bar`'s transaction count (16-byte
// aligned addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   tc::smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(tc::smem_u32(bar))
               : "memory");
}

// Issue the copies of group p (tokens p * TOK ...) into `dst`. Tiles of 16-byte rows
// without swizzle (n = 512 and 1024) hold a group's bytes in their global order, so a
// full group arrives by one bulk copy of its contiguous 64 KiB (the TMA boxes of 16-byte
// rows cost the copy engine one request per row, 4096 per group). A partial group takes
// the boxes, whose rows past the last token read as zero: at n = 512 the block-diagonal
// A operand multiplies the other token's rows by zero, which must not meet stale data.
template <int LOGN, int KR>
__device__ __forceinline__ void load_group(uint8_t *dst, const CUtensorMap *map, const uint16_t *x, uint64_t *bar,
                                           int64_t p, int64_t tokens) {
  using SH = Shape<LOGN, KR>;
  const int64_t t0 = p * SH::TOK;
  const int nvalid = (int)((tokens - t0) < SH::TOK ? (tokens - t0) : SH::TOK);
  if constexpr (SH::LAYOUT == 0) {
    static_assert(SH::TOK * SH::TOKBYTES == kGroupBytes, "a full group is one contiguous range");
    if (nvalid == SH::TOK) {
      tc::mbar_arrive_expect_tx(bar, kGroupBytes);
      bulk_load(dst, x + t0 * (int64_t)(SH::ROWS * SH::B), kGroupBytes, bar);
      return;
    }
  }
  if constexpr (SH::PAIR) {  // whole boxes of two tokens; rows past the last token read as zero
    const int nbox = (nvalid + 1) / 2;
    tc::mbar_arrive_expect_tx(bar, (uint32_t)nbox * SH::BOXBYTES);
    for (int i = 0; i < nbox; ++i)
      tc::tma_load_2d(dst + i * SH::BOXBYTES, map, bar, 0, (int)((t0 + 2 * i) * SH::ROWS));
    return;
  }
  tc::mbar_arrive_expect_tx(bar, (uint32_t)nvalid * SH::TOKBYTES);
  for (int t = 0; t < nvalid; ++t)
    for (int j = 0; j < SH::BPT; ++j)
      tc::tma_load_2d(dst + (t * SH::BPT + j) * SH::BOXBYTES, map, bar, (j % SH::CBOX) * SH::BOXW,
                      (int)((t0 + t) * SH::ROWS + (j / SH::CBOX) * SH::BOXH));
}

template <int LOGN, int KR, bool SIGNS, bool STORE32, int BITS>
__global__ void __launch_bounds__(kThreads, 1)
    k1_tc_rotate_quant(const __grid_constant__ CUtensorMap xmap, const uint16_t *__restrict__ x, int64_t tokens,
                       float clip, float inv_sqrt_n,
                       const uint32_t *__restrict__ signs, uint8_t *__restrict__ q, float *__restrict__ scales,
                       int stall_test, const __grid_constant__ KronParams kp) {
  using SH = Shape<LOGN, KR>;
  constexpr int B = SH::B, SEG = SH::SEG;
  const float step_per_unit = clip * inv_sqrt_n / (BITS == 4 ? 7.0f : 127.0f);
  static_assert(!(SIGNS && SH::SPLIT), "the sign masks of n = 32768 do not fit in registers");
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, derived from the shared array itself so that accesses
  // through it stay shared-memory accesses
  uint8_t *smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  Shared &S = *reinterpret_cast<Shared *>(smem + kOffBar);
  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31u;
  const int64_t ngroups = (tokens + SH::TOK - 1) / SH::TOK;

  // ------------------------------------------------------------ setup
  // Global memory is touched only after the grids this one depends on have
  // finished (programmatic dependent launch lets this prologue overlap their tail).
  tc::grid_dep_wait();
  int64_t first_issued = 0;  // groups the producer issues before the setup barrier
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&S.full[s], 1);
      tc::mbar_init(&S.sgn[s], 1);
      tc::mbar_init(&S.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(&S.tfull[a], 1);
      tc::mbar_init(&S.tempty[a], 256);
    }
    tc::mbar_init(&S.drain, 1);
    tc::mbar_init(&S.clc, 1);
    for (int j = 0; j < kRing; ++j) tc::mbar_init(&S.gfull[j], 1);
    S.abort = 0;
    S.budget = stall_test ? kStallTestCycles : kTimeoutCycles;
    tc::fence_barrier_init();
    tc::prefetch_tensormap(&xmap);
    // The CTA's own group needs no free slot: start its copies now, so the DRAM
    // latency overlaps the rest of the setup; ask for the next group at once.
    S.gid[0] = blockIdx.x;
    tc::mbar_arrive(&S.gfull[0]);
    load_group<LOGN, KR>(smem + kOffX, &xmap, x, &S.full[0], blockIdx.x, tokens);
    first_issued = 1;
    clc_request(&S.clc_resp, &S.clc);
  }
  tc::grid_dep_launch();
  // H_128 (KRON: H_m (x) H_{b/128}, zero outside its KR x KR corner) as the A operand:
  // K-major, two K blocks of [128 rows m][64 k], 128-byte swizzle.
  auto a_entry = [&](uint32_t m, uint32_t k) -> uint32_t {  // bf16 pattern of A[m][k]
    if constexpr (SH::KRON) {
      if (m >= (uint32_t)KR || k >= (uint32_t)KR) return 0u;
      const uint32_t mask = (uint32_t)kp.bq - 1u;
      const int h = paley_entry((int)(m >> kp.lbq), (int)(k >> kp.lbq), kp) * ((__popc(m & k & mask) & 1) ? -1 : 1);
      return h > 0 ? 0x3F80u : 0xBF80u;
    } else if constexpr (SH::PAIR) {  // H_64 (+) H_64
      if ((m >> 6) != (k >> 6)) return 0u;
      return (__popc(m & k & 63u) & 1) ? 0xBF80u : 0x3F80u;
    } else {
      return (__popc(m & k) & 1) ? 0xBF80u : 0x3F80u;
    }
  };
  for (uint32_t c = threadIdx.x; c < 2048; c += kThreads) {
    const uint32_t kb = c >> 10, m = (c >> 3) & 127u, ch = c & 7u;
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t k0 = kb * 64 + ch * 8 + 2 * j;
      w[j] = a_entry(m, k0) | (a_entry(m, k0 + 1) << 16);
    }

    *reinterpret_cast<uint4 *>(smem + kOffH + kb * 16384 + sw128(m, ch)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  tc::fence_proxy_async_smem();
  if (warp == 1) {
    tc::tmem_alloc(&S.tmem_base, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  // ------------------------------------------------------------ roles
  if (warp == 0) {
    if (lane == 0) {
      int64_t last[kStages] = {-1, -1, -1};
      for (int64_t i = 0; i < first_issued; ++i) last[i] = i;
      bool pending = true;  // a work-stealing request is in flight
      uint32_t clc_phase = 0;
      for (int64_t i = first_issued;; ++i) {
        // the group of step i: the one the last request cancelled, or none
        int64_t p = -1;
        if (pending) {
          if (!wait_bounded(&S.clc, clc_phase, S, true)) break;
          clc_phase ^= 1u;
          p = clc_result(&S.clc_resp);
          if (p >= ngroups) p = -1;
          pending = p >= 0;
          if (pending) clc_request(&S.clc_resp, &S.clc);
        }
        const int st = (int)(i % kStages);
        if (!wait_bounded(&S.empty[st], (uint32_t)((i / kStages) & 1) ^ 1u, S, true)) break;
        S.gid[i % kRing] = p;
        tc::mbar_arrive(&S.gfull[i % kRing]);
        if (p < 0) {
          tc::mbar_arrive(&S.full[st]);  // no copies: the sign warps and the MMA read the end mark
          last[st] = -1;  // its previous copy was consumed before the slot came free
          break;
        }
        load_group<LOGN, KR>(smem + kOffX + st * kGroupBytes, &xmap, x, &S.full[st], p, tokens);
        last[st] = i;
      }
      // every issued copy (and work request) has landed before the CTA can leave
      for (int s = 0; s < kStages; ++s)
        if (last[s] >= 0) wait_bounded(&S.full[s], (uint32_t)((last[s] / kStages) & 1), S, false);
      if (pending) wait_bounded(&S.clc, clc_phase, S, false);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_bf16(128, SH::SPLIT ? 128 : 256, true);
      constexpr uint32_t idesc_neg = idesc | (1u << 13);  // negate A
      const uint32_t sH = tc::smem_u32(smem + kOffH), sX = tc::smem_u32(smem + kOffX);
      for (int64_t i = 0;; ++i) {
        const int st = (int)(i % kStages), acc = (int)(i & 1);
        if (!wait_bounded(SIGNS ? &S.sgn[st] : &S.full[st], (uint32_t)((i / kStages) & 1), S, true)) break;
        if (S.gid[i % kRing] < 0) break;
        if (!wait_bounded(&S.tempty[acc], (uint32_t)((i >> 1) & 1) ^ 1u, S, true)) break;
        tc::tc_fence_after();
        if constexpr (SH::SPLIT) {
          // columns 128 u + b: sum over row blocks v of (-1)^(u v) H_128 X_v
#pragma unroll
          for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int v = 0; v < 2; ++v)
#pragma unroll
              for (int s = 0; s < 8; ++s) {
                const uint64_t ad = tc::smem_desc(sH + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024);
                uint64_t bd = tc::smem_desc(sX + st * kGroupBytes + v * SH::CBOX * SH::BOXBYTES + s * 16 * SH::ROWB,
                                            SH::LBO, SH::SBO);
                bd = (bd & ~(7ull << 61)) | ((uint64_t)SH::LAYOUT << 61);
                tc::umma_bf16(tmem + acc * 256 + u * 128, ad, bd, (u & v) ? idesc_neg : idesc,
                              (v > 0 || s > 0) ? 1u : 0u);
              }
        } else {
#pragma unroll
          for (int s = 0; s < SH::KSTEPS; ++s) {
            // A: 16 columns k of H per step. B: rows a = 16 s .. 16 s + 15 of every box
            // (MN-major: boxes of BOXW columns BOXBYTES apart, 8-row groups 8 ROWB apart).
            const uint64_t ad = tc::smem_desc(sH + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024);
            uint64_t bd = tc::smem_desc(sX + st * kGroupBytes + s * 16 * SH::ROWB, SH::LBO, SH::SBO);
            bd = (bd & ~(7ull << 61)) | ((uint64_t)SH::LAYOUT << 61);
            tc::umma_bf16(tmem + acc * 256, ad, bd, idesc, s > 0 ? 1u : 0u);
          }
        }
        tc::umma_commit(&S.empty[st]);
        // Stall test hook: withhold the first group's completion signal, so the
        // epilogue's wait runs out and the CTA takes its abort path.
        if (!(stall_test && i == 0)) tc::umma_commit(&S.tfull[acc]);
      }
    }
  } else if (warp < 4) {
    if constexpr (SIGNS) {
      // Thread ts flips the signs of chunks ts + 64 j of each group's 64 KiB.
      // Those chunks sit at NPOS distinct positions of a token's tile; their
      // sign words stay in registers for the whole kernel.
      constexpr int NPOS = SH::NPOS;
      const uint32_t ts = threadIdx.x - 64;  // 0..63
      uint4 mk[NPOS];
#pragma unroll
      for (int k = 0; k < NPOS; ++k) {
        const uint32_t pos = ts + 64u * k;  // 16-byte chunk index inside one token's tile
        const uint32_t box = pos / (SH::BOXBYTES / 16), inbox = pos % (SH::BOXBYTES / 16);
        const uint32_t a = inbox / SH::CPR, pc = inbox % SH::CPR;
        const uint32_t ch = SH::ROWB == 128 ? (pc ^ (a & 7u))
                            : SH::ROWB == 64 ? (pc ^ ((a >> 1) & 3u))
                            : SH::ROWB == 32 ? (pc ^ ((a >> 2) & 1u))
                                             : pc;  // 16-byte rows: no swizzle
        const uint32_t e = a * B + box * SH::BOXW + ch * 8u;
        const uint32_t byte = (__ldg(signs + (e >> 5)) >> (e & 31u)) & 0xFFu;
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) w[j] = (((byte >> (2 * j)) & 1u) << 15) | (((byte >> (2 * j + 1)) & 1u) << 31);
        mk[k] = make_uint4(w[0], w[1], w[2], w[3]);
      }
      for (int64_t i = 0;; ++i) {
        const int st = (int)(i % kStages);
        if (ts == 0) {
          int ok = wait_bounded(&S.full[st], (uint32_t)((i / kStages) & 1), S, true) ? 1 : 0;
          if (ok && S.gid[i % kRing] < 0) {
            tc::mbar_arrive(&S.sgn[st]);  // pass the end mark on to the MMA
            ok = 0;
          }
          S.dec[2] = ok;
        }
        tc::named_sync(3, 64);
        if (!S.dec[2]) break;
        uint4 *X = reinterpret_cast<uint4 *>(smem + kOffX + st * kGroupBytes) + ts;
#pragma unroll
        for (int j0 = 0; j0 < SH::SIGN_ITERS; j0 += 4) {
          uint4 x[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) x[u] = X[64 * (j0 + u)];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint4 m = mk[(j0 + u) % NPOS];
            X[64 * (j0 + u)] = make_uint4(x[u].x ^ m.x, x[u].y ^ m.y, x[u].z ^ m.z, x[u].w ^ m.w);
          }
        }
        tc::fence_proxy_async_smem();
        tc::named_sync(3, 64);
        if (ts == 0) tc::mbar_arrive(&S.sgn[st]);
      }
    }
  } else {
    // epilogue warpgroup g: warps 4..7 (g = 0) and 8..11 (g = 1)
    const uint32_t g = (warp - 4) >> 2, wq = warp & 3u, tg = threadIdx.x - 128 - 128 * g;
    const uint32_t row = wq * 32 + lane;  // a' = TMEM lane
    // With one token segment per thread and no diagonal, each thread waits for the
    // step's group and accumulator itself, and the warpgroup meets once per step instead
    // of twice (6 to 9 % less time per launch at n = 16384 on a B200). Elsewhere one
    // thread decides for its warpgroup: with several segments the extra meeting costs
    // nothing measurable, and with a diagonal the sign warps set the pace.
    constexpr bool kOwnWaits = SEG == 1 && !SIGNS;
    for (int64_t i = 0;; ++i) {
      const int acc = (int)(i & 1);
      int64_t p = -1;
      bool have;
      if constexpr (kOwnWaits) {
        const bool ok = wait_bounded(&S.gfull[i % kRing], (uint32_t)((i / kRing) & 1), S, true);
        if (ok) p = S.gid[i % kRing];
        have = ok && p >= 0 && wait_bounded(&S.tfull[acc], (uint32_t)((i >> 1) & 1), S, true);
      } else {
        // the step's group from the producer's ring, then its accumulator
        auto decide = [&](int slot) {
          int ok = wait_bounded(&S.gfull[i % kRing], (uint32_t)((i / kRing) & 1), S, true) ? 1 : 0;
          const int64_t gp = ok ? S.gid[i % kRing] : -1;
          if (gp < 0) ok = 0;
          if (ok) ok = wait_bounded(&S.tfull[acc], (uint32_t)((i >> 1) & 1), S, true) ? 1 : 0;
          S.egid[slot] = gp;
          S.dec[slot] = ok;
        };
        if constexpr (SH::SPLIT) {  // one decision for both warpgroups: they meet at barrier 4 below
          if (threadIdx.x == 128) decide(0);
          tc::named_sync(4, 256);
          if (!S.dec[0]) break;
          p = S.egid[0];
        } else {
          if (tg == 0) decide(g);
          tc::named_sync(1 + g, 128);
          if (!S.dec[g]) break;
          p = S.egid[g];
        }
        have = true;
      }
      float v[kRegs];
      if (have) {
        tc::tc_fence_after();
        {
          uint32_t r[kRegs];
          const uint32_t taddr = tmem + ((wq * 32u) << 16) + (uint32_t)acc * 256u + g * 128u;
          tc::tmem_ld32(taddr, r);
          tc::tmem_ld32(taddr + 32, r + 32);
          tc::tmem_ld32(taddr + 64, r + 64);
          tc::tmem_ld32(taddr + 96, r + 96);
          tc::tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < kRegs; ++k) v[k] = __uint_as_float(r[k]);
        }
        tc::tc_fence_before();
        tc::mbar_arrive(&S.tempty[acc]);
        // second Kronecker factor: H_B over b inside each token segment, in registers
        stage<0>(v);
        stage<1>(v);
        stage<2>(v);
        if constexpr (SH::LOGB > 3) stage<3>(v);
        if constexpr (SH::LOGB > 4) stage<4>(v);
        if constexpr (SH::LOGB > 5) stage<5>(v);
        if constexpr (SH::LOGB > 6) stage<6>(v);
        // per-token max |u|: a tree of three-input maxima per segment, then the warp, then the warpgroup
#pragma unroll
        for (int sg = 0; sg < SEG; ++sg) {
          float mx[B / 8];
#pragma unroll
          for (int k = 0; k < B / 8; ++k) {
            const float *w = v + sg * B + 8 * k;
            mx[k] = fmax3(fmax3(fabsf(w[0]), fabsf(w[1]), fabsf(w[2])), fmax3(fabsf(w[3]), fabsf(w[4]), fabsf(w[5])),
                          fmaxf(fabsf(w[6]), fabsf(w[7])));
          }
#pragma unroll
          for (int h = B / 16; h >= 1; h >>= 1)
#pragma unroll
            for (int k = 0; k < h; ++k) mx[k] = fmaxf(mx[k], mx[k + h]);
          const uint32_t wm = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(mx[0]));
          if (lane == 0) S.wmax[g][i & 1][wq][sg] = __uint_as_float(wm);
        }
      }
      // The warpgroup (both, for one n = 32768 token) meets here on every step; with
      // their own waits, its threads all leave when any of them has no group to finish.
      if constexpr (kOwnWaits) {
        if (!(SH::SPLIT ? bar_red_and(4, 256, have) : bar_red_and(1 + g, 128, have))) break;
      } else if constexpr (SH::SPLIT) {
        tc::named_sync(4, 256);
      } else {
        tc::named_sync(1 + g, 128);
      }
#pragma unroll
      for (int sg = 0; sg < SEG; ++sg) {
        float mu;
        if constexpr (SH::PAIR)  // the token of this thread's row: warps 0-1 or 2-3
          mu = fmaxf(S.wmax[g][i & 1][wq & 2u][sg], S.wmax[g][i & 1][(wq & 2u) + 1][sg]);
        else
          mu = fmaxf(fmaxf(S.wmax[g][i & 1][0][sg], S.wmax[g][i & 1][1][sg]),
                     fmaxf(S.wmax[g][i & 1][2][sg], S.wmax[g][i & 1][3][sg]));
        if constexpr (SH::SPLIT)
          mu = fmaxf(mu, fmaxf(fmaxf(S.wmax[g ^ 1][i & 1][0][0], S.wmax[g ^ 1][i & 1][1][0]),
                               fmaxf(S.wmax[g ^ 1][i & 1][2][0], S.wmax[g ^ 1][i & 1][3][0])));
        // step = max(clip m / qmax, 1e-8) (m in the transform's units times 1/sqrt(n)), and
        // 1 / step for the codes; a few ulp from the correctly rounded forms, far inside
        // the step tolerance, and the codes' pre-round values move by ~1e-7 of a step
        const float s = fmaxf(mu * step_per_unit, 1e-8f);
        const uint64_t cq = pair(inv_sqrt_n * rcp_approx(s));
        const int64_t token = SH::SPLIT ? p
                              : SH::PAIR ? p * SH::TOK + 2 * (g * SEG + sg) + (row >> 6)
                                         : p * SH::TOK + g * SEG + sg;
        if (token >= tokens) continue;
        if (SH::KRON && row >= (uint32_t)KR) continue;  // TMEM lanes past the tile's rows hold zeros
        const uint32_t orow = SH::SPLIT ? 128u * g + row : SH::PAIR ? (row & 63u) : row;  // output row of B values
        uint8_t *dst = q + token * (SH::OUTB * (BITS / 4)) + orow * (B * BITS / 8);
        if constexpr (BITS == 8 && B == 8) {  // 8 code bytes per row segment
          uint32_t w2[2];
          codes8_int8(v + sg * B, cq, w2[0], w2[1]);
          __stcs(reinterpret_cast<uint2 *>(dst), make_uint2(w2[0], w2[1]));
        } else if constexpr (BITS == 4 && B == 8) {  // 4 code bytes per row segment
          __stcs(reinterpret_cast<unsigned int *>(dst), codes8(v + sg * B, cq));
        } else if constexpr (BITS == 8 && B == 16) {  // 16 code bytes per row segment
          uint32_t w4[4];
          codes8_int8(v + sg * B, cq, w4[0], w4[1]);
          codes8_int8(v + sg * B + 8, cq, w4[2], w4[3]);
          __stcs(reinterpret_cast<uint4 *>(dst), make_uint4(w4[0], w4[1], w4[2], w4[3]));
        } else if constexpr (BITS == 8) {
          // one code byte per value: 32 bytes (8 words) at a time
#pragma unroll
          for (int c8 = 0; c8 < B / 32; ++c8) {
            uint32_t w8[8];
#pragma unroll
            for (int h = 0; h < 4; ++h) codes8_int8(v + sg * B + 32 * c8 + 8 * h, cq, w8[2 * h], w8[2 * h + 1]);
            if constexpr (STORE32) {
              st_v8_cs(dst + 32 * c8, w8);
            } else {
              __stcs(reinterpret_cast<uint4 *>(dst + 32 * c8), make_uint4(w8[0], w8[1], w8[2], w8[3]));
              __stcs(reinterpret_cast<uint4 *>(dst + 32 * c8) + 1, make_uint4(w8[4], w8[5], w8[6], w8[7]));
            }
          }
        } else {
          uint32_t words[B / 8];
#pragma unroll
          for (int wi = 0; wi < B / 8; ++wi) words[wi] = codes8(v + sg * B + 8 * wi, cq);
          if constexpr (B == 16) {  // 8 code bytes per row segment
            __stcs(reinterpret_cast<uint2 *>(dst), make_uint2(words[0], words[1]));
          } else if constexpr (STORE32 && B >= 64) {
#pragma unroll
            for (int w8 = 0; w8 < B / 64; ++w8) st_v8_cs(dst + 32 * w8, words + 8 * w8);
          } else {
#pragma unroll
            for (int w4 = 0; w4 < B / 32; ++w4)
              __stcs(reinterpret_cast<uint4 *>(dst) + w4,
                     make_uint4(words[4 * w4], words[4 * w4 + 1], words[4 * w4 + 2], words[4 * w4 + 3]));
          }
        }
        if ((SH::PAIR ? (tg & 63u) : tg) == 0 && (!SH::SPLIT || g == 0)) scales[token] = s;
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
    tc::tmem_dealloc(tmem, 512);
  }
}

template <int LOGN, int KR, bool SIGNS, bool STORE32, int BITS>
cudaError_t launch_tc(const void *x, int64_t tokens, float clip, const uint32_t *signs, uint8_t *q, float *scales,
                      cudaStream_t stream, int stall_test, const KronParams &kp) {
  using SH = Shape<LOGN, KR>;
  auto fn = tensor_map_encoder();
  if (!fn) return cudaErrorNotSupported;
  CUtensorMap map;
  const cuuint64_t dims[2] = {(cuuint64_t)SH::B, (cuuint64_t)tokens * SH::ROWS};
  const cuuint64_t strides[1] = {(cuuint64_t)SH::B * 2};
  const cuuint32_t box[2] = {(cuuint32_t)SH::BOXW, (cuuint32_t)SH::BOXH};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(x), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  SH::ROWB == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                  : SH::ROWB == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                  : SH::ROWB == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                   : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  auto kern = k1_tc_rotate_quant<LOGN, KR, SIGNS, STORE32, BITS>;
  int slots = 0;
  cudaError_t err = resident_slots(reinterpret_cast<const void *>(kern), kThreads, (int)kSmemBytes, &slots);
  if (err != cudaSuccess) return err;
  // One CTA per group: the resident ones take the groups of CTAs that have not started
  // yet (cluster launch control), so the groups spread over the SMs as they free up.
  const int64_t grid = (tokens + SH::TOK - 1) / SH::TOK;
  const float inv_sqrt_n = (float)(1.0 / std::sqrt((double)SH::ROWS * SH::B));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, map, static_cast<const uint16_t *>(x), tokens, clip, inv_sqrt_n, signs, q,
                            scales, stall_test, kp);
}

template <int LOGN, int BITS>
cudaError_t launch_n(const void *x, int64_t tokens, float clip, const uint32_t *signs, uint8_t *q, float *scales,
                     cudaStream_t stream, int stall_test) {
  const bool a32 = (reinterpret_cast<uintptr_t>(q) & 31u) == 0;  // 32-byte stores need 32-byte alignment
  const KronParams none = {};
  if constexpr (Shape<LOGN>::SPLIT) {
    if (signs) return cudaErrorInvalidValue;
  } else if (signs) {
    return a32 ? launch_tc<LOGN, 0, true, true, BITS>(x, tokens, clip, signs, q, scales, stream, stall_test, none)
               : launch_tc<LOGN, 0, true, false, BITS>(x, tokens, clip, signs, q, scales, stream, stall_test, none);
  }
  return a32 ? launch_tc<LOGN, 0, false, true, BITS>(x, tokens, clip, nullptr, q, scales, stream, stall_test, none)
             : launch_tc<LOGN, 0, false, false, BITS>(x, tokens, clip, nullptr, q, scales, stream, stall_test, none);
}

// n = 128 KR: 16-byte code stores (the output need only be 16-byte aligned), with or
// without the diagonal.
template <int KR, int BITS>
cudaError_t launch_kron_rows(const void *x, int64_t tokens, float clip, const uint32_t *signs, uint8_t *q,
                             float *scales, cudaStream_t stream, int stall_test, const KronParams &kp) {
  return signs ? launch_tc<14, KR, true, false, BITS>(x, tokens, clip, signs, q, scales, stream, stall_test, kp)
               : launch_tc<14, KR, false, false, BITS>(x, tokens, clip, nullptr, q, scales, stream, stall_test, kp);
}

// ============================================================================ n = 128, 256
// Tokens as the MMA's M. A token row of n = 128 V (V = 1, 2) is V chunks x_v of 128
// and H_n D x = [sum_v (-1)^(u v) H_128 D_v x_v]_u. The MMA computes, for 128 tokens
// at once, Y_v[t][a'] = sum_a X_v[t][a] B_v[a][a'] with A = X_v (K-major, as TMA loads
// it) and B_v = D_v H_128 (the diagonal folded into the constant operand, so it costs
// nothing per token); at n = 256 the epilogue forms the halves Y_0 + Y_1 and Y_0 - Y_1.
// Each epilogue thread owns one token (one TMEM lane): max, step and codes with no
// butterflies and no cross-thread reduction.
//   warp 0      TMA producer: four [128 token][64 element] boxes per group (64 KiB)
//   warp 1      TMEM owner and MMA issuer; two accumulators of 256 columns
//   warps 2-9   epilogue, two warpgroups: n = 128, warpgroup g takes token tile g of
//               every group; n = 256, warpgroup g takes the groups on accumulator g
//               and reads it twice (maximum first, codes second)
constexpr int kThreadsS = 320;

template <int NB>
struct SmallLayout {
  static constexpr int kStages = NB == 2 ? 2 : 3;
  static constexpr uint32_t kOffB = 0;  // B operand(s): 32 KiB each
  static constexpr uint32_t kOffX = 32768u * NB;
  static constexpr uint32_t kOffBar = kOffX + kStages * kGroupBytes;
  static constexpr uint32_t kSmemBytes = kOffBar + 1024 + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory per block");
};

template <int ST>
struct SharedS {
  uint64_t full[ST], empty[ST], tfull[2], tempty[2], drain;
  uint32_t tmem_base;
  int abort;
  int dec[2];
  long long budget;
};

__device__ __forceinline__ float absmax32(const uint32_t *r, float m) {
#pragma unroll
  for (int k = 0; k < 32; ++k) m = fmaxf(m, fabsf(__uint_as_float(r[k])));
  return m;
}

template <int V, bool SIGNS, bool STORE32, int BITS>
__global__ void __launch_bounds__(kThreadsS, 1)
    k1_tcs_rotate_quant(const __grid_constant__ CUtensorMap xmap, int64_t tokens, float clip, float inv_sqrt_n,
                        const uint32_t *__restrict__ signs, uint8_t *__restrict__ q, float *__restrict__ scales) {
  constexpr int TOKG = 256 / V;  // tokens per group
  constexpr int NB = (SIGNS && V == 2) ? 2 : 1;
  using L = SmallLayout<NB>;
  constexpr int ST = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  SharedS<ST> &S = *reinterpret_cast<SharedS<ST> *>(smem + L::kOffBar);
  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31u;
  const int64_t ngroups = (tokens + TOKG - 1) / TOKG;
  auto issue = [&](int st, int64_t p) {  // four boxes of group p into stage st
    tc::mbar_arrive_expect_tx(&S.full[st], kGroupBytes);
    uint8_t *dst = smem + L::kOffX + st * kGroupBytes;
#pragma unroll
    for (int b4 = 0; b4 < 4; ++b4) {  // box b4 = 2 t + (k >= 64): operand t, K half
      const int x = V == 1 ? 64 * (b4 & 1) : 64 * b4;
      const int y = (int)(p * TOKG) + (V == 1 ? 128 * (b4 >> 1) : 0);
      tc::tma_load_2d(dst + b4 * 16384, &xmap, &S.full[st], x, y);
    }
  };

  tc::grid_dep_wait();
  int first_issued = 0;
  if (threadIdx.x == 0) {
    for (int s2 = 0; s2 < ST; ++s2) {
      tc::mbar_init(&S.full[s2], 1);
      tc::mbar_init(&S.empty[s2], 1);
    }
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(&S.tfull[a], 1);
      tc::mbar_init(&S.tempty[a], V == 1 ? 256 : 128);
    }
    tc::mbar_init(&S.drain, 1);
    S.abort = 0;
    S.budget = kTimeoutCycles;
    tc::fence_barrier_init();
    tc::prefetch_tensormap(&xmap);
    for (int i = 0; i < ST; ++i) {
      const int64_t p = blockIdx.x + i * (int64_t)gridDim.x;
      if (p >= ngroups) break;
      issue(i, p);
      first_issued = i + 1;
    }
  }
  tc::grid_dep_launch();
  // B_v = D_v H_128 as the K-major B operand [n = a'][k = a]: entry d_v[a] H[a'][a]
  for (uint32_t c = threadIdx.x; c < 2048u * NB; c += kThreadsS) {
    const uint32_t v = c >> 11, kb = (c >> 10) & 1u, m = (c >> 3) & 127u, ch = c & 7u;
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t k0 = kb * 64 + ch * 8 + 2 * j;
      uint32_t lo = (__popc(m & k0) & 1) ? 0xBF80u : 0x3F80u;
      uint32_t hi = (__popc(m & (k0 + 1)) & 1) ? 0xBF80u : 0x3F80u;
      if constexpr (SIGNS) {
        const uint32_t e0 = 128u * v + k0;
        lo ^= ((__ldg(signs + (e0 >> 5)) >> (e0 & 31u)) & 1u) << 15;
        hi ^= ((__ldg(signs + ((e0 + 1) >> 5)) >> ((e0 + 1) & 31u)) & 1u) << 15;
      }
      w[j] = lo | (hi << 16);
    }
    *reinterpret_cast<uint4 *>(smem + L::kOffB + v * 32768u + kb * 16384u + sw128(m, ch)) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
  tc::fence_proxy_async_smem();
  if (warp == 1) {
    tc::tmem_alloc(&S.tmem_base, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      int64_t last[ST];
      for (int s2 = 0; s2 < ST; ++s2) last[s2] = s2 < first_issued ? s2 : -1;
      for (int64_t i = first_issued;; ++i) {
        const int64_t p = blockIdx.x + i * (int64_t)gridDim.x;
        if (p >= ngroups) break;
        const int st = (int)(i % ST);
        if (!wait_bounded(&S.empty[st], (uint32_t)((i / ST) & 1) ^ 1u, S, true)) break;
        issue(st, p);
        last[st] = i;
      }
      for (int s2 = 0; s2 < ST; ++s2)
        if (last[s2] >= 0) wait_bounded(&S.full[s2], (uint32_t)((last[s2] / ST) & 1), S, false);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_bf16(128, 128, false);  // A and B K-major
      const uint32_t sB = tc::smem_u32(smem + L::kOffB), sX = tc::smem_u32(smem + L::kOffX);
      for (int64_t i = 0;; ++i) {
        const int64_t p = blockIdx.x + i * (int64_t)gridDim.x;
        if (p >= ngroups) break;
        const int st = (int)(i % ST), acc = (int)(i & 1);
        if (!wait_bounded(&S.full[st], (uint32_t)((i / ST) & 1), S, true)) break;
        if (!wait_bounded(&S.tempty[acc], (uint32_t)((i >> 1) & 1) ^ 1u, S, true)) break;
        tc::tc_fence_after();
#pragma unroll
        for (int t = 0; t < 2; ++t)  // V = 1: token tile t; V = 2: input chunk t
#pragma unroll
          for (int s2 = 0; s2 < 8; ++s2) {
            const uint32_t xa = sX + st * kGroupBytes + (2 * t + (s2 >> 2)) * 16384 + (s2 & 3) * 32;
            const uint32_t ba = sB + (NB == 2 ? t * 32768 : 0) + (s2 >> 2) * 16384 + (s2 & 3) * 32;
            tc::umma_bf16(tmem + acc * 256 + t * 128, tc::smem_desc(xa, 16, 1024), tc::smem_desc(ba, 16, 1024),
                          idesc, s2 > 0 ? 1u : 0u);
          }
        tc::umma_commit(&S.empty[st]);
        tc::umma_commit(&S.tfull[acc]);
      }
    }
  } else {
    const uint32_t g = (warp - 2) >> 2, tg = threadIdx.x - 64 - 128 * g;
    const uint32_t row = (warp & 3u) * 32 + lane;
    const uint32_t lane_base = tmem + (((warp & 3u) * 32u) << 16);
    for (int64_t i = (V == 1 ? 0 : g);; i += (V == 1 ? 1 : 2)) {
      const int64_t p = blockIdx.x + i * (int64_t)gridDim.x;
      if (p >= ngroups) break;
      const int acc = (int)(i & 1);
      if (tg == 0) S.dec[g] = wait_bounded(&S.tfull[acc], (uint32_t)((i >> 1) & 1), S, true) ? 1 : 0;
      tc::named_sync(1 + g, 128);
      if (!S.dec[g]) break;
      tc::tc_fence_after();
      const int64_t token = p * TOKG + (V == 1 ? 128 * g : 0) + row;
      const bool live = token < tokens;
      constexpr float QMAX = BITS == 4 ? 7.0f : 127.0f;
      const float step_per_unit = clip * inv_sqrt_n / QMAX;
      uint8_t *dst = q + token * (int64_t)(16 * V * BITS);
      // 32 code bytes at dst + off: one 32-byte store when aligned, else two 16-byte ones
      auto put32 = [&](int off, const uint32_t *w) {
        if constexpr (STORE32) {
          st_v8_cs(dst + off, w);
        } else {
          __stcs(reinterpret_cast<uint4 *>(dst + off), make_uint4(w[0], w[1], w[2], w[3]));
          __stcs(reinterpret_cast<uint4 *>(dst + off) + 1, make_uint4(w[4], w[5], w[6], w[7]));
        }
      };
      float s;
      if constexpr (V == 1) {
        uint32_t r[128];
        const uint32_t taddr = lane_base + (uint32_t)acc * 256u + g * 128u;
        tc::tmem_ld32(taddr, r);
        tc::tmem_ld32(taddr + 32, r + 32);
        tc::tmem_ld32(taddr + 64, r + 64);
        tc::tmem_ld32(taddr + 96, r + 96);
        tc::tmem_wait_ld();
        tc::tc_fence_before();
        tc::mbar_arrive(&S.tempty[acc]);
        float mu = 0.0f;
#pragma unroll
        for (int c = 0; c < 4; ++c) mu = absmax32(r + 32 * c, mu);
        s = fmaxf(mu * step_per_unit, 1e-8f);  // as in the large-n kernel
        const uint64_t cq = pair(inv_sqrt_n * rcp_approx(s));
        if constexpr (BITS == 8) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t w8[8];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              float f[8];
#pragma unroll
              for (int k = 0; k < 8; ++k) f[k] = __uint_as_float(r[32 * c + 8 * h + k]);
              codes8_int8(f, cq, w8[2 * h], w8[2 * h + 1]);
            }
            if (live) put32(32 * c, w8);
          }
        } else {
          uint32_t words[16];
#pragma unroll
          for (int wi = 0; wi < 16; ++wi) {
            float f[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) f[k] = __uint_as_float(r[8 * wi + k]);
            words[wi] = codes8(f, cq);
          }
          if (live) {
#pragma unroll
            for (int w8 = 0; w8 < 2; ++w8) {
              if constexpr (STORE32) {
                st_v8_cs(dst + 32 * w8, words + 8 * w8);
              } else {
                __stcs(reinterpret_cast<uint4 *>(dst + 32 * w8),
                       make_uint4(words[8 * w8], words[8 * w8 + 1], words[8 * w8 + 2], words[8 * w8 + 3]));
                __stcs(reinterpret_cast<uint4 *>(dst + 32 * w8) + 1,
                       make_uint4(words[8 * w8 + 4], words[8 * w8 + 5], words[8 * w8 + 6], words[8 * w8 + 7]));
              }
            }
          }
        }
      } else {
        const uint32_t taddr = lane_base + (uint32_t)acc * 256u;
        float mu = 0.0f;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {  // pass 1: |Y0 + Y1| and |Y0 - Y1|
          uint32_t a[32], b[32];
          tc::tmem_ld32(taddr + 32 * c, a);
          tc::tmem_ld32(taddr + 128 + 32 * c, b);
          tc::tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const float y0 = __uint_as_float(a[k]), y1 = __uint_as_float(b[k]);
            mu = fmax3(mu, fabsf(y0 + y1), fabsf(y0 - y1));
          }
        }
        s = fmaxf(mu * step_per_unit, 1e-8f);  // as in the large-n kernel
        const uint64_t cq = pair(inv_sqrt_n * rcp_approx(s));
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {  // pass 2: codes of outputs 32c.. of both halves
          uint32_t a[32], b[32];
          if constexpr (BITS == 8) {
            uint32_t w0[8], w1[8];
            tc::tmem_ld32(taddr + 32 * c, a);
            tc::tmem_ld32(taddr + 128 + 32 * c, b);
            tc::tmem_wait_ld();
#pragma unroll
            for (int wi = 0; wi < 4; ++wi) {
              float f0[8], f1[8];
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                const float y0 = __uint_as_float(a[8 * wi + k]), y1 = __uint_as_float(b[8 * wi + k]);
                f0[k] = y0 + y1;
                f1[k] = y0 - y1;
              }
              codes8_int8(f0, cq, w0[2 * wi], w0[2 * wi + 1]);
              codes8_int8(f1, cq, w1[2 * wi], w1[2 * wi + 1]);
            }
            if (live) {
              put32(32 * c, w0);
              put32(128 + 32 * c, w1);
            }
          } else {
            uint32_t w0[4], w1[4];
            tc::tmem_ld32(taddr + 32 * c, a);
            tc::tmem_ld32(taddr + 128 + 32 * c, b);
            tc::tmem_wait_ld();
#pragma unroll
            for (int wi = 0; wi < 4; ++wi) {
              float f0[8], f1[8];
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                const float y0 = __uint_as_float(a[8 * wi + k]), y1 = __uint_as_float(b[8 * wi + k]);
                f0[k] = y0 + y1;
                f1[k] = y0 - y1;
              }
              w0[wi] = codes8(f0, cq);
              w1[wi] = codes8(f1, cq);
            }
            if (live) {
              __stcs(reinterpret_cast<uint4 *>(dst + 16 * c), make_uint4(w0[0], w0[1], w0[2], w0[3]));
              __stcs(reinterpret_cast<uint4 *>(dst + 64 + 16 * c), make_uint4(w1[0], w1[1], w1[2], w1[3]));
            }
          }
        }
        tc::tc_fence_before();
        tc::mbar_arrive(&S.tempty[acc]);
      }
      if (live) scales[token] = s;
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) {
      tc::umma_commit(&S.drain);
      wait_bounded(&S.drain, 0, S, false);
    }
    __syncwarp();
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

template <int V, bool SIGNS, bool STORE32, int BITS>
cudaError_t launch_tcs(const void *x, int64_t tokens, float clip, const uint32_t *signs, uint8_t *q, float *scales,
                       cudaStream_t stream) {
  auto fn = tensor_map_encoder();
  if (!fn) return cudaErrorNotSupported;
  CUtensorMap map;
  const cuuint64_t dims[2] = {(cuuint64_t)(128 * V), (cuuint64_t)tokens};
  const cuuint64_t strides[1] = {(cuuint64_t)(256 * V)};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(x), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  auto kern = k1_tcs_rotate_quant<V, SIGNS, STORE32, BITS>;
  constexpr uint32_t smem_bytes = SmallLayout<(SIGNS && V == 2) ? 2 : 1>::kSmemBytes;
  int slots = 0;
  cudaError_t err = resident_slots(reinterpret_cast<const void *>(kern), kThreadsS, (int)smem_bytes, &slots);
  if (err != cudaSuccess) return err;
  const int64_t ngroups = (tokens + 256 / V - 1) / (256 / V);
  const int64_t grid = ngroups < slots ? ngroups : slots;
  const float inv_sqrt_n = (float)(1.0 / std::sqrt((double)(128 * V)));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreadsS);
  cfg.dynamicSmemBytes = smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, map, tokens, clip, inv_sqrt_n, signs, q, scales);
}

template <int V, int BITS>
cudaError_t launch_small(const void *x, int64_t tokens, float clip, const uint32_t *signs, uint8_t *q, float *scales,
                         cudaStream_t stream) {
  // 32-byte stores need 32-byte alignment; INT4 at n = 256 stores 16-byte pieces
  constexpr bool W = V == 1 || BITS == 8;
  const bool a32 = W && (reinterpret_cast<uintptr_t>(q) & 31u) == 0;
  if (signs)
    return a32 ? launch_tcs<V, true, W, BITS>(x, tokens, clip, signs, q, scales, stream)
               : launch_tcs<V, true, false, BITS>(x, tokens, clip, signs, q, scales, stream);
  return a32 ? launch_tcs<V, false, W, BITS>(x, tokens, clip, nullptr, q, scales, stream)
             : launch_tcs<V, false, false, BITS>(x, tokens, clip, nullptr, q, scales, stream);
}

std::atomic<int> g_stall_test{0};

template <int BITS>
cudaError_t launch_tc_bits(int log_n, const void *x, int64_t tokens, float clip, const uint32_t *signs, uint8_t *q,
                           float *scales, cudaStream_t stream, int stall) {
  switch (log_n) {
    case 7: return launch_small<1, BITS>(x, tokens, clip, signs, q, scales, stream);
    case 8: return launch_small<2, BITS>(x, tokens, clip, signs, q, scales, stream);
    case 9: return launch_n<9, BITS>(x, tokens, clip, signs, q, scales, stream, stall);
    case 10: return launch_n<10, BITS>(x, tokens, clip, signs, q, scales, stream, stall);
    case 11: return launch_n<11, BITS>(x, tokens, clip, signs, q, scales, stream, stall);
    case 12: return launch_n<12, BITS>(x, tokens, clip, signs, q, scales, stream, stall);
    case 13: return launch_n<13, BITS>(x, tokens, clip, signs, q, scales, stream, stall);
    case 14: return launch_n<14, BITS>(x, tokens, clip, signs, q, scales, stream, stall);
    case 15: return launch_n<15, BITS>(x, tokens, clip, signs, q, scales, stream, stall);
    default: return cudaErrorInvalidValue;
  }
}

template <int BITS>
cudaError_t launch_kron_bits(int rows, const void *x, int64_t tokens, float clip, const uint32_t *signs, uint8_t *q,
                             float *scales, cudaStream_t stream, int stall, const KronParams &kp) {
  switch (rows) {
    case 16: return launch_kron_rows<16, BITS>(x, tokens, clip, signs, q, scales, stream, stall, kp);
    case 32: return launch_kron_rows<32, BITS>(x, tokens, clip, signs, q, scales, stream, stall, kp);
    case 48: return launch_kron_rows<48, BITS>(x, tokens, clip, signs, q, scales, stream, stall, kp);
    case 64: return launch_kron_rows<64, BITS>(x, tokens, clip, signs, q, scales, stream, stall, kp);
    case 80: return launch_kron_rows<80, BITS>(x, tokens, clip, signs, q, scales, stream, stall, kp);
    case 96: return launch_kron_rows<96, BITS>(x, tokens, clip, signs, q, scales, stream, stall, kp);
    case 112: return launch_kron_rows<112, BITS>(x, tokens, clip, signs, q, scales, stream, stall, kp);
    case 128: return launch_kron_rows<128, BITS>(x, tokens, clip, signs, q, scales, stream, stall, kp);
    default: return cudaErrorInvalidValue;
  }
}

bool is_prime(int v) {
  if (v < 2) return false;
  for (int d = 2; d * d <= v; ++d)
    if (v % d == 0) return false;
  return true;
}

}  // namespace

// Paley's construction applies to m when q = m - 1 is a prime = 3 mod 4 (type I) or
// q = m/2 - 1 is a prime = 1 mod 4 (type II); type I is taken when both do.
int paley_type(int m) {
  if (m >= 4 && (m - 1) % 4 == 3 && is_prime(m - 1)) return 1;
  if (m >= 12 && m % 4 == 0 && (m / 2 - 1) % 4 == 1 && is_prime(m / 2 - 1)) return 2;
  return 0;
}

bool kron_supported(int m, int64_t n) {
  if (!paley_type(m) || n <= 0 || n % m != 0) return false;
  const int64_t b = n / m;
  if (b < 128 || (b & (b - 1)) != 0) return false;
  const int64_t rows = n / 128;
  return rows >= 16 && rows <= 128 && rows % 16 == 0;
}

cudaError_t launch_rotate_quant_kron(int m, int n, int bits, const void *x, int64_t tokens, float clip,
                                     const uint32_t *signs, uint8_t *q, float *scales, cudaStream_t stream) {
  if (!kron_supported(m, n)) return cudaErrorInvalidValue;
  KronParams kp = {};
  kp.m = m;
  kp.type = paley_type(m);
  kp.q = kp.type == 1 ? m - 1 : m / 2 - 1;
  kp.bq = (n / m) / 128;  // a power of two: n / m = 2^k with 2^k >= 128
  while ((1 << kp.lbq) < kp.bq) ++kp.lbq;
  for (int a = 1; a < kp.q; ++a) {  // the nonzero squares mod q
    const int sq = (a * a) % kp.q;
    kp.qr[sq >> 5] |= 1u << (sq & 31);
  }
  const int rows = n / 128;
  const int stall = g_stall_test.load(std::memory_order_relaxed);
  if (bits == 4) return launch_kron_bits<4>(rows, x, tokens, clip, signs, q, scales, stream, stall, kp);
  if (bits == 8) return launch_kron_bits<8>(rows, x, tokens, clip, signs, q, scales, stream, stall, kp);
  return cudaErrorInvalidValue;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// The tensor-core kernel pays a per-CTA setup (H tile, TMEM, first copies) that
// only pays off with at least about one MMA group per SM; smaller batches (decode)
// go to the CUDA-core kernel, which needs no setup.
bool tc_rotate_quant_supported(int log_n, int64_t tokens, uint32_t flags, bool has_signs) {
  if ((flags & kNoRotate) || tokens <= 0) return false;
  if (log_n == 7 || log_n == 8) {  // tokens as M: 256 / V tokens per group
    if (tokens >= (int64_t(1) << 31)) return false;
    const int64_t tok_per_group = log_n == 7 ? 256 : 128;
    return (flags & kTensorCores) || tokens >= 128 * tok_per_group;
  }
  if (log_n < 9 || log_n > 15) return false;
  if (log_n == 15 && has_signs) return false;  // its sign masks do not fit the sign warps' registers
  const int64_t rows_per_token = log_n == 15 ? 256 : log_n == 9 ? 64 : 128;
  if (tokens * rows_per_token >= (int64_t(1) << 31)) return false;
  // tokens per MMA group: one at n = 32768, 256 / (n / 128) below, 64 at n = 512 (two per box)
  const int64_t tok_per_group = log_n == 15 ? 1 : int64_t(256) >> (log_n - 7);
  return (flags & kTensorCores) || tokens >= 128 * tok_per_group;
}

cudaError_t launch_rotate_quant_tc(int log_n, int bits, const void *x, int64_t tokens, float clip,
                                   const uint32_t *signs, uint8_t *q, float *scales, cudaStream_t stream) {
  const int stall = g_stall_test.load(std::memory_order_relaxed);
  if (bits == 4) return launch_tc_bits<4>(log_n, x, tokens, clip, signs, q, scales, stream, stall);
  if (bits == 8) return launch_tc_bits<8>(log_n, x, tokens, clip, signs, q, scales, stream, stall);
  return cudaErrorInvalidValue;
}

void set_stall_test(int enable) { g_stall_test.store(enable ? 1 : 0, std::memory_order_relaxed); }

cudaError_t read_device_status(unsigned int *status, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(status, g_device_status, sizeof(unsigned int));
  if (e != cudaSuccess || !reset) return e;
  const unsigned int zero = 0u;
  return cudaMemcpyToSymbol(g_device_status, &zero, sizeof(unsigned int));
}

}  // namespace spin
