// k3_tc.cu -- dequantise + inverse rotation on the tensor cores: for n = 512 to
// 32768 the first Kronecker factor runs on tcgen05 (below; at n = 512 two 64-row
// token rows share a tile and the factor is H_64 (+) H_64); for n = 128 and 256
// the whole transform does (rows as the MMA's M, further down).
//
// "Rotations: QuaRot, SpinQuant and incoherence", widget "Try it": rotate,
// quantize, rotate back; section "Hadamard matrices": H_n / sqrt(n) is
// orthogonal and symmetric, so D H_n / sqrt(n) undoes H_n D / sqrt(n), and the
// Sylvester H_n is a Kronecker product of smaller Sylvester matrices.
// "SpinQuant Guide: Learned Rotations for 4-Bit LLMs", section "End-to-End
// Implementation": dequantised value = code * scale.
//
// out = D H_n v / sqrt(n) with v = s (c - z): s and z are constant over a row, so
// out = (s / sqrt(n)) D H_n (c - z), and c - z is a small integer vector. A row of
// n = 128 B values is the 128 x B matrix C[a][b] (e = B a + b), and
// H_n (c - z) = vec(H_128 C' H_B):
//   1. Converter warps expand the packed nibbles of a group (32768 elements:
//      256 / B rows, or one row at n = 32768) into fp16 integers c - z + 1024 + z'
//      (exact; the epilogue removes the constant from matrix row 0, the only row
//      H_128 maps it to), written as the MMA's MN-major B operand with the 64- or
//      128-byte swizzle.
//   2. tcgen05.mma (kind::f16, fp16 H = +-1 as the K-major A operand, fp32
//      accumulate in TMEM) computes H_128 C' exactly: every partial sum is an
//      integer below 2^24.
//   3. Each epilogue thread owns one TMEM lane (row a') over 128 columns, runs the
//      log2(B) butterfly stages of H_B in registers (still exact), multiplies by
//      s / sqrt(n) and flips the signs of D (its row's sign words stay in
//      registers). Output rows of 64 bytes or more go through a swizzled staging
//      tile per warp and a TMA tensor store of the warp's 32 rows (whole lines);
//      narrower rows are stored from registers.
// n = 32768 is H_2 (x) H_128 (x) H_128: a row is 256 x 128, the MMA accumulates
// H_128 C'_0 + H_128 C'_1 and H_128 C'_0 - H_128 C'_1 (negate-A bit) into the two
// 128-column halves, and epilogue warpgroup g writes output rows 128 g + a'.
//
// Roles (384 threads, one CTA per SM, persistent over groups):
//   warps 0, 2, 3  converters: codes -> fp16 operand (two-stage ring of 64 KiB);
//                  thread 0 also issues each group's 16 KiB bulk copy of codes
//                  into a three-stage ring (two stages where the output staging
//                  tiles take the third's space)
//   warp 1         TMEM owner and MMA issuer
//   warps 4-11     epilogue, two warpgroups over TMEM columns 0-127 and 128-255
// (setmaxnreg moves registers from warps 0-3 to the epilogue warpgroups).
// Every mbarrier wait is bounded by a clock budget; on expiry the CTA records a
// status (read by spin_device_status), drains its copies and MMAs, frees TMEM and
// returns.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <type_traits>

#include "spin_launch.h"
#include "spin_tile.cuh"
#include "tc_ptx.cuh"

namespace spin {

// Nonzero once a tensor-core dequantise launch gave up on a wait (see spin_device_status).
__device__ unsigned int g_dequant_status = 0u;

namespace {

constexpr int kThreads = 384;
constexpr int kOStages = 2;                        // fp16 operand ring
constexpr uint32_t kCodeBytes = 16384;             // codes of one group (32768 nibbles)
constexpr uint32_t kOpBytes = 65536;               // fp16 operand of one group
constexpr uint32_t kOffH = 0;                      // A operand: H_128 in fp16, K-major, 2 x 16 KiB
constexpr uint32_t kOffO = 32768;                  // operand ring
constexpr uint32_t kStageBytes = 4096;             // output staging per epilogue warp (TMA-store shapes)

// Shared-memory layout. Shapes whose output rows are written by TMA tensor stores
// (`ts`) give up one codes stage (two groups of lead time still cover the DRAM
// latency) for a 4 KiB staging tile per epilogue warp.
template <bool TS>
struct Layout {
  static constexpr int CS = TS ? 2 : 3;              // codes ring stages
  static constexpr uint32_t kOffC = kOffO + kOStages * kOpBytes;
  static constexpr uint32_t kOffS = kOffC + CS * kCodeBytes;  // 8 staging tiles (TS)
  static constexpr uint32_t kOffBar = kOffS + (TS ? 8u * kStageBytes : 0u);
  static constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;  // + alignment slack
  static_assert(kSmemBytes <= 232448, "shared memory per block");
};
constexpr long long kTimeoutCycles = 4000000000LL;     // about two seconds
constexpr int kLaunchRegs = 168;                       // registers per thread at launch (65536 / 384, rounded)
constexpr int kRegsLow = 104, kRegsHigh = 200;         // after the split: warps 0-3, warps 4-11
static_assert(kRegsLow * 128 + kRegsHigh * 256 == kLaunchRegs * kThreads, "register split must add up");

template <int LOGN>
struct Shape {
  static constexpr bool SPLIT = LOGN == 15;
  // n = 512 (PAIR): a row is 64 x 8 and each 128-row operand tile holds two consecutive
  // rows (matrix rows 0-63 and 64-127); the A operand is H_64 (+) H_64.
  static constexpr bool PAIR = LOGN == 9;
  static constexpr int B = SPLIT ? 128 : PAIR ? 8 : 1 << (LOGN - 7);  // columns per row
  static constexpr int LOGB = SPLIT ? 7 : PAIR ? 3 : LOGN - 7;
  static constexpr int ROWS = SPLIT ? 256 : PAIR ? 64 : 128;  // matrix rows per token row
  static constexpr int TPT = PAIR ? 2 : 1;          // token rows per 128-row tile
  static constexpr int TOK = SPLIT ? 1 : TPT * 256 / B;  // token rows per group
  static constexpr int SEG = SPLIT ? 1 : 128 / B;   // column segments per epilogue thread
  static constexpr int BOXW = B < 64 ? B : 64;      // operand tile width (columns)
  static constexpr int ROWB = BOXW * 2;             // bytes per operand tile row
  static constexpr int CBOX = B / BOXW;             // column tiles per 128-row block
  static constexpr int BPT = PAIR ? 1 : CBOX * ROWS / 128;  // tiles per token row (PAIR: per pair)
  static constexpr uint32_t BOXBYTES = 128u * ROWB; // bytes per tile
  static constexpr uint32_t LAYOUT = ROWB == 128 ? 2u : ROWB == 64 ? 4u : ROWB == 32 ? 6u : 0u;  // UMMA swizzle
  // MN-major B operand strides: swizzled tiles step by box along N and by 8 rows along
  // K; the no-swizzle layout (16-byte rows, one 8 x 16 B core matrix per 8 rows) swaps
  // the roles of the two offsets, its leading offset stepping along K.
  static constexpr uint32_t LBO = LAYOUT == 0 ? 8u * ROWB : BOXBYTES;
  static constexpr uint32_t SBO = LAYOUT == 0 ? BOXBYTES : 8u * ROWB;
  static constexpr int WPT = (1 << LOGN) / 8;       // code words (8 nibbles) per token row
  // Output rows of at least 64 bytes (bf16 from n = 4096, fp32 from n = 2048) go out
  // through TMA tensor stores from a swizzled staging tile: a warp's 32 rows of a row
  // segment are one contiguous range, written as whole lines. Narrower rows are
  // stored from registers (their warp stores are contiguous already).
  template <bool F32>
  static constexpr bool ts() { return !PAIR && B * (F32 ? 4 : 2) >= 64; }
  static_assert(LOGN >= 9 && LOGN <= 15, "tensor-core dequantise covers n = 512 .. 32768");
};

struct Shared {
  uint64_t cfull[3], ofull[kOStages], oempty[kOStages], tfull[2], tempty[2], drain;
  uint32_t tmem_base;
  int abort;
  int dec[3];
  long long budget;
};
static_assert(sizeof(Shared) <= 256, "barrier area");

// One bulk copy global -> shared that completes `bar`'s transaction count (16-byte
// aligned addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   tc::smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(tc::smem_u32(bar))
               : "memory");
}

// Instruction descriptor for kind::f16 with fp16 A and B (format 0), fp32 accumulator,
// A K-major, B MN-major (`b_mn`).
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, bool b_mn) {
  return (1u << 4) | ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
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
      atomicOr(&g_dequant_status, 1u);
      return false;
    }
  }
}

// Eight 32-bit words to global memory: one 32-byte streaming store when `wide`
// (32-byte aligned destination), else two 16-byte ones.
template <bool WIDE>
__device__ __forceinline__ void store8(void *p, uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, uint32_t w4,
                                       uint32_t w5, uint32_t w6, uint32_t w7) {
  if constexpr (WIDE) {
    asm volatile("st.global.cs.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w0), "r"(w1),
                 "r"(w2), "r"(w3), "r"(w4), "r"(w5), "r"(w6), "r"(w7)
                 : "memory");
  } else {
    __stcs(reinterpret_cast<uint4 *>(p), make_uint4(w0, w1, w2, w3));
    __stcs(reinterpret_cast<uint4 *>(p) + 1, make_uint4(w4, w5, w6, w7));
  }
}

// TMA tensor store of a staged box (3-D map: element, piece, row) to global memory,
// tracked by the issuing thread's bulk group.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap *map, const void *src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(tc::smem_u32(src)), "r"(x), "r"(y), "r"(z)
               : "memory");
}

// (a0, a1) <- (a0, a1) * (m, m), one packed multiply
__device__ __forceinline__ void mul2(float &a0, float &a1, float m) {
  uint64_t A, M, R;
  asm("mov.b64 %0, {%1, %2};" : "=l"(A) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %1};" : "=l"(M) : "f"(m));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(R) : "l"(A), "l"(M));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(R));
}

// Eight nibbles u (element 2j in the low nibble of byte j; unsigned after the caller's
// sign fix-up) -> eight fp16 values 1024 + u: a byte permute puts each nibble under the
// exponent of 1024 (one unit per ulp). The epilogue removes the constant. The halves
// come out in element order 0, 2, 4, 6, 1, 3, 5, 7 (two permutes fewer than natural
// order): a permutation of the index bits inside each 8-column group, which the
// butterflies of H_B leave as it is (H is unchanged by a bit permutation applied to
// row and column indices alike); the epilogue reads element e of a group from column
// pos8(e).
__device__ __forceinline__ uint4 expand8(uint32_t w) {
  const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;  // even, odd elements
  return make_uint4(__byte_perm(lo, 0x64646464u, 0x4140), __byte_perm(lo, 0x64646464u, 0x4342),
                    __byte_perm(hi, 0x64646464u, 0x4140), __byte_perm(hi, 0x64646464u, 0x4342));
}
// column of element e within an 8-column group, as expand8 lays them out
__host__ __device__ constexpr int pos8(int e) { return (e >> 1) | ((e & 1) << 2); }

template <int LOGN, bool SIGNS, bool F32, bool STORE32>
__global__ void __launch_bounds__(kThreads, 1)
    k3_tc_dequant_inverse(const __grid_constant__ CUtensorMap omap, const uint8_t *__restrict__ codes, int64_t rows, float inv_sqrt_n,
                          const void *__restrict__ scale, const __half *__restrict__ zero,
                          const uint32_t *__restrict__ signs, void *__restrict__ out, int asym) {
  using SH = Shape<LOGN>;
  constexpr int B = SH::B, SEG = SH::SEG;
  constexpr bool TS = SH::template ts<F32>();
  using LY = Layout<TS>;
  constexpr int kCStages = LY::CS;
  constexpr uint32_t kOffC = LY::kOffC, kOffBar = LY::kOffBar;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, derived from the shared array itself so that accesses
  // through it stay shared-memory accesses
  uint8_t *smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  Shared &S = *reinterpret_cast<Shared *>(smem + kOffBar);
  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31u;
  const int64_t ngroups = (rows + SH::TOK - 1) / SH::TOK;

  // ------------------------------------------------------------ setup
  tc::grid_dep_wait();
  int64_t first_issued = 0;
  auto issue = [&](int64_t i, int64_t p) {  // codes of group p into codes stage i % kCStages
    const int cs = (int)(i % kCStages);
    const int64_t t0 = p * SH::TOK;
    const int nvalid = (int)((rows - t0) < SH::TOK ? (rows - t0) : SH::TOK);
    const uint32_t bytes = (uint32_t)nvalid * (uint32_t)(SH::WPT * 4);
    tc::mbar_arrive_expect_tx(&S.cfull[cs], bytes);
    bulk_load(smem + kOffC + cs * kCodeBytes, codes + t0 * (int64_t)(SH::WPT * 4), bytes, &S.cfull[cs]);
  };
  if (threadIdx.x == 0) {
    for (int s = 0; s < kCStages; ++s) tc::mbar_init(&S.cfull[s], 1);
    for (int s = 0; s < kOStages; ++s) {
      tc::mbar_init(&S.ofull[s], 1);
      tc::mbar_init(&S.oempty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(&S.tfull[a], 1);
      tc::mbar_init(&S.tempty[a], 256);
    }
    tc::mbar_init(&S.drain, 1);
    S.abort = 0;
    S.budget = kTimeoutCycles;
    tc::fence_barrier_init();
    for (int64_t i = 0; i < kCStages; ++i) {  // the first stages need no free slot
      const int64_t p = blockIdx.x + i * (int64_t)gridDim.x;
      if (p >= ngroups) break;
      issue(i, p);
      first_issued = i + 1;
    }
  }
  tc::grid_dep_launch();
  // H_128 in fp16 as the A operand: K-major, two K blocks of [128 rows m][64 k], 128-byte swizzle.
  for (uint32_t c = threadIdx.x; c < 2048; c += kThreads) {
    const uint32_t kb = c >> 10, m = (c >> 3) & 127u, ch = c & 7u;
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t k0 = kb * 64 + ch * 8 + 2 * j;
      auto entry = [&](uint32_t k) -> uint32_t {  // fp16 +-1 of H_128, or of H_64 (+) H_64
        if (SH::PAIR && (m >> 6) != (k >> 6)) return 0u;
        return (__popc(m & k & (SH::PAIR ? 63u : 127u)) & 1) ? 0xBC00u : 0x3C00u;
      };
      w[j] = entry(k0) | (entry(k0 + 1) << 16);
    }
    *reinterpret_cast<uint4 *>(smem + kOffH + kb * 16384 + m * 128u + ((ch ^ (m & 7u)) << 4)) =
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

  // ------------------------------------------------------------ roles
  // Registers: warps 0-3 (converters, MMA) need few, the epilogue's 128 values per
  // thread many. kRegsLow x 128 + kRegsHigh x 256 equals the launch's kLaunchRegs x 384
  // (the launcher checks the compiled count), so the increase never waits for
  // registers that are not there.
  if (warp < 4) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow) : "memory");
  else asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh) : "memory");
  if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(128, SH::SPLIT ? 128 : 256, true);
      constexpr uint32_t idesc_neg = idesc | (1u << 13);  // negate A
      const uint32_t sH = tc::smem_u32(smem + kOffH), sO = tc::smem_u32(smem + kOffO);
      for (int64_t i = 0;; ++i) {
        const int64_t p = blockIdx.x + i * (int64_t)gridDim.x;
        if (p >= ngroups) break;
        const int os = (int)(i % kOStages), acc = (int)(i & 1);
        if (!wait_bounded(&S.ofull[os], (uint32_t)((i / kOStages) & 1), S, true)) break;
        if (!wait_bounded(&S.tempty[acc], (uint32_t)((i >> 1) & 1) ^ 1u, S, true)) break;
        tc::tc_fence_after();
        if constexpr (SH::SPLIT) {
          // columns 128 u + b: sum over row blocks v of (-1)^(u v) H_128 C'_v
#pragma unroll
          for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int v = 0; v < 2; ++v)
#pragma unroll
              for (int s = 0; s < 8; ++s) {
                const uint64_t ad = tc::smem_desc(sH + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024);
                uint64_t bd = tc::smem_desc(sO + os * kOpBytes + v * SH::CBOX * SH::BOXBYTES + s * 16 * SH::ROWB,
                                            SH::LBO, SH::SBO);
                bd = (bd & ~(7ull << 61)) | ((uint64_t)SH::LAYOUT << 61);
                tc::umma_bf16(tmem + acc * 256 + u * 128, ad, bd, (u & v) ? idesc_neg : idesc,
                              (v > 0 || s > 0) ? 1u : 0u);
              }
        } else {
#pragma unroll
          for (int s = 0; s < 8; ++s) {
            const uint64_t ad = tc::smem_desc(sH + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024);
            uint64_t bd = tc::smem_desc(sO + os * kOpBytes + s * 16 * SH::ROWB, SH::LBO, SH::SBO);
            bd = (bd & ~(7ull << 61)) | ((uint64_t)SH::LAYOUT << 61);
            tc::umma_bf16(tmem + acc * 256, ad, bd, idesc, s > 0 ? 1u : 0u);
          }
        }
        tc::umma_commit(&S.oempty[os]);
        tc::umma_commit(&S.tfull[acc]);
      }
    }
  } else if (warp < 4) {
    // Converters (warps 0, 2, 3): converter c expands the quads (four code words, 32
    // consecutive elements of one matrix row) of slots c, c + 96, ... < 1024 of the
    // group. A slot's bits are, from the bottom: the half of a 64-column tile row (when
    // the tile is 64 wide), the row a (7 bits), the column tile, then the token row (or
    // the 128-row block at n = 32768); so the eight lanes of a 16-byte store phase write
    // eight different bank groups of the swizzled tiles. Converter 0 (thread 0) also
    // refills each codes stage with the group kCStages steps ahead as soon as the group
    // in it has been converted.
    constexpr uint32_t kConv = 96;
    const uint32_t cid = warp == 0 ? lane : threadIdx.x - 32;
    int64_t last[3] = {-1, -1, -1};  // converter 0: last group index issued per stage
    for (int64_t i = 0; i < first_issued; ++i) last[i] = i;
    for (int64_t i = 0;; ++i) {
      const int64_t p = blockIdx.x + i * (int64_t)gridDim.x;
      if (p >= ngroups) break;
      const int cs = (int)(i % kCStages), os = (int)(i % kOStages);
      if (cid == 0) {
        int ok = wait_bounded(&S.cfull[cs], (uint32_t)((i / kCStages) & 1), S, true) ? 1 : 0;
        if (ok) ok = wait_bounded(&S.oempty[os], (uint32_t)((i / kOStages) & 1) ^ 1u, S, true) ? 1 : 0;
        S.dec[2] = ok;
      }
      tc::named_sync(3, kConv);
      if (!S.dec[2]) break;
      const uint4 *cw = reinterpret_cast<const uint4 *>(smem + kOffC + cs * kCodeBytes);
      uint8_t *op = smem + kOffO + os * kOpBytes;
      const uint32_t flip = asym ? 0u : 0x88888888u;
      if constexpr (SH::B <= 16) {
        // 16- and 32-byte tile rows: one code word (8 elements) -> one 16-byte chunk.
        // Chunk c is chunk (c & (B/8 - 1)) of tile row (c / (B/8)) & 127 of tile
        // c / (128 B/8); consecutive lanes fill consecutive 16-byte slots of a tile (a
        // 128-byte store phase touches eight different bank groups), and read
        // consecutive code words: element e of token row t is word t WPT + e / 8, and
        // a tile's words are contiguous (PAIR: a tile is two token rows of 64 words).
        constexpr uint32_t CPRW = SH::B / 8;  // chunks per tile row
        const uint32_t *cwords = reinterpret_cast<const uint32_t *>(cw);
#pragma unroll 4
        for (uint32_t c = cid; c < 4096u; c += kConv) {
          const uint32_t tile = c / (128u * CPRW), inrow = c % (128u * CPRW);
          const uint32_t a = inrow / CPRW, cr = inrow % CPRW;
          const uint32_t w = cwords[c] ^ flip;  // the tile's words are contiguous: word c
          const uint32_t sx = SH::ROWB == 32 ? ((a >> 2) & 1u) : 0u;  // 32-byte swizzle
          *reinterpret_cast<uint4 *>(op + tile * SH::BOXBYTES + a * SH::ROWB + ((cr ^ sx) << 4)) = expand8(w);
        }
      } else {
#pragma unroll 2
      for (uint32_t q = cid; q < 1024u; q += kConv) {
        constexpr uint32_t HB = SH::BOXW / 32, LHB = HB == 2 ? 1 : 0;  // quads per tile row
        const uint32_t h = q & (HB - 1), a = (q >> LHB) & 127u, rest = q >> (LHB + 7);
        const uint32_t jc = rest % SH::CBOX, blk = rest / SH::CBOX;  // column tile, token row or row block
        const uint32_t t = SH::SPLIT ? 0u : blk, rb = SH::SPLIT ? blk : 0u;
        const uint32_t e = B * (128u * rb + a) + SH::BOXW * jc + 32u * h;  // first element in the token row
        const uint4 w = cw[(t * SH::WPT + e / 8u) / 4u];
        const uint32_t c0 = 4u * h;                          // first 16-byte chunk in the tile row
        uint8_t *rowp = op + (t * SH::BPT + rb * SH::CBOX + jc) * SH::BOXBYTES + a * SH::ROWB;
        const uint32_t sx = SH::ROWB == 128 ? (a & 7u) : ((a >> 1) & 3u);
        const uint32_t ws[4] = {w.x ^ flip, w.y ^ flip, w.z ^ flip, w.w ^ flip};
#pragma unroll
        for (int u = 0; u < 4; ++u) *reinterpret_cast<uint4 *>(rowp + (((c0 + u) ^ sx) << 4)) = expand8(ws[u]);
      }
      }
      tc::fence_proxy_async_smem();
      tc::named_sync(3, kConv);
      if (cid == 0) {
        tc::mbar_arrive(&S.ofull[os]);
        const int64_t inext = i + kCStages, pn = blockIdx.x + inext * (int64_t)gridDim.x;
        if (pn < ngroups && !*reinterpret_cast<volatile int *>(&S.abort)) {
          tc::fence_proxy_async_smem();  // every converter's reads of the stage come before the copy
          issue(inext, pn);
          last[cs] = inext;
        }
      }
    }
    if (cid == 0)  // every issued copy has landed before the CTA can leave
      for (int s2 = 0; s2 < kCStages; ++s2)
        if (last[s2] >= 0) wait_bounded(&S.cfull[s2], (uint32_t)((last[s2] / kCStages) & 1), S, false);
  } else {
    // epilogue warpgroup g: warps 4..7 (g = 0) and 8..11 (g = 1)
    const uint32_t g = (warp - 4) >> 2, wq = warp & 3u;
    const uint32_t row = wq * 32 + lane;  // a' = TMEM lane
    const uint32_t orow = SH::SPLIT ? 128u * g + row : SH::PAIR ? (row & 63u) : row;  // output matrix row
    // this row's sign bits (the same for every token row): B / 32 words, or for B < 32
    // the word holding them, shifted so that bit k is element orow B + k
    constexpr int NSW = B >= 32 ? B / 32 : 1;
    uint32_t sw[NSW];
#pragma unroll
    for (int k = 0; k < NSW; ++k)
      sw[k] = SIGNS ? (__ldg(signs + (orow * B) / 32 + k) >> (B >= 32 ? 0u : (orow * B) & 31u)) : 0u;
    // The thread's token row in segment sg of group pp is first_token(pp) + sg TSTEP
    // (PAIR: the warp's half of the tile picks the odd or even token rows).
    constexpr int TSTEP = SH::PAIR ? 2 : 1;
    auto first_token = [&](int64_t pp) -> int64_t {
      return SH::SPLIT ? pp : SH::PAIR ? pp * SH::TOK + 2 * g * SEG + (wq >> 1) : pp * SH::TOK + g * SEG;
    };
    // The row steps (and zero points) of a group are loaded one group ahead, so their
    // DRAM latency hides behind the previous group's work: raw bits (fp32 step, or fp16
    // step in the low and fp16 zero in the high half). With 8 or more segments per thread
    // (n <= 2048) lane sg loads segment sg's and each thread takes them by shuffle when
    // the group starts; otherwise every thread loads its few segments' itself.
    constexpr bool LANES = SEG >= 8;
    constexpr int NST = LANES ? 1 : SEG;  // raw steps a thread prefetches
    auto load_steps = [&](int64_t pp, uint32_t (&dst)[NST]) {
#pragma unroll
      for (int j = 0; j < NST; ++j) {
        const int sg = LANES ? (int)lane : j;
        const int64_t token = first_token(pp) + (int64_t)sg * TSTEP;
        dst[j] = 0u;
        if (sg < SEG && pp < ngroups && token < rows)
          dst[j] = asym ? (uint32_t)__ldg(static_cast<const unsigned short *>(scale) + token) |
                              ((uint32_t)__ldg(reinterpret_cast<const unsigned short *>(zero) + token) << 16)
                        : __float_as_uint(__ldg(static_cast<const float *>(scale) + token));
      }
    };
    uint32_t step_next[NST];
    load_steps(blockIdx.x, step_next);
    for (int64_t i = 0;; ++i) {
      const int64_t p = blockIdx.x + i * (int64_t)gridDim.x;
      if (p >= ngroups) break;
      uint32_t step_raw[SEG];
#pragma unroll
      for (int sg = 0; sg < SEG; ++sg)
        step_raw[sg] = LANES ? __shfl_sync(0xffffffffu, step_next[0], sg) : step_next[LANES ? 0 : sg];
      load_steps(p + gridDim.x, step_next);
      const int64_t tok0 = first_token(p);
      // segments 0 .. nseg - 1 hold token rows below `rows` (the same for the warp)
      const int nseg = rows - tok0 >= (int64_t)SEG * TSTEP ? SEG : (int)((rows - tok0 + TSTEP - 1) / TSTEP);
      const int acc = (int)(i & 1);
      // every thread sleeps on the accumulator's barrier itself (no block-level barrier
      // between the epilogue warps)
      if (!wait_bounded(&S.tfull[acc], (uint32_t)((i >> 1) & 1), S, true)) break;
      tc::tc_fence_after();
      float v[kRegs];
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
      // The operand carried every value plus 1024 + K (K = 8 for symmetric codes, else
      // the row's zero point). H_128 of a constant is nonzero only in matrix row 0
      // (128 times it; twice that in the top half at n = 32768, nothing in the bottom
      // half), so the thread holding row 0 takes it out before H_B; all exact integers.
      // (PAIR: H_64 (+) H_64 puts 64 times it in rows 0 and 64, one per token row.)
      if ((SH::PAIR ? (row & 63u) : row) == 0 && (!SH::SPLIT || g == 0)) {
#pragma unroll
        for (int sg = 0; sg < SEG; ++sg) {
          const float K = asym ? __half2float(__ushort_as_half((unsigned short)(step_raw[sg] >> 16))) : 8.0f;
          const float corr = (SH::SPLIT ? 256.0f : SH::PAIR ? 64.0f : 128.0f) * (1024.0f + K);
#pragma unroll
          for (int k = 0; k < B; ++k) v[sg * B + k] -= corr;
        }
      }
      // second Kronecker factor: H_B over b inside each token row's segment
      stage<0>(v);
      stage<1>(v);
      stage<2>(v);
      if constexpr (SH::LOGB > 3) stage<3>(v);
      if constexpr (SH::LOGB > 4) stage<4>(v);
      if constexpr (SH::LOGB > 5) stage<5>(v);
      if constexpr (SH::LOGB > 6) stage<6>(v);
      if constexpr (TS) {
        // A warp's 32 rows of a row segment are one contiguous range of the output. Each
        // piece (128 or 64 bytes of every row) is written into the warp's staging tile
        // with the TMA swizzle (row `lane` at lane x OROWB, 16-byte chunk c at position
        // c ^ (row bits), so the eight lanes of a store phase hit eight bank groups),
        // then one lane issues the tensor store that writes it out as whole lines.
        constexpr int OE = F32 ? 4 : 2;                  // output bytes per element
        constexpr int OROWB = B * OE >= 128 ? 128 : 64;  // staged bytes per row (the swizzle span)
        constexpr int PE = OROWB / OE;                   // elements per piece
        constexpr int NP = B / PE;                       // pieces per row segment
        constexpr int CH = OROWB / 16;                   // 16-byte chunks per staged row
        uint8_t *stg = smem + LY::kOffS + (warp - 4) * kStageBytes;
        const uint32_t srow = tc::smem_u32(stg) + lane * (uint32_t)OROWB;
        const uint32_t swz = OROWB == 128 ? (lane & 7u) : ((lane >> 1) & 3u);
        const int orow0 = (SH::SPLIT ? 128 * (int)g : 0) + 32 * (int)wq;
#pragma unroll
        for (int sg = 0; sg < SEG; ++sg) {
          if (sg >= nseg) break;  // the same for the whole warpgroup
          const int64_t token = tok0 + sg;
          const float s = asym ? __half2float(__ushort_as_half((unsigned short)step_raw[sg]))
                               : __uint_as_float(step_raw[sg]);
          const float m = s * inv_sqrt_n;
          const float *w = v + sg * B;
#pragma unroll
          for (int pc = 0; pc < NP; ++pc) {
            uint32_t wv[CH * 4];
#pragma unroll
            for (int u = 0; u < PE; u += 2) {
              const int k = pc * PE + u;  // element of the row segment (even)
              float o0 = w[(k & ~7) + pos8(k & 7)], o1 = w[(k & ~7) + pos8((k + 1) & 7)];
              mul2(o0, o1, m);
              if constexpr (SIGNS) {
                const uint32_t sb = B >= 32 ? sw[k >> 5] >> (k & 31) : sw[0] >> k;
                o0 = __uint_as_float(__float_as_uint(o0) ^ ((sb & 1u) << 31));
                o1 = __uint_as_float(__float_as_uint(o1) ^ (((sb >> 1) & 1u) << 31));
              }
              if constexpr (F32) {
                wv[u] = __float_as_uint(o0);
                wv[u + 1] = __float_as_uint(o1);
              } else {
                wv[u >> 1] = pack_bf16x2(o0, o1);
              }
            }
            if (lane == 0) tc::bulk_wait_read0();  // the tile's previous piece has been read out
            __syncwarp();
#pragma unroll
            for (int c = 0; c < CH; ++c)
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(srow + ((c ^ swz) << 4)),
                           "r"(wv[4 * c]), "r"(wv[4 * c + 1]), "r"(wv[4 * c + 2]), "r"(wv[4 * c + 3])
                           : "memory");
            tc::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_3d(&omap, stg, 0, pc, (int)(token * SH::ROWS) + orow0);
              tc::bulk_commit();
            }
          }
        }
      } else {
        // first element of this thread's row in segment 0; segment sg starts sg TSTEP
        // token rows further (a constant offset the compiler folds into the stores)
        const int64_t off0 = tok0 * (int64_t)(B * SH::ROWS) + (int64_t)orow * B;
#pragma unroll
        for (int sg = 0; sg < SEG; ++sg) {
          if (sg >= nseg) break;
          const float s = asym ? __half2float(__ushort_as_half((unsigned short)step_raw[sg]))
                               : __uint_as_float(step_raw[sg]);
          const float m = s * inv_sqrt_n;
          const float *w = v + sg * B;
          const int64_t off = off0 + (int64_t)sg * TSTEP * (B * SH::ROWS);
          // one 8 (fp32) or 16 (bf16; 8 when B = 8) element piece at a time, in element
          // order: scale, diagonal sign, store
          constexpr int P = (F32 || B == 8) ? 8 : 16;
#pragma unroll
          for (int k = 0; k < B; k += P) {
            float o[P];
#pragma unroll
            for (int u = 0; u < P; u += 2) {
              o[u] = w[k + (u & ~7) + pos8(u & 7)];
              o[u + 1] = w[k + (u & ~7) + pos8((u + 1) & 7)];
              mul2(o[u], o[u + 1], m);
            }
            if constexpr (SIGNS) {
              const uint32_t sb = B >= 32 ? sw[k >> 5] >> (k & 31) : sw[0] >> k;
#pragma unroll
              for (int u = 0; u < P; ++u) o[u] = __uint_as_float(__float_as_uint(o[u]) ^ (((sb >> u) & 1u) << 31));
            }
            if constexpr (F32) {
              store8<STORE32>(static_cast<float *>(out) + off + k, __float_as_uint(o[0]), __float_as_uint(o[1]),
                              __float_as_uint(o[2]), __float_as_uint(o[3]), __float_as_uint(o[4]),
                              __float_as_uint(o[5]), __float_as_uint(o[6]), __float_as_uint(o[7]));
            } else if constexpr (P == 8) {  // 8 bf16: one 16-byte store
              __stcs(reinterpret_cast<uint4 *>(static_cast<uint16_t *>(out) + off + k),
                     make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                                pack_bf16x2(o[6], o[7])));
            } else {
              store8<STORE32>(static_cast<uint16_t *>(out) + off + k, pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]),
                              pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]), pack_bf16x2(o[8], o[9]),
                              pack_bf16x2(o[10], o[11]), pack_bf16x2(o[12], o[13]), pack_bf16x2(o[14], o[15]));
            }
          }
        }
      }
    }
    if constexpr (TS)
      if (lane == 0) tc::bulk_wait0();  // every tensor store has completed before the CTA leaves
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

template <int LOGN, bool SIGNS, bool F32, bool STORE32>
cudaError_t launch_tc(const uint8_t *codes, int64_t rows, const void *scale, const void *zero,
                      const uint32_t *signs, void *out, bool asym, cudaStream_t stream) {
  using SH = Shape<LOGN>;
  auto kern = k3_tc_dequant_inverse<LOGN, SIGNS, F32, STORE32>;
  static cudaError_t checked = [&] {  // the register split assumes this count at launch
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, reinterpret_cast<const void *>(kern));
    if (e != cudaSuccess) return e;
    return fa.numRegs == kLaunchRegs ? cudaSuccess : cudaErrorInvalidConfiguration;
  }();
  if (checked != cudaSuccess) return checked;
  constexpr bool TS = SH::template ts<F32>();
  constexpr uint32_t kSmemBytes = Layout<TS>::kSmemBytes;
  // Output map for the tensor stores: (element within a 128- or 64-byte piece, piece
  // within a matrix row, matrix row = token row x rows-per-token + a'), boxes of one
  // piece x 32 rows, swizzled like the staging tile.
  CUtensorMap omap;
  std::memset(&omap, 0, sizeof(omap));
  if constexpr (TS) {
    constexpr int OE = F32 ? 4 : 2, OROWB = SH::B * OE >= 128 ? 128 : 64, PE = OROWB / OE;
    if (rows * SH::ROWS >= (int64_t(1) << 31)) return cudaErrorInvalidValue;  // row coordinates are 32-bit
    auto fn = tensor_map_encoder();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[3] = {(cuuint64_t)PE, (cuuint64_t)(SH::B / PE), (cuuint64_t)(rows * SH::ROWS)};
    const cuuint64_t strides[2] = {(cuuint64_t)OROWB, (cuuint64_t)SH::B * OE};
    const cuuint32_t box[3] = {(cuuint32_t)PE, 1, 32};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(&omap, F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, out, dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    OROWB == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  }
  int slots = 0;
  cudaError_t err = resident_slots(reinterpret_cast<const void *>(kern), kThreads, (int)kSmemBytes, &slots);
  if (err != cudaSuccess) return err;
  const int64_t ngroups = (rows + SH::TOK - 1) / SH::TOK;
  const int64_t grid = ngroups < slots ? ngroups : slots;
  const float inv_sqrt_n = (float)(1.0 / std::sqrt((double)(1 << LOGN)));
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
  return cudaLaunchKernelEx(&cfg, kern, omap, codes, rows, inv_sqrt_n, scale, static_cast<const __half *>(zero),
                            signs, out, asym ? 1 : 0);
}

template <int LOGN, bool SIGNS>
cudaError_t launch_s(const uint8_t *codes, int64_t rows, const void *scale, const void *zero, const uint32_t *signs,
                     void *out, bool asym, bool f32, cudaStream_t stream) {
  const bool a32 = (reinterpret_cast<uintptr_t>(out) & 31u) == 0;  // 32-byte stores need 32-byte alignment
  if (f32)
    return a32 ? launch_tc<LOGN, SIGNS, true, true>(codes, rows, scale, zero, signs, out, asym, stream)
               : launch_tc<LOGN, SIGNS, true, false>(codes, rows, scale, zero, signs, out, asym, stream);
  return a32 ? launch_tc<LOGN, SIGNS, false, true>(codes, rows, scale, zero, signs, out, asym, stream)
             : launch_tc<LOGN, SIGNS, false, false>(codes, rows, scale, zero, signs, out, asym, stream);
}

template <int LOGN>
cudaError_t launch_n(const uint8_t *codes, int64_t rows, const void *scale, const void *zero, const uint32_t *signs,
                     void *out, bool asym, bool f32, cudaStream_t stream) {
  return signs ? launch_s<LOGN, true>(codes, rows, scale, zero, signs, out, asym, f32, stream)
               : launch_s<LOGN, false>(codes, rows, scale, zero, nullptr, out, asym, f32, stream);
}


// ============================================================================ n = 128, 256
// Tokens as the MMA's M. A row of n = 128 V (V = 1, 2) is V chunks c_v of 128
// codes, and H_n (c - z) = [sum_v (-1)^(u v) H_128 (c_v - z)]_u. For 128 rows at
// once the MMA computes Y_v[t][a'] = sum_a C'_v[t][a] H[a'][a] with A = C'_v (the
// rows' fp16 integers 1024 + u, K-major) and B = H_128 (K-major, fp16 +-1, built
// once). The constant 1024 + K of every element lands only in column 0 of each
// Y_v (128 times it), which the epilogue takes out; at n = 256 it then forms
// Y_0 + Y_1 and Y_0 - Y_1. Each epilogue thread owns one row (one TMEM lane) and
// writes it in element order: scale, diagonal sign, store.
//   warp 0      bulk copies of each group's codes (128 rows) into a codes ring
//   warp 1      TMEM owner and MMA issuer; two accumulators of 128 V columns
//   warps 2-5   converters: codes -> fp16 operand ring (two stages)
//   warps 6-9   epilogue
constexpr int kThreadsS = 320;

template <int V>
struct SmallLayout {
  static constexpr int kCS = V == 1 ? 4 : 3;              // codes stages
  static constexpr int kAS = 2;                           // operand stages
  static constexpr uint32_t kCodeBytes = 8192u * V;       // 128 rows of codes
  static constexpr uint32_t kOpBytes = 32768u * V;        // 128 rows of fp16 operand
  static constexpr uint32_t kOffB = 0;                    // H_128, fp16, K-major, 2 x 16 KiB
  static constexpr uint32_t kOffC = 32768;
  static constexpr uint32_t kOffA = kOffC + kCS * kCodeBytes;
  static constexpr uint32_t kOffBar = kOffA + kAS * kOpBytes;
  static constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory per block");
};

template <int CS, int AS>
struct SharedS {
  uint64_t cfull[CS], cempty[CS], afull[AS], aempty[AS], tfull[2], tempty[2], drain;
  uint32_t tmem_base;
  int abort;
  int dec[2];
  long long budget;
};

template <int V, bool SIGNS, bool F32, bool STORE32>
__global__ void __launch_bounds__(kThreadsS, 1)
    k3_tcs_dequant_inverse(const uint8_t *__restrict__ codes, int64_t rows, float inv_sqrt_n,
                           const void *__restrict__ scale, const __half *__restrict__ zero,
                           const uint32_t *__restrict__ signs, void *__restrict__ out, int asym) {
  using L = SmallLayout<V>;
  constexpr int CS = L::kCS, AS = L::kAS;
  constexpr int N = 128 * V;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  SharedS<CS, AS> &S = *reinterpret_cast<SharedS<CS, AS> *>(smem + L::kOffBar);
  static_assert(sizeof(SharedS<CS, AS>) <= 256, "barrier area");
  const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31u;
  const int64_t ngroups = (rows + 127) / 128;
  auto issue = [&](int cs, int64_t p) {  // codes of group p into codes stage cs
    const int64_t t0 = p * 128;
    const uint32_t nvalid = (uint32_t)((rows - t0) < 128 ? (rows - t0) : 128);
    const uint32_t bytes = nvalid * (uint32_t)(N / 2);
    tc::mbar_arrive_expect_tx(&S.cfull[cs], bytes);
    bulk_load(smem + L::kOffC + cs * L::kCodeBytes, codes + t0 * (int64_t)(N / 2), bytes, &S.cfull[cs]);
  };

  tc::grid_dep_wait();
  int first_issued = 0;
  if (threadIdx.x == 0) {
    for (int s2 = 0; s2 < CS; ++s2) {
      tc::mbar_init(&S.cfull[s2], 1);
      tc::mbar_init(&S.cempty[s2], 128);
    }
    for (int s2 = 0; s2 < AS; ++s2) {
      tc::mbar_init(&S.afull[s2], 128);
      tc::mbar_init(&S.aempty[s2], 1);
    }
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(&S.tfull[a], 1);
      tc::mbar_init(&S.tempty[a], 128);
    }
    tc::mbar_init(&S.drain, 1);
    S.abort = 0;
    S.budget = kTimeoutCycles;
    tc::fence_barrier_init();
    for (int i = 0; i < CS; ++i) {  // the first stages need no free slot
      const int64_t p = blockIdx.x + i * (int64_t)gridDim.x;
      if (p >= ngroups) break;
      issue(i, p);
      first_issued = i + 1;
    }
  }
  tc::grid_dep_launch();
  // H_128 in fp16 as the B operand [n = a'][k = a], K-major, two K blocks of 64 with
  // the 128-byte swizzle; physical K position p of an 8-column group holds element
  // e = 2 (p & 3) + (p >> 2), the order expand8 writes the codes in.
  for (uint32_t c = threadIdx.x; c < 2048; c += kThreadsS) {
    const uint32_t kb = c >> 10, m = (c >> 3) & 127u, ch = c & 7u;
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t p0 = 2 * j, p1 = 2 * j + 1;
      const uint32_t k0 = kb * 64 + ch * 8 + 2 * (p0 & 3u) + (p0 >> 2);
      const uint32_t k1 = kb * 64 + ch * 8 + 2 * (p1 & 3u) + (p1 >> 2);
      const uint32_t lo = (__popc(m & k0) & 1) ? 0xBC00u : 0x3C00u;
      const uint32_t hi = (__popc(m & k1) & 1) ? 0xBC00u : 0x3C00u;
      w[j] = lo | (hi << 16);
    }
    *reinterpret_cast<uint4 *>(smem + L::kOffB + kb * 16384 + m * 128u + ((ch ^ (m & 7u)) << 4)) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
  tc::fence_proxy_async_smem();
  if (warp == 1) {
    tc::tmem_alloc(&S.tmem_base, 256 * V);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      int64_t last[CS];
      for (int s2 = 0; s2 < CS; ++s2) last[s2] = s2 < first_issued ? s2 : -1;
      for (int64_t i = first_issued;; ++i) {
        const int64_t p = blockIdx.x + i * (int64_t)gridDim.x;
        if (p >= ngroups) break;
        const int cs = (int)(i % CS);
        if (!wait_bounded(&S.cempty[cs], (uint32_t)((i / CS) & 1) ^ 1u, S, true)) break;
        tc::fence_proxy_async_smem();  // the converters' reads of the stage come before the copy
        issue(cs, p);
        last[cs] = i;
      }
      for (int s2 = 0; s2 < CS; ++s2)  // every issued copy has landed before the CTA can leave
        if (last[s2] >= 0) wait_bounded(&S.cfull[s2], (uint32_t)((last[s2] / CS) & 1), S, false);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(128, 128, false);  // A and B K-major
      const uint32_t sB = tc::smem_u32(smem + L::kOffB), sA = tc::smem_u32(smem + L::kOffA);
      for (int64_t i = 0;; ++i) {
        const int64_t p = blockIdx.x + i * (int64_t)gridDim.x;
        if (p >= ngroups) break;
        const int as = (int)(i % AS), acc = (int)(i & 1);
        if (!wait_bounded(&S.afull[as], (uint32_t)((i / AS) & 1), S, true)) break;
        if (!wait_bounded(&S.tempty[acc], (uint32_t)((i >> 1) & 1) ^ 1u, S, true)) break;
        tc::tc_fence_after();
#pragma unroll
        for (int v = 0; v < V; ++v)
#pragma unroll
          for (int s2 = 0; s2 < 8; ++s2) {
            const uint32_t aa = sA + as * L::kOpBytes + v * 32768 + (s2 >> 2) * 16384 + (s2 & 3) * 32;
            const uint32_t ba = sB + (s2 >> 2) * 16384 + (s2 & 3) * 32;
            tc::umma_bf16(tmem + acc * (128 * V) + v * 128, tc::smem_desc(aa, 16, 1024),
                          tc::smem_desc(ba, 16, 1024), idesc, s2 > 0 ? 1u : 0u);
          }
        tc::umma_commit(&S.aempty[as]);
        tc::umma_commit(&S.tfull[acc]);
      }
    }
  } else if (warp < 6) {
    // Converters. One 16-byte read covers 32 consecutive codes of a row: the read
    // phases take 128 contiguous bytes. Lane (row t, chunk v, quarter qd) writes the
    // four 8-code groups of its quarter in the order j ^ (qd & 2) ^ v, so the eight
    // lanes of a 16-byte store phase hit eight different bank groups of the swizzled
    // rows.
    const uint32_t cid = threadIdx.x - 64, cw = cid >> 5;
    const uint32_t flip = asym ? 0u : 0x88888888u;
    for (int64_t i = 0;; ++i) {
      const int64_t p = blockIdx.x + i * (int64_t)gridDim.x;
      if (p >= ngroups) break;
      const int cs = (int)(i % CS), as = (int)(i % AS);
      if (cid == 0) {
        int ok = wait_bounded(&S.cfull[cs], (uint32_t)((i / CS) & 1), S, true) ? 1 : 0;
        if (ok) ok = wait_bounded(&S.aempty[as], (uint32_t)((i / AS) & 1) ^ 1u, S, true) ? 1 : 0;
        S.dec[0] = ok;
      }
      tc::named_sync(1, 128);
      if (!S.dec[0]) break;
      const uint8_t *cb = smem + L::kOffC + cs * L::kCodeBytes;
      uint8_t *ab = smem + L::kOffA + as * L::kOpBytes;
      constexpr int RPI = 32 / (4 * V);  // rows per warp and iteration
#pragma unroll 2
      for (int it = 0; it < 128 / (4 * RPI); ++it) {
        const uint32_t t = (uint32_t)(it * 4 + cw) * RPI + (lane / (4 * V));
        const uint32_t u = lane & (4 * V - 1), v = u >> 2, qd = u & 3u;
        const uint4 w = *reinterpret_cast<const uint4 *>(cb + t * (N / 2) + u * 16);
        const uint32_t ws[4] = {w.x ^ flip, w.y ^ flip, w.z ^ flip, w.w ^ flip};
        uint8_t *rowp = ab + v * 32768 + (qd >> 1) * 16384 + t * 128;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t jj = (uint32_t)j ^ (qd & 2u) ^ v;
          const uint32_t word = (jj & 2u) ? ((jj & 1u) ? ws[3] : ws[2]) : ((jj & 1u) ? ws[1] : ws[0]);
          const uint32_t ch = (qd & 1u) * 4u + jj;
          *reinterpret_cast<uint4 *>(rowp + ((ch ^ (t & 7u)) << 4)) = expand8(word);
        }
      }
      tc::mbar_arrive(&S.cempty[cs]);
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&S.afull[as]);
    }
  } else {
    const uint32_t row = (warp & 3u) * 32 + lane;
    const uint32_t lane_base = tmem + (((warp & 3u) * 32u) << 16);
    // a row's step (fp32; or fp16 step | fp16 zero << 16), loaded one group ahead
    auto load_step = [&](int64_t pp) -> uint32_t {
      const int64_t token = pp * 128 + row;
      if (pp >= ngroups || token >= rows) return 0u;
      return asym ? (uint32_t)__ldg(static_cast<const unsigned short *>(scale) + token) |
                        ((uint32_t)__ldg(reinterpret_cast<const unsigned short *>(zero) + token) << 16)
                  : __float_as_uint(__ldg(static_cast<const float *>(scale) + token));
    };
    uint32_t step_next = load_step(blockIdx.x);
    for (int64_t i = 0;; ++i) {
      const int64_t p = blockIdx.x + i * (int64_t)gridDim.x;
      if (p >= ngroups) break;
      const uint32_t step_raw = step_next;
      step_next = load_step(p + gridDim.x);
      const int acc = (int)(i & 1);
      // every epilogue thread sleeps on the accumulator's barrier itself (no meeting point)
      if (!wait_bounded(&S.tfull[acc], (uint32_t)((i >> 1) & 1), S, true)) break;
      tc::tc_fence_after();
      const int64_t token = p * 128 + row;
      const bool live = token < rows;
      const float s = asym ? __half2float(__ushort_as_half((unsigned short)step_raw)) : __uint_as_float(step_raw);
      const float K = asym ? __half2float(__ushort_as_half((unsigned short)(step_raw >> 16))) : 8.0f;
      const float corr = 128.0f * (1024.0f + K);  // H_128 of the constant: column 0 only
      const float m = s * inv_sqrt_n;
      const uint32_t taddr = lane_base + (uint32_t)acc * (128u * V);
      const int64_t off = token * (int64_t)N;
      // 32 outputs (elements e0 .., fp32 bit patterns in w, updated in place): scale,
      // sign, store
      auto emit = [&](uint32_t *w, int e0) {
#pragma unroll
        for (int k = 0; k < 32; k += 2) {
          float x0 = __uint_as_float(w[k]), x1 = __uint_as_float(w[k + 1]);
          mul2(x0, x1, m);
          w[k] = __float_as_uint(x0);
          w[k + 1] = __float_as_uint(x1);
        }
        if constexpr (SIGNS) {  // the diagonal's sign word of these 32 elements (the same for every row)
          const uint32_t sb = __ldg(signs + (e0 >> 5));
#pragma unroll
          for (int k = 0; k < 32; ++k) w[k] ^= ((sb >> k) & 1u) << 31;
        }
        if (!live) return;
        if constexpr (F32) {
          float *dst = static_cast<float *>(out) + off + e0;
#pragma unroll
          for (int k = 0; k < 32; k += 8)
            store8<STORE32>(dst + k, w[k], w[k + 1], w[k + 2], w[k + 3], w[k + 4], w[k + 5], w[k + 6], w[k + 7]);
        } else {
          auto f = [&](int k) { return __uint_as_float(w[k]); };
          uint16_t *dst = static_cast<uint16_t *>(out) + off + e0;
#pragma unroll
          for (int k = 0; k < 32; k += 16)
            store8<STORE32>(dst + k, pack_bf16x2(f(k), f(k + 1)), pack_bf16x2(f(k + 2), f(k + 3)),
                            pack_bf16x2(f(k + 4), f(k + 5)), pack_bf16x2(f(k + 6), f(k + 7)),
                            pack_bf16x2(f(k + 8), f(k + 9)), pack_bf16x2(f(k + 10), f(k + 11)),
                            pack_bf16x2(f(k + 12), f(k + 13)), pack_bf16x2(f(k + 14), f(k + 15)));
        }
      };
      // TMEM loads are issued 128 columns at a time and waited for once; the
      // accumulator is released as soon as its last columns are in registers
      if constexpr (V == 1) {
        uint32_t r[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) tc::tmem_ld32(taddr + 32 * c, r + 32 * c);
        tc::tmem_wait_ld();
        tc::tc_fence_before();
        tc::mbar_arrive(&S.tempty[acc]);
        r[0] = __float_as_uint(__uint_as_float(r[0]) - corr);
#pragma unroll
        for (int c = 0; c < 4; ++c) emit(r + 32 * c, 32 * c);
      } else {
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {  // chunks 2h and 2h + 1 of both halves
          uint32_t a[64], b[64];
          tc::tmem_ld32(taddr + 64 * h, a);
          tc::tmem_ld32(taddr + 64 * h + 32, a + 32);
          tc::tmem_ld32(taddr + 128 + 64 * h, b);
          tc::tmem_ld32(taddr + 128 + 64 * h + 32, b + 32);
          tc::tmem_wait_ld();
          if (h == 1) {
            tc::tc_fence_before();
            tc::mbar_arrive(&S.tempty[acc]);
          } else {
            a[0] = __float_as_uint(__uint_as_float(a[0]) - corr);
            b[0] = __float_as_uint(__uint_as_float(b[0]) - corr);
          }
#pragma unroll
          for (int k = 0; k < 64; ++k) {  // the H_2 halves, in place
            const float y0 = __uint_as_float(a[k]), y1 = __uint_as_float(b[k]);
            a[k] = __float_as_uint(y0 + y1);
            b[k] = __float_as_uint(y0 - y1);
          }
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            emit(a + 32 * cc, 64 * h + 32 * cc);
            emit(b + 32 * cc, 128 + 64 * h + 32 * cc);
          }
        }
      }
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
    tc::tmem_dealloc(tmem, 256 * V);
  }
}

template <int V, bool SIGNS, bool F32, bool STORE32>
cudaError_t launch_tcs(const uint8_t *codes, int64_t rows, const void *scale, const void *zero,
                       const uint32_t *signs, void *out, bool asym, cudaStream_t stream) {
  auto kern = k3_tcs_dequant_inverse<V, SIGNS, F32, STORE32>;
  constexpr uint32_t smem_bytes = SmallLayout<V>::kSmemBytes;
  int slots = 0;
  cudaError_t err = resident_slots(reinterpret_cast<const void *>(kern), kThreadsS, (int)smem_bytes, &slots);
  if (err != cudaSuccess) return err;
  const int64_t ngroups = (rows + 127) / 128;
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
  return cudaLaunchKernelEx(&cfg, kern, codes, rows, inv_sqrt_n, scale, static_cast<const __half *>(zero), signs,
                            out, asym ? 1 : 0);
}

template <int V>
cudaError_t launch_small(const uint8_t *codes, int64_t rows, const void *scale, const void *zero,
                         const uint32_t *signs, void *out, bool asym, bool f32, cudaStream_t stream) {
  const bool a32 = (reinterpret_cast<uintptr_t>(out) & 31u) == 0;  // 32-byte stores need 32-byte alignment
  auto go = [&](auto sg, auto fp) {  // sg, fp: std::integral_constant<bool, ...>
    return a32 ? launch_tcs<V, decltype(sg)::value, decltype(fp)::value, true>(codes, rows, scale, zero, signs, out,
                                                                             asym, stream)
               : launch_tcs<V, decltype(sg)::value, decltype(fp)::value, false>(codes, rows, scale, zero, signs, out,
                                                                              asym, stream);
  };
  using T = std::true_type;
  using F = std::false_type;
  if (signs) return f32 ? go(T{}, T{}) : go(T{}, F{});
  return f32 ? go(F{}, T{}) : go(F{}, F{});
}

}  // namespace

bool tc_dequant_supported(int log_n, int64_t rows, uint32_t flags) {
  if ((flags & kNoRotate) || rows <= 0) return false;
  if (log_n < 7 || log_n > 15) return false;
  if (rows * (int64_t(1) << log_n) >= (int64_t(1) << 40)) return false;
  // rows per MMA group: 128 at n = 128 and 256, 64 at n = 512 (two per tile), 256 / (n / 128)
  // from n = 1024, one at n = 32768
  const int64_t rows_per_group = log_n <= 8 ? 128 : log_n == 15 ? 1 : int64_t(256) >> (log_n - 7);
  return (flags & kTensorCores) || rows >= 128 * rows_per_group;
}

cudaError_t launch_dequant_inverse_tc(int log_n, const uint8_t *codes, int64_t rows, int mode, const void *scale,
                                      const void *zero, const uint32_t *signs, void *out, int out_dtype,
                                      cudaStream_t stream) {
  const bool asym = mode == 1, f32 = out_dtype == 1;
  switch (log_n) {
    case 7: return launch_small<1>(codes, rows, scale, zero, signs, out, asym, f32, stream);
    case 8: return launch_small<2>(codes, rows, scale, zero, signs, out, asym, f32, stream);
    case 9: return launch_n<9>(codes, rows, scale, zero, signs, out, asym, f32, stream);
    case 10: return launch_n<10>(codes, rows, scale, zero, signs, out, asym, f32, stream);
    case 11: return launch_n<11>(codes, rows, scale, zero, signs, out, asym, f32, stream);
    case 12: return launch_n<12>(codes, rows, scale, zero, signs, out, asym, f32, stream);
    case 13: return launch_n<13>(codes, rows, scale, zero, signs, out, asym, f32, stream);
    case 14: return launch_n<14>(codes, rows, scale, zero, signs, out, asym, f32, stream);
    case 15: return launch_n<15>(codes, rows, scale, zero, signs, out, asym, f32, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t read_dequant_status(unsigned int *status, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(status, g_dequant_status, sizeof(unsigned int));
  if (e != cudaSuccess || !reset) return e;
  const unsigned int zero = 0u;
  return cudaMemcpyToSymbol(g_dequant_status, &zero, sizeof(unsigned int));
}

}  // namespace spin
