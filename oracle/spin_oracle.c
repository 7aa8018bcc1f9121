/*
 * spin_oracle.c -- plain, slow, fp64 CPU oracle for the online Hadamard
 * rotation path (SpinQuant's R3 and R4 rotations and the quantisers that
 * follow them).
 *
 * TEST INFRASTRUCTURE ONLY. The test suite, the smoke check and the CPU
 * baseline leg of the benchmark are the only users of this file. The CUDA
 * library shares no code, header, table or helper with it, and it includes
 * nothing from the CUDA library.
 *
 * Every value is carried in IEEE binary64. Rounding to the storage formats
 * (bfloat16, binary16, binary32) is done once, at the point where the method
 * stores a value, by the explicit round-to-nearest-even converters below.
 *
 * Sources (web pages about SpinQuant, cited by title and section):
 *  [RQ]  "Rotations: QuaRot, SpinQuant and incoherence", section "Hadamard
 *        matrices" (Sylvester recursion, orthogonality of H_n/sqrt(n),
 *        randomised Hadamard (1/sqrt n) H_n diag(+-1), Kronecker products),
 *        section "Why it's free: computational invariance" (O(d log d)
 *        transform with no matrix multiply), example "a hidden state with an
 *        outlier channel" (per-token 4-bit step max/7), widget "Try it"
 *        (rotate -> quantize -> rotate back).
 *  [SG]  "SpinQuant Guide: Learned Rotations for 4-Bit LLMs", section "The
 *        Outlier Curse in 4-Bit Weight-Activation Quantization" (INT4 range
 *        [-8, 7], step = max|x| / (2^(b-1) - 1); at b = 8 the per-token INT8
 *        activations of W4A8), section "End-to-End
 *        Implementation" (scale clamped below at 1e-8, x_dequant = x_quant *
 *        scale; the quantised layer output is the product of the quantised
 *        activations and weights), section "RoPE Compatibility with 4-Bit KV
 *        Caching" (RoPE rotates 2-D coordinate pairs; KV cache stored as 4-bit),
 *        section "Production Engineering and Cluster Deployment Best Practices"
 *        (W R^T baked offline into packed INT4 weights for an INT4 GEMM).
 *  [SW]  "SpinQuant, when rotations are worth learning", section "Four
 *        rotation sites, two of them free" (R3: Hadamard on Q and K after
 *        RoPE; R4: Hadamard on the down-projection input), section "Paper vs.
 *        code" (power-of-two head dim required by the fast transform),
 *        section "The math, slowly" (RMSNorm commutes with rotations).
 *
 * Readings where the pages are silent (each is also listed in the design
 * notes): rotate-half RoPE pairing (p, p + d/2) with inv_freq = theta^(-2p/d);
 * asymmetric INT4 with an integer zero point whose range is widened to
 * include 0; codes of element 2j in the low nibble of byte j; the diagonal is
 * applied before the transform; the asymmetric quantiser divides by the
 * fp16-rounded scale; for n = m 2^k that is not a power of two, the small factor
 * H_m is Paley's (type I or II, a named published construction: the pages give
 * none), the product is H_m (x) H_{2^k} with the H_m index as the high part of
 * the element index, and the diagonal again comes first; the W4A4 GEMM's weights
 * are quantised per output channel by the activations' symmetric INT4 rule (the
 * pages' listing uses one scale per tensor), each row first rotated by the same R.
 */
#include <fenv.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_NO_ROTATE 1u
#define ORC_METHOD_FWHT 0
#define ORC_METHOD_EXPLICIT 1

/* ------------------------------------------------------------------ */
/* Storage-format converters (exact decode, round-to-nearest-even encode) */
/* ------------------------------------------------------------------ */

int orc_rounding_is_nearest(void) { return fegetround() == FE_TONEAREST; }

double orc_rne(double v) { return nearbyint(v); } /* ties to even under FE_TONEAREST */

double orc_bf16_to_f64(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* Round x to the nearest value with `sig` significant bits whose exponent is
 * at least `min_exp` (the subnormal quantum), ties to even. Exact in fp64. */
static double round_to_grid(double a, int sig, int min_quantum_exp) {
  int e;
  frexp(a, &e);             /* a in [2^(e-1), 2^e) */
  int q = (e - 1) - (sig - 1); /* quantum of the binade */
  if (q < min_quantum_exp) q = min_quantum_exp;
  return ldexp(nearbyint(ldexp(a, -q)), q);
}

uint16_t orc_f64_to_bf16(double x) {
  if (isnan(x)) return 0x7FC0;
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  double a = fabs(x);
  if (a == 0.0) return sign;
  if (isinf(a)) return sign | 0x7F80;
  double v = round_to_grid(a, 8, -133);
  if (v >= 0x1p128) return sign | 0x7F80;
  float f = (float)v; /* exact: v has <= 8 significant bits */
  uint32_t u;
  memcpy(&u, &f, 4);
  return sign | (uint16_t)((u >> 16) & 0x7FFF);
}

double orc_f16_to_f64(uint16_t h) {
  int s = (h >> 15) & 1, e = (h >> 10) & 0x1F, m = h & 0x3FF;
  double v;
  if (e == 0) v = ldexp((double)m, -24);
  else if (e == 31) v = m ? NAN : INFINITY;
  else v = ldexp((double)(m | 0x400), e - 25);
  return s ? -v : v;
}

uint16_t orc_f64_to_f16(double x) {
  if (isnan(x)) return 0x7E00;
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  double a = fabs(x);
  if (a == 0.0) return sign;
  if (isinf(a)) return sign | 0x7C00;
  double v = round_to_grid(a, 11, -24);
  if (v >= 65536.0) return sign | 0x7C00;
  if (v < 0x1p-14) return sign | (uint16_t)ldexp(v, 24); /* subnormal */
  int e;
  frexp(v, &e);
  int E = e - 1; /* v in [2^E, 2^(E+1)), E in [-14, 15] */
  uint16_t mant = (uint16_t)(ldexp(v, 10 - E) - 1024.0);
  return sign | (uint16_t)((E + 15) << 10) | mant;
}

float orc_f64_to_f32(double x) { return (float)x; } /* C conversion: RNE under FE_TONEAREST */

/* ------------------------------------------------------------------ */
/* Hadamard matrices [RQ "Hadamard matrices"]                          */
/* ------------------------------------------------------------------ */

/* Sylvester recursion, written out: H_1 = [1], H_2m = [[H_m, H_m], [H_m, -H_m]].
 * H is n*n row-major int8. */
void orc_sylvester_matrix(int n, int8_t *H) {
  H[0] = 1;
  for (int m = 1; m < n; m *= 2)
    for (int i = 0; i < m; i++)
      for (int j = 0; j < m; j++) {
        int8_t h = H[(size_t)i * n + j];
        H[(size_t)i * n + j + m] = h;
        H[(size_t)(i + m) * n + j] = h;
        H[(size_t)(i + m) * n + j + m] = (int8_t)-h;
      }
}

/* Entry (i, j) of the Sylvester matrix of any power-of-two order: unrolling
 * the recursion bit by bit, every level whose row and column halves are both
 * the lower-right block contributes one factor -1. */
int orc_hadamard_entry(uint64_t i, uint64_t j) {
  uint64_t both = i & j;
  int parity = 0;
  while (both) {
    parity ^= (int)(both & 1u);
    both >>= 1;
  }
  return parity ? -1 : 1;
}

/* y = H_n x (unnormalised) as n explicit sums, O(n^2). */
void orc_wht_explicit(const double *x, int n, double *y) {
  for (int i = 0; i < n; i++) {
    double acc = 0.0;
    for (int j = 0; j < n; j++) acc += orc_hadamard_entry((uint64_t)i, (uint64_t)j) * x[j];
    y[i] = acc;
  }
}

/* In-place textbook fast Walsh-Hadamard transform, unnormalised, natural
 * (Sylvester) order: log2(n) passes of butterflies (a, b) -> (a + b, a - b)
 * [RQ "Why it's free"]. */
void orc_fwht(double *x, int n) {
  for (int h = 1; h < n; h *= 2)
    for (int i = 0; i < n; i += 2 * h)
      for (int j = i; j < i + h; j++) {
        double a = x[j], b = x[j + h];
        x[j] = a + b;
        x[j + h] = a - b;
      }
}

static int is_pow2(int n) { return n > 0 && (n & (n - 1)) == 0; }

static int sign_bit(const uint32_t *signs, int j) {
  return signs ? (int)((signs[j >> 5] >> (j & 31)) & 1u) : 0;
}

/* y = H_n D x / sqrt(n), D = diag(+-1) from the bitmask (bit j set -> -1)
 * [RQ "Hadamard matrices": randomised Hadamard (1/sqrt n) H_n diag(+-1)]. */
int orc_rotate(const double *x, int n, const uint32_t *signs, int method, double *y) {
  if (!is_pow2(n)) return -1;
  double *t = (double *)malloc(sizeof(double) * (size_t)n);
  if (!t) return -2;
  for (int j = 0; j < n; j++) t[j] = sign_bit(signs, j) ? -x[j] : x[j];
  if (method == ORC_METHOD_EXPLICIT) {
    orc_wht_explicit(t, n, y);
  } else {
    orc_fwht(t, n);
    memcpy(y, t, sizeof(double) * (size_t)n);
  }
  double r = sqrt((double)n);
  for (int i = 0; i < n; i++) y[i] = y[i] / r;
  free(t);
  return 0;
}

/* ------------------------------------------------------------------ */
/* Sizes that are not powers of two: H_m (x) H_b, b a power of two       */
/* ------------------------------------------------------------------ */

/* [RQ "Hadamard matrices"]: sizes that are not powers of two use a Kronecker
 * product of a small known Hadamard matrix with a Sylvester one. The pages give
 * no small matrix, so H_m comes from Paley's construction (R. E. A. C. Paley,
 * "On orthogonal matrices", 1933) for a prime q:
 *   type I,  q = 3 (mod 4), m = q + 1:   H = I + S,  S = [[0, 1^T], [-1, Q]];
 *   type II, q = 1 (mod 4), m = 2(q + 1): H = S (x) [[1, -1], [-1, -1]] + I (x) [[1, 1], [1, -1]],
 *            S = [[0, 1^T], [1, Q]];
 * with the Jacobsthal matrix Q[i][j] = chi(j - i), chi the quadratic character
 * mod q (chi(0) = 0). */

double orc_quant_sym_int4(const double *y, int n, double clip, double *pre, int8_t *codes);

static int is_prime(int64_t q) {
  if (q < 2) return 0;
  for (int64_t d = 2; d * d <= q; d++)
    if (q % d == 0) return 0;
  return 1;
}

/* Quadratic character of a mod an odd prime q by Euler's criterion:
 * a^((q-1)/2) = 1 (residue), q - 1 (non-residue), 0 (a = 0 mod q). */
int orc_legendre(int64_t a, int64_t q) {
  int64_t r = ((a % q) + q) % q;
  if (r == 0) return 0;
  int64_t e = (q - 1) / 2, acc = 1, b = r;
  while (e > 0) {
    if (e & 1) acc = (acc * b) % q;
    b = (b * b) % q;
    e >>= 1;
  }
  return acc == 1 ? 1 : -1;
}

/* The Paley type (1 or 2) that gives a Hadamard matrix of order m, or 0. */
int orc_paley_type(int m) {
  if (m >= 4 && (m - 1) % 4 == 3 && is_prime(m - 1)) return 1;
  if (m >= 12 && m % 4 == 0 && (m / 2 - 1) % 4 == 1 && is_prime(m / 2 - 1)) return 2;
  return 0;
}

/* H (m x m, row-major, entries +-1) by Paley's construction; -1 if m has none. */
int orc_paley_hadamard(int m, int8_t *H) {
  const int type = orc_paley_type(m);
  if (!type) return -1;
  const int q = type == 1 ? m - 1 : m / 2 - 1, k = q + 1;
  int8_t *S = (int8_t *)malloc((size_t)k * (size_t)k);
  if (!S) return -2;
  for (int i = 0; i < k; i++)
    for (int j = 0; j < k; j++) {
      int v;
      if (i == 0 && j == 0) v = 0;
      else if (i == 0) v = 1;
      else if (j == 0) v = type == 1 ? -1 : 1;
      else v = orc_legendre((int64_t)(j - 1) - (int64_t)(i - 1), q);
      S[i * k + j] = (int8_t)v;
    }
  if (type == 1) {
    for (int i = 0; i < k; i++)
      for (int j = 0; j < k; j++) H[i * m + j] = (int8_t)(S[i * k + j] + (i == j ? 1 : 0));
  } else {
    static const int A[2][2] = {{1, -1}, {-1, -1}}, B[2][2] = {{1, 1}, {1, -1}};
    for (int i = 0; i < k; i++)
      for (int j = 0; j < k; j++)
        for (int u = 0; u < 2; u++)
          for (int v = 0; v < 2; v++)
            H[(2 * i + u) * m + (2 * j + v)] = (int8_t)(S[i * k + j] * A[u][v] + (i == j ? B[u][v] : 0));
  }
  free(S);
  return 0;
}

/* y = (H_m (x) H_b) D x / sqrt(m b) for a row of n = m b values, element e = b i + j
 * (i the H_m index, j the Sylvester one; D first, as for powers of two): H_b on each
 * of the m blocks of b, then H_m across the blocks, both written out plainly. */
int orc_rotate_kron(const double *x, int m, int b, const uint32_t *signs, double *y) {
  if (!is_pow2(b)) return -1;
  int8_t *H = (int8_t *)malloc((size_t)m * (size_t)m);
  double *t = (double *)malloc(sizeof(double) * (size_t)m * (size_t)b);
  if (!H || !t) {
    free(H); free(t);
    return -2;
  }
  if (orc_paley_hadamard(m, H)) {
    free(H); free(t);
    return -1;
  }
  const int n = m * b;
  for (int e = 0; e < n; e++) t[e] = sign_bit(signs, e) ? -x[e] : x[e];
  for (int i = 0; i < m; i++) orc_fwht(t + (size_t)i * b, b);
  for (int i = 0; i < m; i++)
    for (int j = 0; j < b; j++) {
      double acc = 0.0;
      for (int k = 0; k < m; k++) acc += H[i * m + k] * t[(size_t)k * b + j];
      y[(size_t)i * b + j] = acc;
    }
  const double r = sqrt((double)n);
  for (int e = 0; e < n; e++) y[e] = y[e] / r;
  free(H); free(t);
  return 0;
}

/* R4 for n = m b: the Kronecker rotation, then the per-token INT4 quantiser. */
int orc_r4_row_kron(const uint16_t *x, int m, int b, double clip, const uint32_t *signs, double *y_out,
                    double *pre, int8_t *codes, double *scale64, float *scale32) {
  const int n = m * b;
  double *xd = (double *)malloc(sizeof(double) * (size_t)n);
  double *y = (double *)malloc(sizeof(double) * (size_t)n);
  if (!xd || !y) {
    free(xd); free(y);
    return -2;
  }
  for (int e = 0; e < n; e++) xd[e] = orc_bf16_to_f64(x[e]);
  int rc = orc_rotate_kron(xd, m, b, signs, y);
  if (!rc) {
    double s = orc_quant_sym_int4(y, n, clip, pre, codes);
    if (y_out) memcpy(y_out, y, sizeof(double) * (size_t)n);
    if (scale64) *scale64 = s;
    *scale32 = (float)s;
  }
  free(xd); free(y);
  return rc;
}

void orc_pack_nibbles(const int32_t *codes, int n, uint8_t *packed);

/* Many rows of n = m b through orc_r4_row_kron (INT4 codes packed two per byte,
 * element 2j in the low nibble, and fp32 steps); rows spread over `threads`. */
int orc_r4_rows_kron(const uint16_t *x, int64_t tokens, int m, int b, double clip, const uint32_t *signs,
                     uint8_t *packed, float *scales, int threads) {
  const int n = m * b;
  int rc = 0;
#pragma omp parallel for schedule(dynamic, 8) num_threads(threads > 0 ? threads : 1) reduction(| : rc)
  for (int64_t t = 0; t < tokens; t++) {
    int8_t *codes = (int8_t *)malloc((size_t)n);
    int32_t *c32 = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
    int r = (codes && c32) ? orc_r4_row_kron(x + t * n, m, b, clip, signs, NULL, NULL, codes, NULL, scales + t) : -2;
    if (r == 0) {
      for (int j = 0; j < n; j++) c32[j] = codes[j];
      orc_pack_nibbles(c32, n, packed + t * (n / 2));
    }
    free(codes); free(c32);
    rc |= r;
  }
  return rc ? -1 : 0;
}

/* ------------------------------------------------------------------ */
/* Quantisers                                                          */
/* ------------------------------------------------------------------ */

static double clampd(double v, double lo, double hi) { return v < lo ? lo : (v > hi ? hi : v); }

/* Symmetric per-token INT4 [SG "The Outlier Curse"; RQ "a hidden state with an
 * outlier channel"]: s = max(clip * max|y| / 7, 1e-8), q = clamp(rne(y/s), -8, 7).
 * `pre` (nullable) receives y/s before rounding. Returns s in fp64. */
double orc_quant_sym_int4(const double *y, int n, double clip, double *pre, int8_t *codes) {
  double m = 0.0;
  for (int j = 0; j < n; j++) m = fmax(m, fabs(y[j]));
  double s = clip * m / 7.0;
  if (s < 1e-8) s = 1e-8; /* the guide's clamp of the scale at 1e-8 */
  for (int j = 0; j < n; j++) {
    double p = y[j] / s;
    if (pre) pre[j] = p;
    codes[j] = (int8_t)clampd(nearbyint(p), -8.0, 7.0);
  }
  return s;
}

/* Symmetric per-token INT8, the same rule at b = 8 bits [SG "The Outlier Curse":
 * signed b-bit range [-2^(b-1), 2^(b-1) - 1], step = max|x| / (2^(b-1) - 1); the
 * A8 of the W4A8 decoding figure in "SpinQuant, when rotations are worth
 * learning", section "Measured effects"]: s = max(clip * max|y| / 127, 1e-8),
 * q = clamp(rne(y/s), -128, 127). `pre` (nullable) receives y/s. Returns s. */
double orc_quant_sym_int8(const double *y, int n, double clip, double *pre, int8_t *codes) {
  double m = 0.0;
  for (int j = 0; j < n; j++) m = fmax(m, fabs(y[j]));
  double s = clip * m / 127.0;
  if (s < 1e-8) s = 1e-8;
  for (int j = 0; j < n; j++) {
    double p = y[j] / s;
    if (pre) pre[j] = p;
    codes[j] = (int8_t)clampd(nearbyint(p), -128.0, 127.0);
  }
  return s;
}

/* Codes and zero point of one asymmetric INT4 group for a given fp16 step s16
 * (the steps of the asymmetric rule that follow the step's rounding):
 * lo = min(clip*min x, 0), z = clamp(rne(-lo/s), 0, 15), q = clamp(rne(x/s) + z, 0, 15);
 * a step of 0 becomes s = 1, z = 0. `pre` (nullable) receives x/s + z before rounding.
 * Returns the fp16 pattern of the step actually used (s16, or 1.0 for a zero step). */
uint16_t orc_quant_asym_int4_at(const double *x, int n, double clip, uint16_t s16, double *pre,
                                uint8_t *codes, uint16_t *z16) {
  double mn = x[0];
  for (int j = 1; j < n; j++) mn = fmin(mn, x[j]);
  double lo = fmin(clip * mn, 0.0);
  double s = orc_f16_to_f64(s16);
  double z;
  if (s == 0.0) {
    s16 = 0x3C00; /* 1.0 */
    s = 1.0;
    z = 0.0;
  } else {
    z = clampd(nearbyint(-lo / s), 0.0, 15.0) + 0.0; /* + 0.0 maps -0 to +0 */
  }
  for (int j = 0; j < n; j++) {
    double p = x[j] / s + z;
    if (pre) pre[j] = p;
    codes[j] = (uint8_t)clampd(nearbyint(x[j] / s) + z, 0.0, 15.0);
  }
  *z16 = orc_f64_to_f16(z);
  return s16;
}

double orc_asym_unrounded_scale(const double *x, int n, double clip);

/* The asymmetric zero point before its rounding, -lo/s with lo = min(clip*min x, 0)
 * and s the given fp16 step (a zero step counts as 1), and the codes for that
 * step and a given integer zero point z: q = clamp(rne(x/s) + z, 0, 15); `pre`
 * (nullable) receives x/s + z. Used to check a zero point whose rounding sits on
 * a .5 tie against the oracle's own result for the other rounding. */
double orc_asym_codes_at(const double *x, int n, double clip, uint16_t s16, double z, double *pre,
                         uint8_t *codes) {
  double mn = x[0];
  for (int j = 1; j < n; j++) mn = fmin(mn, x[j]);
  double lo = fmin(clip * mn, 0.0);
  double s = orc_f16_to_f64(s16);
  if (s == 0.0) s = 1.0;
  for (int j = 0; j < n; j++) {
    if (pre) pre[j] = x[j] / s + z;
    codes[j] = (uint8_t)clampd(nearbyint(x[j] / s) + z, 0.0, 15.0);
  }
  return -lo / s;
}

/* Asymmetric INT4 over one group (reading of "KV cache stored as 4-bit INT4";
 * the pages give no formula): lo = min(clip*min x, 0), hi = max(clip*max x, 0),
 * s = (hi - lo) / 15 rounded to fp16, then z and the codes as in
 * orc_quant_asym_int4_at. `pre` (nullable) receives x/s + z before rounding. */
void orc_quant_asym_int4(const double *x, int n, double clip, double *pre, uint8_t *codes,
                         uint16_t *s16, uint16_t *z16) {
  uint16_t sh = orc_f64_to_f16(orc_asym_unrounded_scale(x, n, clip));
  *s16 = orc_quant_asym_int4_at(x, n, clip, sh, pre, codes, z16);
}

/* The asymmetric step before its rounding to fp16, (hi - lo) / 15 (used to
 * recognise steps that sit on an fp16 rounding boundary). */
double orc_asym_unrounded_scale(const double *x, int n, double clip) {
  double mn = x[0], mx = x[0];
  for (int j = 1; j < n; j++) {
    mn = fmin(mn, x[j]);
    mx = fmax(mx, x[j]);
  }
  return (fmax(clip * mx, 0.0) - fmin(clip * mn, 0.0)) / 15.0;
}

/* Two codes per byte: element 2j in the low nibble, element 2j+1 in the high
 * nibble, each as a 4-bit two's-complement (signed) or plain (unsigned) field. */
void orc_pack_nibbles(const int32_t *codes, int n, uint8_t *packed) {
  for (int j = 0; j < n / 2; j++)
    packed[j] = (uint8_t)((codes[2 * j] & 0xF) | ((codes[2 * j + 1] & 0xF) << 4));
}

void orc_unpack_nibbles(const uint8_t *packed, int n, int is_signed, int32_t *codes) {
  for (int j = 0; j < n; j++) {
    int v = (packed[j / 2] >> ((j & 1) * 4)) & 0xF;
    if (is_signed && v >= 8) v -= 16;
    codes[j] = v;
  }
}

/* ------------------------------------------------------------------ */
/* R4: rotate the down-projection input, then per-token INT4           */
/* [SW "Four rotation sites"; RQ "Hadamard matrices"]                   */
/* ------------------------------------------------------------------ */

/* One token row. x: n bf16 bit patterns. Outputs (all nullable except
 * packed/scale32): y (rotated fp64), pre (y/s), codes (int8), packed
 * (n/2 bytes), scale64 (fp64 step), scale32 (step rounded to fp32). With
 * ORC_NO_ROTATE, neither D nor H is applied (direct quantisation). */
int orc_r4_row(const uint16_t *x, int n, double clip, const uint32_t *signs, uint32_t flags,
               int method, double *y_out, double *pre, int8_t *codes_out, uint8_t *packed,
               double *scale64, float *scale32) {
  if (!is_pow2(n) || n < 2) return -1;
  double *xd = (double *)malloc(sizeof(double) * (size_t)n);
  double *y = (double *)malloc(sizeof(double) * (size_t)n);
  int8_t *q = (int8_t *)malloc((size_t)n);
  int32_t *q32 = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
  if (!xd || !y || !q || !q32) {
    free(xd); free(y); free(q); free(q32);
    return -2;
  }
  for (int j = 0; j < n; j++) xd[j] = orc_bf16_to_f64(x[j]);
  if (flags & ORC_NO_ROTATE) memcpy(y, xd, sizeof(double) * (size_t)n);
  else orc_rotate(xd, n, signs, method, y);
  double s = orc_quant_sym_int4(y, n, clip, pre, q);
  for (int j = 0; j < n; j++) q32[j] = q[j];
  orc_pack_nibbles(q32, n, packed);
  if (y_out) memcpy(y_out, y, sizeof(double) * (size_t)n);
  if (codes_out) memcpy(codes_out, q, (size_t)n);
  if (scale64) *scale64 = s;
  *scale32 = (float)s;
  free(xd); free(y); free(q); free(q32);
  return 0;
}

/* One token row through R4 with per-token INT8 codes (one signed byte per
 * element). Outputs as in orc_r4_row; codes (n bytes) is required. */
int orc_r4_row_int8(const uint16_t *x, int n, double clip, const uint32_t *signs, uint32_t flags,
                    int method, double *y_out, double *pre, int8_t *codes, double *scale64,
                    float *scale32) {
  if (!is_pow2(n) || n < 2) return -1;
  double *xd = (double *)malloc(sizeof(double) * (size_t)n);
  double *y = (double *)malloc(sizeof(double) * (size_t)n);
  if (!xd || !y) {
    free(xd); free(y);
    return -2;
  }
  for (int j = 0; j < n; j++) xd[j] = orc_bf16_to_f64(x[j]);
  if (flags & ORC_NO_ROTATE) memcpy(y, xd, sizeof(double) * (size_t)n);
  else orc_rotate(xd, n, signs, method, y);
  double s = orc_quant_sym_int8(y, n, clip, pre, codes);
  if (y_out) memcpy(y_out, y, sizeof(double) * (size_t)n);
  if (scale64) *scale64 = s;
  *scale32 = (float)s;
  free(xd); free(y);
  return 0;
}

/* Many rows with the fast transform (the timed CPU baseline uses this loop). Rows are
 * independent, so `threads` > 1 spreads them over OpenMP threads; each row's arithmetic
 * is the same as with one thread, so the results are identical. */
int orc_r4_rows(const uint16_t *x, int64_t tokens, int n, double clip, const uint32_t *signs,
                uint32_t flags, uint8_t *packed, float *scales, int threads) {
  int rc = 0;
#pragma omp parallel for schedule(dynamic, 16) num_threads(threads > 0 ? threads : 1) reduction(| : rc)
  for (int64_t t = 0; t < tokens; t++) {
    rc |= orc_r4_row(x + t * n, n, clip, signs, flags, ORC_METHOD_FWHT, NULL, NULL, NULL,
                     packed + t * (n / 2), NULL, scales + t);
  }
  return rc ? -1 : 0;
}

/* Threads OpenMP would use by default (the host's cores). */
int orc_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ------------------------------------------------------------------ */
/* W4A4 GEMM on the codes                                               */
/* ------------------------------------------------------------------ */

/* [SG] "End-to-End Implementation": the quantised layer output is the matrix product of
 * the quantised activations and the quantised (rotated) weights, each dequantised as
 * code * scale; "Production Engineering and Cluster Deployment Best Practices": the
 * rotated weights W R^T are quantised offline and stored as packed INT4 nibbles, and
 * the product runs on INT4 tensor cores.
 *   y[t][o] = sum_k (s_x[t] q_x[t][k]) (s_w[o] q_w[o][k]) = s_x[t] s_w[o] sum_k q_x q_w
 * The integer sum is exact (int64); the scales multiply it once, in binary64. Codes are
 * 4-bit two's complement, element 2j in the low nibble of byte j: x [tokens, k/2],
 * w [n_out, k/2] (one row per output channel), y [tokens, n_out]. Rows of y are
 * independent; `threads` spreads them over OpenMP threads. */
int orc_w4a4_gemm(const uint8_t *xq, const float *xs, int64_t tokens, const uint8_t *wq, const float *ws,
                  int n_out, int k, double *y, int threads) {
  if (tokens < 0 || n_out <= 0 || k <= 0 || (k & 1)) return -1;
  int32_t *w = (int32_t *)malloc(sizeof(int32_t) * (size_t)n_out * (size_t)k);
  if (!w) return -1;
  for (int o = 0; o < n_out; o++) orc_unpack_nibbles(wq + (size_t)o * (k / 2), k, 1, w + (size_t)o * k);
  int rc = 0;
#pragma omp parallel for schedule(dynamic, 4) num_threads(threads > 0 ? threads : 1) reduction(| : rc)
  for (int64_t t = 0; t < tokens; t++) {
    int32_t *x = (int32_t *)malloc(sizeof(int32_t) * (size_t)k);
    if (!x) {
      rc |= 1;
      continue;
    }
    orc_unpack_nibbles(xq + (size_t)t * (k / 2), k, 1, x);
    for (int o = 0; o < n_out; o++) {
      const int32_t *wo = w + (size_t)o * k;
      int64_t acc = 0;
      for (int j = 0; j < k; j++) acc += (int64_t)x[j] * wo[j];
      y[(size_t)t * n_out + o] = (double)xs[t] * (double)ws[o] * (double)acc;
    }
    free(x);
  }
  free(w);
  return rc ? -1 : 0;
}

/* ------------------------------------------------------------------ */
/* R3: RoPE, then Hadamard on Q and K; asymmetric INT4 KV cache         */
/* ------------------------------------------------------------------ */

/* Rotate-half RoPE on one head vector of even length d, in place, fp64:
 * for p < d/2, angle a = pos * theta^(-2p/d);
 * (x_p, x_{p+d/2}) <- (x_p cos a - x_{p+d/2} sin a, x_{p+d/2} cos a + x_p sin a).
 * [SG "RoPE Compatibility with 4-Bit KV Caching": RoPE rotates 2-D pairs.] */
void orc_rope_half(double *x, int d, double pos, double theta) {
  int h = d / 2;
  for (int p = 0; p < h; p++) {
    double inv = pow(theta, -2.0 * (double)p / (double)d);
    double a = pos * inv;
    double c = cos(a), s = sin(a);
    double x0 = x[p], x1 = x[p + h];
    x[p] = x0 * c - x1 * s;
    x[p + h] = x1 * c + x0 * s;
  }
}

/* One token of R3 + KV quantisation. Inputs are bf16 bit patterns:
 * q [hq][d], k [hkv][d], v [hkv][d]. Outputs (nullable where marked):
 * q_f64 [hq][d] (rotated Q, fp64, nullable), q_bf16 [hq][d],
 * k_f64 [hkv][d] (rotated K before quantisation, nullable),
 * k_pre/v_pre [hkv][d] (value/s + z before rounding, nullable),
 * k_packed/v_packed [hkv][d/2], k_s/k_z/v_s/v_z [hkv] fp16 bit patterns. */
int orc_r3_token(const uint16_t *q, const uint16_t *k, const uint16_t *v, double pos, double theta,
                 int d, int hq, int hkv, double clip, double *q_f64, uint16_t *q_bf16,
                 double *k_f64, double *k_pre, double *v_pre, uint8_t *k_packed,
                 uint8_t *v_packed, uint16_t *k_s, uint16_t *k_z, uint16_t *v_s, uint16_t *v_z) {
  if (!is_pow2(d) || d < 2) return -1;
  double *t = (double *)malloc(sizeof(double) * (size_t)d);
  double *y = (double *)malloc(sizeof(double) * (size_t)d);
  uint8_t *c = (uint8_t *)malloc((size_t)d);
  int32_t *c32 = (int32_t *)malloc(sizeof(int32_t) * (size_t)d);
  if (!t || !y || !c || !c32) {
    free(t); free(y); free(c); free(c32);
    return -2;
  }
  for (int h = 0; h < hq; h++) {
    for (int j = 0; j < d; j++) t[j] = orc_bf16_to_f64(q[h * d + j]);
    orc_rope_half(t, d, pos, theta);
    orc_rotate(t, d, NULL, ORC_METHOD_FWHT, y);
    for (int j = 0; j < d; j++) {
      if (q_f64) q_f64[h * d + j] = y[j];
      q_bf16[h * d + j] = orc_f64_to_bf16(y[j]);
    }
  }
  for (int h = 0; h < hkv; h++) {
    for (int j = 0; j < d; j++) t[j] = orc_bf16_to_f64(k[h * d + j]);
    orc_rope_half(t, d, pos, theta);
    orc_rotate(t, d, NULL, ORC_METHOD_FWHT, y);
    if (k_f64) memcpy(k_f64 + (size_t)h * d, y, sizeof(double) * (size_t)d);
    orc_quant_asym_int4(y, d, clip, k_pre ? k_pre + (size_t)h * d : NULL, c, &k_s[h], &k_z[h]);
    for (int j = 0; j < d; j++) c32[j] = c[j];
    orc_pack_nibbles(c32, d, k_packed + (size_t)h * (d / 2));

    for (int j = 0; j < d; j++) t[j] = orc_bf16_to_f64(v[h * d + j]);
    orc_quant_asym_int4(t, d, clip, v_pre ? v_pre + (size_t)h * d : NULL, c, &v_s[h], &v_z[h]);
    for (int j = 0; j < d; j++) c32[j] = c[j];
    orc_pack_nibbles(c32, d, v_packed + (size_t)h * (d / 2));
  }
  free(t); free(y); free(c); free(c32);
  return 0;
}

/* Whole R3 batch: q [B,S,hq,d], k/v [B,S,hkv,d], pos [B,S]; cache slot of
 * token (b, s) is cache_offset + s; caches are [B, hkv, cache_len, d/2] and
 * scale/zero arrays [B, hkv, cache_len] fp16. q_out [B,S,hq,d] bf16. Slots
 * outside [cache_offset, cache_offset + S) are not written. Tokens are
 * independent and write disjoint slots, so `threads` > 1 spreads them over
 * OpenMP threads with identical results. */
int orc_r3_batch(const uint16_t *q, const uint16_t *k, const uint16_t *v, const int32_t *pos,
                 double theta, int d, int B, int S, int hq, int hkv, double clip, uint16_t *q_out,
                 uint8_t *k_cache, uint8_t *v_cache, uint16_t *k_scale, uint16_t *k_zero,
                 uint16_t *v_scale, uint16_t *v_zero, int cache_len, int cache_offset, int threads) {
  if (cache_offset < 0 || cache_offset + S > cache_len) return -1;
  int rc = 0;
#pragma omp parallel for schedule(dynamic, 8) num_threads(threads > 0 ? threads : 1) reduction(| : rc)
  for (int64_t tok = 0; tok < (int64_t)B * S; tok++) {
    int b = (int)(tok / S), s = (int)(tok % S);
    uint8_t *kp = (uint8_t *)malloc((size_t)hkv * d / 2), *vp = (uint8_t *)malloc((size_t)hkv * d / 2);
    uint16_t *ks = (uint16_t *)malloc(2 * (size_t)hkv), *kz = (uint16_t *)malloc(2 * (size_t)hkv);
    uint16_t *vs = (uint16_t *)malloc(2 * (size_t)hkv), *vz = (uint16_t *)malloc(2 * (size_t)hkv);
    int r = (kp && vp && ks && kz && vs && vz) ? 0 : -2;
    if (r == 0)
      r = orc_r3_token(q + (size_t)tok * hq * d, k + (size_t)tok * hkv * d, v + (size_t)tok * hkv * d,
                       (double)pos[tok], theta, d, hq, hkv, clip, NULL, q_out + (size_t)tok * hq * d, NULL,
                       NULL, NULL, kp, vp, ks, kz, vs, vz);
    if (r == 0) {
      int slot = cache_offset + s;
      for (int h = 0; h < hkv; h++) {
        size_t row = ((size_t)b * hkv + h) * cache_len + slot;
        memcpy(k_cache + row * (d / 2), kp + (size_t)h * (d / 2), (size_t)d / 2);
        memcpy(v_cache + row * (d / 2), vp + (size_t)h * (d / 2), (size_t)d / 2);
        k_scale[row] = ks[h];
        k_zero[row] = kz[h];
        v_scale[row] = vs[h];
        v_zero[row] = vz[h];
      }
    }
    free(kp); free(vp); free(ks); free(kz); free(vs); free(vz);
    rc |= r;
  }
  return rc ? -1 : 0;
}

/* ------------------------------------------------------------------ */
/* Dequantise and rotate back [RQ "Try it": rotate -> quantize -> rotate */
/* back; SG: x_dequant = x_quant * scale]                               */
/* ------------------------------------------------------------------ */

/* mode 0: symmetric signed codes, value = q * scale.
 * mode 1: asymmetric unsigned codes, value = (q - zero) * scale.
 * Unless ORC_NO_ROTATE: out = D H_n value / sqrt(n) (the inverse of
 * H_n D / sqrt(n), since that matrix is orthogonal and D H_n / sqrt(n) is
 * its transpose). */
int orc_dequant_inverse_row(const uint8_t *packed, int n, int mode, double scale, double zero,
                            const uint32_t *signs, uint32_t flags, int method, double *out) {
  if (!is_pow2(n) || n < 2) return -1;
  int32_t *c = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
  double *v = (double *)malloc(sizeof(double) * (size_t)n);
  if (!c || !v) {
    free(c); free(v);
    return -2;
  }
  orc_unpack_nibbles(packed, n, mode == 0, c);
  for (int j = 0; j < n; j++) v[j] = ((double)c[j] - (mode == 0 ? 0.0 : zero)) * scale;
  if (flags & ORC_NO_ROTATE) {
    memcpy(out, v, sizeof(double) * (size_t)n);
  } else {
    if (method == ORC_METHOD_EXPLICIT) orc_wht_explicit(v, n, out);
    else {
      orc_fwht(v, n);
      memcpy(out, v, sizeof(double) * (size_t)n);
    }
    double r = sqrt((double)n);
    for (int j = 0; j < n; j++) {
      out[j] = out[j] / r;
      if (sign_bit(signs, j)) out[j] = -out[j];
    }
  }
  free(c); free(v);
  return 0;
}

/* Many rows through orc_dequant_inverse_row with the fast transform: codes
 * [rows, n/2], scale [rows] (fp64 values), zero [rows] (mode 1; NULL for mode 0),
 * out [rows, n] fp64. Rows are independent; `threads` > 1 spreads them over
 * OpenMP threads with identical results. */
int orc_dequant_inverse_rows(const uint8_t *packed, int64_t rows, int n, int mode, const double *scale,
                             const double *zero, const uint32_t *signs, uint32_t flags, double *out,
                             int threads) {
  int rc = 0;
#pragma omp parallel for schedule(dynamic, 16) num_threads(threads > 0 ? threads : 1) reduction(| : rc)
  for (int64_t r = 0; r < rows; r++)
    rc |= orc_dequant_inverse_row(packed + r * (n / 2), n, mode, scale[r], zero ? zero[r] : 0.0, signs, flags,
                                  ORC_METHOD_FWHT, out + r * n);
  return rc ? -1 : 0;
}

/* ------------------------------------------------------------------ */
/* Decode attention over the 4-bit KV cache ["SpinQuant Guide", the KV4 */
/* serving diagram: rotated keys stored in the cache as INT4, then a     */
/* "Fused INT4 Dot Product" with the rotated queries; "SpinQuant: rotate */
/* before you round", "Deployment implications": a rotation only pays   */
/* once the runtime has KV4 kernels]                                    */
/* ------------------------------------------------------------------ */

/* One decode step of one batch row. q: [hq][d] bf16 bit patterns (queries after
 * RoPE and R3, as the R3 kernel writes them). Cache of one batch row: k_codes,
 * v_codes [hkv][cache_len][d/2] (unsigned nibbles, element 2j low), k_s, k_z,
 * v_s, v_z [hkv][cache_len] fp16 patterns; slots 0 .. len-1 are attended.
 * Query head h reads kv head h / (hq / hkv). In fp64, plainly:
 *   khat_j = (code - z) s,  score_j = (q . khat_j) * softmax_scale,
 *   p = exp(score - max score) / sum,  out_h = sum_j p_j vhat_j.
 * Since R3 rotates q and k by the same orthogonal H/sqrt(d), q . k is the
 * unrotated product; V is not rotated, so out is in the value basis.
 * out: [hq][d] fp64. Returns 0, or -1 for bad sizes. */
int orc_decode_attention(const uint16_t *q, const uint8_t *k_codes, const uint8_t *v_codes,
                         const uint16_t *k_s, const uint16_t *k_z, const uint16_t *v_s, const uint16_t *v_z,
                         int hq, int hkv, int d, int cache_len, int len, double softmax_scale, double *out) {
  if (hq <= 0 || hkv <= 0 || hq % hkv != 0 || d < 2 || (d & 1) || len <= 0 || len > cache_len) return -1;
  double *sc = (double *)malloc(sizeof(double) * (size_t)len);
  double *qd = (double *)malloc(sizeof(double) * (size_t)d);
  int32_t *c = (int32_t *)malloc(sizeof(int32_t) * (size_t)d);
  if (!sc || !qd || !c) {
    free(sc); free(qd); free(c);
    return -2;
  }
  const int group = hq / hkv;
  for (int h = 0; h < hq; h++) {
    const int g = h / group;
    for (int i = 0; i < d; i++) qd[i] = orc_bf16_to_f64(q[(size_t)h * d + i]);
    double mx = -INFINITY;
    for (int j = 0; j < len; j++) {
      const size_t row = (size_t)g * cache_len + j;
      orc_unpack_nibbles(k_codes + row * (d / 2), d, 0, c);
      const double s = orc_f16_to_f64(k_s[row]), z = orc_f16_to_f64(k_z[row]);
      double dot = 0.0;
      for (int i = 0; i < d; i++) dot += qd[i] * (((double)c[i] - z) * s);
      sc[j] = dot * softmax_scale;
      if (sc[j] > mx) mx = sc[j];
    }
    double den = 0.0;
    for (int j = 0; j < len; j++) {
      sc[j] = exp(sc[j] - mx);
      den += sc[j];
    }
    for (int i = 0; i < d; i++) out[(size_t)h * d + i] = 0.0;
    for (int j = 0; j < len; j++) {
      const size_t row = (size_t)g * cache_len + j;
      orc_unpack_nibbles(v_codes + row * (d / 2), d, 0, c);
      const double s = orc_f16_to_f64(v_s[row]), z = orc_f16_to_f64(v_z[row]);
      const double p = sc[j] / den;
      for (int i = 0; i < d; i++) out[(size_t)h * d + i] += p * (((double)c[i] - z) * s);
    }
  }
  free(sc); free(qd); free(c);
  return 0;
}

/* Batch of decode steps: q [B][hq][d]; caches [B][hkv][cache_len][d/2] and
 * [B][hkv][cache_len]; lens [B] (slots attended per batch row); out [B][hq][d].
 * Rows are independent; `threads` > 1 spreads them over OpenMP threads. */
int orc_decode_attention_batch(const uint16_t *q, const uint8_t *k_codes, const uint8_t *v_codes,
                               const uint16_t *k_s, const uint16_t *k_z, const uint16_t *v_s,
                               const uint16_t *v_z, const int32_t *lens, int B, int hq, int hkv, int d,
                               int cache_len, double softmax_scale, double *out, int threads) {
  int rc = 0;
#pragma omp parallel for schedule(dynamic, 1) num_threads(threads > 0 ? threads : 1) reduction(| : rc)
  for (int b = 0; b < B; b++) {
    const size_t cb = (size_t)b * hkv * cache_len;
    rc |= orc_decode_attention(q + (size_t)b * hq * d, k_codes + cb * (d / 2), v_codes + cb * (d / 2),
                               k_s + cb, k_z + cb, v_s + cb, v_z + cb, hq, hkv, d, cache_len, lens[b],
                               softmax_scale, out + (size_t)b * hq * d);
  }
  return rc ? -1 : 0;
}

/* ------------------------------------------------------------------ */
/* Self-test helpers: RMSNorm [SW "The math, slowly"; RQ "Computational */
/* invariance"]                                                         */
/* ------------------------------------------------------------------ */

void orc_rmsnorm(const double *h, int d, double eps, double *out) {
  double ss = 0.0;
  for (int i = 0; i < d; i++) ss += h[i] * h[i];
  double r = sqrt(ss / d + eps);
  for (int i = 0; i < d; i++) out[i] = h[i] / r;
}

/* Mean squared difference of two fp64 vectors. */
double orc_mse(const double *a, const double *b, int64_t n) {
  double acc = 0.0;
  for (int64_t i = 0; i < n; i++) {
    double d = a[i] - b[i];
    acc += d * d;
  }
  return n ? acc / (double)n : 0.0;
}
