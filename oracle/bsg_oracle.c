/*
 * bsg_oracle.c -- plain fp64 CPU reference for the block-scaled grouped GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls this file; only the
 * tests, the smoke check and the CPU-baseline leg of the benchmark do.  It shares no code, header,
 * table or helper with the CUDA library.
 *
 * What it computes (the definition, written out with no blocking, fusion or reordering):
 *
 *   FP8 variant -- "[flashinfer] FlashInfer FP8 GEMM 최적화: 윈도우 세그먼트 KG1 프로그램", introduction
 *   and section 1 (kernel signature): E4M3 A[M,K] x B[G,N,K], FP32 scales per 128-element K block
 *   (a_scale per row and K block, b_scale per 128x128 block of B[g]), BF16 output, rows grouped by
 *   m_indices:
 *
 *     C[m,n] = bf16( sum_{kb < K/128} a_scale[m,kb] * b_scale[g,n/128,kb]
 *                                     * sum_{k in kb} e4m3(A[m,k]) * e4m3(B[g,n,k]) ),  g = m_indices[m]
 *
 *   NVFP4 variant -- "[onnxruntime] ... NVFP4 QMoE를 위한 네이티브 FP4xFP4 Prefill", section 1 (native
 *   FP4xFP4 grouped GEMM): E2M1 codes, one E4M3 scale per 16 K elements, an FP32 per-tensor factor:
 *
 *     C[m,n] = bf16( alpha[g] * sum_{j < K/16} ue4m3(sfa[m,j]) * ue4m3(sfb[g,n,j])
 *                                      * sum_{k in block j} e2m1(A[m,k]) * e2m1(B[g,n,k]) )
 *
 *   Every code is decoded from its bit fields.  Each inner block sum is formed in fp64, where it is
 *   exact (E4M3 products carry at most 8 significant bits, 128 of them need at most 42 bits; E2M1
 *   block sums are multiples of 1/4 below 600).  The result is rounded ONCE, fp64 -> bf16,
 *   round-to-nearest-even.  Rows whose m_indices value is negative or >= G are not written.
 *
 * Parity pins (tests/test_oracle_*.py): full decode tables against the format definitions and an
 * independent library decoder; bf16 rounding against fp32-exact library conversion and hand-checked
 * double-rounding cases; exact integer-grid products; grouped == G dense GEMMs; an exact rational
 * brute force; an fp64 library matmul of dequantised operands.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- element decoders ---------- */

/* E4M3 (the "FN" variant, max 448, no infinities): sign bit 7, exponent bits 6..3 (bias 7),
 * mantissa bits 2..0.  Exponent 0 is subnormal: m * 2^-9.  Exponent 15 with mantissa 7 is NaN. */
double bsg_oracle_dec_e4m3(uint8_t code) {
  int s = (code >> 7) & 1;
  int e = (code >> 3) & 0xF;
  int m = code & 0x7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) {
    v = ldexp((double)m, -9);
  } else {
    v = ldexp(1.0 + (double)m / 8.0, e - 7);
  }
  return s ? -v : v;
}

/* E2M1: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0.  Exponent 0 is subnormal: m * 0.5. */
double bsg_oracle_dec_e2m1(uint8_t nibble) {
  int s = (nibble >> 3) & 1;
  int e = (nibble >> 1) & 0x3;
  int m = nibble & 0x1;
  double v;
  if (e == 0) {
    v = 0.5 * (double)m;
  } else {
    v = ldexp(1.0 + (double)m / 2.0, e - 1);
  }
  return s ? -v : v;
}

/* Element k of a packed E2M1 row: two codes per byte, the lower-K element in the low nibble. */
static double e2m1_at(const uint8_t* row, int64_t k) {
  uint8_t byte = row[k / 2];
  uint8_t nib = (k % 2 == 0) ? (uint8_t)(byte & 0xF) : (uint8_t)(byte >> 4);
  return bsg_oracle_dec_e2m1(nib);
}

/* ---------------------------------------------------------------- fp64 -> bf16, RNE ---------- */

/* bf16: 1 sign, 8 exponent (bias 127), 7 mantissa bits.  The value is rounded once, directly from
 * the double, to the nearest bf16 (ties to the even mantissa), so no double rounding through fp32.
 * Overflow goes to +-Inf; NaN maps to the canonical quiet NaN with the input's sign. */
uint16_t bsg_oracle_bf16_from_f64(double x) {
  uint16_t sign = signbit(x) ? 0x8000u : 0u;
  double a = fabs(x);
  if (isnan(x)) return (uint16_t)(sign | 0x7FC0u);
  if (isinf(x)) return (uint16_t)(sign | 0x7F80u);
  if (a == 0.0) return sign;
  int e2;
  frexp(a, &e2);           /* a = f * 2^e2 with f in [0.5, 1): the leading bit has weight 2^(e2-1) */
  int lead = e2 - 1;
  if (lead < -126) lead = -126; /* subnormal range: fixed spacing 2^-133 */
  double ulp = ldexp(1.0, lead - 7);
  double q = a / ulp;     /* exact: division by a power of two */
  double r = nearbyint(q); /* default rounding mode: nearest, ties to even */
  double v = r * ulp;      /* exact */
  if (v >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80u);
  /* encode v exactly */
  if (v < ldexp(1.0, -126)) {
    /* subnormal (or rounded up to the smallest normal, handled by the general branch below) */
    uint32_t mant = (uint32_t)(v / ldexp(1.0, -133));
    return (uint16_t)(sign | mant);
  }
  int ev;
  double f = frexp(v, &ev); /* v = f * 2^ev, f in [0.5,1) */
  uint32_t biased = (uint32_t)(ev - 1 + 127);
  uint32_t mant = (uint32_t)((f * 2.0 - 1.0) * 128.0); /* exact: 7 fraction bits */
  return (uint16_t)(sign | (biased << 7) | mant);
}

/* ---------------------------------------------------------------- the two GEMMs -------------- */

static int routed_expert(const int32_t* m_indices, int64_t m, int64_t G) {
  int64_t g = m_indices ? (int64_t)m_indices[m] : 0;
  if (g < 0 || g >= G) return -1;
  return (int)g;
}

/*
 * FP8 grouped GEMM.  Operands: A uint8[M,K], B uint8[G,N,K], a_scale f32[M,K/128],
 * b_scale f32[G,ceil(N/128),K/128], m_indices int32[M] (NULL means every row goes to expert 0).
 * rows: which rows of C to compute (NULL = all M rows, in order); n_rows their count.
 * out_f64 (nullable) receives the unrounded sums, out_bf16 (nullable) the rounded result, both laid
 * out [n_rows, N]; entries of rows that are not routed are left untouched.
 * Returns 0, or -1 for an invalid size.
 */
int bsg_oracle_fp8_grouped(const uint8_t* A, const uint8_t* B, const float* a_scale,
                           const float* b_scale, const int32_t* m_indices, int64_t M, int64_t N,
                           int64_t K, int64_t G, const int64_t* rows, int64_t n_rows,
                           double* out_f64, uint16_t* out_bf16) {
  if (M < 0 || N <= 0 || K <= 0 || K % 128 != 0 || G <= 0) return -1;
  const int64_t KB = K / 128;
  const int64_t NB = (N + 127) / 128;
  if (!rows) n_rows = M;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < n_rows; ++i) {
    int64_t m = rows ? rows[i] : i;
    if (m < 0 || m >= M) continue;
    int g = routed_expert(m_indices, m, G);
    if (g < 0) continue;
    const uint8_t* arow = A + m * K;
    for (int64_t n = 0; n < N; ++n) {
      const uint8_t* brow = B + ((int64_t)g * N + n) * K;
      double acc = 0.0;
      for (int64_t kb = 0; kb < KB; ++kb) {
        double partial = 0.0;
        for (int64_t k = kb * 128; k < kb * 128 + 128; ++k)
          partial += bsg_oracle_dec_e4m3(arow[k]) * bsg_oracle_dec_e4m3(brow[k]);
        double sa = (double)a_scale[m * KB + kb];
        double sb = (double)b_scale[((int64_t)g * NB + n / 128) * KB + kb];
        acc += sa * sb * partial;
      }
      if (out_f64) out_f64[i * N + n] = acc;
      if (out_bf16) out_bf16[i * N + n] = bsg_oracle_bf16_from_f64(acc);
    }
  }
  return 0;
}

/*
 * NVFP4 grouped GEMM.  Operands: A uint8[M,K/2] (packed E2M1), B uint8[G,N,K/2], sfa uint8[M,K/16]
 * (E4M3 scale codes), sfb uint8[G,N,K/16], alpha f32[G], m_indices int32[M] (NULL: all rows to
 * expert 0).  rows / n_rows / out_f64 / out_bf16 as for the FP8 variant.
 * Returns 0, or -1 for an invalid size.
 */
int bsg_oracle_nvfp4(const uint8_t* A, const uint8_t* B, const uint8_t* sfa, const uint8_t* sfb,
                     const float* alpha, const int32_t* m_indices, int64_t M, int64_t N, int64_t K,
                     int64_t G, const int64_t* rows, int64_t n_rows, double* out_f64,
                     uint16_t* out_bf16) {
  if (M < 0 || N <= 0 || K <= 0 || K % 16 != 0 || G <= 0) return -1;
  const int64_t KS = K / 16;
  if (!rows) n_rows = M;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < n_rows; ++i) {
    int64_t m = rows ? rows[i] : i;
    if (m < 0 || m >= M) continue;
    int g = routed_expert(m_indices, m, G);
    if (g < 0) continue;
    const uint8_t* arow = A + m * (K / 2);
    for (int64_t n = 0; n < N; ++n) {
      const uint8_t* brow = B + ((int64_t)g * N + n) * (K / 2);
      double acc = 0.0;
      for (int64_t j = 0; j < KS; ++j) {
        double block = 0.0;
        for (int64_t k = j * 16; k < j * 16 + 16; ++k) block += e2m1_at(arow, k) * e2m1_at(brow, k);
        double s = bsg_oracle_dec_e4m3(sfa[m * KS + j]) *
                   bsg_oracle_dec_e4m3(sfb[((int64_t)g * N + n) * KS + j]);
        acc += s * block;
      }
      acc = (double)alpha[g] * acc;
      if (out_f64) out_f64[i * N + n] = acc;
      if (out_bf16) out_bf16[i * N + n] = bsg_oracle_bf16_from_f64(acc);
    }
  }
  return 0;
}

/* ---------------------------------------------------------------- activation quantisers ---- */

/*
 * The step just before the GEMM: BF16 activations quantised per row block into the GEMM's input
 * formats, optionally gathering the rows first (the MoE "expand" that puts each expert's tokens in
 * contiguous runs; row m of the output is row src_rows[m] of the input).  Written from the format
 * definitions and the quantisation recipe of the two GEMMs' inputs:
 *
 *   FP8, per 1 x 128 block:  scale = amax / 448;  code = e4m3_rne_satfinite(x / scale)
 *   NVFP4, per 1 x 16 block, global scale gs:
 *       s = ue4m3_rne_satfinite((amax16 / 6) / gs);  code = e2m1_rne_satfinite(x / (dec(s) * gs))
 *
 * Every operation is the IEEE fp32 one (each division and product correctly rounded, no fused
 * multiply-add): the quotient x / scale is formed once per element as a single correctly rounded fp32
 * division, and the encoder then rounds that fp32 value to the code.  The code is an integer decided
 * in fp32, so a GPU that reaches the same fp32 quotient reaches the same code.  A block whose scale is
 * zero (every element zero) gets all-zero codes.  The encoders round to the nearest representable
 * value, ties to the even code, and saturate at the largest finite magnitude (448, 6).
 */

/* fp32 -> E4M3 (FN) code: RNE, saturating at +-448; NaN -> 0x7F with the sign. */
uint8_t bsg_oracle_enc_e4m3(float x) {
  uint8_t sign = signbit(x) ? 0x80u : 0u;
  double a = fabs((double)x);
  if (isnan(x)) return (uint8_t)(sign | 0x7Fu);
  if (a >= 448.0) return (uint8_t)(sign | 0x7Eu);
  if (a < ldexp(1.0, -6)) {
    /* subnormal spacing 2^-9; a result of 8 quanta is the smallest normal, code 0x08 */
    double r = nearbyint(a / ldexp(1.0, -9));
    return (uint8_t)(sign | (uint8_t)r);
  }
  int e2;
  frexp(a, &e2);                         /* a in [2^(e2-1), 2^e2) */
  int e = e2 - 1;
  double r = nearbyint(a / ldexp(1.0, e - 3)); /* 8..16 quanta of the binade */
  int code = (e + 6) * 8 + (int)r;       /* (e + 7) << 3 | (r - 8); r = 16 carries into the exponent */
  if (code > 0x7E) code = 0x7E;
  return (uint8_t)(sign | (uint8_t)code);
}

/* fp32 -> E2M1 code (0..15): RNE on the magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}, saturating at +-6. */
uint8_t bsg_oracle_enc_e2m1(float x) {
  uint8_t sign = signbit(x) ? 0x8u : 0u;
  double a = fabs((double)x);
  int code;
  if (a >= 6.0) {
    code = 7;
  } else if (a < 2.0) {
    code = (int)nearbyint(a / 0.5);      /* quantum 0.5: codes 0..4 */
  } else if (a < 4.0) {
    code = 2 + (int)nearbyint(a);        /* quantum 1: codes 4..6 */
  } else {
    code = 4 + (int)nearbyint(a / 2.0);  /* quantum 2: codes 6..7 */
  }
  return (uint8_t)(sign | (uint8_t)code);
}

static float bf16_bits_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof(f));
  return f;
}

/* X bf16 bits [M_in, K]; src_rows int32 [M] or NULL (output row m = input row m, M_in >= M).
 * A uint8 [M, K] E4M3 codes; scale f32 [M, K/128].  Output rows whose source is outside
 * [0, M_in) are left untouched.  Returns 0, or -1 for an invalid size. */
int bsg_oracle_quant_fp8_rows(const uint16_t* X, const int32_t* src_rows, int64_t M_in, int64_t M, int64_t K,
                              uint8_t* A, float* scale) {
  if (M < 0 || M_in < 0 || K <= 0 || K % 128 != 0) return -1;
  const int64_t KB = K / 128;
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    int64_t src = src_rows ? (int64_t)src_rows[m] : m;
    if (src < 0 || src >= M_in) continue;
    const uint16_t* x = X + src * K;
    for (int64_t kb = 0; kb < KB; ++kb) {
      float amax = 0.0f;
      for (int64_t k = 0; k < 128; ++k) {
        float v = fabsf(bf16_bits_to_f32(x[kb * 128 + k]));
        if (v > amax) amax = v;
      }
      volatile float s = amax / 448.0f;
      scale[m * KB + kb] = s;
      for (int64_t k = 0; k < 128; ++k) {
        if (!(s > 0.0f)) {               /* zero block: zero codes */
          A[m * K + kb * 128 + k] = 0;
          continue;
        }
        float v = bf16_bits_to_f32(x[kb * 128 + k]);
        volatile float q = v / s;
        A[m * K + kb * 128 + k] = bsg_oracle_enc_e4m3(q);
      }
    }
  }
  return 0;
}

/* X bf16 bits [M_in, K]; gs the global scale (> 0); A uint8 [M, K/2] packed E2M1 (lower-K element
 * in the low nibble); sf uint8 [M, K/16] UE4M3 codes.  src_rows as above.  Returns 0 or -1. */
int bsg_oracle_quant_nvfp4_rows(const uint16_t* X, const int32_t* src_rows, float gs, int64_t M_in, int64_t M,
                                int64_t K, uint8_t* A, uint8_t* sf) {
  if (M < 0 || M_in < 0 || K <= 0 || K % 16 != 0) return -1;
  const int64_t KS = K / 16;
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    int64_t src = src_rows ? (int64_t)src_rows[m] : m;
    if (src < 0 || src >= M_in) continue;
    const uint16_t* x = X + src * K;
    for (int64_t j = 0; j < KS; ++j) {
      float amax = 0.0f;
      for (int64_t k = 0; k < 16; ++k) {
        float v = fabsf(bf16_bits_to_f32(x[j * 16 + k]));
        if (v > amax) amax = v;
      }
      volatile float t = amax / 6.0f;
      volatile float t2 = (gs > 0.0f) ? t / gs : 0.0f;
      uint8_t sc = bsg_oracle_enc_e4m3(t2);
      sf[m * KS + j] = sc;
      volatile float denom = (float)bsg_oracle_dec_e4m3(sc) * gs;
      uint8_t codes[16];
      for (int64_t k = 0; k < 16; ++k) {
        if (!(denom > 0.0f)) {           /* zero scale: zero codes */
          codes[k] = 0;
          continue;
        }
        float v = bf16_bits_to_f32(x[j * 16 + k]);
        volatile float q = v / denom;
        codes[k] = bsg_oracle_enc_e2m1(q);
      }
      for (int64_t k = 0; k < 16; k += 2)
        A[m * (K / 2) + (j * 16 + k) / 2] = (uint8_t)(codes[k] | (codes[k + 1] << 4));
    }
  }
  return 0;
}

/* ---------------------------------------------------------------- MoE expand permutation ---- */

/*
 * The MoE "expand" that precedes the activation quantiser and the grouped GEMM (the expanded input
 * rows of the ONNX Runtime page, "[onnxruntime] ONNX Runtime: Blackwell (SM120+)에서 NVFP4 QMoE를 위한
 * 네이티브 FP4xFP4 Prefill 최적화", section 1): every token t has top_k expert choices
 * expert_ids[t, k]; the T * top_k (token, choice) entries are laid out expert by expert so that each
 * expert's rows form one contiguous run of the GEMM's A.  Written as a plain stable counting sort of
 * the entries, taken in token-major order i = t * top_k + k, by their expert:
 *
 *   count[g]          = number of entries with expert g                 (g in [0, G))
 *   expert_offsets[g] = count[0] + ... + count[g - 1];  expert_offsets[G] = entries placed
 *   entry i with expert g in [0, G) goes to the next free position p of g's run, in increasing i:
 *       src_rows[p] = t,  m_indices[p] = g,  dst_rows[i] = p
 *   an entry whose expert is outside [0, G) is dropped: dst_rows[i] = -1
 *   positions p in [expert_offsets[G], T * top_k) hold src_rows[p] = m_indices[p] = -1
 *
 * so the GEMM skips those rows and the quantiser leaves them untouched.  dst_rows is the inverse
 * map a later combine needs (row dst_rows[t, k] of the GEMM's output belongs to token t, choice k).
 * Returns 0, or -1 for an invalid size.
 */
int bsg_oracle_moe_permute(const int32_t* expert_ids, int64_t T, int64_t top_k, int64_t G, int32_t* src_rows,
                           int32_t* m_indices, int32_t* dst_rows, int32_t* expert_offsets) {
  if (T < 0 || top_k < 1 || G < 1) return -1;
  const int64_t n = T * top_k;
  int64_t* next = (int64_t*)calloc((size_t)G, sizeof(int64_t));
  if (!next) return -1;
  for (int64_t i = 0; i < n; ++i) {
    const int32_t g = expert_ids[i];
    if (g >= 0 && g < G) next[g] += 1;
  }
  int64_t run = 0;
  for (int64_t g = 0; g < G; ++g) {
    const int64_t c = next[g];
    expert_offsets[g] = (int32_t)run;
    next[g] = run;
    run += c;
  }
  expert_offsets[G] = (int32_t)run;
  for (int64_t i = 0; i < n; ++i) {
    const int32_t g = expert_ids[i];
    if (g >= 0 && g < G) {
      const int64_t p = next[g]++;
      src_rows[p] = (int32_t)(i / top_k);
      m_indices[p] = g;
      dst_rows[i] = (int32_t)p;
    } else {
      dst_rows[i] = -1;
    }
  }
  for (int64_t p = run; p < n; ++p) {
    src_rows[p] = -1;
    m_indices[p] = -1;
  }
  free(next);
  return 0;
}

/* Threads the OpenMP loops above may use (for the timed CPU baseline). */
int bsg_oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void bsg_oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}
