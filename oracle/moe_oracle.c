/*
 * moe_oracle.c -- plain, slow, obviously-correct CPU reference for one
 * FP8 x FP4 Mixture-of-Experts layer forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link
 * or call this file: only the tests, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, table or helper with the CUDA
 * library; every codebook below is rebuilt here from its bit definition.
 *
 * Sources (web pages describing DeepGEMM's "Public Release 26/04"):
 *   [EXPLAINER] "DeepSeek DeepGEMM 2026年4月重磅更新：Mega MoE融合算子、FP4精度与极致性能优化"
 *               (chenxutan.com) -- section 3.1 (the five-step MoE pipeline),
 *               3.3 (buffer fields x / x_sf / topk_idx / topk_weights, BF16 y),
 *               4.1 (E4M3 / E2M1 bit layouts), 4.2 (UE8M0 scale factors,
 *               four per 32-bit int; FP32 accumulation), 9.2 (top-k + softmax
 *               router), 11.1 (per-block fine-grained scaling).
 *   [OVERVIEW]  "DeepGEMM: DeepSeek 把大模型核心算子打包成一座 CUDA 训练场"
 *               (zevenfang.github.io) -- section 4 (SM100 takes packed UE8M0
 *               scale factors), section 5 (Mega MoE = dispatch, linear1
 *               FP8xFP4, SwiGLU, linear2 FP8xFP4, combine).
 *
 * Readings taken where the pages are silent (each is listed with its reason
 * in the design notes of this repository):
 *   - FP8 activations x FP4 weights; W1 rows [0,I) are gate, [I,2I) are up.
 *   - one UE8M0 scale per 1x32 block along K for x, W1, W2 and the
 *     SwiGLU output; the scale exponent is the smallest e with
 *     qmax * 2^e >= amax (qmax 448 for E4M3), amax == 0 gives e = 0,
 *     e is clamped to [-127, 127].
 *   - SwiGLU(g, u) = silu(g) * u with silu(z) = z / (1 + exp(-z)).
 *   - the SwiGLU output is rounded to float, then requantised to E4M3
 *     (round to nearest even, saturating) with the rule above; linear2
 *     consumes the decoded requantised values.
 *   - the top-k weight multiplies the linear2 output of its slot; the
 *     weighted outputs are summed in slot order in double and y is the one
 *     BF16 round-to-nearest-even of that sum.  The fused operator keeps the
 *     expert outputs on chip up to the combine ([EXPLAINER] 3.2), so no
 *     intermediate rounding other than the FP8 requantisation of the
 *     SwiGLU output is part of the definition.
 *   - topk_idx == -1 means "slot unused"; any other id outside [0, E) is
 *     counted as invalid and skipped.
 *   - rows of one expert are ordered by ascending flattened index t*k+s.
 *
 * Parity pins (tests/test_oracle_*.py): codebook round trips and closed
 * forms, brute-force nearest-code search for the encoder, exhaustive scale
 * boundaries, the SwiGLU closed form, hand-worked MoE examples in
 * tests/golden/, a dense-FFN special case and a masked all-experts
 * formulation written independently in numpy, and invariants.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* Codebooks, from the bit definitions ([EXPLAINER] 4.1).                   */
/* ------------------------------------------------------------------------ */

/* E2M1: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit.  Exponent
 * field 0 is subnormal: value = m * 0.5.  No Inf / NaN. */
double orc_e2m1_value(unsigned code) {
  code &= 0xF;
  unsigned s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
  double mag = (e == 0) ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, (int)e - 1);
  return s ? -mag : mag;
}

/* E4M3 ("e4m3fn"): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits.
 * Exponent field 0 is subnormal: m/8 * 2^-6.  S.1111.111 is NaN; no Inf. */
double orc_e4m3_value(unsigned code) {
  code &= 0xFF;
  unsigned s = (code >> 7) & 1, e = (code >> 3) & 0xF, m = code & 7;
  if (e == 15 && m == 7) return NAN;
  double mag = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, (int)e - 7);
  return s ? -mag : mag;
}

/* UE8M0: unsigned 8-bit exponent, value 2^(b-127); 0xFF is NaN. */
double orc_ue8m0_value(unsigned b) {
  b &= 0xFF;
  if (b == 255) return NAN;
  return ldexp(1.0, (int)b - 127);
}

/* Round half to even of a non-negative double to an integer-valued double. */
static double rne_nonneg(double v) {
  double f = floor(v);
  double d = v - f;
  if (d > 0.5) return f + 1.0;
  if (d < 0.5) return f;
  return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* E4M3 encoder: nearest representable value, ties to the even code,
 * magnitudes beyond 448 saturate to 448 (no Inf in this format).  All
 * steps are exact in double: v / 2^e and (m - 1) * 8 are exact. */
unsigned orc_e4m3_encode(double v) {
  unsigned sign = (signbit(v) ? 0x80u : 0u);
  double a = fabs(v);
  if (a >= 448.0) return sign | 0x7Eu;
  if (a < ldexp(1.0, -6)) {                  /* subnormal grid, step 2^-9 */
    double q = rne_nonneg(a / ldexp(1.0, -9)); /* 0..8; 8 is the first normal */
    return sign | (unsigned)q;
  }
  int ex;
  double fr = frexp(a, &ex);                 /* a = fr * 2^ex, fr in [0.5,1) */
  int e = ex - 1;                            /* a = m * 2^e, m in [1,2) */
  double m = ldexp(fr, 1);
  double mq = rne_nonneg((m - 1.0) * 8.0);   /* 0..8 */
  if (mq == 8.0) { mq = 0.0; e += 1; }
  int ef = e + 7;
  if (ef > 15 || (ef == 15 && mq == 7.0)) return sign | 0x7Eu;
  return sign | (unsigned)((ef << 3) | (int)mq);
}

/* Block scale exponent: smallest integer e with qmax * 2^e >= amax; amax
 * of 0 gives 0; result clamped to [-127, 127] ([EXPLAINER] 11.1: one scale
 * per block, chosen from the block's absolute maximum). */
int orc_block_exponent(double amax, double qmax) {
  if (!(amax > 0.0)) return 0;
  int e = (int)ceil(log2(amax / qmax)) - 2;  /* start below, walk up exactly */
  while (ldexp(qmax, e) < amax) e++;
  while (ldexp(qmax, e - 1) >= amax) e--;
  if (e < -127) e = -127;
  if (e > 127) e = 127;
  return e;
}

/* silu(z) = z * sigmoid(z) = z / (1 + exp(-z)). */
double orc_silu(double z) { return z / (1.0 + exp(-z)); }

/* BF16 round-to-nearest-even of a double (through the exact float of the
 * same value when representable; ties decided on the double). */
uint16_t orc_bf16_rne(double v) {
  if (isnan(v)) return 0x7FC0;
  unsigned sign = signbit(v) ? 0x8000u : 0u;
  double a = fabs(v);
  if (a == 0.0) return (uint16_t)sign;
  /* bf16 has 8 significant bits; exponent range as fp32. */
  int ex;
  frexp(a, &ex);                 /* a in [2^(ex-1), 2^ex) */
  int e = ex - 1;
  if (e < -126) e = -126;        /* subnormal grid below 2^-126 */
  double ulp = ldexp(1.0, e - 7);
  double q = rne_nonneg(a / ulp) * ulp;
  if (q >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80u); /* overflow -> Inf */
  float f = (float)q;            /* exact: q has <= 8 significant bits */
  uint32_t bits;
  memcpy(&bits, &f, 4);
  return (uint16_t)(sign | (bits >> 16));
}

/* Requantise one block of n floats: amax over the block, E4M3 scale
 * exponent with qmax = 448, codes = E4M3(a / 2^e).  Writes n codes and the
 * UE8M0 byte (e + 127). */
void orc_requant_block(const float* a, int n, uint8_t* codes, uint8_t* sbyte) {
  double amax = 0.0;
  for (int i = 0; i < n; ++i) {
    double v = fabs((double)a[i]);
    if (v > amax) amax = v;
  }
  int e = orc_block_exponent(amax, 448.0);
  for (int i = 0; i < n; ++i) codes[i] = (uint8_t)orc_e4m3_encode(ldexp((double)a[i], -e));
  *sbyte = (uint8_t)(e + 127);
}

/* ------------------------------------------------------------------------ */
/* Plan: counting sort of assignments by expert ([EXPLAINER] 3.1: dispatch */
/* sends each token to its experts' contiguous regions).                   */
/* ------------------------------------------------------------------------ */

/* Returns the number of invalid ids (not -1 and outside [0,E)).
 *   counts[E]   assignments per expert
 *   offs[E+1]   exclusive prefix of counts
 *   poffs[E+1]  exclusive prefix of counts rounded up to a multiple of bm
 *   row_of[T*k] padded row of each assignment, -1 when skipped
 *   src_of[P]   assignment index t*k+s of each padded row, -1 for padding
 * P = poffs[E]; src_of must hold at least P entries (p_cap). */
int orc_plan(int T, int k, int E, int bm, const int32_t* topk_idx, int32_t* counts,
             int32_t* offs, int32_t* poffs, int32_t* row_of, int32_t* src_of, int p_cap) {
  int R = T * k, bad = 0;
  if (E <= 0 || T < 0 || k <= 0 || bm <= 0) return -1;
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int i = 0; i < R; ++i) {
    int e = topk_idx[i];
    if (e >= 0 && e < E) counts[e]++;
    else if (e != -1) bad++;
  }
  offs[0] = 0;
  poffs[0] = 0;
  for (int e = 0; e < E; ++e) {
    offs[e + 1] = offs[e] + counts[e];
    poffs[e + 1] = poffs[e] + (counts[e] + bm - 1) / bm * bm;
  }
  int P = poffs[E];
  for (int r = 0; r < P && r < p_cap; ++r) src_of[r] = -1;
  int* fill = (int*)calloc((size_t)E, sizeof(int));
  for (int i = 0; i < R; ++i) {            /* ascending i: stable */
    int e = topk_idx[i];
    if (e >= 0 && e < E) {
      int r = poffs[e] + fill[e]++;
      row_of[i] = r;
      if (r < p_cap) src_of[r] = i;
    } else {
      row_of[i] = -1;
    }
  }
  free(fill);
  return bad;
}

/* ------------------------------------------------------------------------ */
/* The layer forward ([EXPLAINER] 3.1 and 3.3; [OVERVIEW] 5).               */
/* ------------------------------------------------------------------------ */
/* Canonical layouts (all row-major):
 *   x      u8  [T, H]        E4M3 codes
 *   x_sf   i32 [T, H/128]    byte j (little-endian) of word i is the UE8M0
 *                            scale of K-block 4i+j (32 elements per block)
 *   topk_idx i32 [T, k], topk_w f32 [T, k]
 *   w1     u8  [E, 2I, H/2]  E2M1 codes, two per byte, low nibble = even k
 *   w1_sf  u8  [E, 2I, H/32] UE8M0
 *   w2     u8  [E, H, I/2],  w2_sf u8 [E, H, I/32]
 * Computes y for the tokens in token_list (n_list of them) into
 * y_out [n_list, H] (bf16 bits) and, when acc_out is not NULL, the double
 * sum of the weighted slot outputs before the final rounding [n_list, H].
 * Returns the number of invalid expert ids met. */

static inline double x_value(const uint8_t* x, const int32_t* x_sf, int H, int t, int h) {
  uint32_t word = (uint32_t)x_sf[(size_t)t * (H / 128) + h / 128];
  unsigned sb = (word >> (8 * ((h / 32) % 4))) & 0xFF;
  return orc_e4m3_value(x[(size_t)t * H + h]) * orc_ue8m0_value(sb);
}

static inline double w_value(const uint8_t* w, const uint8_t* w_sf, int N, int K, int e, int n,
                             int kk) {
  size_t row = (size_t)e * N + n;
  uint8_t byte = w[row * (K / 2) + kk / 2];
  unsigned code = (kk & 1) ? (byte >> 4) : (byte & 0xF);
  return orc_e2m1_value(code) * orc_ue8m0_value(w_sf[row * (K / 32) + kk / 32]);
}

int orc_moe_forward(int T, int H, int I, int E, int k, const uint8_t* x, const int32_t* x_sf,
                    const int32_t* topk_idx, const float* topk_w, const uint8_t* w1,
                    const uint8_t* w1_sf, const uint8_t* w2, const uint8_t* w2_sf,
                    const int32_t* token_list, int n_list, uint16_t* y_out, double* acc_out,
                    int nthreads) {
  (void)T;
  int bad = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : bad)
  for (int li = 0; li < n_list; ++li) {
    int t = token_list[li];
    double* xd = (double*)malloc(sizeof(double) * (size_t)H);
    double* g = (double*)malloc(sizeof(double) * 2 * (size_t)I);
    float* af = (float*)malloc(sizeof(float) * (size_t)I);
    double* ad = (double*)malloc(sizeof(double) * (size_t)I);
    uint8_t* q = (uint8_t*)malloc((size_t)I);
    double* acc = (double*)calloc((size_t)H, sizeof(double));
    for (int h = 0; h < H; ++h) xd[h] = x_value(x, x_sf, H, t, h);
    for (int s = 0; s < k; ++s) {
      int e = topk_idx[(size_t)t * k + s];
      if (e == -1) continue;
      if (e < 0 || e >= E) { bad++; continue; }
      /* linear1: g[j] = sum_h x[h] * W1[e][j][h], j < 2I */
      for (int j = 0; j < 2 * I; ++j) {
        double sum = 0.0;
        for (int h = 0; h < H; ++h) sum += xd[h] * w_value(w1, w1_sf, 2 * I, H, e, j, h);
        g[j] = sum;
      }
      /* SwiGLU: a[j] = silu(gate[j]) * up[j], rounded to float */
      for (int j = 0; j < I; ++j) af[j] = (float)(orc_silu(g[j]) * g[I + j]);
      /* requantise per 1x32 block, then decode */
      for (int b = 0; b < I / 32; ++b) {
        uint8_t sb;
        orc_requant_block(af + 32 * b, 32, q + 32 * b, &sb);
        for (int j = 32 * b; j < 32 * b + 32; ++j) ad[j] = orc_e4m3_value(q[j]) * orc_ue8m0_value(sb);
      }
      /* linear2, weighted, combined in double: acc[n] += w * sum_j a[j] * W2[e][n][j] */
      double wt = (double)topk_w[(size_t)t * k + s];
      for (int n = 0; n < H; ++n) {
        double sum = 0.0;
        for (int j = 0; j < I; ++j) sum += ad[j] * w_value(w2, w2_sf, H, I, e, n, j);
        acc[n] += wt * sum;
      }
    }
    for (int n = 0; n < H; ++n) {
      y_out[(size_t)li * H + n] = orc_bf16_rne(acc[n]);
      if (acc_out) acc_out[(size_t)li * H + n] = acc[n];
    }
    free(xd); free(g); free(af); free(ad); free(q); free(acc);
  }
  return bad;
}

/* ------------------------------------------------------------------------ */
/* FP8 x FP4 GEMM, dense and masked grouped ([EXPLAINER] 4.3: A FP8 [M, K]  */
/* with block scales, B FP4 [N, K/2] packed with UE8M0 scales, D BF16;     */
/* [OVERVIEW] 2 and [DAILY] "3. MoE模型专属优化": the masked grouped layout */
/* for CUDA-graph decode, where only the device knows each group's rows).  */
/* ------------------------------------------------------------------------ */
/* Layouts: a u8 [G, M, K] E4M3, a_sf i32 [G, M, K/128] (byte j of word i =
 * UE8M0 scale of K-block 4i+j, as x_sf), b u8 [G, N, K/2] E2M1 (low nibble
 * = even k), b_sf u8 [G, N, K/32], d u16 [G, M, N] BF16 bits.
 * D[g][m][n] = BF16_RNE( sum_k A[g][m][k] * B[g][n][k] ), decoded values,
 * summed in double, for m < rows_g where rows_g = masked_m[g] (clamped to
 * [0, M]) or M when masked_m is NULL.  Rows m >= rows_g are not written. */
void orc_gemm(int G, int M, int N, int K, const uint8_t* a, const int32_t* a_sf,
              const int32_t* masked_m, const uint8_t* b, const uint8_t* b_sf, uint16_t* d,
              int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
  for (int g = 0; g < G; ++g) {
    int rows = masked_m ? masked_m[g] : M;
    if (rows < 0) rows = 0;
    if (rows > M) rows = M;
    const uint8_t* ag = a + (size_t)g * M * K;
    const int32_t* asg = a_sf + (size_t)g * M * (K / 128);
#pragma omp parallel for schedule(dynamic, 1)
    for (int m = 0; m < rows; ++m) {
      double* ad = (double*)malloc(sizeof(double) * (size_t)K);
      for (int kk = 0; kk < K; ++kk) ad[kk] = x_value(ag, asg, K, m, kk);
      for (int n = 0; n < N; ++n) {
        double sum = 0.0;
        for (int kk = 0; kk < K; ++kk) sum += ad[kk] * w_value(b, b_sf, N, K, g, n, kk);
        d[((size_t)g * M + m) * N + n] = orc_bf16_rne(sum);
      }
      free(ad);
    }
  }
}

int orc_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* FP4 indexer: MQA logits with FP8 queries and FP4 keys ([EXPLAINER] 5.1   */
/* and 5.2, the fp8_fp4_mqa_logits call; [NEWS] "FP4 Indexer").             */
/* ------------------------------------------------------------------------ */
/* Readings (each with its reason in the design notes):
 *   - q is FP8 E4M3 and kv is FP4 E2M1, both with one UE8M0 scale per 1x32
 *     block along the head dimension (the library's fp8_fp4_* naming: FP8
 *     first operand, FP4 second);
 *   - logits[i][j] = sum_h weights[i][h] * max(0, sum_d q[i][h][d] * k[j][d])
 *     (the page's formula has a two-index logit and per-head weights; the
 *     softmax inside its ReLU is dropped);
 *   - only keys ks[i] <= j < ke[i] are scored; with clean != 0 every other
 *     entry of row i is -inf, otherwise it is not written;
 *   - the output is FP32 (the cleaned entries are -inf, which no FP4 code
 *     holds).
 * Layouts: q u8 [S, Hh, D] E4M3; q_sf i32 [S, Hh, D/128] (byte j of word i =
 * scale of block 4i+j, as x_sf); kv u8 [N, D/2] E2M1 (low nibble = even d);
 * kv_sf u8 [N, D/32]; weights f32 [S, Hh]; ks, ke i32 [S]; logits f32 [S, N].
 * When mag is not NULL, mag[i][j] = sum_h |weights[i][h]| * sum_d |q[i][h][d] * k[j][d]|
 * (the size of every product that enters the logit: a comparison with a
 * lower-precision computation scales its tolerance by it). */
void orc_mqa_logits(int S, int Hh, int D, int N, const uint8_t* q, const int32_t* q_sf,
                    const uint8_t* kv, const uint8_t* kv_sf, const float* weights,
                    const int32_t* ks, const int32_t* ke, int clean, float* logits, double* mag,
                    int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
#pragma omp parallel for schedule(dynamic, 1)
  for (int i = 0; i < S; ++i) {
    double* qd = (double*)malloc(sizeof(double) * (size_t)Hh * D);
    double* kd = (double*)malloc(sizeof(double) * (size_t)D);
    for (int h = 0; h < Hh; ++h)
      for (int d = 0; d < D; ++d)
        qd[(size_t)h * D + d] = x_value(q, q_sf, D, i * Hh + h, d);
    int lo = ks[i] < 0 ? 0 : ks[i];
    int hi = ke[i] > N ? N : ke[i];
    for (int j = 0; j < N; ++j) {
      float* out = logits + (size_t)i * N + j;
      if (j < lo || j >= hi) {
        if (clean) *out = -INFINITY;
        if (mag) mag[(size_t)i * N + j] = 0.0;
        continue;
      }
      for (int d = 0; d < D; ++d) kd[d] = w_value(kv, kv_sf, N, D, 0, j, d);
      double acc = 0.0, m = 0.0;
      for (int h = 0; h < Hh; ++h) {
        double s = 0.0, sa = 0.0;
        for (int d = 0; d < D; ++d) {
          s += qd[(size_t)h * D + d] * kd[d];
          sa += fabs(qd[(size_t)h * D + d] * kd[d]);
        }
        double w = (double)weights[(size_t)i * Hh + h];
        if (s > 0.0) acc += w * s;
        m += fabs(w) * sa;
      }
      *out = (float)acc;
      if (mag) mag[(size_t)i * N + j] = m;
    }
    free(qd);
    free(kd);
  }
}
