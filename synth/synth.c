/*
 * synth.c -- seeded synthetic inputs for the FP8 x FP4 MoE layer.
 *
 * Input preparation only: it draws the workloads' random tensors and casts
 * them to the storage formats the layer consumes (E4M3 activations with one
 * UE8M0 scale per 1x32 block, E2M1 weights with one UE8M0 scale per 1x32
 * block, int32 top-k ids and fp32 top-k weights).  It holds none of the
 * layer's own arithmetic (no GEMM, no SwiGLU, no requantisation of the
 * intermediate, no combine); both the CUDA library's tests and the CPU
 * oracle consume its output.  Its casts are written here a third time (by
 * nearest-value search over codebooks built from the bit definitions), so
 * they share nothing with either side.
 *
 * Random numbers: counter-based.  Draw i of (seed, stream) is the splitmix64
 * finaliser applied to (seed ^ stream << 40 ^ i) + 0x9E3779B97F4A7C15; two
 * 53-bit uniforms make one Box-Muller pair (cos branch for even i, sin for
 * odd i; computed in single precision).  Streams: 1 = x, 2 = W1,
 * 3 = W2, 4 = router logits, 5 = the random expert ranking behind the
 * Zipf bias.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define TWO_PI 6.283185307179586476925286766559

static inline uint64_t draw_u64(uint64_t seed, uint64_t stream, uint64_t i) {
  uint64_t z = (seed ^ (stream << 40) ^ i) + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

/* uniform in (0, 1): (53-bit integer + 0.5) / 2^53 */
static inline double draw_unif(uint64_t seed, uint64_t stream, uint64_t i) {
  return ((double)(draw_u64(seed, stream, i) >> 11) + 0.5) * 0x1.0p-53;
}

/* normals n[2p], n[2p+1] of (seed, stream) */
static inline void draw_normal_pair(uint64_t seed, uint64_t stream, uint64_t p, double* n0,
                                    double* n1) {
  /* single-precision transcendental functions: ample for synthetic data */
  float u1 = (float)draw_unif(seed, stream, 2 * p), u2 = (float)draw_unif(seed, stream, 2 * p + 1);
  if (u1 <= 0.0f) u1 = 0x1.0p-30f;
  float r = sqrtf(-2.0f * logf(u1));
  float th = (float)TWO_PI * u2;
  *n0 = (double)(r * cosf(th));
  *n1 = (double)(r * sinf(th));
}

static inline double draw_normal(uint64_t seed, uint64_t stream, uint64_t i) {
  double a, b;
  draw_normal_pair(seed, stream, i >> 1, &a, &b);
  return (i & 1) ? b : a;
}

/* ---- codebooks for the casts (magnitudes of the positive codes) -------- */
static double g_e4m3_mag[127];  /* codes 0x00..0x7E */
static double g_e2m1_mag[8];    /* codes 0..7 */
static int g_tables_ready = 0;

static void build_tables(void) {
  if (g_tables_ready) return;
  for (int c = 0; c < 127; ++c) {
    int e = (c >> 3) & 0xF, m = c & 7;
    g_e4m3_mag[c] = e ? ldexp(1.0 + m / 8.0, e - 7) : ldexp(m / 8.0, -6);
  }
  for (int c = 0; c < 8; ++c) {
    int e = (c >> 1) & 3, m = c & 1;
    g_e2m1_mag[c] = e ? ldexp(1.0 + m / 2.0, e - 1) : 0.5 * m;
  }
  g_tables_ready = 1;
}

/* nearest entry of an ascending table; ties go to the even code; values
 * beyond the last entry take the last entry (saturating cast). */
static inline int nearest_code(const double* mag, int n, double a) {
  if (a >= mag[n - 1]) return n - 1;
  int lo = 0, hi = n - 1;                       /* mag[lo] <= a < mag[hi] */
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (mag[mid] <= a) lo = mid; else hi = mid;
  }
  double dl = a - mag[lo], dh = mag[hi] - a;
  if (dl < dh) return lo;
  if (dh < dl) return hi;
  return (lo & 1) ? hi : lo;
}

/* smallest e with qmax * 2^e >= amax (0 for amax == 0), clamped to +-127 */
static inline int cast_exponent(double amax, double qmax) {
  if (!(amax > 0.0)) return 0;
  int ex;
  frexp(amax / qmax, &ex);                     /* amax/qmax in [2^(ex-1), 2^ex) */
  int e = ex - 1;
  while (ldexp(qmax, e) < amax) e++;
  while (ldexp(qmax, e - 1) >= amax) e--;
  if (e < -127) e = -127;
  if (e > 127) e = 127;
  return e;
}

/* x: [T, H] E4M3 codes, x_sf: [T, H/128] int32 (byte j = scale of block 4i+j) */
void synth_x(int T, int H, uint64_t seed, uint8_t* x, int32_t* x_sf) {
  build_tables();
#pragma omp parallel for schedule(static)
  for (int t = 0; t < T; ++t) {
    double v[32];
    for (int b = 0; b < H / 32; ++b) {
      uint64_t base = (uint64_t)t * H + (uint64_t)b * 32;
      for (int i = 0; i < 32; i += 2) draw_normal_pair(seed, 1, (base + i) >> 1, &v[i], &v[i + 1]);
      double amax = 0;
      for (int i = 0; i < 32; ++i) amax = fmax(amax, fabs(v[i]));
      int e = cast_exponent(amax, 448.0);
      const double inv = ldexp(1.0, -e);         /* exact power of two */
      for (int i = 0; i < 32; ++i) {
        double a = v[i] * inv;
        int c = nearest_code(g_e4m3_mag, 127, fabs(a));
        x[base + i] = (uint8_t)(c | (a < 0 ? 0x80 : 0));
      }
      uint32_t* word = (uint32_t*)&x_sf[(size_t)t * (H / 128) + b / 4];
      uint32_t sh = 8u * (uint32_t)(b % 4);
      *word = (*word & ~(0xFFu << sh)) | ((uint32_t)(e + 127) << sh);
    }
  }
}

/* W: [E, N, K] drawn N(0, std^2), cast to E2M1 per 1x32 block along K.
 * Out: w [E, N, K/2] (low nibble = even k), w_sf [E, N, K/32] UE8M0. */
void synth_w(int E, int N, int K, uint64_t seed, uint64_t stream, double std, uint8_t* w,
             uint8_t* w_sf) {
  build_tables();
  int64_t rows = (int64_t)E * N;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    double v[32];
    for (int b = 0; b < K / 32; ++b) {
      uint64_t base = (uint64_t)r * K + (uint64_t)b * 32;
      for (int i = 0; i < 32; i += 2) {
        draw_normal_pair(seed, stream, (base + i) >> 1, &v[i], &v[i + 1]);
        v[i] *= std;
        v[i + 1] *= std;
      }
      double amax = 0;
      for (int i = 0; i < 32; ++i) amax = fmax(amax, fabs(v[i]));
      int e = cast_exponent(amax, 6.0);
      const double inv = ldexp(1.0, -e);         /* exact power of two */
      uint8_t* dst = w + (size_t)r * (K / 2) + (size_t)b * 16;
      for (int i = 0; i < 32; i += 2) {
        double a0 = v[i] * inv, a1 = v[i + 1] * inv;
        int c0 = nearest_code(g_e2m1_mag, 8, fabs(a0)) | (a0 < 0 ? 8 : 0);
        int c1 = nearest_code(g_e2m1_mag, 8, fabs(a1)) | (a1 < 0 ? 8 : 0);
        dst[i / 2] = (uint8_t)(c0 | (c1 << 4));
      }
      w_sf[(size_t)r * (K / 32) + b] = (uint8_t)(e + 127);
    }
  }
}

/* Router: logits[t][e] ~ N(0,1) (stream 4) plus an optional per-expert bias
 * b_e = -zipf_s * ln(rank_e), rank a seeded random permutation of 1..E
 * (stream 5).  Top-k by descending biased logit, ties to the lower expert
 * index.  Weights over the chosen k: mode 0 = softmax of the chosen logits,
 * mode 1 = sigmoid of the chosen logits divided by their sum. */
void synth_routing(int T, int E, int k, uint64_t seed, int mode, double zipf_s, int32_t* idx,
                   float* wts) {
  double* bias = (double*)calloc((size_t)E, sizeof(double));
  if (zipf_s > 0) {
    int* rank = (int*)malloc(sizeof(int) * (size_t)E);
    for (int e = 0; e < E; ++e) rank[e] = e + 1;
    for (int i = E - 1; i > 0; --i) {
      int j = (int)floor(draw_unif(seed, 5, (uint64_t)i) * (i + 1));
      if (j > i) j = i;
      int tmp = rank[i]; rank[i] = rank[j]; rank[j] = tmp;
    }
    for (int e = 0; e < E; ++e) bias[e] = -zipf_s * log((double)rank[e]);
    free(rank);
  }
#pragma omp parallel for schedule(static)
  for (int t = 0; t < T; ++t) {
    double* lg = (double*)malloc(sizeof(double) * (size_t)E);
    char* used = (char*)calloc((size_t)E, 1);
    double chosen[64];
    for (int e = 0; e < E; ++e) lg[e] = draw_normal(seed, 4, (uint64_t)t * E + e) + bias[e];
    for (int s = 0; s < k; ++s) {
      int best = -1;
      for (int e = 0; e < E; ++e)
        if (!used[e] && (best < 0 || lg[e] > lg[best])) best = e;
      used[best] = 1;
      idx[(size_t)t * k + s] = best;
      chosen[s] = lg[best];
    }
    double sum = 0, vals[64];
    if (mode == 0) {
      double mx = chosen[0];
      for (int s = 1; s < k; ++s) mx = fmax(mx, chosen[s]);
      for (int s = 0; s < k; ++s) { vals[s] = exp(chosen[s] - mx); sum += vals[s]; }
    } else {
      for (int s = 0; s < k; ++s) { vals[s] = 1.0 / (1.0 + exp(-chosen[s])); sum += vals[s]; }
    }
    for (int s = 0; s < k; ++s) wts[(size_t)t * k + s] = (float)(vals[s] / sum);
    free(lg);
    free(used);
  }
  free(bias);
}
