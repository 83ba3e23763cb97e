/*
 * awq_oracle.c -- CPU ORACLE for the W4A16 AWQ linear layer.  TEST INFRASTRUCTURE ONLY.
 *
 * Plain, single-threaded, slow and obviously correct.  It shares no code with the CUDA library: the
 * fp16 conversions, the quantizer, the packed layout and the matmul are written here from the IEEE 754
 * definitions, from the pages and from the prose layout description in the library's public header.
 * Only the test suite, the smoke check and the CPU-baseline leg of the benchmark may load it.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC (x86-64 SSE2 arithmetic, so
 * every float / double operation below is one correctly rounded IEEE operation).
 *
 * Sources (web pages on AWQ, cited by title and section):
 *   [AWQ/GPTQ]  "AWQ and GPTQ algorithms" (jsqmd.com): section 2.1 (2) importance E[|X_j|] over the
 *               calibration data; section 2.1 (3) multiply salient weight channels by s and divide the
 *               activations by s at inference (equivalent before rounding); section 1.1 W4A16.
 *   [LLM-AWQ]   "LLM-AWQ academic impact" (CSDN mirror), "quantization flow": w_bit 4, group size 128.
 *   [AutoAWQ]   "LLM quantization speed-up" (bjdmk.com.cn), "quantization parameters": group 128,
 *               zero-point quantization.
 * Readings where the pages are silent (the same ones the public header states):
 *   - grid: asymmetric min/max round-to-nearest over each group of 128 channels of one output row:
 *     scale = max((max - min)/15, 1e-5) rounded to fp16, zero = clamp(rint(-min/scale), 0, 15),
 *     q = clamp(rint(w/scale) + zero, 0, 15); fp32 arithmetic, rint = half to even;
 *   - the AWQ scale exponent is 0.5: s = fp16((mean_r |x_rj|)^0.5), computed in fp64;
 *   - activations: x' = fp16(x / s) with the division in fp64.
 *
 * Parity pins (each function is checked by tests/test_oracle_pins.py against something other than
 * itself): numpy's float16 conversions, closed forms of the grid, the round-trip bound, q = z gives 0,
 * s = 1 equals plain RTN, an independent unpacker, neutrality of the scaling in fp64, and brute-force
 * matmuls.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------------------------------ */
/* IEEE binary16 conversions, from the definition of the format (1 sign, 5 exponent, 10 fraction bits,
 * bias 15, subnormals k * 2^-24).                                                                   */

/* Exact widening of a binary16 bit pattern to double. */
double oracle_f16_to_f64(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1F;
  int f = h & 0x3FF;
  double v;
  if (e == 0x1F) {
    v = f ? NAN : INFINITY;
  } else if (e == 0) {
    v = ldexp((double)f, -24); /* subnormal: f * 2^-24 */
  } else {
    v = ldexp((double)(1024 + f), e - 25); /* (1 + f/1024) * 2^(e-15) */
  }
  return sign ? -v : v;
}

float oracle_f16_to_f32(uint16_t h) { return (float)oracle_f16_to_f64(h); }

/* Round a double to the nearest binary16, ties to even, in ONE rounding step. */
uint16_t oracle_f64_to_f16(double d) {
  uint64_t b;
  memcpy(&b, &d, sizeof b);
  uint16_t sign = (uint16_t)((b >> 63) << 15);
  int e = (int)((b >> 52) & 0x7FF);
  uint64_t m = b & ((1ULL << 52) - 1);
  if (e == 0x7FF) return (uint16_t)(sign | 0x7C00 | (m ? 0x200 : 0)); /* Inf or (quiet) NaN */
  if (e == 0) return sign;            /* zero or a double subnormal: far below half of 2^-24 */
  int E = e - 1023;                   /* value = S * 2^(E - 52), S = 2^52 + m */
  if (E > 15) return (uint16_t)(sign | 0x7C00);
  uint64_t S = (1ULL << 52) | m;
  int qexp = (E > -14 ? E : -14) - 10; /* exponent of one unit in the last place of the result */
  int r = 52 + qexp - E;              /* bits of S below that unit */
  if (r >= 54) return sign;           /* value < half the smallest subnormal */
  uint64_t k = S >> r;
  uint64_t rem = S & ((1ULL << r) - 1);
  uint64_t half = 1ULL << (r - 1);
  if (rem > half || (rem == half && (k & 1))) k += 1;
  uint32_t out;
  if (E >= -14) {
    out = ((uint32_t)(E + 14) << 10) + (uint32_t)k; /* k in [1024, 2048]; 2048 carries into exponent */
  } else {
    out = (uint32_t)k; /* subnormal; k == 1024 is exactly the smallest normal */
  }
  if (out >= 0x7C00) return (uint16_t)(sign | 0x7C00);
  return (uint16_t)(sign | out);
}

/* float -> binary16: widening to double is exact, so this is one rounding of the float's value. */
uint16_t oracle_f32_to_f16(float f) { return oracle_f64_to_f16((double)f); }

void oracle_f64_to_f16_array(const double* d, size_t n, uint16_t* h) {
  for (size_t i = 0; i < n; ++i) h[i] = oracle_f64_to_f16(d[i]);
}

/* ------------------------------------------------------------------------------------------------ */
/* Step a1: per-channel AWQ scale ([AWQ/GPTQ] 2.1 (2), exponent 0.5).                               */
void oracle_act_scale(const uint16_t* xcal, int R, int K, uint16_t* s) {
  for (int j = 0; j < K; ++j) {
    double sum = 0.0;
    for (int r = 0; r < R; ++r) sum += fabs(oracle_f16_to_f64(xcal[(size_t)r * K + j]));
    double mean = sum / (double)R;
    s[j] = oracle_f64_to_f16(sqrt(mean));
  }
}

/* The scale at exponent alpha, for the scale search ([AWQ/GPTQ] 2.1 (3), [LLM-AWQ] "quantization flow"
 * stage 1): s_j = fp16((mean_r |xcal_rj|)^alpha), mean and power in fp64 (alpha = 0 gives s = 1). */
void oracle_act_pow(const uint16_t* xcal, int R, int K, double alpha, uint16_t* s) {
  for (int j = 0; j < K; ++j) {
    double sum = 0.0;
    for (int r = 0; r < R; ++r) sum += fabs(oracle_f16_to_f64(xcal[(size_t)r * K + j]));
    double mean = sum / (double)R;
    s[j] = oracle_f64_to_f16(alpha == 0.0 ? 1.0 : pow(mean, alpha));
  }
}

/* Step a7: activations divided by s ([AWQ/GPTQ] 2.1 (3)). */
void oracle_inv_scale(const uint16_t* x, const uint16_t* s, int M, int K, uint16_t* xp) {
  for (int m = 0; m < M; ++m)
    for (int k = 0; k < K; ++k) {
      size_t i = (size_t)m * K + k;
      xp[i] = oracle_f64_to_f16(oracle_f16_to_f64(x[i]) / oracle_f16_to_f64(s[k]));
    }
}

/* ------------------------------------------------------------------------------------------------ */
/* Steps a2-a5: fold s into W and quantize each (row, group) with the asymmetric grid of w_bit bits,
 * qmax = 2^w_bit - 1 (15 for the pages' 4 bits; 7 for the 3-bit grid):
 *   W [N][K] fp16, s [K] fp16 or NULL (= 1).  Outputs, unpacked: q [N][K] codes 0..qmax,
 *   sc [N][K/g] fp16 scales, z [N][K/g] zeros 0..qmax.                                               */
void oracle_quantize_bits(const uint16_t* W, const uint16_t* s, int N, int K, int g, int w_bit, uint8_t* q,
                          uint16_t* sc, uint8_t* z) {
  const float qmax = (float)((1 << w_bit) - 1);
  int G = K / g;
  float* wp = (float*)malloc(sizeof(float) * (size_t)g);
  for (int n = 0; n < N; ++n) {
    for (int gi = 0; gi < G; ++gi) {
      /* a2: w' = W * s in fp32 (exact) */
      for (int e = 0; e < g; ++e) {
        int k = gi * g + e;
        float w = oracle_f16_to_f32(W[(size_t)n * K + k]);
        float sk = s ? oracle_f16_to_f32(s[k]) : 1.0f;
        wp[e] = w * sk;
      }
      /* a3: group min and max */
      float mn = wp[0], mx = wp[0];
      for (int e = 1; e < g; ++e) {
        if (wp[e] < mn) mn = wp[e];
        if (wp[e] > mx) mx = wp[e];
      }
      /* a4: scale (fp16) and zero point */
      float range = mx - mn;
      float sc32 = range / qmax;
      if (sc32 < 1e-5f) sc32 = 1e-5f;
      uint16_t sch = oracle_f32_to_f16(sc32);
      float S = oracle_f16_to_f32(sch);
      float zf = rintf(-mn / S);
      if (zf < 0.0f) zf = 0.0f;
      if (zf > qmax) zf = qmax;
      int zi = (int)zf;
      sc[(size_t)n * G + gi] = sch;
      z[(size_t)n * G + gi] = (uint8_t)zi;
      /* a5: codes */
      for (int e = 0; e < g; ++e) {
        float r = rintf(wp[e] / S);
        float v = r + (float)zi;
        if (v < 0.0f) v = 0.0f;
        if (v > qmax) v = qmax;
        q[(size_t)n * K + gi * g + e] = (uint8_t)(int)v;
      }
    }
  }
  free(wp);
}

void oracle_quantize(const uint16_t* W, const uint16_t* s, int N, int K, int g, uint8_t* q, uint16_t* sc,
                     uint8_t* z) {
  oracle_quantize_bits(W, s, N, K, g, 4, q, sc, z);
}

/* ------------------------------------------------------------------------------------------------ */
/* Step a6: write the packed layout described in the public header (prose), from unpacked q, sc, z.
 * Rows N .. N_pad-1 are zero.                                                                       */
static int round_up32(int n) { return (n + 31) / 32 * 32; }

void oracle_pack(const uint8_t* q, const uint16_t* sc, const uint8_t* z, int N, int K, int g,
                 uint32_t* qweight, uint16_t* scales, uint32_t* qzeros) {
  int G = K / g;
  int Np = round_up32(N);
  int KC = K / 32;
  memset(qweight, 0, sizeof(uint32_t) * (size_t)Np * K / 8);
  memset(scales, 0, sizeof(uint16_t) * (size_t)G * Np);
  memset(qzeros, 0, sizeof(uint32_t) * (size_t)G * Np / 8);
  /* nibble position of channel offset e inside a word: even e -> e/2, odd e -> 4 + e/2 */
  for (int n = 0; n < N; ++n) {
    int rb = n / 32, r = n % 32;
    for (int k = 0; k < K; ++k) {
      int kc = k / 32, j = (k % 32) / 8, e = k % 8;
      int p = (e % 2 == 0) ? e / 2 : 4 + e / 2;
      size_t word = ((size_t)rb * KC + kc) * 128 + (size_t)r * 4 + j;
      qweight[word] |= (uint32_t)(q[(size_t)n * K + k] & 0xF) << (4 * p);
    }
    for (int gi = 0; gi < G; ++gi) {
      size_t unit = (size_t)rb * G + gi; /* unit-major scales and zeros */
      scales[unit * 32 + r] = sc[(size_t)n * G + gi];
      qzeros[unit * 4 + r / 8] |= (uint32_t)(z[(size_t)n * G + gi] & 0xF) << (4 * (r % 8));
    }
  }
}

/* Independent decoder of the packed layout (used to pin oracle_pack by round trip).  It walks the
 * packed words in storage order and asks, for every nibble, which (row, channel) it belongs to. */
void oracle_unpack(const uint32_t* qweight, const uint16_t* scales, const uint32_t* qzeros, int N, int K,
                   int g, uint8_t* q, uint16_t* sc, uint8_t* z) {
  int G = K / g;
  int Np = round_up32(N);
  size_t nwords = (size_t)Np * K / 8;
  static const int chan_of_nibble[8] = {0, 2, 4, 6, 1, 3, 5, 7};
  for (size_t w = 0; w < nwords; ++w) {
    size_t tile = w / 128;            /* 512-byte tile index = rb * (K/32) + kc */
    int within = (int)(w % 128);      /* 32 rows x 4 words */
    int r = within / 4, j = within % 4;
    int rb = (int)(tile / (size_t)(K / 32)), kc = (int)(tile % (size_t)(K / 32));
    int n = rb * 32 + r;
    for (int p = 0; p < 8; ++p) {
      int k = kc * 32 + j * 8 + chan_of_nibble[p];
      uint8_t code = (uint8_t)((qweight[w] >> (4 * p)) & 0xF);
      if (n < N) q[(size_t)n * K + k] = code;
    }
  }
  /* scales and zeros: walk the units in storage order */
  for (size_t unit = 0; unit < (size_t)(Np / 32) * G; ++unit) {
    int rb = (int)(unit / (size_t)G), gi = (int)(unit % (size_t)G);
    for (int r = 0; r < 32; ++r) {
      int n = rb * 32 + r;
      if (n >= N) continue;
      sc[(size_t)n * G + gi] = scales[unit * 32 + r];
      z[(size_t)n * G + gi] = (uint8_t)((qzeros[unit * 4 + r / 8] >> (4 * (r % 8))) & 0xF);
    }
  }
}

/* ------------------------------------------------------------------------------------------------ */
/* Exact dequantization: Wq = (q - z) * S in fp32 (|q - z| <= 15 times an 11-bit significand: exact). */
void oracle_dequant(const uint8_t* q, const uint16_t* sc, const uint8_t* z, int N, int K, int g, float* Wq) {
  int G = K / g;
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k) {
      int gi = k / g;
      float S = oracle_f16_to_f32(sc[(size_t)n * G + gi]);
      int d = (int)q[(size_t)n * K + k] - (int)z[(size_t)n * G + gi];
      Wq[(size_t)n * K + k] = (float)d * S;
    }
}

/* y[m][n] = sum_k x'[m][k] * Wq[n][k], plain triple loop accumulated in fp64. */
void oracle_linear_f64(const uint16_t* xp, const float* Wq, int M, int N, int K, double* y) {
  for (int m = 0; m < M; ++m)
    for (int n = 0; n < N; ++n) {
      double acc = 0.0;
      for (int k = 0; k < K; ++k)
        acc += oracle_f16_to_f64(xp[(size_t)m * K + k]) * (double)Wq[(size_t)n * K + k];
      y[(size_t)m * N + n] = acc;
    }
}

/* Sampled outputs straight from the unpacked quantization: y for the listed (m, n) pairs, fp64. */
void oracle_linear_pairs_f64(const uint16_t* xp, const uint8_t* q, const uint16_t* sc, const uint8_t* z,
                             int M, int N, int K, int g, const int32_t* ms, const int32_t* ns, int count,
                             double* out) {
  int G = K / g;
  (void)M;
  (void)N;
  for (int i = 0; i < count; ++i) {
    int m = ms[i], n = ns[i];
    double acc = 0.0;
    for (int k = 0; k < K; ++k) {
      int gi = k / g;
      double S = oracle_f16_to_f64(sc[(size_t)n * G + gi]);
      int d = (int)q[(size_t)n * K + k] - (int)z[(size_t)n * G + gi];
      acc += oracle_f16_to_f64(xp[(size_t)m * K + k]) * ((double)d * S);
    }
    out[i] = acc;
  }
}

/* ------------------------------------------------------------------------------------------------ */
/* GPTQ ([AWQ/GPTQ] section 3.1: minimise ||W X - W_hat X||_F^2 over the calibration activations, the
 * Hessian H = X^T X, columns quantized block by block (128 columns) with each column's quantization error
 * compensated in the columns not yet quantized through the inverse Hessian, the inverse obtained through
 * Cholesky factorisations, and lazy batch updates of the columns after the block; section 3.3: 1e-6 added
 * to the diagonal against a singular Hessian).  Everything in fp64 except the grid, which is the same fp32
 * asymmetric min/max grid as awq_pack (s = 1) applied to the current weights rounded to fp32.              */

/* In-place Cholesky of the symmetric positive definite n x n matrix A (row major): on return the lower
 * triangle holds L with A = L L^T and the strict upper triangle is zero.  Returns 0, or -1 if A is not
 * positive definite. */
int oracle_cholesky_lower(double* A, int n) {
  for (int j = 0; j < n; ++j) {
    double d = A[(size_t)j * n + j];
    for (int k = 0; k < j; ++k) d -= A[(size_t)j * n + k] * A[(size_t)j * n + k];
    if (!(d > 0.0)) return -1;
    double ljj = sqrt(d);
    A[(size_t)j * n + j] = ljj;
    for (int i = j + 1; i < n; ++i) {
      double v = A[(size_t)i * n + j];
      for (int k = 0; k < j; ++k) v -= A[(size_t)i * n + k] * A[(size_t)j * n + k];
      A[(size_t)i * n + j] = v / ljj;
    }
    for (int i = 0; i < j; ++i) A[(size_t)i * n + j] = 0.0;
  }
  return 0;
}

/* U, upper triangular with H^-1 = U^T U: H = L L^T (Cholesky), H^-1 = L^-T L^-1 (L^-1 by forward
 * substitution), then U = (Cholesky factor of H^-1)^T.  H is n x n row major (not modified). */
int oracle_gptq_u(const double* H, int n, double* U) {
  double* L = (double*)malloc(sizeof(double) * (size_t)n * n);
  double* Li = (double*)calloc((size_t)n * n, sizeof(double));
  if (!L || !Li) { free(L); free(Li); return -1; }
  memcpy(L, H, sizeof(double) * (size_t)n * n);
  int rc = oracle_cholesky_lower(L, n);
  if (rc == 0) {
    for (int c = 0; c < n; ++c) /* column c of L^-1: solve L x = e_c */
      for (int i = c; i < n; ++i) {
        double v = (i == c) ? 1.0 : 0.0;
        for (int k = c; k < i; ++k) v -= L[(size_t)i * n + k] * Li[(size_t)k * n + c];
        Li[(size_t)i * n + c] = v / L[(size_t)i * n + i];
      }
    for (int i = 0; i < n; ++i) /* H^-1 = L^-T L^-1 */
      for (int j = 0; j < n; ++j) {
        double v = 0.0;
        for (int k = (i > j ? i : j); k < n; ++k) v += Li[(size_t)k * n + i] * Li[(size_t)k * n + j];
        U[(size_t)i * n + j] = v;
      }
    rc = oracle_cholesky_lower(U, n);
    if (rc == 0)
      for (int i = 0; i < n; ++i) /* transpose the lower factor into the upper triangle */
        for (int j = i + 1; j < n; ++j) {
          U[(size_t)i * n + j] = U[(size_t)j * n + i];
          U[(size_t)j * n + i] = 0.0;
        }
  }
  free(L);
  free(Li);
  return rc;
}

/* The grid of one group (the awq_pack grid with s = 1) on the fp32 values v[0 .. g-1]. */
static void grid_params(const float* v, int g, uint16_t* sch, float* S, int* zi) {
  float mn = v[0], mx = v[0];
  for (int e = 1; e < g; ++e) {
    if (v[e] < mn) mn = v[e];
    if (v[e] > mx) mx = v[e];
  }
  float sc32 = (mx - mn) / 15.0f;
  if (sc32 < 1e-5f) sc32 = 1e-5f;
  *sch = oracle_f32_to_f16(sc32);
  *S = oracle_f16_to_f32(*sch);
  float zf = rintf(-mn / *S);
  if (zf < 0.0f) zf = 0.0f;
  if (zf > 15.0f) zf = 15.0f;
  *zi = (int)zf;
}

/* GPTQ of W [N][K] fp16 on calibration rows xcal [R][K] fp16 at group size g; outputs unpacked like
 * oracle_quantize (q [N][K], sc [N][K/g] fp16, z [N][K/g]).  Returns 0, or -1 if H is not positive
 * definite. */
int oracle_gptq(const uint16_t* W, const uint16_t* xcal, int N, int K, int R, int g, double damp, uint8_t* q,
                uint16_t* sc, uint8_t* z) {
  const int B = 128, G = K / g;
  double* H = (double*)calloc((size_t)K * K, sizeof(double));
  double* U = (double*)malloc(sizeof(double) * (size_t)K * K);
  double* Wc = (double*)malloc(sizeof(double) * (size_t)N * K);
  double* E = (double*)malloc(sizeof(double) * (size_t)N * B);
  float* gv = (float*)malloc(sizeof(float) * (size_t)g);
  float* S = (float*)malloc(sizeof(float) * (size_t)N);
  int* zz = (int*)malloc(sizeof(int) * (size_t)N);
  double* gx = (double*)malloc(sizeof(double) * (size_t)K);
  int rc = -1;
  if (!H || !U || !Wc || !E || !gv || !S || !zz || !gx) goto out;
  for (int r = 0; r < R; ++r) { /* H = X^T X, rows in order */
    for (int j = 0; j < K; ++j) gx[j] = oracle_f16_to_f64(xcal[(size_t)r * K + j]);
    for (int i = 0; i < K; ++i) {
      double xi = gx[i];
      if (xi == 0.0) continue;
      for (int j = 0; j < K; ++j) H[(size_t)i * K + j] += xi * gx[j];
    }
  }
  for (int i = 0; i < K; ++i) H[(size_t)i * K + i] += damp;
  if (oracle_gptq_u(H, K, U) != 0) goto out;
  for (size_t i = 0; i < (size_t)N * K; ++i) Wc[i] = oracle_f16_to_f64(W[i]);
  for (int b0 = 0; b0 < K; b0 += B) {
    int b1 = b0 + B < K ? b0 + B : K;
    for (int i = b0; i < b1; ++i) {
      if (i % g == 0) { /* a group starts: its grid from the current weights of its g columns */
        for (int n = 0; n < N; ++n) {
          for (int e = 0; e < g; ++e) gv[e] = (float)Wc[(size_t)n * K + i + e];
          grid_params(gv, g, &sc[(size_t)n * G + i / g], &S[n], &zz[n]);
          z[(size_t)n * G + i / g] = (uint8_t)zz[n];
        }
      }
      double d = U[(size_t)i * K + i];
      for (int n = 0; n < N; ++n) {
        double w = Wc[(size_t)n * K + i];
        float v = rintf((float)w / S[n]) + (float)zz[n];
        if (v < 0.0f) v = 0.0f;
        if (v > 15.0f) v = 15.0f;
        int code = (int)v;
        q[(size_t)n * K + i] = (uint8_t)code;
        double err = (w - (double)(code - zz[n]) * (double)S[n]) / d;
        for (int j = i + 1; j < b1; ++j) Wc[(size_t)n * K + j] -= err * U[(size_t)i * K + j];
        E[(size_t)n * B + (i - b0)] = err;
      }
    }
    for (int n = 0; n < N; ++n) /* lazy batch update of the columns after the block */
      for (int j = b1; j < K; ++j) {
        double v = 0.0;
        for (int t = 0; t < b1 - b0; ++t) v += E[(size_t)n * B + t] * U[(size_t)(b0 + t) * K + j];
        Wc[(size_t)n * K + j] -= v;
      }
  }
  rc = 0;
out:
  free(H); free(U); free(Wc); free(E); free(gv); free(S); free(zz); free(gx);
  return rc;
}

/* ------------------------------------------------------------------------------------------------ */
/* The packed 3-bit layout (the public header's prose, "3-BIT LAYOUT"): per 32-row block rb, 32-channel
 * chunk kc and row r, three 32-bit words at word (rb * (K/32) + kc) * 96 + 3 r:
 *   word 0: the low 2 bits of channels 0..15 of the chunk, word 1: of channels 16..31.  Channel 8j + 2p + h
 *           (j = 0..3 the 8-channel group, p = 0..3 the pair, h = 0..1) sits at bit 8 (j % 2) + 2p + 16h of
 *           word j / 2;
 *   word 2: the high bit of channel 8j + 2p + h at bit 4j + p + 16h.
 * Scales and zeros: exactly as the 4-bit layout (unit major, 64 B and 16 B per unit).                   */
void oracle_pack3(const uint8_t* q, const uint16_t* sc, const uint8_t* z, int N, int K, int g,
                  uint32_t* qweight, uint16_t* scales, uint32_t* qzeros) {
  int G = K / g;
  int Np = round_up32(N);
  int KC = K / 32;
  memset(qweight, 0, sizeof(uint32_t) * (size_t)Np * KC * 3);
  memset(scales, 0, sizeof(uint16_t) * (size_t)G * Np);
  memset(qzeros, 0, sizeof(uint32_t) * (size_t)G * Np / 8);
  for (int n = 0; n < N; ++n) {
    int rb = n / 32, r = n % 32;
    for (int k = 0; k < K; ++k) {
      int kc = k / 32, c = k % 32, j = c / 8, p = (c % 8) / 2, h = c % 2;
      uint32_t code = q[(size_t)n * K + k] & 7u;
      size_t base = ((size_t)rb * KC + kc) * 96 + (size_t)r * 3;
      qweight[base + (size_t)(j / 2)] |= (code & 3u) << (8 * (j % 2) + 2 * p + 16 * h);
      qweight[base + 2] |= (code >> 2) << (4 * j + p + 16 * h);
    }
    for (int gi = 0; gi < G; ++gi) {
      size_t unit = (size_t)rb * G + gi;
      scales[unit * 32 + r] = sc[(size_t)n * G + gi];
      qzeros[unit * 4 + r / 8] |= (uint32_t)(z[(size_t)n * G + gi] & 0xF) << (4 * (r % 8));
    }
  }
}

/* Independent decoder of the 3-bit layout: walks every stored word and asks which (row, channel) each of
 * its bits belongs to. */
void oracle_unpack3(const uint32_t* qweight, int N, int K, uint8_t* q) {
  int Np = round_up32(N);
  int KC = K / 32;
  size_t nwords = (size_t)Np * KC * 3;
  memset(q, 0, (size_t)N * K);
  for (size_t w = 0; w < nwords; ++w) {
    size_t tile = w / 96;
    int within = (int)(w % 96), r = within / 3, kind = within % 3;
    int rb = (int)(tile / (size_t)KC), kc = (int)(tile % (size_t)KC);
    int n = rb * 32 + r;
    if (n >= N) continue;
    for (int bit = 0; bit < 32; ++bit) {
      uint32_t v = (qweight[w] >> bit) & 1u;
      int h = bit / 16, b = bit % 16, c, shift;
      if (kind < 2) { /* low bits: b = 8 (j % 2) + 2p + t, t the bit of the 2-bit field */
        int jj = b / 8, p = (b % 8) / 2, t = b % 2;
        c = 8 * (2 * kind + jj) + 2 * p + h;
        shift = t;
      } else { /* high bit: b = 4j + p */
        int j = b / 4, p = b % 4;
        c = 8 * j + 2 * p + h;
        shift = 2;
      }
      q[(size_t)n * K + kc * 32 + c] |= (uint8_t)(v << shift);
    }
  }
}
