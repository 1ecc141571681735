/*
 * zq_oracle.c -- plain, slow, obviously-correct CPU oracle for causal prefill
 * attention in FP8 e4m3 / BF16 (fp64 arithmetic unless a step fixes a
 * precision).
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check and the CPU-baseline
 * leg of the benchmark may load this library.  It shares no code, header,
 * table or constant generator with the CUDA path.
 *
 * Sources (web pages re-reporting the same ZYFA announcement):
 *   [P1] "Zyphra ZYFA : FlashAttention en FP8 pour l'AMD MI355X, jusqu'a
 *        1,76 fois plus rapide" (lefilia.fr); paragraphs 1-3.
 *   [P2] "Zyphra rilascia ZYFA, kernel di attenzione FP8 ottimizzati per le
 *        GPU AMD" (aicronaca.it); sections "Che cosa ha annunciato Zyphra",
 *        "I numeri dichiarati e il confronto con AITER",
 *        "Perche l'FP8 non basta da solo", "Limiti e questioni aperte".
 *   [P3] "Zyphra ZYFA ... FP8 FlashAttention for AMD MI355X up to 1.76x"
 *        (ai4bro.com); sections TL;DR, "What is ZYFA",
 *        "Why FP8 attention underperforms", "How ZYFA works", "How accurate".
 *
 * Functions:
 *   zo_e4m3_decode / zo_e4m3_encode_rne_sat   OCP e4m3fn codec (bias 7,
 *        max 448, 0x7F/0xFF NaN).  [P3 TL;DR: "FP8 e4m3"]
 *   zo_fwht128_f32      unnormalised 128-point Walsh-Hadamard transform in
 *        fp32, butterflies at strides 1,2,...,64.  [P2 "Perche l'FP8 non
 *        basta da solo": Hadamard rotation of Q and K]
 *   zo_fwht64_f32       the same for 64 points (strides 1..32); the d = 192
 *        rotation uses it, scaled by fl32(sqrt 2), on channels 128..191.
 *   zo_quantize_fp8     per-tensor amax quantiser (R3).
 *   zo_attn_ref         exact fp64 softmax(QK^T*scale + causal mask)V (R1).
 *   zo_leanp_code       Lean P byte for a log2-domain value (used by R2).
 *   zo_attn_fp8_emul    scalar emulation of the FP8 P path: per-(row,64-key
 *        block) power-of-2 scaling, exact-exp2 or Lean P rounding, division
 *        by the sum of the rounded probabilities (R2).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int zo_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Thread count for the parallel loops that follow (n <= 0: leave as is).
 * Returns the count now in effect.  Only timing uses it (the single-thread
 * rate of the CPU baseline); results do not depend on it. */
int zo_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
  return omp_get_max_threads();
#else
  (void)n;
  return 1;
#endif
}

/* ------------------------------------------------------------------ */
/* e4m3fn codec                                                        */
/* ------------------------------------------------------------------ */

/* Value of an e4m3fn byte: sign bit, 4-bit exponent (bias 7), 3-bit mantissa.
 * Exponent field 0 encodes subnormals m * 2^-9.  0x7F / 0xFF are NaN. */
double zo_e4m3_decode(uint8_t b) {
  int sign = (b >> 7) & 1;
  int ex = (b >> 3) & 0xF;
  int man = b & 7;
  double v;
  if (ex == 0xF && man == 7) return NAN;
  if (ex == 0)
    v = ldexp((double)man, -9);
  else
    v = ldexp(1.0 + man / 8.0, ex - 7);
  return sign ? -v : v;
}

/* Round a real value to the nearest e4m3fn value (ties to even mantissa),
 * saturating to +-448 ("satfinite"); NaN maps to 0x7F.
 * Normal binade [2^ex, 2^(ex+1)), ex >= -6, holds 8 values spaced 2^(ex-3);
 * below 2^-6 the subnormals are spaced 2^-9.  a / spacing is exact in fp64,
 * so nearbyint (ties to even) rounds it; code = 8*(ex+7) + (count - 8) for a
 * normal binade and code = count for the subnormal range, and a count that
 * rounds up to the next binade lands on the next code by construction. */
uint8_t zo_e4m3_encode_rne_sat(double x) {
  if (isnan(x)) return 0x7F;
  uint8_t sign = signbit(x) ? 0x80 : 0;
  double a = fabs(x);
  if (a >= 448.0) return sign | 0x7E;
  int code;
  if (a < 0.015625) { /* 2^-6 */
    code = (int)nearbyint(ldexp(a, 9));
  } else {
    int ex;
    frexp(a, &ex); /* a = f * 2^ex, f in [0.5, 1) */
    ex -= 1;       /* a in [2^ex, 2^(ex+1)) */
    double cnt = nearbyint(ldexp(a, 3 - ex)); /* in [8, 16] */
    code = 8 * (ex + 7) + (int)cnt - 8;
  }
  if (code > 0x7E) code = 0x7E;
  return sign | (uint8_t)code;
}

/* ------------------------------------------------------------------ */
/* Hadamard rotation and quantiser (R3)                                */
/* ------------------------------------------------------------------ */

/* In-place unnormalised FWHT of 128 fp32 values (Sylvester ordering):
 * for h = 1,2,4,...,64 replace each pair (x[j], x[j+h]) by (a+b, a-b). */
void zo_fwht128_f32(float* x) {
  for (int h = 1; h < 128; h <<= 1)
    for (int i = 0; i < 128; i += 2 * h)
      for (int j = i; j < i + h; ++j) {
        float a = x[j], b = x[j + h];
        x[j] = a + b;
        x[j + h] = a - b;
      }
}

/* In-place unnormalised FWHT of 64 fp32 values, as above with h < 64. */
void zo_fwht64_f32(float* x) {
  for (int h = 1; h < 64; h <<= 1)
    for (int i = 0; i < 64; i += 2 * h)
      for (int j = i; j < i + h; ++j) {
        float a = x[j], b = x[j + h];
        x[j] = a + b;
        x[j + h] = a - b;
      }
}

/* The rotation of one d-channel vector: H128 on every 128-channel slice;
 * for d = 192 (the MLA query/key width) the last 64 channels get
 * sqrt(2) * H64 instead, each value multiplied by fl32(sqrt 2) after the
 * butterflies.  Then (R q).(R k) = 128 q.k for every slice (up to the fp32
 * rounding of sqrt 2), so one descale factor 2^-3.5 per tensor undoes the
 * rotation in QK^T for d = 128 and d = 192 alike. */
static void rotate_vec(float* x, int d) {
  int c = 0;
  for (; c + 128 <= d; c += 128) zo_fwht128_f32(x + c);
  if (c < d) {
    zo_fwht64_f32(x + c);
    for (int j = 0; j < 64; ++j) {
      volatile float y = x[c + j] * 1.41421356237309504880f; /* fl32(sqrt 2), one rounding */
      x[c + j] = y;
    }
  }
}

static float bf16_bits_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* Per-tensor FP8 quantiser.  x has n_vec vectors of d channels, fp32
 * (x_dtype 0) or bf16 bits (x_dtype 1).  With hadamard != 0 (d % 128 == 0,
 * or d == 192) every vector is rotated first (rotate_vec).
 *   amax    = max |x|                       (exact)
 *   inv     = fl32(448 / amax)
 *   q       = e4m3_rne_sat(fl32(x * inv))
 *   descale = fl32(amax / 448)   [ * fl32(2^-3.5) in fp32 when rotated ]
 * amax == 0 gives inv = 1 and descale = 0 semantics: q = 0, descale = 0.
 * Returns 0, or -1 for an unsupported argument. */
int zo_quantize_fp8(const void* x, int x_dtype, int64_t n_vec, int d, int hadamard,
                    uint8_t* out, float* descale) {
  if (n_vec < 0 || d <= 0 || (hadamard && d % 128 && d != 192)) return -1;
  int64_t n = n_vec * (int64_t)d;
  float* t = (float*)malloc(sizeof(float) * (size_t)(n > 0 ? n : 1));
  if (!t) return -1;
#pragma omp parallel for
  for (int64_t i = 0; i < n; ++i)
    t[i] = x_dtype == 0 ? ((const float*)x)[i] : bf16_bits_to_f32(((const uint16_t*)x)[i]);
  if (hadamard) {
#pragma omp parallel for
    for (int64_t v = 0; v < n_vec; ++v) rotate_vec(t + v * d, d);
  }
  float amax = 0.0f;
#pragma omp parallel for reduction(max : amax)
  for (int64_t i = 0; i < n; ++i) {
    float a = fabsf(t[i]);
    if (a > amax) amax = a;
  }
  volatile float inv_v = amax > 0.0f ? 448.0f / amax : 1.0f;
  float inv = inv_v;
#pragma omp parallel for
  for (int64_t i = 0; i < n; ++i) {
    volatile float s = t[i] * inv; /* one fp32 rounding of the product */
    out[i] = zo_e4m3_encode_rne_sat((double)s);
  }
  volatile float ds = amax / 448.0f;
  if (hadamard) {
    volatile float r = 0.08838834764831845f; /* fl32(2^-3.5) */
    ds = ds * r;
  }
  *descale = ds;
  free(t);
  return 0;
}

/* ------------------------------------------------------------------ */
/* Attention                                                          */
/* ------------------------------------------------------------------ */

/* Rows to evaluate: either all (rows == NULL) or a list of flat row ids
 * r = (b * Hq + h) * Sq + i.  Layouts: q (B,Sq,Hq,dqk), k (B,Sk,Hkv,dqk),
 * v (B,Sk,Hkv,dv), o (nrows, dv) in row-list order, lse (nrows). */
typedef struct {
  int B, Sq, Sk, Hq, Hkv, dqk, dv, causal;
  double scale;
} zo_shape;

static void row_coords(const zo_shape* s, int64_t r, int* b, int* h, int* i) {
  *i = (int)(r % s->Sq);
  int64_t bh = r / s->Sq;
  *h = (int)(bh % s->Hq);
  *b = (int)(bh / s->Hq);
}

/* Last visible key for query i: bottom-right causal alignment
 * (key c visible iff c <= i + Sk - Sq); all keys when not causal. */
static int last_key(const zo_shape* s, int i) {
  if (!s->causal) return s->Sk - 1;
  int L = i + s->Sk - s->Sq;
  return L < s->Sk - 1 ? L : s->Sk - 1;
}

static const double* qrow(const zo_shape* s, const double* q, int b, int i, int h) {
  return q + (((int64_t)b * s->Sq + i) * s->Hq + h) * s->dqk;
}
static const double* krow(const zo_shape* s, const double* k, int b, int c, int g) {
  return k + (((int64_t)b * s->Sk + c) * s->Hkv + g) * s->dqk;
}
static const double* vrow(const zo_shape* s, const double* v, int b, int c, int g) {
  return v + (((int64_t)b * s->Sk + c) * s->Hkv + g) * s->dv;
}

/* R1: exact attention in fp64.  [P3 TL;DR: causal forward (prefill)
 * attention; P1 para 2 / P2 "I numeri dichiarati": error measured against
 * an fp64 reference.]  GQA: query head h reads kv head h / (Hq / Hkv).
 * A row with no visible key gives o = 0, lse = -inf. */
int zo_attn_ref(const double* q, const double* k, const double* v, int B, int Sq, int Sk,
                int Hq, int Hkv, int dqk, int dv, double scale, int causal,
                const int64_t* rows, int64_t nrows, double* o, double* lse) {
  if (B <= 0 || Sq <= 0 || Sk <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv) return -1;
  zo_shape s = {B, Sq, Sk, Hq, Hkv, dqk, dv, causal, scale};
  int64_t n = rows ? nrows : (int64_t)B * Hq * Sq;
#pragma omp parallel
  {
    double* sc = (double*)malloc(sizeof(double) * (size_t)Sk);
#pragma omp for schedule(dynamic, 16)
    for (int64_t t = 0; t < n; ++t) {
      int b, h, i;
      row_coords(&s, rows ? rows[t] : t, &b, &h, &i);
      int g = h / (Hq / Hkv);
      int L = last_key(&s, i);
      double* orow = o + t * dv;
      for (int e = 0; e < dv; ++e) orow[e] = 0.0;
      if (L < 0) {
        lse[t] = -INFINITY;
        continue;
      }
      const double* qi = qrow(&s, q, b, i, h);
      double m = -INFINITY;
      for (int c = 0; c <= L; ++c) {
        const double* kc = krow(&s, k, b, c, g);
        double dot = 0.0;
        for (int e = 0; e < dqk; ++e) dot += qi[e] * kc[e];
        sc[c] = scale * dot;
        if (sc[c] > m) m = sc[c];
      }
      double l = 0.0;
      for (int c = 0; c <= L; ++c) {
        double p = exp(sc[c] - m);
        l += p;
        const double* vc = vrow(&s, v, b, c, g);
        for (int e = 0; e < dv; ++e) orow[e] += p * vc[e];
      }
      for (int e = 0; e < dv; ++e) orow[e] /= l;
      lse[t] = m + log(l);
    }
    free(sc);
  }
  return 0;
}

/* Lean P code for a log2-domain value z = y - e (P1 para 3: an e4m3 pattern
 * read as an integer grows by 8 per doubling, so 8*z plus the exponent bias
 * 56 = 7*8 gives the pattern of 2^z; P2 "Perche l'FP8 non basta da solo":
 * 2^x from a multiply-add and an integer conversion).  Rounding of 8*z is
 * half-to-even; the code is clamped to the finite range [0, 126]. */
int zo_leanp_code(double z) {
  double t = 8.0 * z;
  double r = nearbyint(t); /* default rounding mode: ties to even */
  double c = r + 56.0;
  if (c < 0.0) c = 0.0;
  if (c > 126.0) c = 126.0;
  return (int)c;
}

/* R2: FP8 P-path emulation.  For each row, y_c = s_c * log2(e).
 *   block_scale = 1: for each 64-key block j of visible keys,
 *       e_j = ceil(max_{c in j} y_c) - T     [P1 para 3: each block of 64
 *       keys scaled by a power of 2; P3 "How ZYFA works" item 3: scaled
 *       before rounding]
 *   block_scale = 0 ("running"): keys are taken in tiles of 128; for tile t,
 *       e_t = ceil(max of y over tiles 0..t) - T, shared by its two blocks.
 *   p~_c = round_e4m3(2^(y_c - e))            (mode 0, exact exp2)
 *        = decode(leanp_code(y_c - e))        (mode 1, Lean P)
 *        = 2^(y_c - e) unrounded              (mode 2, rounding off: a pin)
 *   E = max e;  L = sum_c 2^(e(c) - E) p~_c;  N = sum_c 2^(e(c) - E) p~_c v_c
 *   o = N / L  [P1 para 3: divide by the sum of the rounded probabilities;
 *   P2 "Perche l'FP8 non basta da solo": an extra matrix instruction for
 *   that sum]
 *   lse = ln L + E ln 2   (natural log, in the units of the scores s)
 * Optionally returns p~ (fp64) for single-row debugging via pdump (Sk
 * values for row rows[0] or row 0). */
int zo_attn_fp8_emul(const double* q, const double* k, const double* v, int B, int Sq, int Sk,
                     int Hq, int Hkv, int dqk, int dv, double scale, int causal, int mode,
                     int block_scale, int T, const int64_t* rows, int64_t nrows, double* o,
                     double* lse, double* pdump) {
  if (B <= 0 || Sq <= 0 || Sk <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv) return -1;
  if (mode < 0 || mode > 2) return -1;
  zo_shape s = {B, Sq, Sk, Hq, Hkv, dqk, dv, causal, scale};
  int64_t n = rows ? nrows : (int64_t)B * Hq * Sq;
  const double LOG2E = 1.4426950408889634;
#pragma omp parallel
  {
    double* y = (double*)malloc(sizeof(double) * (size_t)Sk);
    double* pt = (double*)malloc(sizeof(double) * (size_t)Sk);
    int* ec = (int*)malloc(sizeof(int) * (size_t)Sk);
#pragma omp for schedule(dynamic, 16)
    for (int64_t t = 0; t < n; ++t) {
      int b, h, i;
      row_coords(&s, rows ? rows[t] : t, &b, &h, &i);
      int g = h / (Hq / Hkv);
      int L = last_key(&s, i);
      double* orow = o + t * dv;
      for (int e = 0; e < dv; ++e) orow[e] = 0.0;
      if (L < 0) {
        lse[t] = -INFINITY;
        if (pdump && t == 0)
          for (int c = 0; c < Sk; ++c) pdump[c] = 0.0;
        continue;
      }
      const double* qi = qrow(&s, q, b, i, h);
      for (int c = 0; c <= L; ++c) {
        const double* kc = krow(&s, k, b, c, g);
        double dot = 0.0;
        for (int e = 0; e < dqk; ++e) dot += qi[e] * kc[e];
        y[c] = scale * dot * LOG2E;
      }
      /* exponent per key */
      if (block_scale) {
        for (int j0 = 0; j0 <= L; j0 += 64) {
          int j1 = j0 + 63 < L ? j0 + 63 : L;
          double bm = -INFINITY;
          for (int c = j0; c <= j1; ++c)
            if (y[c] > bm) bm = y[c];
          int e = (int)ceil(bm) - T;
          for (int c = j0; c <= j1; ++c) ec[c] = e;
        }
      } else {
        double run = -INFINITY;
        for (int t0 = 0; t0 <= L; t0 += 128) {
          int t1 = t0 + 127 < L ? t0 + 127 : L;
          for (int c = t0; c <= t1; ++c)
            if (y[c] > run) run = y[c];
          int e = (int)ceil(run) - T;
          for (int c = t0; c <= t1; ++c) ec[c] = e;
        }
      }
      int E = ec[0];
      for (int c = 0; c <= L; ++c)
        if (ec[c] > E) E = ec[c];
      double Lsum = 0.0;
      for (int c = 0; c <= L; ++c) {
        double z = y[c] - ec[c];
        double p;
        if (mode == 0)
          p = zo_e4m3_decode(zo_e4m3_encode_rne_sat(exp2(z)));
        else if (mode == 1)
          p = zo_e4m3_decode((uint8_t)zo_leanp_code(z));
        else
          p = exp2(z);
        pt[c] = p;
        double w = ldexp(p, ec[c] - E);
        Lsum += w;
        const double* vc = vrow(&s, v, b, c, g);
        for (int e = 0; e < dv; ++e) orow[e] += w * vc[e];
      }
      for (int e = 0; e < dv; ++e) orow[e] /= Lsum;
      lse[t] = log(Lsum) + E * log(2.0);
      /* lse is in units of the natural-log scores; y = s*log2(e) so
         ln(sum 2^(y - E)) + E ln 2 = ln(sum e^s). */
      if (pdump && t == 0) {
        for (int c = 0; c < Sk; ++c) pdump[c] = c <= L ? pt[c] : 0.0;
      }
    }
    free(y);
    free(pt);
    free(ec);
  }
  return 0;
}

/* Exact dequantisation of e4m3 bytes times a per-tensor descale (fp64). */
void zo_dequant_e4m3(const uint8_t* x, int64_t n, double descale, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = zo_e4m3_decode(x[i]) * descale;
}
