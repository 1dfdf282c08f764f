/*
 * moe_oracle.c -- plain, slow CPU oracle of the quantized routed-expert MoE
 * call.  TEST INFRASTRUCTURE ONLY (see moe_oracle.h): loaded by tests/,
 * __graft_entry__.smoke() and bench.py's CPU legs, never by the product.
 *
 * Build: gcc -O2 -std=c11 -fopenmp -ffp-contract=off -fPIC -shared
 * (-ffp-contract=off keeps every fp32 operation a separate rounding step,
 *  which the routing sigmoid's specification requires).
 *
 * Floating point: the fixed-precision steps (routing, weight and activation
 * quantization, the mid quantization decision) run in fp32 exactly as the
 * method states them; the two contractions and the combine accumulate in
 * fp64.  Each function names the passage or external specification it
 * follows.
 */
#include "moe_oracle.h"

#include <math.h>
#include <omp.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* Codecs.  OCP Microscaling Formats (MX) v1.0 spec, sections 5.1-5.3
 * (E2M1 element, E8M0 scale); OCP 8-bit Floating Point spec (E4M3 with
 * bias 7, max 448, no infinities, 0x7F/0xFF NaN).                      */

double orc_e2m1_value(uint8_t code) {
  int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
  double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
  return s ? -mag : mag;
}

double orc_e4m3_value(uint8_t code) {
  int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
  if (e == 15 && m == 7) return NAN;
  double mag = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
  return s ? -mag : mag;
}

double orc_e8m0_value(uint8_t code) {
  if (code == 0xFF) return NAN;
  return ldexp(1.0, (int)code - 127);
}

/* Round |v| to the nearest multiple of the quantum of its binade, ties to an
 * even multiple (= even mantissa), then saturate.  `emin` is the smallest
 * normal exponent, `mbits` the mantissa width.                            */
static double rne_to_grid(double a, int emin, int mbits, double maxval) {
  if (a == 0.0) return 0.0;
  int ex;
  frexp(a, &ex);               /* a = f * 2^ex, f in [0.5, 1) */
  int E = ex - 1;              /* floor(log2 a)               */
  if (E < emin) E = emin;      /* subnormal range shares emin's quantum */
  double q = ldexp(1.0, E - mbits);
  double r = rint(a / q) * q;  /* a/q is exact (q a power of two) */
  return r > maxval ? maxval : r;
}

uint8_t orc_e2m1_encode(double v) {
  uint8_t sign = signbit(v) ? 8 : 0;
  double r = rne_to_grid(fabs(v), 0, 1, 6.0);
  uint8_t code;
  if (r < 1.0) {
    code = (uint8_t)(r * 2.0);              /* 0 or 0.5 */
  } else {
    int ex;
    double f = frexp(r, &ex);               /* r = 2f * 2^(ex-1) */
    int E = ex - 1, mant = (int)((2.0 * f - 1.0) * 2.0);
    code = (uint8_t)(((E + 1) << 1) | mant);
  }
  return (uint8_t)(code | sign);
}

uint8_t orc_e4m3_encode(double v) {
  uint8_t sign = signbit(v) ? 0x80 : 0;
  double r = rne_to_grid(fabs(v), -6, 3, 448.0);
  uint8_t code;
  if (r < ldexp(1.0, -6)) {
    code = (uint8_t)(r * 512.0);            /* subnormal: m * 2^-9 */
  } else {
    int ex;
    double f = frexp(r, &ex);
    int E = ex - 1, mant = (int)((2.0 * f - 1.0) * 8.0);
    code = (uint8_t)(((E + 7) << 3) | mant);
  }
  return (uint8_t)(code | sign);
}

uint16_t orc_bf16_encode(float v) {
  uint32_t u;
  memcpy(&u, &v, 4);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;                      /* round to nearest, ties even */
  return (uint16_t)(u >> 16);
}

float orc_bf16_value(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* OCP MX v1.0, section 6.3 (conversion to MX): shared exponent
 * floor(log2(amax)) - emax_elem, emax_elem = 2 for E2M1.                 */
uint8_t orc_mx_scale_code(float amax) {
  if (!(amax > 0.0f)) return 0;
  int ex;
  frexp((double)amax, &ex);
  int e = (ex - 1) - 2;
  if (e < -127) e = -127;
  if (e > 127) e = 127;
  return (uint8_t)(e + 127);
}

/* The mid scale of the FP8 mid hand-off is a power of two (the pages fix an
 * fp32 scale per 128-block but not its value; this build takes the smallest
 * power of two that keeps the block inside E4M3's range).                  */
float orc_pow2_scale_e4m3(float amax) {
  if (!(amax > 0.0f)) return 1.0f;
  int ex;
  double f = 2.0 * frexp((double)amax, &ex);  /* amax = f * 2^E, f in [1,2) */
  int E = ex - 1;
  int k = (f <= 1.75) ? E - 8 : E - 7;         /* 448 = 1.75 * 2^8          */
  if (k < -126) k = -126;
  if (k > 127) k = 127;
  return (float)ldexp(1.0, k);
}

void orc_quant_mxfp4(const float* w, int64_t rows, int32_t K,
                     uint8_t* packed, uint8_t* scales) {
  int32_t nb = K / 32;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int32_t b = 0; b < nb; ++b) {
      const float* v = w + r * K + (int64_t)b * 32;
      float amax = 0.0f;
      for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
      uint8_t c = orc_mx_scale_code(amax);
      double X = ldexp(1.0, (int)c - 127);
      scales[r * nb + b] = c;
      uint8_t* out = packed + r * (K / 2) + (int64_t)b * 16;
      for (int i = 0; i < 16; ++i) {
        uint8_t lo = orc_e2m1_encode((double)v[2 * i] / X);
        uint8_t hi = orc_e2m1_encode((double)v[2 * i + 1] / X);
        out[i] = (uint8_t)(lo | (hi << 4));
      }
    }
  }
}

void orc_quant_fp8_block128(const float* w, int32_t rows, int32_t K,
                            uint8_t* q, float* scales) {
  int32_t rb = rows / 128, kb = K / 128;
#pragma omp parallel for schedule(static)
  for (int32_t bi = 0; bi < rb * kb; ++bi) {
    int32_t r0 = (bi / kb) * 128, k0 = (bi % kb) * 128;
    float amax = 0.0f;
    for (int r = 0; r < 128; ++r)
      for (int c = 0; c < 128; ++c)
        amax = fmaxf(amax, fabsf(w[(int64_t)(r0 + r) * K + k0 + c]));
    float s = (amax > 0.0f) ? amax / 448.0f : 1.0f;   /* fp32 division */
    scales[bi] = s;
    for (int r = 0; r < 128; ++r)
      for (int c = 0; c < 128; ++c) {
        int64_t i = (int64_t)(r0 + r) * K + k0 + c;
        float t = w[i] / s;                             /* fp32 division */
        q[i] = orc_e4m3_encode((double)t);
      }
  }
}

void orc_quant_fp8_pow2_row(const float* v, int32_t K, uint8_t* q, float* scales) {
  for (int32_t b = 0; b < K / 128; ++b) {
    float amax = 0.0f;
    for (int i = 0; i < 128; ++i) amax = fmaxf(amax, fabsf(v[b * 128 + i]));
    float s = orc_pow2_scale_e4m3(amax);
    scales[b] = s;
    for (int i = 0; i < 128; ++i)
      q[b * 128 + i] = orc_e4m3_encode((double)v[b * 128 + i] / (double)s);
  }
}

/* ------------------------------------------------------------------ */
/* Routing ("glm53: FP8 mid hand-off", commit "per-row up/gate jobs at 4
 * rows": top-8 rounds, a tied round broken by expert ID).                 */

static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

float orc_exp_spec(float x) {
  /* Cody & Waite (1980) argument reduction, two-part ln 2. */
  const float LOG2E = 0x1.715476p+0f;
  const float C1 = 0x1.63p-1f;           /* 0.693359375, 9 significant bits */
  const float C2 = -0x1.bd0106p-13f;
  const float K2 = 0x1p-1f, K3 = 0x1.555556p-3f, K4 = 0x1.555556p-5f,
              K5 = 0x1.111112p-7f, K6 = 0x1.6c16c2p-10f, K7 = 0x1.a01a02p-13f;
  if (x < -87.0f) x = -87.0f;
  if (x > 88.0f) x = 88.0f;
  float n = rintf(x * LOG2E);
  float r = x - n * C1;
  r = r - n * C2;
  float p = K7;
  p = p * r + K6;
  p = p * r + K5;
  p = p * r + K4;
  p = p * r + K3;
  p = p * r + K2;
  p = p * r + 1.0f;
  p = p * r + 1.0f;
  float two_n = f32_from_bits((uint32_t)((int)n + 127) << 23);
  return p * two_n;
}

float orc_sigmoid_spec(float l) {
  float e = orc_exp_spec(-l);
  float d = 1.0f + e;
  return 1.0f / d;
}

void orc_route(int32_t M, int32_t E, int32_t k, const float* logits,
               const float* bias, float routed_scale,
               int32_t* topk_ids, float* topk_w) {
#pragma omp parallel
  {
    float* s = (float*)malloc(sizeof(float) * E);
    float* sel = (float*)malloc(sizeof(float) * E);
    unsigned char* taken = (unsigned char*)malloc(E);
#pragma omp for schedule(static)
    for (int32_t t = 0; t < M; ++t) {
      for (int32_t e = 0; e < E; ++e) {
        s[e] = orc_sigmoid_spec(logits[(int64_t)t * E + e]);
        sel[e] = bias ? s[e] + bias[e] : s[e];
        taken[e] = 0;
      }
      for (int32_t j = 0; j < k; ++j) {
        int32_t best = -1;
        for (int32_t e = 0; e < E; ++e)       /* ascending IDs: strict > keeps */
          if (!taken[e] && (best < 0 || sel[e] > sel[best])) best = e;  /* the lower ID on ties */
        taken[best] = 1;
        topk_ids[(int64_t)t * k + j] = best;
      }
      float denom = 0.0f;
      for (int32_t j = 0; j < k; ++j) denom += s[topk_ids[(int64_t)t * k + j]];
      for (int32_t j = 0; j < k; ++j) {
        float q = s[topk_ids[(int64_t)t * k + j]] / denom;
        topk_w[(int64_t)t * k + j] = q * routed_scale;
      }
    }
    free(s); free(sel); free(taken);
  }
}

void orc_align(int32_t M, int32_t k, int32_t E, const int32_t* topk_ids,
               int32_t* counts, int32_t* offsets, int32_t* sorted_pairs,
               int32_t* inv) {
  int64_t P = (int64_t)M * k;
  int32_t* cursor = (int32_t*)malloc(sizeof(int32_t) * (E + 1));
  for (int32_t e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t p = 0; p < P; ++p) counts[topk_ids[p]]++;
  offsets[0] = 0;
  for (int32_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  for (int32_t e = 0; e < E; ++e) cursor[e] = offsets[e];
  for (int64_t p = 0; p < P; ++p) {
    int32_t pos = cursor[topk_ids[p]]++;
    sorted_pairs[pos] = (int32_t)p;
    inv[p] = pos;
  }
  free(cursor);
}

void orc_quant_act_row(int32_t wfmt, const uint16_t* x_row, int32_t H,
                       uint8_t* q, void* s) {
  float* xf = (float*)malloc(sizeof(float) * H);
  for (int32_t h = 0; h < H; ++h) xf[h] = orc_bf16_value(x_row[h]);
  if (wfmt == ORC_W_MXFP4)
    orc_quant_mxfp4(xf, 1, H, q, (uint8_t*)s);
  else
    orc_quant_fp8_pow2_row(xf, H, q, (float*)s);
  free(xf);
}

/* ------------------------------------------------------------------ */
/* Forward.  Weight dequantization is decode(code) * scale, exact in fp64. */

static double deq_w13(const orc_shape_t* sh, const uint8_t* w, const void* s,
                      int32_t e, int32_t n, int32_t h) {
  int64_t H = sh->H, N2 = 2 * (int64_t)sh->I;
  if (sh->wfmt == ORC_W_MXFP4) {
    uint8_t byte = w[((int64_t)e * N2 + n) * (H / 2) + h / 2];
    uint8_t code = (h & 1) ? (byte >> 4) : (byte & 15);
    uint8_t sc = ((const uint8_t*)s)[((int64_t)e * N2 + n) * (H / 32) + h / 32];
    return orc_e2m1_value(code) * orc_e8m0_value(sc);
  } else {
    uint8_t code = w[((int64_t)e * N2 + n) * H + h];
    float sc = ((const float*)s)[((int64_t)e * (N2 / 128) + n / 128) * (H / 128) + h / 128];
    return orc_e4m3_value(code) * (double)sc;
  }
}

static double deq_w2(const orc_shape_t* sh, const uint8_t* w, const void* s,
                     int32_t e, int32_t h, int32_t i) {
  int64_t H = sh->H, I = sh->I;
  if (sh->wfmt == ORC_W_MXFP4) {
    uint8_t byte = w[((int64_t)e * H + h) * (I / 2) + i / 2];
    uint8_t code = (i & 1) ? (byte >> 4) : (byte & 15);
    uint8_t sc = ((const uint8_t*)s)[((int64_t)e * H + h) * (I / 32) + i / 32];
    return orc_e2m1_value(code) * orc_e8m0_value(sc);
  } else {
    uint8_t code = w[((int64_t)e * H + h) * I + i];
    float sc = ((const float*)s)[((int64_t)e * (H / 128) + h / 128) * (I / 128) + i / 128];
    return orc_e4m3_value(code) * (double)sc;
  }
}

int orc_forward_tokens(const orc_shape_t* sh, const uint16_t* x,
                       const int32_t* topk_ids, const float* topk_w,
                       const uint8_t* w13, const void* s13,
                       const uint8_t* w2, const void* s2,
                       int32_t ntok, const int32_t* toks,
                       uint8_t* midq, float* midqs, double* ref,
                       uint16_t* out) {
  const int32_t M = sh->M, H = sh->H, I = sh->I, E = sh->E, k = sh->topk;
  if (M < 1 || H < 128 || I < 128 || H % 128 || I % 128 || k < 1 || k > E) return -1;
  if (sh->wfmt != ORC_W_MXFP4 && sh->wfmt != ORC_W_FP8_BLOCK128) return -1;
  if (!toks) ntok = M;

  double* xd = (double*)malloc(sizeof(double) * H);
  uint8_t* xq = (uint8_t*)malloc(H);
  float* xs = (float*)malloc(sizeof(float) * (H / 32 + 1));
  double* g = (double*)malloc(sizeof(double) * 2 * I);
  float* mid = (float*)malloc(sizeof(float) * I);
  double* mdq = (double*)malloc(sizeof(double) * I);
  double* y = (double*)malloc(sizeof(double) * H);
  double* acc = (double*)malloc(sizeof(double) * H);

  for (int32_t n = 0; n < ntok; ++n) {
    int32_t t = toks ? toks[n] : n;
    if (t < 0 || t >= M) return -1;
    /* activation quantization of x[t] and its dequantized values */
    const uint16_t* xr = x + (int64_t)t * H;
    if (sh->wfmt == ORC_W_MXFP4) {
      uint8_t* xsc = (uint8_t*)xs;
      orc_quant_act_row(sh->wfmt, xr, H, xq, xsc);
      for (int32_t h = 0; h < H; ++h) {
        uint8_t code = (h & 1) ? (xq[h / 2] >> 4) : (xq[h / 2] & 15);
        xd[h] = orc_e2m1_value(code) * orc_e8m0_value(xsc[h / 32]);
      }
    } else {
      orc_quant_act_row(sh->wfmt, xr, H, xq, xs);
      for (int32_t h = 0; h < H; ++h) xd[h] = orc_e4m3_value(xq[h]) * (double)xs[h / 128];
    }
    for (int32_t h = 0; h < H; ++h) acc[h] = 0.0;

    for (int32_t j = 0; j < k; ++j) {
      int32_t e = topk_ids[(int64_t)t * k + j];
      if (e < 0 || e >= E) return -1;
      /* GEMM1: rows [0, I) gate, [I, 2I) up */
#pragma omp parallel for schedule(static)
      for (int32_t r = 0; r < 2 * I; ++r) {
        double a = 0.0;
        for (int32_t h = 0; h < H; ++h) a += xd[h] * deq_w13(sh, w13, s13, e, r, h);
        g[r] = a;
      }
      /* SwiGLU on the fp32 accumulator values */
      for (int32_t i = 0; i < I; ++i) {
        float gate = (float)g[i], up = (float)g[I + i];
        double gd = (double)gate;
        mid[i] = (float)(gd / (1.0 + exp(-gd)) * (double)up);
      }
      /* mid quantized once per (pair, 128-block) */
      int64_t prow = (int64_t)n * k + j;
      for (int32_t b = 0; b < I / 128; ++b) {
        float amax = 0.0f;
        for (int32_t i = 0; i < 128; ++i) amax = fmaxf(amax, fabsf(mid[b * 128 + i]));
        float s = orc_pow2_scale_e4m3(amax);
        if (midqs) midqs[prow * (I / 128) + b] = s;
        for (int32_t i = 0; i < 128; ++i) {
          uint8_t c = orc_e4m3_encode((double)mid[b * 128 + i] / (double)s);
          if (midq) midq[prow * I + b * 128 + i] = c;
          mdq[b * 128 + i] = orc_e4m3_value(c) * (double)s;
        }
      }
      /* GEMM2 */
#pragma omp parallel for schedule(static)
      for (int32_t h = 0; h < H; ++h) {
        double a = 0.0;
        for (int32_t i = 0; i < I; ++i) a += mdq[i] * deq_w2(sh, w2, s2, e, h, i);
        y[h] = a;
      }
      double wj = (double)topk_w[(int64_t)t * k + j];
      for (int32_t h = 0; h < H; ++h) acc[h] += wj * y[h];
    }
    for (int32_t h = 0; h < H; ++h) {
      if (ref) ref[(int64_t)n * H + h] = acc[h];
      if (out) out[(int64_t)n * H + h] = orc_bf16_encode((float)acc[h]);
    }
  }
  free(xd); free(xq); free(xs); free(g); free(mid); free(mdq); free(y); free(acc);
  return 0;
}

/* Thread count of the OpenMP loops above (timing only: the results do not
 * depend on it).  Returns the previous count; n <= 0 leaves it unchanged.  */
int orc_set_threads(int n) {
  int prev = omp_get_max_threads();
  if (n > 0) omp_set_num_threads(n);
  return prev;
}
