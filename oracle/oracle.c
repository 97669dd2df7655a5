/*
 * oracle.c -- plain, slow CPU oracle for SageSLA attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check and the benchmark's
 * CPU-baseline leg may load this file's library.  The CUDA library shares no
 * code, header, table or constant with it.
 *
 * What it follows (page title, section):
 *   - "揭秘TurboDiffusion：如何让视频生成实现百倍加速？", 支柱一 SageAttention:
 *     attention is quantised to INT8 and a smoothing step handles outliers.
 *   - same page, 支柱二 SLA: only the most important block interactions are
 *     computed exactly; a light linear-attention component covers the rest;
 *     the two stack as "SageSLA".
 *   - "TurboDiffusion跨模态：图文音视频多模态融合探索", 2.2 SLA: linear part is a
 *     kernel-function approximation (phi); sla_topk 0.05/0.1/0.15.
 *   - 量子位 news (aiho.net), 技术解密 1: "异常值平滑" (outlier smoothing).
 * Everything the pages leave open (block size 64, the INT8/FP8 formats and
 * scale granularity, mean-pooled block scores, ties to the lower index,
 * phi = elu+1, the d x d projection) is taken in its plainest reading; the
 * readings are listed in the design notes of the repository.
 *
 * Floating point: fp64 everywhere, except where a float decides an integer
 * that the GPU must reproduce bit for bit (INT8/FP8 codes, the block mask);
 * those decisions are taken in fp32, the precision of the kernels.
 *
 * Parity pins (tests/test_oracle_*.py): dense vs brute force and vs torch
 * SDPA; smoothing invariance; emulation == dense with quantisation off;
 * closed forms for the quantised path (uniform scores, constant V, a
 * two-key worked example); e4m3 encoder exhaustive vs torch's cast; int8
 * quantiser closed forms; mask vs brute-force sort and constructed ties;
 * linear branch vs per-token sum and closed forms; W8A8 linear vs integer
 * matmul at unit scales and vs the matmul of the dequantised operands;
 * QK RMSNorm vs its fp64 definition, power-of-two closed forms, and the
 * coupling of the heads of a token.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_QBLK 64 /* quantisation block of Q and K: 64 tokens */

int orc_version(void) { return 3; }

int orc_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

static float bf16_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* ------------------------------------------------------------------------ */
/* FP8 E4M3 (OCP 8-bit floating point spec, "E4M3FN"): 1 sign, 4 exponent   */
/* bits with bias 7, 3 mantissa bits, no infinities, S.1111.111 = NaN,      */
/* largest finite 448 = 1.75 * 2^8, smallest normal 2^-6, subnormals        */
/* m * 2^-9.  Encoding: round to nearest, ties to even, saturate to +-448.  */
/* ------------------------------------------------------------------------ */
uint8_t orc_e4m3_encode(float x) {
  if (isnan(x)) return 0x7F;
  uint8_t sign = signbit(x) ? 0x80 : 0x00;
  double a = fabs((double)x);
  if (a >= 448.0) return sign | 0x7E;
  double quantum;
  if (a < ldexp(1.0, -6)) {
    quantum = ldexp(1.0, -9);
  } else {
    quantum = ldexp(1.0, ilogb(a) - 3);
  }
  double r = nearbyint(a / quantum) * quantum; /* exact scaling; RNE */
  if (r > 448.0) r = 448.0;
  if (r == 0.0) return sign;
  if (r < ldexp(1.0, -6)) {
    int m = (int)(r / ldexp(1.0, -9));
    return sign | (uint8_t)m;
  }
  int e = ilogb(r);
  int m = (int)(r / ldexp(1.0, e - 3)) - 8;
  return sign | (uint8_t)(((e + 7) << 3) | m);
}

double orc_e4m3_decode(uint8_t c) {
  int s = c >> 7, e = (c >> 3) & 0xF, m = c & 7;
  double v;
  if (e == 0xF && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m, -9);
  else
    v = ldexp(1.0 + m / 8.0, e - 7);
  return s ? -v : v;
}

void orc_e4m3_encode_array(const float* x, uint8_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(x[i]);
}
void orc_e4m3_decode_array(const uint8_t* c, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_decode(c[i]);
}

/* Symmetric INT8 code: x * (127/amax) in fp32, rounded half to even,
 * clamped to [-127, 127].  mult = fl32(127/amax) is computed by the caller. */
int8_t orc_int8_code(float x, float mult) {
  float p = x * mult;
  float r = nearbyintf(p);
  if (r > 127.f) r = 127.f;
  if (r < -127.f) r = -127.f;
  return (int8_t)r;
}
/* Same with a symmetric range of +-qmax (127: INT8; 7: the INT4 variant). */
static int8_t orc_qcode(float x, float mult, int qmax) {
  float p = x * mult;
  float r = nearbyintf(p);
  if (r > (float)qmax) r = (float)qmax;
  if (r < -(float)qmax) r = -(float)qmax;
  return (int8_t)r;
}
void orc_int8_code_array(const float* x, float mult, int8_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_int8_code(x[i], mult);
}

/* phi(x) = elu(x) + 1: x + 1 for x > 0, exp(x) otherwise (always > 0). */
static double phi(double x) { return x > 0.0 ? x + 1.0 : exp(x); }
double orc_phi(double x) { return phi(x); }

/* k = clamp(ceil(topk * Nb), 1, Nb): at least the fraction topk of the key
 * blocks is computed exactly.  topk arrives as fp32, so the product is shrunk
 * by one part in 10^6 before the ceiling: 0.3f * 10 -> 3, not 4. */
int orc_topk_count(int nb, float topk) {
  double t = (double)topk * (double)nb;
  t -= t * 1e-6;
  int k = (int)ceil(t);
  if (k < 1) k = 1;
  if (k > nb) k = nb;
  return k;
}

/* ------------------------------------------------------------------------ */
/* Dense softmax attention in fp64: out = softmax(q k^T / sqrt(d)) v, per   */
/* (b,h), over the N tokens.  Inputs are fp64 [BH][N][d].                   */
/* ------------------------------------------------------------------------ */
void orc_dense_attn(const double* q, const double* k, const double* v, int BH, int N, int d,
                    double* out) {
  const double sc = 1.0 / sqrt((double)d);
#pragma omp parallel for collapse(2) schedule(dynamic, 16)
  for (int bh = 0; bh < BH; ++bh) {
    for (int r = 0; r < N; ++r) {
      const double* qr = q + ((int64_t)bh * N + r) * d;
      const double* kb = k + (int64_t)bh * N * d;
      const double* vb = v + (int64_t)bh * N * d;
      double* s = (double*)malloc(sizeof(double) * N);
      double m = -INFINITY;
      for (int n = 0; n < N; ++n) {
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += qr[c] * kb[(int64_t)n * d + c];
        s[n] = acc * sc;
        if (s[n] > m) m = s[n];
      }
      double l = 0.0;
      for (int n = 0; n < N; ++n) {
        s[n] = exp(s[n] - m);
        l += s[n];
      }
      double* o = out + ((int64_t)bh * N + r) * d;
      for (int c = 0; c < d; ++c) o[c] = 0.0;
      for (int n = 0; n < N; ++n)
        for (int c = 0; c < d; ++c) o[c] += s[n] * vb[(int64_t)n * d + c];
      for (int c = 0; c < d; ++c) o[c] /= l;
      free(s);
    }
  }
}

/* Same, from bf16 bit patterns (exact in fp64). */
void orc_dense_attn_bf16(const uint16_t* q, const uint16_t* k, const uint16_t* v, int BH, int N,
                         int d, double* out) {
  int64_t E = (int64_t)BH * N * d;
  double* qd = (double*)malloc(sizeof(double) * E);
  double* kd = (double*)malloc(sizeof(double) * E);
  double* vd = (double*)malloc(sizeof(double) * E);
  for (int64_t i = 0; i < E; ++i) {
    qd[i] = bf16_f32(q[i]);
    kd[i] = bf16_f32(k[i]);
    vd[i] = bf16_f32(v[i]);
  }
  orc_dense_attn(qd, kd, vd, BH, N, d, out);
  free(qd);
  free(kd);
  free(vd);
}

/* ------------------------------------------------------------------------ */
/* Step 1+2+3: smoothing and quantisation of one (b,h).                     */
/*  mu[c]   = fl32( (sum_n K[n,c] in fp64) / N )                              */
/*  ks      = fl32(K - mu)                                                  */
/*  per 64-token block t: amax = max |x| over its valid tokens and d;        */
/*     s = fl32(amax/127), mult = fl32(127/amax), code = int8(x*mult);       */
/*     amax == 0 -> s = 1, codes 0.                                         */
/*  V per channel: amax_c over the N tokens; s_v = fl32(amax/448),          */
/*     mult_v = fl32(448/amax), code = e4m3(fl32(v*mult_v)); 0 -> s_v = 1.   */
/* Codes are [N][d]; scales are per 64-token block (ceil(N/64)).            */
/* ------------------------------------------------------------------------ */
/* mu[c] = fl32((sum over the N tokens of K[n,c], in fp64) / N). */
static void smooth_mean(const uint16_t* k, int N, int d, float* mu) {
  for (int c = 0; c < d; ++c) {
    double acc = 0.0;
    for (int n = 0; n < N; ++n) acc += (double)bf16_f32(k[(int64_t)n * d + c]);
    mu[c] = (float)(acc / (double)N);
  }
}

/* qmax = 127 (INT8) or 7 (the INT4 variant); q_per_token != 0: one Q scale
 * per token (sq has N entries) instead of one per 64-token block. */
static void quant_head(const uint16_t* q, const uint16_t* k, const uint16_t* v, int N, int d,
                       float* mu, float* ks_out /* [N][d] or NULL */, int8_t* q8, int8_t* k8,
                       uint8_t* v8, float* sq, float* sk, float* sv, int qmax, int q_per_token) {
  const float fq = (float)qmax;
  smooth_mean(k, N, d, mu);
  float* ks = ks_out ? ks_out : (float*)malloc(sizeof(float) * (int64_t)N * d);
  for (int n = 0; n < N; ++n)
    for (int c = 0; c < d; ++c) ks[(int64_t)n * d + c] = bf16_f32(k[(int64_t)n * d + c]) - mu[c];

  int nq = (N + ORC_QBLK - 1) / ORC_QBLK;
  for (int t = 0; t < nq; ++t) {
    int n0 = t * ORC_QBLK, n1 = n0 + ORC_QBLK < N ? n0 + ORC_QBLK : N;
    float aq = 0.f, ak = 0.f;
    for (int n = n0; n < n1; ++n)
      for (int c = 0; c < d; ++c) {
        float xq = fabsf(bf16_f32(q[(int64_t)n * d + c]));
        float xk = fabsf(ks[(int64_t)n * d + c]);
        if (xq > aq) aq = xq;
        if (xk > ak) ak = xk;
      }
    float mq = aq > 0.f ? fq / aq : 0.f;
    float mk = ak > 0.f ? fq / ak : 0.f;
    if (!q_per_token) sq[t] = aq > 0.f ? aq / fq : 1.f;
    sk[t] = ak > 0.f ? ak / fq : 1.f;
    for (int n = n0; n < n1; ++n) {
      float mqn = mq;
      if (q_per_token) { /* the row's own absmax over its d channels */
        float an = 0.f;
        for (int c = 0; c < d; ++c) {
          float x = fabsf(bf16_f32(q[(int64_t)n * d + c]));
          if (x > an) an = x;
        }
        mqn = an > 0.f ? fq / an : 0.f;
        sq[n] = an > 0.f ? an / fq : 1.f;
      }
      for (int c = 0; c < d; ++c) {
        q8[(int64_t)n * d + c] = orc_qcode(bf16_f32(q[(int64_t)n * d + c]), mqn, qmax);
        k8[(int64_t)n * d + c] = orc_qcode(ks[(int64_t)n * d + c], mk, qmax);
      }
    }
  }
  for (int c = 0; c < d; ++c) {
    float a = 0.f;
    for (int n = 0; n < N; ++n) {
      float x = fabsf(bf16_f32(v[(int64_t)n * d + c]));
      if (x > a) a = x;
    }
    float mv = a > 0.f ? 448.f / a : 0.f;
    sv[c] = a > 0.f ? a / 448.f : 1.f;
    for (int n = 0; n < N; ++n) {
      float x = bf16_f32(v[(int64_t)n * d + c]) * mv;
      v8[(int64_t)n * d + c] = orc_e4m3_encode(x);
    }
  }
  if (!ks_out) free(ks);
}

void orc_quant(const uint16_t* q, const uint16_t* k, const uint16_t* v, int BH, int N, int d,
               float* mu, int8_t* q8, int8_t* k8, uint8_t* v8, float* sq, float* sk, float* sv) {
  int nq = (N + ORC_QBLK - 1) / ORC_QBLK;
#pragma omp parallel for schedule(dynamic, 1)
  for (int bh = 0; bh < BH; ++bh) {
    int64_t o = (int64_t)bh * N * d;
    quant_head(q + o, k + o, v + o, N, d, mu + (int64_t)bh * d, NULL, q8 + o, k8 + o, v8 + o,
               sq + (int64_t)bh * nq, sk + (int64_t)bh * nq, sv + (int64_t)bh * d, 127, 0);
  }
}

/* ------------------------------------------------------------------------ */
/* Step 4+5: mean pooling and the block mask (fp32, the kernels' precision, */
/* because the mask is an integer decision the GPU reproduces).             */
/*  qbar_i = mean of Q over the valid rows of block i (fp32, sequential);   */
/*  kbar_j = mean of ks over the valid rows of block j;                     */
/*  sbar_ij = fl32(dot(qbar_i, kbar_j)) * fl32(1/sqrt(d)), dot sequential.  */
/*  S_i = the k largest sbar_i., ties to the lower j, sorted ascending.     */
/* ------------------------------------------------------------------------ */
static void pool_head(const uint16_t* q, const float* ks, int N, int d, int block, float* qbar,
                      float* kbar) {
  int nb = (N + block - 1) / block;
  for (int i = 0; i < nb; ++i) {
    int n0 = i * block, n1 = n0 + block < N ? n0 + block : N;
    float cnt = (float)(n1 - n0);
    for (int c = 0; c < d; ++c) {
      float aq = 0.f, ak = 0.f;
      for (int n = n0; n < n1; ++n) {
        aq += bf16_f32(q[(int64_t)n * d + c]);
        ak += ks[(int64_t)n * d + c];
      }
      qbar[(int64_t)i * d + c] = aq / cnt;
      kbar[(int64_t)i * d + c] = ak / cnt;
    }
  }
}

typedef struct {
  float s;
  int j;
} orc_sj;

static int cmp_desc_lowj(const void* a, const void* b) {
  const orc_sj* x = (const orc_sj*)a;
  const orc_sj* y = (const orc_sj*)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  return x->j - y->j;
}
static int cmp_int(const void* a, const void* b) { return *(const int*)a - *(const int*)b; }

static void mask_rows(const float* qbar, const float* kbar, int nb, int d, int kc, int32_t* idx,
                      float* scores /* [nb][nb] or NULL */) {
  const float rs = 1.0f / sqrtf((float)d);
  orc_sj* row = (orc_sj*)malloc(sizeof(orc_sj) * nb);
  for (int i = 0; i < nb; ++i) {
    for (int j = 0; j < nb; ++j) {
      float acc = 0.f;
      for (int c = 0; c < d; ++c) acc += qbar[(int64_t)i * d + c] * kbar[(int64_t)j * d + c];
      row[j].s = acc * rs;
      row[j].j = j;
      if (scores) scores[(int64_t)i * nb + j] = row[j].s;
    }
    qsort(row, nb, sizeof(orc_sj), cmp_desc_lowj);
    int32_t* out = idx + (int64_t)i * kc;
    for (int t = 0; t < kc; ++t) out[t] = row[t].j;
    qsort(out, kc, sizeof(int32_t), cmp_int);
  }
  free(row);
}

/* Pooled means and mask for all heads.  qbar/kbar [BH][Nb][d], idx
 * [BH][Nb][k], scores [BH][Nb][Nb] (optional). */
void orc_mask(const uint16_t* q, const uint16_t* k, int BH, int N, int d, int block, float topk,
              float* qbar, float* kbar, int32_t* idx, float* scores) {
  int nb = (N + block - 1) / block;
  int kc = orc_topk_count(nb, topk);
#pragma omp parallel for schedule(dynamic, 1)
  for (int bh = 0; bh < BH; ++bh) {
    int64_t o = (int64_t)bh * N * d;
    float* mu = (float*)malloc(sizeof(float) * d);
    float* ks = (float*)malloc(sizeof(float) * (int64_t)N * d);
    smooth_mean(k + o, N, d, mu);
    for (int n = 0; n < N; ++n)
      for (int c = 0; c < d; ++c)
        ks[(int64_t)n * d + c] = bf16_f32(k[o + (int64_t)n * d + c]) - mu[c];
    float* qb = qbar + (int64_t)bh * nb * d;
    float* kb = kbar + (int64_t)bh * nb * d;
    pool_head(q + o, ks, N, d, block, qb, kb);
    mask_rows(qb, kb, nb, d, kc, idx + (int64_t)bh * nb * kc,
              scores ? scores + (int64_t)bh * nb * nb : NULL);
    free(ks);
    free(mu);
  }
}

/* Pooled block scores in fp64 (same definition, fp64 arithmetic from the
 * fp64 smoothed keys) for the near-tie analysis. */
void orc_block_scores_f64(const uint16_t* q, const uint16_t* k, int BH, int N, int d, int block,
                          double* scores) {
  int nb = (N + block - 1) / block;
#pragma omp parallel for schedule(dynamic, 1)
  for (int bh = 0; bh < BH; ++bh) {
    int64_t o = (int64_t)bh * N * d;
    double* mu = (double*)malloc(sizeof(double) * d);
    double* qb = (double*)malloc(sizeof(double) * (int64_t)nb * d);
    double* kb = (double*)malloc(sizeof(double) * (int64_t)nb * d);
    for (int c = 0; c < d; ++c) {
      double acc = 0.0;
      for (int n = 0; n < N; ++n) acc += (double)bf16_f32(k[o + (int64_t)n * d + c]);
      mu[c] = acc / (double)N;
    }
    for (int i = 0; i < nb; ++i) {
      int n0 = i * block, n1 = n0 + block < N ? n0 + block : N;
      for (int c = 0; c < d; ++c) {
        double aq = 0.0, ak = 0.0;
        for (int n = n0; n < n1; ++n) {
          aq += bf16_f32(q[o + (int64_t)n * d + c]);
          ak += bf16_f32(k[o + (int64_t)n * d + c]) - mu[c];
        }
        qb[(int64_t)i * d + c] = aq / (n1 - n0);
        kb[(int64_t)i * d + c] = ak / (n1 - n0);
      }
    }
    for (int i = 0; i < nb; ++i)
      for (int j = 0; j < nb; ++j) {
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += qb[(int64_t)i * d + c] * kb[(int64_t)j * d + c];
        scores[((int64_t)bh * nb + i) * nb + j] = acc / sqrt((double)d);
      }
    free(mu);
    free(qb);
    free(kb);
  }
}

/* ------------------------------------------------------------------------ */
/* Steps 6-8: the sparse softmax branch, the linear branch, the projection. */
/* ------------------------------------------------------------------------ */
#define ORC_NOQUANT 1 /* test switch: no quantisation anywhere (reduction to dense) */
/* Alternative readings, kept only so that a test can measure how far the
 * result moves between readings the pages leave open; the method's reading
 * is flags = 0. */
#define ORC_ALT_WALK128 2 /* update the running max once per 128 keys of the list */
#define ORC_ALT_LSUM_P 4  /* row sum over the unquantised P instead of P~        */
/* SageAttention2++ variants (量子位 news, 技术解密 1: codes of 8 and, further,
 * 4 bits, and a quantisation calibrated per thread): one Q scale per token (the unit
 * a softmax thread owns) instead of per 64-token block, and Q/K codes in
 * +-7 (4-bit) instead of +-127. */
#define ORC_Q_PER_TOKEN 8
#define ORC_QK_INT4 16

typedef struct {
  int N, d, block, nb, kc;
  const uint16_t *q, *k, *v, *w;
  const int8_t *q8, *k8;
  const uint8_t* v8;
  const float *sq, *sk, *sv, *mu;
  const double *h, *z; /* per key block: h_j [d][d], z_j [d] (linear) */
  int flags;
} orc_head;

/* One query block i: rows n in [i*block, min((i+1)*block, N)). */
static void emul_qblock(const orc_head* H, int i, const int32_t* sel, double* out) {
  const int N = H->N, d = H->d, block = H->block, kc = H->kc;
  const double rsd = 1.0 / sqrt((double)d);
  int n0 = i * block, n1 = n0 + block < N ? n0 + block : N;
  double* o = (double*)malloc(sizeof(double) * d);
  /* The walk visits the selected key blocks of the list in ascending order,
   * one block at a time: the running max is updated once per block and that
   * block's P is quantised against it (ORC_ALT_WALK128: 128 keys at a time). */
  const int per_tile = (H->flags & ORC_ALT_WALK128) && 128 / block > 1 ? 128 / block : 1;
  double* sc = (double*)malloc(sizeof(double) * (size_t)per_tile * block);
  double* Hc = NULL;
  double* Zc = NULL;
  uint8_t* in_s = (uint8_t*)calloc(H->nb, 1);
  for (int t = 0; t < kc; ++t) in_s[sel[t]] = 1;
  if (H->w) {
    /* H_i = sum over key blocks NOT selected of h_j; Z_i likewise. */
    Hc = (double*)calloc((size_t)d * d, sizeof(double));
    Zc = (double*)calloc((size_t)d, sizeof(double));
    for (int j = 0; j < H->nb; ++j) {
      if (in_s[j]) continue;
      const double* hj = H->h + (int64_t)j * d * d;
      const double* zj = H->z + (int64_t)j * d;
      for (int e = 0; e < d * d; ++e) Hc[e] += hj[e];
      for (int c = 0; c < d; ++c) Zc[c] += zj[c];
    }
  }
  for (int n = n0; n < n1; ++n) {
    /* --- sparse softmax branch: online over the selected blocks, ascending --- */
    double m = -INFINITY, l = 0.0;
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    for (int t0 = 0; t0 < kc; t0 += per_tile) {
      const int t1 = t0 + per_tile < kc ? t0 + per_tile : kc;
      /* scores of the walk unit (one key block; keys past N are not scored) */
      double mj = -INFINITY;
      for (int t = t0; t < t1; ++t) {
        const int j = sel[t];
        const int k0 = j * block, k1 = k0 + block < N ? k0 + block : N;
        for (int kk = k0; kk < k1; ++kk) {
          double s;
          if (H->flags & ORC_NOQUANT) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c)
              acc += (double)bf16_f32(H->q[(int64_t)n * d + c]) *
                     ((double)bf16_f32(H->k[(int64_t)kk * d + c]) - (double)H->mu[c]);
            s = acc * rsd;
          } else {
            int64_t acc = 0;
            for (int c = 0; c < d; ++c)
              acc += (int64_t)H->q8[(int64_t)n * d + c] * (int64_t)H->k8[(int64_t)kk * d + c];
            s = (double)acc * (double)H->sq[(H->flags & ORC_Q_PER_TOKEN) ? n : n / ORC_QBLK] *
                (double)H->sk[kk / ORC_QBLK] * rsd;
          }
          sc[(t - t0) * block + (kk - k0)] = s;
          if (s > mj) mj = s;
        }
      }
      /* new running max; O and l move to it (alpha = 0 on the first unit) */
      const double mnew = mj > m ? mj : m;
      const double alpha = exp(m - mnew);
      l *= alpha;
      for (int c = 0; c < d; ++c) o[c] *= alpha;
      for (int t = t0; t < t1; ++t) {
        const int j = sel[t];
        const int k0 = j * block, k1 = k0 + block < N ? k0 + block : N;
        for (int kk = k0; kk < k1; ++kk) {
          const double p = exp(sc[(t - t0) * block + (kk - k0)] - mnew);
          if (H->flags & ORC_NOQUANT) {
            l += p;
            for (int c = 0; c < d; ++c) o[c] += p * (double)bf16_f32(H->v[(int64_t)kk * d + c]);
          } else {
            /* P~ = e4m3(P*448): the FP8 probabilities; the row sum l is taken
             * over the same quantised values that weight V, so a constant V
             * passes through unchanged. */
            const double pq = orc_e4m3_decode(orc_e4m3_encode((float)(p * 448.0)));
            l += (H->flags & ORC_ALT_LSUM_P) ? p * 448.0 : pq;
            for (int c = 0; c < d; ++c) o[c] += pq * orc_e4m3_decode(H->v8[(int64_t)kk * d + c]);
          }
        }
      }
      m = mnew;
    }
    double* orow = out + (int64_t)n * d;
    for (int c = 0; c < d; ++c) {
      double sv = (H->flags & ORC_NOQUANT) ? 1.0 : (double)H->sv[c];
      orow[c] = o[c] * sv / l;
    }
    /* --- linear branch: phi(q) H_i / phi(q) Z_i, then y = O_l W^T --- */
    if (H->w) {
      double* fq = (double*)malloc(sizeof(double) * d);
      for (int c = 0; c < d; ++c) fq[c] = phi((double)bf16_f32(H->q[(int64_t)n * d + c]));
      double den = 0.0;
      for (int c = 0; c < d; ++c) den += fq[c] * Zc[c];
      double* ol = (double*)calloc((size_t)d, sizeof(double));
      if (den > 0.0) {
        for (int ck = 0; ck < d; ++ck)
          for (int cv = 0; cv < d; ++cv) ol[cv] += fq[ck] * Hc[(int64_t)ck * d + cv];
        for (int cv = 0; cv < d; ++cv) ol[cv] /= den;
      }
      for (int co = 0; co < d; ++co) {
        double y = 0.0;
        for (int cv = 0; cv < d; ++cv) y += ol[cv] * (double)bf16_f32(H->w[(int64_t)co * d + cv]);
        orow[co] += y;
      }
      free(ol);
      free(fq);
    }
  }
  free(in_s);
  free(o);
  free(sc);
  free(Hc);
  free(Zc);
}

/* Per key block j: h_j[ck][cv] = sum_{n in j, n < N} phi(k_n[ck]) v_n[cv],
 * z_j[ck] = sum phi(k_n[ck]); from the original (unsmoothed) bf16 K, V. */
static void linear_blocks(const uint16_t* k, const uint16_t* v, int N, int d, int block, double* h,
                          double* z) {
  int nb = (N + block - 1) / block;
  for (int j = 0; j < nb; ++j) {
    double* hj = h + (int64_t)j * d * d;
    double* zj = z + (int64_t)j * d;
    memset(hj, 0, sizeof(double) * d * d);
    memset(zj, 0, sizeof(double) * d);
    int k0 = j * block, k1 = k0 + block < N ? k0 + block : N;
    for (int n = k0; n < k1; ++n)
      for (int ck = 0; ck < d; ++ck) {
        double f = phi((double)bf16_f32(k[(int64_t)n * d + ck]));
        zj[ck] += f;
        for (int cv = 0; cv < d; ++cv) hj[(int64_t)ck * d + cv] += f * (double)bf16_f32(v[(int64_t)n * d + cv]);
      }
  }
}

/*
 * The whole SageSLA path for all heads.
 *   q,k,v   bf16 bits [BH][N][d]; w bf16 bits [d][d] row-major (y = x W^T),
 *           NULL = linear branch off.
 *   idx_override  [BH][Nb][k] sorted block lists to use instead of the
 *           oracle's own mask (NULL = own mask).
 *   qsel    [BH][Nb] flags: compute only the query blocks flagged (NULL = all).
 *   out     fp64 [BH][N][d]; rows of unflagged blocks are left untouched.
 *   idx_out [BH][Nb][k] the mask used (NULL = not returned).
 * Returns k, or -1 on bad arguments.
 */
int orc_sagesla(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* w, int BH,
                int N, int d, int block, float topk, const int32_t* idx_override,
                const uint8_t* qsel, int flags, double* out, int32_t* idx_out) {
  if (BH < 1 || N < 1 || d < 1 || d > 1024 || block < 1 || !(topk > 0.f) || topk > 1.f) return -1;
  int nb = (N + block - 1) / block;
  int kc = orc_topk_count(nb, topk);
  int nq = (N + ORC_QBLK - 1) / ORC_QBLK;
#pragma omp parallel for schedule(dynamic, 1)
  for (int bh = 0; bh < BH; ++bh) {
    int64_t o = (int64_t)bh * N * d;
    orc_head Hd;
    memset(&Hd, 0, sizeof(Hd));
    Hd.N = N;
    Hd.d = d;
    Hd.block = block;
    Hd.nb = nb;
    Hd.kc = kc;
    Hd.q = q + o;
    Hd.k = k + o;
    Hd.v = v + o;
    Hd.w = w;
    Hd.flags = flags;
    float* mu = (float*)malloc(sizeof(float) * d);
    float* ks = (float*)malloc(sizeof(float) * (int64_t)N * d);
    int8_t* q8 = (int8_t*)malloc((size_t)N * d);
    int8_t* k8 = (int8_t*)malloc((size_t)N * d);
    uint8_t* v8 = (uint8_t*)malloc((size_t)N * d);
    float* sq = (float*)malloc(sizeof(float) * (nq > N ? nq : N));
    float* sk = (float*)malloc(sizeof(float) * nq);
    float* sv = (float*)malloc(sizeof(float) * d);
    quant_head(Hd.q, Hd.k, Hd.v, N, d, mu, ks, q8, k8, v8, sq, sk, sv, (flags & ORC_QK_INT4) ? 7 : 127,
               (flags & ORC_Q_PER_TOKEN) != 0);
    Hd.q8 = q8;
    Hd.k8 = k8;
    Hd.v8 = v8;
    Hd.sq = sq;
    Hd.sk = sk;
    Hd.sv = sv;
    Hd.mu = mu;
    int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (int64_t)nb * kc);
    if (idx_override) {
      memcpy(idx, idx_override + (int64_t)bh * nb * kc, sizeof(int32_t) * (int64_t)nb * kc);
    } else {
      float* qb = (float*)malloc(sizeof(float) * (int64_t)nb * d);
      float* kb = (float*)malloc(sizeof(float) * (int64_t)nb * d);
      pool_head(Hd.q, ks, N, d, block, qb, kb);
      mask_rows(qb, kb, nb, d, kc, idx, NULL);
      free(qb);
      free(kb);
    }
    if (idx_out) memcpy(idx_out + (int64_t)bh * nb * kc, idx, sizeof(int32_t) * (int64_t)nb * kc);
    double* h = NULL;
    double* z = NULL;
    if (w) {
      h = (double*)malloc(sizeof(double) * (int64_t)nb * d * d);
      z = (double*)malloc(sizeof(double) * (int64_t)nb * d);
      linear_blocks(Hd.k, Hd.v, N, d, block, h, z);
      Hd.h = h;
      Hd.z = z;
    }
    for (int i = 0; i < nb; ++i) {
      if (qsel && !qsel[(int64_t)bh * nb + i]) continue;
      emul_qblock(&Hd, i, idx + (int64_t)i * kc, out + o);
    }
    free(mu);
    free(ks);
    free(q8);
    free(k8);
    free(v8);
    free(sq);
    free(sk);
    free(sv);
    free(idx);
    free(h);
    free(z);
  }
  return kc;
}

/* Linear branch alone, straight from its per-token definition, for the
 * identity pin: for row r of block i, num = sum over valid tokens n of key
 * blocks not in S_i of (phi(q_r).phi(k_n)) v_n, den = sum of phi(q_r).phi(k_n);
 * O_l = num/den (0 when no such token).  fp64 inputs [N][d]; out [N][d]. */
void orc_linear_direct(const double* q, const double* k, const double* v, int N, int d, int block,
                       int kc, const int32_t* idx, double* out) {
  int nb = (N + block - 1) / block;
#pragma omp parallel for schedule(dynamic, 4)
  for (int r = 0; r < N; ++r) {
    int i = r / block;
    uint8_t* in_s = (uint8_t*)calloc(nb, 1);
    for (int t = 0; t < kc; ++t) in_s[idx[(int64_t)i * kc + t]] = 1;
    double den = 0.0;
    double* num = out + (int64_t)r * d;
    for (int c = 0; c < d; ++c) num[c] = 0.0;
    for (int n = 0; n < N; ++n) {
      if (in_s[n / block]) continue;
      double a = 0.0;
      for (int c = 0; c < d; ++c) a += phi(q[(int64_t)r * d + c]) * phi(k[(int64_t)n * d + c]);
      den += a;
      for (int c = 0; c < d; ++c) num[c] += a * v[(int64_t)n * d + c];
    }
    for (int c = 0; c < d; ++c) num[c] = den > 0.0 ? num[c] / den : 0.0;
    free(in_s);
  }
}

/* ------------------------------------------------------------------------ */
/* W8A8 linear layer ("揭秘TurboDiffusion：如何让视频生成实现百倍加速？",   */
/* 支柱三 W8A8线性层量化; 量子位 news, 技术解密 4): weights and activations   */
/* are both INT8, quantised in blocks of 128 x 128, and y = x W^T (W is     */
/* [N][K], the nn.Linear convention).  Reading (the pages give only the     */
/* block size): one fp32 scale per 128 x 128 block, the same symmetric      */
/* quantiser as Q and K above (s = fl32(amax/127), code = RNE(fl32(x *      */
/* fl32(127/amax))) clamped to +-127; amax = 0 -> s = 1, codes 0); a last    */
/* block of rows shorter than 128 is quantised over its valid rows.          */
/*   y[m][n] = sum over 128-wide K blocks kb of                              */
/*             s_x[m/128][kb] * s_w[n/128][kb] * (exact integer dot on kb).  */
/* ------------------------------------------------------------------------ */
#define ORC_WBLK 128

/* a: bf16 [rows][cols] (cols a multiple of 128); q: int8 [rows][cols];
 * s: fp32 [ceil(rows/128)][cols/128]. */
void orc_w8a8_quant(const uint16_t* a, int rows, int cols, int8_t* q, float* s) {
  const int nrb = (rows + ORC_WBLK - 1) / ORC_WBLK, ncb = cols / ORC_WBLK;
  for (int rb = 0; rb < nrb; ++rb)
    for (int cb = 0; cb < ncb; ++cb) {
      const int r0 = rb * ORC_WBLK, r1 = r0 + ORC_WBLK < rows ? r0 + ORC_WBLK : rows;
      const int c0 = cb * ORC_WBLK;
      float amax = 0.f;
      for (int r = r0; r < r1; ++r)
        for (int c = c0; c < c0 + ORC_WBLK; ++c) {
          float x = fabsf(bf16_f32(a[(int64_t)r * cols + c]));
          if (x > amax) amax = x;
        }
      const float mult = amax > 0.f ? 127.f / amax : 0.f;
      s[(int64_t)rb * ncb + cb] = amax > 0.f ? amax / 127.f : 1.f;
      for (int r = r0; r < r1; ++r)
        for (int c = c0; c < c0 + ORC_WBLK; ++c)
          q[(int64_t)r * cols + c] = orc_int8_code(bf16_f32(a[(int64_t)r * cols + c]), mult);
    }
}

/* y: fp64 [M][N] from the codes and scales of x [M][K] and W [N][K]. */
void orc_w8a8_gemm(const int8_t* qx, const float* sx, const int8_t* qw, const float* sw, int M, int N, int K,
                   double* y) {
  const int nkb = K / ORC_WBLK;
#pragma omp parallel for schedule(static)
  for (int m = 0; m < M; ++m)
    for (int n = 0; n < N; ++n) {
      double acc = 0.0;
      for (int kb = 0; kb < nkb; ++kb) {
        int64_t dot = 0;
        for (int k = kb * ORC_WBLK; k < (kb + 1) * ORC_WBLK; ++k)
          dot += (int64_t)qx[(int64_t)m * K + k] * (int64_t)qw[(int64_t)n * K + k];
        acc += (double)sx[(int64_t)(m / ORC_WBLK) * nkb + kb] * (double)sw[(int64_t)(n / ORC_WBLK) * nkb + kb] *
               (double)dot;
      }
      y[(int64_t)m * N + n] = acc;
    }
}

/* ------------------------------------------------------------------------ */
/* QK RMSNorm before the path ("thu-ml/TurboDiffusion" radar page §二 step 5:  */
/* the DiT's norms run in its own kernels; 量子位 news, 技术解密 4: custom      */
/* RMSNorm kernels).  Reading: per token, over the model dimension (all H   */
/* heads x d channels), y = x / sqrt(mean(x^2) + eps) * gamma, gamma of     */
/* length H*d; the mean in fp64, inv = fl32(1/sqrt(mean + eps)), then       */
/* y = bf16(fl32(fl32(x * inv) * gamma)) -- the normalised activations are  */
/* bf16, the DiT's activation type.  x, y: bf16 [B][H][N][d].               */
/* ------------------------------------------------------------------------ */
void orc_rmsnorm_bf16(const uint16_t* x, const uint16_t* gamma, int B, int H, int N, int d, double eps,
                      uint16_t* y) {
#pragma omp parallel for schedule(static)
  for (int64_t bn = 0; bn < (int64_t)B * N; ++bn) {
    const int b = (int)(bn / N), n = (int)(bn % N);
    double ss = 0.0;
    for (int h = 0; h < H; ++h)
      for (int c = 0; c < d; ++c) {
        const double v = bf16_f32(x[(((int64_t)b * H + h) * N + n) * d + c]);
        ss += v * v;
      }
    const float inv = (float)(1.0 / sqrt(ss / ((double)H * d) + eps));
    for (int h = 0; h < H; ++h)
      for (int c = 0; c < d; ++c) {
        const int64_t o = (((int64_t)b * H + h) * N + n) * d + c;
        const float t = bf16_f32(x[o]) * inv;
        const float r = t * bf16_f32(gamma[(int64_t)h * d + c]);
        /* round to bf16, nearest even (r is finite) */
        uint32_t u;
        memcpy(&u, &r, 4);
        u += 0x7FFFu + ((u >> 16) & 1u);
        y[o] = (uint16_t)(u >> 16);
      }
  }
}
