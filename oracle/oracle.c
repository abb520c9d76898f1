/*
 * oracle.c -- plain, slow, single-threaded CPU oracle of the routed-expert MoE
 * layer.  TEST INFRASTRUCTURE ONLY (see oracle.h): the product path never
 * links or calls it, and it shares no code with the CUDA kernels.
 *
 * Build: gcc -O2 -std=c99 -ffp-contract=off -fPIC -shared oracle.c -lm
 * (-ffp-contract=off: a*b+c is two roundings unless fmaf() is written.)
 *
 * Page citations are given per function.  The pages describe the engine
 * (colibri) in prose only and print no listing of these steps; where they are
 * silent, the reading taken is stated at the function.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Weight container.                                                         */
/* int4 weights, one fp16 scale per group of 64 along the input dimension:   */
/* "gs64 group-scaled" container of colibri (tantan.ink), "我看到的几个坑";   */
/* gate / up / down of an expert stored next to each other so that one read  */
/* fetches the expert: colibri (tantan.ink), "几个关键工程动作".              */
/* Byte layout (this library's reading; the pages give none):                */
/*   row-major [N][K/2] packed bytes; group g of row n = bytes [32g, 32g+32); */
/*   byte j of a group: low nibble = element 64g+j, high = element 64g+32+j; */
/*   nibble u = w + 8 (offset binary), w in [-8, 7];                         */
/*   then [N][K/64] IEEE fp16 scales; dequantised weight = w * scale.        */
/* ------------------------------------------------------------------------ */

size_t or_matrix_bytes(int N, int K) {
  return (size_t)N * (size_t)(K / 2) + (size_t)N * (size_t)(K / 64) * 2u;
}

size_t or_expert_bytes(int H, int I) {
  return 2u * or_matrix_bytes(I, H) + or_matrix_bytes(H, I);
}

int or_weight(const uint8_t *mat, int N, int K, int n, int k) {
  (void)N;
  int g = k / 64, j = k % 64;
  uint8_t byte = mat[(size_t)n * (size_t)(K / 2) + (size_t)(32 * g + (j % 32))];
  int u = (j < 32) ? (byte & 0x0F) : (byte >> 4);
  return u - 8;
}

float or_half_to_float(uint16_t h) {
  int sign = (h >> 15) & 1;
  int ex = (h >> 10) & 0x1F;
  int man = h & 0x3FF;
  float v;
  if (ex == 0) {
    v = ldexpf((float)man, -24); /* subnormal: man * 2^-24, exact */
  } else if (ex == 31) {
    v = man ? NAN : INFINITY;
  } else {
    v = ldexpf((float)(man + 1024), ex - 25); /* (1024+man) * 2^(ex-15-10) */
  }
  return sign ? -v : v;
}

float or_scale(const uint8_t *mat, int N, int K, int n, int g) {
  const uint8_t *s = mat + (size_t)N * (size_t)(K / 2);
  size_t o = ((size_t)n * (size_t)(K / 64) + (size_t)g) * 2u;
  uint16_t h = (uint16_t)(s[o] | (s[o + 1] << 8)); /* little-endian */
  return or_half_to_float(h);
}

void or_pack_matrix(const int8_t *w, const uint16_t *s16, int N, int K, uint8_t *mat) {
  size_t rowb = (size_t)(K / 2);
  for (int n = 0; n < N; ++n) {
    for (int g = 0; g < K / 64; ++g) {
      for (int j = 0; j < 32; ++j) {
        int lo = w[(size_t)n * K + 64 * g + j] + 8;
        int hi = w[(size_t)n * K + 64 * g + 32 + j] + 8;
        mat[(size_t)n * rowb + 32 * g + j] = (uint8_t)((lo & 0xF) | ((hi & 0xF) << 4));
      }
    }
  }
  uint8_t *s = mat + (size_t)N * rowb;
  for (size_t i = 0; i < (size_t)N * (size_t)(K / 64); ++i) {
    s[2 * i] = (uint8_t)(s16[i] & 0xFF);
    s[2 * i + 1] = (uint8_t)(s16[i] >> 8);
  }
}

/* ------------------------------------------------------------------------ */
/* Q8_0 activations: int8 values in blocks of 32 with one fp32 scale per      */
/* block -- Colibri article (alphamatch.ai), "優化整數核心".                  */
/* Reading: d = amax / 127 (one IEEE division), q = round-half-even(x / d);   */
/* a block with d == 0 quantises to all zeros.                                */
/* ------------------------------------------------------------------------ */

void or_quant_q8_0(const float *x, int64_t n, int8_t *q, float *d) {
  for (int64_t b = 0; b < n / 32; ++b) {
    const float *xb = x + 32 * b;
    float amax = 0.0f;
    for (int i = 0; i < 32; ++i) {
      float a = fabsf(xb[i]);
      if (a > amax) amax = a;
    }
    float db = amax / 127.0f;
    d[b] = db;
    for (int i = 0; i < 32; ++i) {
      int v = 0;
      if (db != 0.0f) {
        float r = rintf(xb[i] / db);
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        v = (int)r;
      }
      q[32 * b + i] = (int8_t)v;
    }
  }
}

/* ------------------------------------------------------------------------ */
/* SiLU, the gate of the SwiGLU expert FFN: SiLU(g) = g / (1 + e^-g).        */
/* e^x is the C library's expf (a library primitive; the pages fix no        */
/* approximation of their own).                                               */
/* ------------------------------------------------------------------------ */

/* SwiGLU expert FFN, SiLU(gate) * up: the experts of the models the pages run
 * (GLM-5.2 MoE layers; colibri (tantan.ink), "它的核心判断"). */
float or_silu(float g) {
  float e = expf(-g);
  float den = 1.0f + e;
  return g / den;
}

void or_silu_n(const float *x, float *y, int64_t n) {
  for (int64_t i = 0; i < n; ++i) y[i] = or_silu(x[i]);
}

/* ------------------------------------------------------------------------ */
/* Router: per-token scores over the routed experts (256 per layer for       */
/* GLM-5.2: colibri (tantan.ink), "它的核心判断"), softmax top-k.             */
/* Fixed order (a reading; the pages give none): 32 chains, chain l sums      */
/* x[h]*Wr[h] for h = 32i + l, i ascending, with fmaf from 0; then for        */
/* off = 16,8,4,2,1 every chain becomes c[l] + c[l^off]; the logit is c[0].   */
/* Routing must not change with placement (colibri deep review, design rule   */
/* "never silently change precision or router semantics"), so both sides    */
/* use this one order and the selected experts are reproducible bit for bit. */
/* ------------------------------------------------------------------------ */

float or_router_logit(const float *x, const float *wr, int H) {
  float c[32], t[32];
  for (int l = 0; l < 32; ++l) {
    float p = 0.0f;
    for (int i = 0; 32 * i + l < H; ++i) p = fmaf(x[32 * i + l], wr[32 * i + l], p);
    c[l] = p;
  }
  for (int off = 16; off >= 1; off >>= 1) {
    for (int l = 0; l < 32; ++l) t[l] = c[l] + c[l ^ off];
    memcpy(c, t, sizeof c);
  }
  return c[0];
}

void or_router_logits(const float *x, const float *Wr, int T, int H, int E, float *logits) {
  for (int t = 0; t < T; ++t)
    for (int e = 0; e < E; ++e)
      logits[(size_t)t * E + e] = or_router_logit(x + (size_t)t * H, Wr + (size_t)e * H, H);
}

/* Top-k: the k largest logits, a tie going to the lower expert index, listed
 * by descending logit.  Weights: softmax over the k kept logits, i.e. the full
 * softmax renormalised over the selection:
 *   m = l[idx0]; e_s = expf(l_s - m) (C library); Z = ((e_0 + e_1) + e_2) + ...;
 *   w_s = e_s / Z. */
void or_topk_softmax(const float *logits, int T, int E, int k, int32_t *idx, float *w) {
  unsigned char *taken = (unsigned char *)malloc((size_t)E);
  float *ev = (float *)malloc(sizeof(float) * (size_t)k);
  for (int t = 0; t < T; ++t) {
    const float *l = logits + (size_t)t * E;
    memset(taken, 0, (size_t)E);
    for (int s = 0; s < k; ++s) {
      int best = -1;
      for (int e = 0; e < E; ++e)
        if (!taken[e] && (best < 0 || l[e] > l[best])) best = e;
      taken[best] = 1;
      idx[(size_t)t * k + s] = best;
    }
    float m = l[idx[(size_t)t * k]];
    float z = 0.0f;
    for (int s = 0; s < k; ++s) {
      ev[s] = expf(l[idx[(size_t)t * k + s]] - m);
      z = (s == 0) ? ev[0] : z + ev[s];
    }
    for (int s = 0; s < k; ++s) w[(size_t)t * k + s] = ev[s] / z;
  }
  free(ev);
  free(taken);
}

/* ------------------------------------------------------------------------ */
/* Batch union: the experts picked by the batch, each listed once, so each is */
/* fetched once -- colibri (tantan.ink), "几个关键工程动作" (Batch union), and */
/* the batched-union MoE of prefill, Colibri article (alphamatch.ai).         */
/* cnt[e] = pairs routed to e; off = exclusive prefix sum (off[E] = T*k);     */
/* uni = experts with cnt > 0 ascending; perm = pair ids p = t*k+s grouped by */
/* expert, ascending p inside each group (a stable counting sort).            */
/* ------------------------------------------------------------------------ */

void or_bucket(const int32_t *idx, int T, int k, int E, int32_t *cnt, int32_t *off,
               int32_t *uni, int32_t *n_uni, int32_t *perm) {
  int P = T * k;
  for (int e = 0; e < E; ++e) cnt[e] = 0;
  for (int p = 0; p < P; ++p) cnt[idx[p]] += 1;
  off[0] = 0;
  for (int e = 0; e < E; ++e) off[e + 1] = off[e] + cnt[e];
  int nu = 0;
  for (int e = 0; e < E; ++e)
    if (cnt[e] > 0) uni[nu++] = e;
  *n_uni = nu;
  int32_t *cur = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E > 0 ? E : 1));
  for (int e = 0; e < E; ++e) cur[e] = off[e];
  for (int p = 0; p < P; ++p) perm[cur[idx[p]]++] = p;
  free(cur);
}

/* ------------------------------------------------------------------------ */
/* int4 x int8 dot products (the integer kernels of the engine: Colibri       */
/* article (alphamatch.ai), "優化整數核心").                                  */
/* Row n of a [N][K] matrix against a Q8_0 vector (q, d), the definition      */
/* written out:                                                               */
/*   S_b = sum over the 32 elements of block b of w*q          (exact int32) */
/*   row value = sum over the groups g = 0 .. K/64-1, in ascending order, of  */
/*               s_g * (S_2g * d_2g + S_2g+1 * d_2g+1)                        */
/* in binary32 with one accumulator, each product and sum rounded once.       */
/* ------------------------------------------------------------------------ */

int32_t or_block_dot(const uint8_t *mat, int N, int K, int n, int b, const int8_t *q) {
  int32_t s = 0;
  for (int i = 0; i < 32; ++i) s += or_weight(mat, N, K, n, 32 * b + i) * (int32_t)q[32 * b + i];
  return s;
}

float or_expert_dot(const uint8_t *mat, int N, int K, int n, const int8_t *q, const float *d) {
  float acc = 0.0f;
  for (int g = 0; g < K / 64; ++g) {
    float s0 = (float)or_block_dot(mat, N, K, n, 2 * g, q);
    float s1 = (float)or_block_dot(mat, N, K, n, 2 * g + 1, q);
    float grp = s0 * d[2 * g] + s1 * d[2 * g + 1];
    acc = acc + or_scale(mat, N, K, n, g) * grp;
  }
  return acc;
}

/* ------------------------------------------------------------------------ */
/* MXFP4 experts (microscaled FP4): in the model-family table of the colibri */
/* deep review (ai-tools-nav), the Kimi K3 row says that family's experts    */
/* come QAT-trained in MXFP4 and are streamed as shipped, with no conversion. */
/* The pages give no finer detail; the format is the OCP Microscaling one:   */
/* blocks of 32 E2M1 elements sharing an E8M0 scale.  Readings stated here:  */
/*  - element value = e2m1(code) * 2^(E - 127); E = 255 (NaN) is outside the */
/*    contract;                                                              */
/*  - [N][K] matrix = N*K/2 packed bytes (two consecutive elements per byte, */
/*    the lower-indexed one in the low nibble), then N*K/32 E8M0 bytes, one  */
/*    per 32-block of a row -- the same byte count as the int4 gs64 layout,  */
/*    and the same blob order gate | up | down;                              */
/*  - activations stay Q8_0, so a block's products 2*e2m1 * q are integers   */
/*    and its sum S_b is exact; the block term is (S_b * d_b) * 2^(E_b-128)  */
/*    (the second factor a power of two), and the row value is the sum of    */
/*    the block terms over b = 0 .. K/32-1 in ascending order, one binary32  */
/*    accumulator.                                                           */
/* ------------------------------------------------------------------------ */
float or_e2m1_value(int code) {
  int sign = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
  /* subnormal when the exponent field is 0: m * 2^-1; else (1 + m/2) * 2^(e-1) */
  float mag = (e == 0) ? 0.5f * (float)m : (1.0f + 0.5f * (float)m) * ldexpf(1.0f, e - 1);
  return sign ? -mag : mag;
}

int or_mx_code(const uint8_t *mat, int N, int K, int n, int k) {
  (void)N;
  uint8_t byte = mat[(size_t)n * (size_t)(K / 2) + (size_t)(k / 2)];
  return (k & 1) ? (byte >> 4) : (byte & 15);
}

int or_mx_scale_exp(const uint8_t *mat, int N, int K, int n, int b) {
  return mat[(size_t)N * (size_t)(K / 2) + (size_t)n * (size_t)(K / 32) + (size_t)b];
}

/* 2^k for any k in [-149, 127], exact (a subnormal power of two below -126). */
static float pow2_any(int k) { return ldexpf(1.0f, k); }

float or_mx_weight(const uint8_t *mat, int N, int K, int n, int k) {
  return or_e2m1_value(or_mx_code(mat, N, K, n, k)) * pow2_any(or_mx_scale_exp(mat, N, K, n, k / 32) - 127);
}

void or_mx_pack_matrix(const uint8_t *codes, const uint8_t *exps, int N, int K, uint8_t *mat) {
  for (int n = 0; n < N; ++n)
    for (int j = 0; j < K / 2; ++j) {
      uint8_t lo = codes[(size_t)n * K + 2 * j] & 15, hi = codes[(size_t)n * K + 2 * j + 1] & 15;
      mat[(size_t)n * (K / 2) + j] = (uint8_t)(lo | (hi << 4));
    }
  memcpy(mat + (size_t)N * (K / 2), exps, (size_t)N * (size_t)(K / 32));
}

int32_t or_mx_block_dot(const uint8_t *mat, int N, int K, int n, int b, const int8_t *q) {
  int32_t s = 0;
  for (int i = 0; i < 32; ++i) {
    int k = 32 * b + i;
    /* 2 * e2m1 is an integer in [-12, 12] */
    int32_t c2 = (int32_t)(2.0f * or_e2m1_value(or_mx_code(mat, N, K, n, k)));
    s += c2 * (int32_t)q[k];
  }
  return s;
}

float or_mx_expert_dot(const uint8_t *mat, int N, int K, int n, const int8_t *q, const float *d) {
  float acc = 0.0f;
  for (int b = 0; b < K / 32; ++b) {
    int32_t sb = or_mx_block_dot(mat, N, K, n, b, q);
    float t = ((float)sb * d[b]) * pow2_any(or_mx_scale_exp(mat, N, K, n, b) - 128);
    acc = acc + t;
  }
  return acc;
}

void or_expert_down(const uint8_t *blob, int H, int I, const int8_t *hq, const float *hd, float *y) {
  const uint8_t *down = blob + 2 * or_matrix_bytes(I, H);
  for (int m = 0; m < H; ++m) y[m] = or_expert_dot(down, H, I, m, hq, hd);
}

/* The same down projection for an MXFP4 blob (same byte offsets). */
void or_mx_expert_down(const uint8_t *blob, int H, int I, const int8_t *hq, const float *hd, float *y) {
  const uint8_t *down = blob + 2 * or_matrix_bytes(I, H);
  for (int m = 0; m < H; ++m) y[m] = or_mx_expert_dot(down, H, I, m, hq, hd);
}

/* Row n of an [N][K] matrix of weight format fmt (OR_FMT_INT4_GS64 or
 * OR_FMT_MXFP4) against the Q8_0 vector (q, d). */
static float fmt_dot(int fmt, const uint8_t *mat, int N, int K, int n, const int8_t *q, const float *d) {
  return fmt == OR_FMT_MXFP4 ? or_mx_expert_dot(mat, N, K, n, q, d) : or_expert_dot(mat, N, K, n, q, d);
}

static void expert_ffn_fmt(int fmt, const uint8_t *blob, int H, int I, const int8_t *xq, const float *xd,
                           float *g, float *u, float *h, int8_t *hq, float *hd, float *y) {
  const uint8_t *gate = blob;
  const uint8_t *up = blob + or_matrix_bytes(I, H);  /* both formats: N*K/2 + N*K/32 bytes */
  float *hh = (float *)malloc(sizeof(float) * (size_t)I);
  int8_t *q = (int8_t *)malloc((size_t)I);
  float *dd = (float *)malloc(sizeof(float) * (size_t)(I / 32));
  for (int n = 0; n < I; ++n) {
    float gv = fmt_dot(fmt, gate, I, H, n, xq, xd);
    float uv = fmt_dot(fmt, up, I, H, n, xq, xd);
    if (g) g[n] = gv;
    if (u) u[n] = uv;
    hh[n] = or_silu(gv) * uv;
  }
  or_quant_q8_0(hh, I, q, dd);
  if (h) memcpy(h, hh, sizeof(float) * (size_t)I);
  if (hq) memcpy(hq, q, (size_t)I);
  if (hd) memcpy(hd, dd, sizeof(float) * (size_t)(I / 32));
  if (y) {
    const uint8_t *down = blob + 2 * or_matrix_bytes(I, H);
    for (int m = 0; m < H; ++m) y[m] = fmt_dot(fmt, down, H, I, m, q, dd);
  }
  free(dd);
  free(q);
  free(hh);
}

void or_expert_ffn(const uint8_t *blob, int H, int I, const int8_t *xq, const float *xd,
                   float *g, float *u, float *h, int8_t *hq, float *hd, float *y) {
  expert_ffn_fmt(OR_FMT_INT4_GS64, blob, H, I, xq, xd, g, u, h, hq, hd, y);
}

void or_mx_expert_ffn(const uint8_t *blob, int H, int I, const int8_t *xq, const float *xd,
                      float *g, float *u, float *h, int8_t *hq, float *hd, float *y) {
  expert_ffn_fmt(OR_FMT_MXFP4, blob, H, I, xq, xd, g, u, h, hq, hd, y);
}

/* ------------------------------------------------------------------------ */
/* The layer: shared expert (part of the resident dense weights, colibri      */
/* (tantan.ink), "它的核心判断") plus the router-weighted routed experts.      */
/* out[t] = y_shared; then for s = 0..k-1: out = out + w[t,s] * y_s, each     */
/* product and sum rounded once (the sum in slot order, shared term first).   */
/* No residual add, no norm: the input is the already normalised hidden       */
/* state (reading).  The shared expert has weight 1 (reading).               */
/* ------------------------------------------------------------------------ */

static int dims_ok(int H, int I, int E, int k) {
  return H > 0 && I > 0 && H % 128 == 0 && I % 128 == 0 && E >= 1 && k >= 1 && k <= E;
}

static void token_forward(int fmt, int H, int I, int E, int k, const float *xt, const float *Wr,
                          const uint8_t *const *blobs, float *out, int8_t *xq_o, float *xd_o,
                          float *logit_o, int32_t *idx_o, float *w_o, int8_t *hq_o,
                          float *hd_o, float *y_o) {
  int8_t *xq = (int8_t *)malloc((size_t)H);
  float *xd = (float *)malloc(sizeof(float) * (size_t)(H / 32));
  float *lg = (float *)malloc(sizeof(float) * (size_t)E);
  int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)k);
  float *w = (float *)malloc(sizeof(float) * (size_t)k);
  float *y = (float *)malloc(sizeof(float) * (size_t)H);
  or_quant_q8_0(xt, H, xq, xd);
  or_router_logits(xt, Wr, 1, H, E, lg);
  or_topk_softmax(lg, 1, E, k, idx, w);
  /* shared expert first (slot k in the trace) */
  expert_ffn_fmt(fmt, blobs[E], H, I, xq, xd, NULL, NULL, NULL, hq_o ? hq_o + (size_t)k * I : NULL,
                 hd_o ? hd_o + (size_t)k * (I / 32) : NULL, y);
  if (y_o) memcpy(y_o + (size_t)k * H, y, sizeof(float) * (size_t)H);
  memcpy(out, y, sizeof(float) * (size_t)H);
  for (int s = 0; s < k; ++s) {
    expert_ffn_fmt(fmt, blobs[idx[s]], H, I, xq, xd, NULL, NULL, NULL,
                   hq_o ? hq_o + (size_t)s * I : NULL, hd_o ? hd_o + (size_t)s * (I / 32) : NULL, y);
    if (y_o) memcpy(y_o + (size_t)s * H, y, sizeof(float) * (size_t)H);
    for (int m = 0; m < H; ++m) out[m] = out[m] + w[s] * y[m];
  }
  if (xq_o) memcpy(xq_o, xq, (size_t)H);
  if (xd_o) memcpy(xd_o, xd, sizeof(float) * (size_t)(H / 32));
  if (logit_o) memcpy(logit_o, lg, sizeof(float) * (size_t)E);
  if (idx_o) memcpy(idx_o, idx, sizeof(int32_t) * (size_t)k);
  if (w_o) memcpy(w_o, w, sizeof(float) * (size_t)k);
  free(y);
  free(w);
  free(idx);
  free(lg);
  free(xd);
  free(xq);
}

static int layer_fmt(int fmt, int H, int I, int E, int k, int T, const float *x, const float *Wr,
                     const uint8_t *const *blobs, float *out, or_layer_trace *tr) {
  if (!dims_ok(H, I, E, k) || T < 0) return -1;
  int32_t *idx_all = (int32_t *)malloc(sizeof(int32_t) * (size_t)(T > 0 ? T * k : 1));
  for (int t = 0; t < T; ++t) {
    size_t tk = (size_t)t * (size_t)(k + 1);
    token_forward(fmt, H, I, E, k, x + (size_t)t * H, Wr, blobs, out + (size_t)t * H,
                  tr && tr->xq ? tr->xq + (size_t)t * H : NULL,
                  tr && tr->xd ? tr->xd + (size_t)t * (H / 32) : NULL,
                  tr && tr->logits ? tr->logits + (size_t)t * E : NULL, idx_all + (size_t)t * k,
                  tr && tr->w ? tr->w + (size_t)t * k : NULL,
                  tr && tr->hq ? tr->hq + tk * I : NULL,
                  tr && tr->hd ? tr->hd + tk * (I / 32) : NULL,
                  tr && tr->y ? tr->y + tk * H : NULL);
  }
  if (tr && tr->idx) memcpy(tr->idx, idx_all, sizeof(int32_t) * (size_t)T * k);
  if (tr && tr->cnt && tr->off && tr->uni && tr->n_uni && tr->perm)
    or_bucket(idx_all, T, k, E, tr->cnt, tr->off, tr->uni, tr->n_uni, tr->perm);
  free(idx_all);
  return 0;
}

int or_moe_layer(int H, int I, int E, int k, int T, const float *x, const float *Wr,
                 const uint8_t *const *blobs, float *out, or_layer_trace *tr) {
  return layer_fmt(OR_FMT_INT4_GS64, H, I, E, k, T, x, Wr, blobs, out, tr);
}

int or_moe_layer_mx(int H, int I, int E, int k, int T, const float *x, const float *Wr,
                    const uint8_t *const *blobs, float *out, or_layer_trace *tr) {
  return layer_fmt(OR_FMT_MXFP4, H, I, E, k, T, x, Wr, blobs, out, tr);
}

static int layer_tokens_fmt(int fmt, int H, int I, int E, int k, const float *x, const float *Wr,
                            const uint8_t *const *blobs, const int32_t *tok, int n_tok, float *out) {
  if (!dims_ok(H, I, E, k) || n_tok < 0) return -1;
  for (int i = 0; i < n_tok; ++i)
    token_forward(fmt, H, I, E, k, x + (size_t)tok[i] * H, Wr, blobs, out + (size_t)i * H, NULL,
                  NULL, NULL, NULL, NULL, NULL, NULL, NULL);
  return 0;
}

int or_moe_layer_tokens(int H, int I, int E, int k, const float *x, const float *Wr,
                        const uint8_t *const *blobs, const int32_t *tok, int n_tok,
                        float *out) {
  return layer_tokens_fmt(OR_FMT_INT4_GS64, H, I, E, k, x, Wr, blobs, tok, n_tok, out);
}

int or_moe_layer_tokens_mx(int H, int I, int E, int k, const float *x, const float *Wr,
                           const uint8_t *const *blobs, const int32_t *tok, int n_tok,
                           float *out) {
  return layer_tokens_fmt(OR_FMT_MXFP4, H, I, E, k, x, Wr, blobs, tok, n_tok, out);
}
