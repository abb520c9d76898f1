/*
 * oracle.h -- plain single-threaded CPU oracle of the routed-expert MoE layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link or
 * call this code: only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference arm use it.  It shares no code with the CUDA path.
 *
 * What it computes (sources, by page and section):
 *  - int4 weights in groups of 64 with one scale per group ("gs64 group-scaled"):
 *    colibri (tantan.ink), section on pitfalls "我看到的几个坑"; colibri deep review
 *    (ai-tools-nav), install notes.
 *  - int8 activations in 32-wide blocks with one scale per block ("Q8_0 style"):
 *    Colibri article (alphamatch.ai), section "優化整數核心".
 *  - batch union of the routed experts, gate/up/down stored side by side:
 *    colibri (tantan.ink), section "几个关键工程动作".
 *  - shared expert in the resident dense part: colibri (tantan.ink), section
 *    "它的核心判断".
 *  - router = softmax over the experts, top-k kept and renormalised; the pages
 *    do not name the router function, this is the layer's definition as stated
 *    for this library.
 * Where the pages are silent (rounding mode, tie-breaks, scale types, the
 * order of every fp32 sum, the nibble layout), the choice is stated at the
 * function that makes it.
 *
 * Arithmetic is IEEE binary32, each operation rounded once; the file is
 * compiled with -ffp-contract=off, so the only fused multiply-adds are the
 * explicit fmaf() of the router's fixed order.  Sums run in the plain order of
 * the definition (index ascending, one accumulator), not in any order a
 * kernel chooses.  e^x is the C library's expf.  Integer dot products are
 * exact (int32).
 *
 * Parity status: every function here is pinned by tests/test_oracle.py
 * (brute force, closed forms, exact-integer special cases, invariants, and a
 * float64 NumPy evaluation within a stated bound).
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Container: bytes of one [N][K] int4 gs64 matrix (packed nibbles, then fp16 scales). */
size_t or_matrix_bytes(int N, int K);
/* Bytes of one expert blob: gate [I][H], up [I][H], down [H][I] back to back. */
size_t or_expert_bytes(int H, int I);

/* Signed weight w in [-8,7] of element (n,k) of a packed matrix. */
int or_weight(const uint8_t *mat, int N, int K, int n, int k);
/* fp32 value of the fp16 scale of group (n, g). */
float or_scale(const uint8_t *mat, int N, int K, int n, int g);
/* Builds a packed matrix from signed weights w[N][K] in [-8,7] and fp16 bit
 * patterns of the scales s16[N][K/64]. */
void or_pack_matrix(const int8_t *w, const uint16_t *s16, int N, int K, uint8_t *mat);
/* fp16 bit pattern -> float (exact). */
float or_half_to_float(uint16_t h);

/* Q8_0: x[n] (n % 32 == 0) -> q[n], d[n/32]. */
void or_quant_q8_0(const float *x, int64_t n, int8_t *q, float *d);

/* SiLU(g) = g / (1 + expf(-g)), expf from the C library. */
float or_silu(float g);
/* Element-wise array form of the above (for sweeps in the tests). */
void or_silu_n(const float *x, float *y, int64_t n);

/* Router logits in the fixed order (32 strided fmaf chains, xor tree). */
float or_router_logit(const float *x, const float *wr, int H);
void or_router_logits(const float *x, const float *Wr, int T, int H, int E, float *logits);
/* Top-k by logit (ties to the lower expert index), softmax over the kept k. */
void or_topk_softmax(const float *logits, int T, int E, int k, int32_t *idx, float *w);

/* Counting sort of the T*k (token, slot) pairs by expert. */
void or_bucket(const int32_t *idx, int T, int k, int E, int32_t *cnt, int32_t *off,
               int32_t *uni, int32_t *n_uni, int32_t *perm);

/* Exact int32 dot of 32-element block b of row n with q[32b .. 32b+32). */
int32_t or_block_dot(const uint8_t *mat, int N, int K, int n, int b, const int8_t *q);
/* Row n of the matrix against the Q8_0 vector (q, d): the sum over the groups
 * g ascending of s_g * (S_2g d_2g + S_2g+1 d_2g+1), one binary32 accumulator. */
float or_expert_dot(const uint8_t *mat, int N, int K, int n, const int8_t *q, const float *d);

/* The down projection of one expert from given Q8_0 codes of h:
 * y[m] = row m of the down matrix against (hq[I], hd[I/32]), m < H. */
void or_expert_down(const uint8_t *blob, int H, int I, const int8_t *hq, const float *hd, float *y);

/* One SwiGLU expert on one token.  Any of the intermediate outputs may be NULL.
 * g[I], u[I], h[I], hq[I], hd[I/32], y[H]. */
void or_expert_ffn(const uint8_t *blob, int H, int I, const int8_t *xq, const float *xd,
                   float *g, float *u, float *h, int8_t *hq, float *hd, float *y);

/* ---- MXFP4 experts (microscaled FP4: 32 E2M1 elements per E8M0 scale).
 * Matrix [N][K]: N*K/2 bytes, two consecutive elements per byte (lower index
 * in the low nibble), then N*K/32 E8M0 exponent bytes; value = e2m1(code) *
 * 2^(E-127).  Blob = gate | up | down as for int4 gs64, same byte count. */
#define OR_FMT_INT4_GS64 0
#define OR_FMT_MXFP4 1
/* E2M1 value of a 4-bit code (sign, 2 exponent bits with bias 1, 1 mantissa bit). */
float or_e2m1_value(int code);
int or_mx_code(const uint8_t *mat, int N, int K, int n, int k);
int or_mx_scale_exp(const uint8_t *mat, int N, int K, int n, int b);
float or_mx_weight(const uint8_t *mat, int N, int K, int n, int k);
/* codes[N][K] (0..15), exps[N][K/32] -> packed matrix. */
void or_mx_pack_matrix(const uint8_t *codes, const uint8_t *exps, int N, int K, uint8_t *mat);
/* Exact int32 sum over block b of row n: sum 2*e2m1(code) * q. */
int32_t or_mx_block_dot(const uint8_t *mat, int N, int K, int n, int b, const int8_t *q);
/* Row n against the Q8_0 vector: block terms (S_b * d_b) * 2^(E_b - 128) summed
 * over b ascending, one binary32 accumulator. */
float or_mx_expert_dot(const uint8_t *mat, int N, int K, int n, const int8_t *q, const float *d);
/* The down projection of an MXFP4 expert from given Q8_0 codes of h. */
void or_mx_expert_down(const uint8_t *blob, int H, int I, const int8_t *hq, const float *hd, float *y);
void or_mx_expert_ffn(const uint8_t *blob, int H, int I, const int8_t *xq, const float *xd,
                      float *g, float *u, float *h, int8_t *hq, float *hd, float *y);

/* Intermediates of a full layer call (all optional, NULL to skip). */
typedef struct or_layer_trace {
  int8_t *xq;      /* [T][H]      */
  float *xd;       /* [T][H/32]   */
  float *logits;   /* [T][E]      */
  int32_t *idx;    /* [T][k]      */
  float *w;        /* [T][k]      */
  int32_t *cnt;    /* [E]         */
  int32_t *off;    /* [E+1]       */
  int32_t *uni;    /* [E]         */
  int32_t *n_uni;  /* [1]         */
  int32_t *perm;   /* [T*k]       */
  int8_t *hq;      /* [T][k+1][I]   pair (t,s), slot k = shared expert */
  float *hd;       /* [T][k+1][I/32] */
  float *y;        /* [T][k+1][H]   */
} or_layer_trace;

/* The whole layer.  blobs[e] for e < E are the routed experts, blobs[E] is the
 * shared expert.  Returns 0, or -1 on a shape it does not accept. */
int or_moe_layer(int H, int I, int E, int k, int T, const float *x, const float *Wr,
                 const uint8_t *const *blobs, float *out, or_layer_trace *trace);

/* The whole layer with MXFP4 expert blobs (routing, SwiGLU, Q8_0 of h and the
 * combine exactly as or_moe_layer). */
int or_moe_layer_mx(int H, int I, int E, int k, int T, const float *x, const float *Wr,
                    const uint8_t *const *blobs, float *out, or_layer_trace *trace);

/* Token subset variant: only rows tok[0..n_tok) of x are evaluated; out is
 * [n_tok][H].  Used to time and check a bounded sample of a large batch
 * (routing of a token does not depend on other tokens). */
int or_moe_layer_tokens(int H, int I, int E, int k, const float *x, const float *Wr,
                        const uint8_t *const *blobs, const int32_t *tok, int n_tok,
                        float *out);
/* The same with MXFP4 expert blobs. */
int or_moe_layer_tokens_mx(int H, int I, int E, int k, const float *x, const float *Wr,
                           const uint8_t *const *blobs, const int32_t *tok, int n_tok,
                           float *out);

#ifdef __cplusplus
}
#endif
#endif
