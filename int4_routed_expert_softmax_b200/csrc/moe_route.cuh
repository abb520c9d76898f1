// moe_route.cuh -- device pieces of the routing step shared by the routing
// kernels (moe_kernels.cu) and the fused batch-1 kernel (moe_fused.cu): the
// batch union of up to 32 (token, slot) pairs in registers, the warp top-k
// (ties to the lower expert index) and the softmax over the kept logits.
#pragma once

#include <climits>

#include "moe_device.cuh"

namespace moe {

// =====================================================================
// The same counting sort for P = T*k <= 32 pairs, in registers: lane p holds
// pair p; its position is the number of pairs before it in (expert, pair id)
// order; the union follows from comparisons.  Counts and offsets of all E
// experts: bucket_small_counts (any number of warps).
// =====================================================================
__device__ inline void bucket_small_counts(int E, int P, const int *s_pairs, int32_t *cnt, int32_t *off, int warp,
                                    int nwarps) {
  const int lane = threadIdx.x & 31;
  for (int e = warp * 32 + lane; e < E; e += nwarps * 32) {
    int c = 0, o = 0;
    for (int q = 0; q < P; ++q) {
      const int eq = s_pairs[q];  // every lane reads the same word
      c += eq == e ? 1 : 0;
      o += eq < e ? 1 : 0;
    }
    cnt[e] = c;
    off[e] = o;
  }
}

__device__ inline void bucket_small(int E, int k, int T, const int32_t *idx, int32_t *cnt, int32_t *off,
                             int32_t *uni, int32_t *n_uni, int32_t *perm, int32_t *pos,
                             int32_t *pair_tok) {
  const int lane = threadIdx.x & 31;
  const int P = T * k;
  const int ep = lane < P ? idx[lane] : INT_MAX;
  int rank = 0, first = 1, below = 0;  // below: distinct experts smaller than ep
  for (int q = 0; q < P; ++q) {
    const int eq = __shfl_sync(0xffffffffu, ep, q);
    rank += (eq < ep || (eq == ep && q < lane)) ? 1 : 0;
    if (eq == ep && q < lane) first = 0;
  }
  // distinct experts below ep: pairs q that are the first of their expert
  const int fl = (lane < P) ? first : 0;
  const unsigned firsts = __ballot_sync(0xffffffffu, fl);
  for (int q = 0; q < P; ++q) {
    const int eq = __shfl_sync(0xffffffffu, ep, q);
    below += (((firsts >> q) & 1u) && eq < ep) ? 1 : 0;
  }
  const int nu = __popc(firsts);
  if (lane < P) {
    perm[rank] = lane;
    if (pos) pos[lane] = rank;
    if (pair_tok) pair_tok[rank] = lane / k;
    if (first) uni[below] = ep;
  }
  if (lane == 0) {
    off[E] = P;
    *n_uni = nu;
    uni[nu] = E;
  }
  if (pair_tok)
    for (int t = lane; t < T; t += 32) pair_tok[P + t] = t;
}

// =====================================================================
// The same stable counting sort by a single warp (no block barriers), for
// the decode batches (P = T*k <= 512 pairs): counts by shared-memory atomics,
// offsets and the union by a warp scan over the experts, positions chunk by
// chunk with match.any among the lanes of one expert (pairs of an expert stay
// in pair order).  s_work: >= 2E ints of shared memory; idx may live in shared
// memory.
// =====================================================================
__device__ inline void bucket_warp(int E, int k, int T, const int32_t *idx, int *s_work, int32_t *cnt,
                            int32_t *off, int32_t *uni, int32_t *n_uni, int32_t *perm,
                            int32_t *pos, int32_t *pair_tok) {
  const int lane = threadIdx.x & 31;
  const int P = T * k;
  int *s_cnt = s_work;      // [E]
  int *s_cur = s_work + E;  // [E]
  for (int e = lane; e < E; e += 32) s_cnt[e] = 0;
  __syncwarp();
  for (int p = lane; p < P; p += 32) atomicAdd(&s_cnt[idx[p]], 1);
  __syncwarp();
  // exclusive scans of the counts and of the union flags; lane owns a range
  const int per = (E + 31) / 32;
  const int b0 = min(E, lane * per), b1 = min(E, b0 + per);
  int lc = 0, lf = 0;
  for (int e = b0; e < b1; ++e) {
    lc += s_cnt[e];
    lf += s_cnt[e] > 0 ? 1 : 0;
  }
  int ic = lc, jf = lf;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int vc = __shfl_up_sync(0xffffffffu, ic, o);
    const int vf = __shfl_up_sync(0xffffffffu, jf, o);
    if (lane >= o) {
      ic += vc;
      jf += vf;
    }
  }
  int run = ic - lc, runf = jf - lf;
  for (int e = b0; e < b1; ++e) {
    const int c = s_cnt[e];
    cnt[e] = c;
    off[e] = run;
    s_cur[e] = run;
    run += c;
    if (c > 0) uni[runf++] = e;
  }
  const int nu = __shfl_sync(0xffffffffu, jf, 31);
  if (lane == 0) {
    off[E] = P;
    *n_uni = nu;
    uni[nu] = E;  // the shared expert follows the union
  }
  __syncwarp();
  const unsigned lt = (1u << lane) - 1u;
  for (int c0 = 0; c0 < P; c0 += 32) {
    const int p = c0 + lane;
    const bool has = p < P;
    const int e = has ? idx[p] : -1 - lane;  // distinct dummies never match
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int base = has ? s_cur[e] : 0;
    __syncwarp();
    if (has && lane == __ffs(peers) - 1) s_cur[e] = base + __popc(peers);
    if (has) {
      const int q = base + __popc(peers & lt);
      perm[q] = p;
      if (pos) pos[p] = q;
      if (pair_tok) pair_tok[q] = p / k;
    }
    __syncwarp();
  }
  if (pair_tok)
    for (int t = lane; t < T; t += 32) pair_tok[P + t] = t;
}

// =====================================================================
// Top-k of one token's logits by one warp (E <= 1024, k <= 32): lane s ends
// holding slot s (expert, logit); ties go to the lower expert index.
// Selection by a bitwise radix search for the k-th largest logit: logits map
// to order-preserving unsigned keys (-0 taken as +0 so that equal values tie);
// 32 halving steps with a warp-wide count (redux) find the k-th largest key;
// every key above it is kept, and keys equal to it are taken in ascending
// expert index until k are kept; the kept k are then ranked by (logit
// descending, index ascending).  scratch: 128 words of shared memory per warp.
// =====================================================================
__device__ __forceinline__ uint32_t order_key(float v) {
  if (v == 0.0f) v = 0.0f;  // -0 == +0
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
// The logit of a key (-0 comes back as +0, equal in every later use).
__device__ __forceinline__ float key_value(uint32_t kk) {
  return __uint_as_float((kk & 0x80000000u) ? (kk & 0x7FFFFFFFu) : ~kk);
}

template <int NPER>
__device__ __forceinline__ void warp_topk_radix(const float *lg, int E, int k, int lane, int &e_sel,
                                                float &l_sel, uint32_t *scratch) {
  float v[NPER];
  uint32_t key[NPER];
#pragma unroll
  for (int j = 0; j < NPER; ++j) {
    const int e = lane + 32 * j;
    v[j] = e < E ? __ldcg(lg + e) : 0.0f;
    key[j] = e < E ? order_key(v[j]) : 0u;  // absent entries never reach the top k (k <= E)
  }
  uint32_t pre = 0u;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = pre | (1u << bit);
    int c = 0;  // keys >= cand over the warp: one vote per held key (absent keys are 0 < cand)
#pragma unroll
    for (int j = 0; j < NPER; ++j) c += __popc(__ballot_sync(0xffffffffu, key[j] >= cand));
    if (c >= k) pre = cand;
  }
  // pre = k-th largest key: keep > pre, then == pre by ascending index
  int gt = 0;
#pragma unroll
  for (int j = 0; j < NPER; ++j) gt += (lane + 32 * j < E && key[j] > pre) ? 1 : 0;
  const int need = k - (int)__reduce_add_sync(0xffffffffu, (unsigned)gt);
  const unsigned lt = (1u << lane) - 1u;
  int eq_before = 0, sel_before = 0;
  uint32_t *s_key = scratch, *s_e = scratch + 32;
#pragma unroll
  for (int j = 0; j < NPER; ++j) {
    const int e = lane + 32 * j;
    const bool valid = e < E;
    const bool eq = valid && key[j] == pre;
    const unsigned beq = __ballot_sync(0xffffffffu, eq);
    const bool keep = valid && (key[j] > pre || (eq && eq_before + __popc(beq & lt) < need));
    eq_before += __popc(beq);
    const unsigned bk = __ballot_sync(0xffffffffu, keep);
    if (keep) {
      const int at = sel_before + __popc(bk & lt);  // compaction in index order
      s_key[at] = key[j];
      s_e[at] = (uint32_t)e;
    }
    sel_before += __popc(bk);
  }
  __syncwarp();
  e_sel = 0;
  l_sel = 0.0f;
  if (lane < k) {
    const uint32_t mk = s_key[lane];
    const int me = (int)s_e[lane];
    int rank = 0;
    for (int i = 0; i < k; ++i) {
      const uint32_t ok = s_key[i];
      const int oe = (int)s_e[i];
      rank += (ok > mk || (ok == mk && oe < me)) ? 1 : 0;
    }
    scratch[64 + rank] = (uint32_t)me;
    scratch[96 + rank] = mk;
  }
  __syncwarp();
  if (lane < k) {
    e_sel = (int)scratch[64 + lane];
    l_sel = key_value(scratch[96 + lane]);
  }
  __syncwarp();
}

// The same selection for small k by k rounds of a warp argmax: each lane keeps
// its NPER keys in registers; a round takes each lane's best live key (the
// lowest index among equal keys), the warp's largest key, and among the lanes
// holding it the lowest expert index -- so round r yields the r-th largest
// logit, ties to the lower index, as the radix selection does.
template <int NPER>
__device__ __forceinline__ void warp_topk_rounds(const float *lg, int E, int k, int lane, int &e_sel,
                                                 float &l_sel) {
  uint32_t key[NPER];
  uint32_t live = 0u;  // bit j: entry lane + 32 j present and not yet taken
#pragma unroll
  for (int j = 0; j < NPER; ++j) {
    const int e = lane + 32 * j;
    key[j] = e < E ? order_key(__ldcg(lg + e)) : 0u;
    if (e < E) live |= 1u << j;
  }
  e_sel = 0;
  l_sel = 0.0f;
  for (int r = 0; r < k; ++r) {
    uint32_t bk = 0u;
    int bj = -1;
#pragma unroll
    for (int j = 0; j < NPER; ++j)
      if (((live >> j) & 1u) && (bj < 0 || key[j] > bk)) {
        bk = key[j];
        bj = j;
      }
    const uint32_t m = __reduce_max_sync(0xffffffffu, bj >= 0 ? bk : 0u);
    const uint32_t cand = (bj >= 0 && bk == m) ? (uint32_t)(lane + 32 * bj) : 0xFFFFFFFFu;
    const uint32_t win = __reduce_min_sync(0xffffffffu, cand);
    if (win != 0xFFFFFFFFu && lane == (int)(win & 31u)) live &= ~(1u << (win >> 5));
    if (lane == r) {
      e_sel = (int)win;
      l_sel = key_value(m);
    }
  }
}

__device__ __forceinline__ void warp_topk(const float *lg, int E, int k, int lane, int &e_sel,
                                          float &l_sel, uint32_t *scratch) {
  const int nper = (E + 31) >> 5;
  if (k <= 12 && nper <= 8) {
    if (nper <= 4) warp_topk_rounds<4>(lg, E, k, lane, e_sel, l_sel);
    else warp_topk_rounds<8>(lg, E, k, lane, e_sel, l_sel);
    return;
  }
  if (nper <= 1) warp_topk_radix<1>(lg, E, k, lane, e_sel, l_sel, scratch);
  else if (nper <= 2) warp_topk_radix<2>(lg, E, k, lane, e_sel, l_sel, scratch);
  else if (nper <= 4) warp_topk_radix<4>(lg, E, k, lane, e_sel, l_sel, scratch);
  else if (nper <= 8) warp_topk_radix<8>(lg, E, k, lane, e_sel, l_sel, scratch);
  else if (nper <= 16) warp_topk_radix<16>(lg, E, k, lane, e_sel, l_sel, scratch);
  else warp_topk_radix<32>(lg, E, k, lane, e_sel, l_sel, scratch);
}

// softmax over the k kept logits held one per lane; writes idx / w of token t.
__device__ __forceinline__ void warp_softmax_store(int t, int k, int lane, int e_sel, float l_sel,
                                                   int32_t *idx, float *w, int32_t *counts,
                                                   int *s_idx) {
  const float m = __shfl_sync(0xffffffffu, l_sel, 0);
  const float ev = (lane < k) ? expf(__fsub_rn(l_sel, m)) : 0.0f;
  float z = __shfl_sync(0xffffffffu, ev, 0);
  for (int s = 1; s < k; ++s) z = fadd(z, __shfl_sync(0xffffffffu, ev, s));
  if (lane < k) {
    idx[(size_t)t * k + lane] = e_sel;
    w[(size_t)t * k + lane] = fdiv(ev, z);
    if (s_idx) s_idx[t * k + lane] = e_sel;
    if (counts) atomicAdd(counts + e_sel, 1);
  }
}

}  // namespace moe
