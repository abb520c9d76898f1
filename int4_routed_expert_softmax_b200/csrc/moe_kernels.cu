// moe_kernels.cu -- sm_100a kernels of the routed-expert MoE layer, decode
// (GEMV) path plus the routing kernels shared by every path.
//
// The layer (per token t):
//   x -> Q8_0 (32-wide blocks, fp32 scale)           Colibri (alphamatch.ai), 優化整數核心
//   logits = x . Wr, top-k, softmax over the k kept  router over 256 experts, tantan.ink 它的核心判断
//   batch union of the selected experts               tantan.ink 几个关键工程动作 (Batch union)
//   per expert: g, u = int4 gs64 x Q8_0 dots; h = SiLU(g) * u; h -> Q8_0;
//               y = int4 down x Q8_0(h)              gs64 container, tantan.ink 我看到的几个坑
//   out = y_shared + sum_s w_s * y_s                  shared expert, tantan.ink 它的核心判断
//
// Decode design (B200): the expert weights are the only large operand
// (20,054,016 B per expert at H=6144, I=2048), so the two FFN kernels are
// persistent, one CTA per SM, and stream weight rows through a ring of
// shared-memory stages filled by TMA bulk copies (cp.async.bulk, completion
// on mbarriers) issued by one producer thread; eight consumer warps unpack
// nibbles in registers and run dp4a integer dots per 32-block.  The fp32
// steps that decide integer codes follow one fixed order (see moe_device.cuh).
#include <climits>
#include <cstdio>

#include "moe_device.cuh"

namespace moe {

// =====================================================================
// Q8_0 quantisation: one warp per 32-block (lane = element).
// =====================================================================
__global__ void __launch_bounds__(256) k_quant(QuantArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t b = gw; b < a.nblk; b += nw) {
    const float v = a.x[b * 32 + lane];
    const float d = fdiv(warp_max(fabsf(v)), 127.0f);
    a.q[b * 32 + lane] = (int8_t)q8_code(v, d);
    if (lane == 0) a.d[b] = d;
  }
}

cudaError_t launch_quant(const QuantArgs &a, cudaStream_t s) {
  if (a.nblk == 0) return cudaSuccess;
  int64_t blocks = (a.nblk + 7) / 8;
  if (blocks > 148 * 16) blocks = 148 * 16;
  k_quant<<<(unsigned)blocks, 256, 0, s>>>(a);
  return cudaGetLastError();
}

// =====================================================================
// Block-wide exclusive scan of n <= 1024 ints (one CTA, any warp count).
// scratch: >= 33 ints of shared memory.  Returns the total.
// =====================================================================
__device__ int block_exclusive_scan(const int *in, int *out, int n, int *scratch) {
  const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
  const int per = (n + nt - 1) / nt;
  const int b0 = min(n, tid * per), b1 = min(n, b0 + per);
  int local = 0;
  for (int i = b0; i < b1; ++i) local += in[i];
  int incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int w = 0; w < (nt + 31) / 32; ++w) {
      const int v = scratch[w];
      scratch[w] = run;
      run += v;
    }
    scratch[32] = run;
  }
  __syncthreads();
  int run = scratch[warp] + incl - local;
  for (int i = b0; i < b1; ++i) {
    const int v = in[i];
    out[i] = run;
    run += v;
  }
  const int total = scratch[32];
  __syncthreads();
  return total;
}

// =====================================================================
// Stable counting sort of P = T*k pairs by expert, one CTA.
// s_idx: the pairs' experts in shared memory (or global), s_work: >= 3E+40
// ints of shared memory.  Writes cnt, off, uni (+ shared slot E), n_uni,
// perm, pos and pair_tok (routed positions, then T shared positions).
// =====================================================================
__device__ void bucket_block(int E, int k, int T, const int32_t *idx, int *s_work, int32_t *cnt,
                             int32_t *off, int32_t *uni, int32_t *n_uni, int32_t *perm,
                             int32_t *pos, int32_t *pair_tok) {
  const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
  const int P = T * k;
  int *s_cnt = s_work;           // [E]
  int *s_off = s_work + E;       // [E]  (exclusive)
  int *s_cur = s_work + 2 * E;   // [E]  running cursors
  int *scratch = s_work + 3 * E; // [40]
  for (int e = tid; e < E; e += nt) s_cnt[e] = 0;
  __syncthreads();
  for (int p = tid; p < P; p += nt) atomicAdd(&s_cnt[idx[p]], 1);
  __syncthreads();
  block_exclusive_scan(s_cnt, s_off, E, scratch);
  for (int e = tid; e < E; e += nt) {
    cnt[e] = s_cnt[e];
    off[e] = s_off[e];
    s_cur[e] = (s_cnt[e] > 0) ? 1 : 0;  // flags for the union scan
  }
  if (tid == 0) off[E] = P;
  __syncthreads();
  const int nu = block_exclusive_scan(s_cur, s_cur, E, scratch);
  for (int e = tid; e < E; e += nt)
    if (s_cnt[e] > 0) uni[s_cur[e]] = e;
  if (tid == 0) {
    *n_uni = nu;
    uni[nu] = E;  // the shared expert follows the union
  }
  __syncthreads();
  for (int e = tid; e < E; e += nt) s_cur[e] = s_off[e];
  __syncthreads();
  // stable placement: chunks of nt pairs in order; inside a chunk, warps take
  // turns; inside a warp, lanes with equal experts are ranked by lane.
  const int nwarps = (nt + 31) / 32;
  for (int c0 = 0; c0 < P; c0 += nt) {
    const int p = c0 + tid;
    const bool has = p < P;
    const int e = has ? idx[p] : -1 - lane;  // distinct dummies never match
    for (int w = 0; w < nwarps; ++w) {
      if (warp == w) {
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const unsigned lt = (1u << lane) - 1u;
        const int leader = __ffs(peers) - 1;
        int base = 0;
        if (has) base = s_cur[e];
        __syncwarp();
        if (has && lane == leader) s_cur[e] = base + __popc(peers);
        if (has) {
          const int q = base + __popc(peers & lt);
          perm[q] = p;
          if (pos) pos[p] = q;
          if (pair_tok) pair_tok[q] = p / k;
        }
      }
      __syncthreads();
    }
  }
  if (pair_tok)
    for (int t = tid; t < T; t += nt) pair_tok[P + t] = t;
}

// =====================================================================
// The same stable counting sort by a single warp (no block barriers): for
// the decode batch (P = T*k <= 512 pairs).  s_work: >= 2E ints of shared
// memory; idx may live in shared memory.
// =====================================================================
__device__ void bucket_warp(int E, int k, int T, const int32_t *idx, int *s_work, int32_t *cnt,
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
// holding slot s (expert, logit).  Ties go to the lower expert index.
// =====================================================================
__device__ __forceinline__ void warp_topk(const float *lg, int E, int k, int lane, int &e_sel,
                                          float &l_sel) {
  float v[32];
  const int nper = (E + 31) >> 5;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const int e = lane + 32 * j;
    v[j] = (j < nper && e < E) ? __ldcg(lg + e) : 0.0f;
  }
  unsigned taken = 0u;
  e_sel = 0;
  l_sel = 0.0f;
  for (int s = 0; s < k; ++s) {
    float bv = 0.0f;
    int be = INT_MAX;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int e = lane + 32 * j;
      if (j < nper && e < E && !((taken >> j) & 1u)) {
        if (be == INT_MAX || v[j] > bv) {
          bv = v[j];
          be = e;
        }
      }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oe = __shfl_xor_sync(0xffffffffu, be, off);
      if (oe != INT_MAX && (be == INT_MAX || ov > bv || (ov == bv && oe < be))) {
        bv = ov;
        be = oe;
      }
    }
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    if (lane == s) {
      e_sel = be;
      l_sel = bv;
    }
  }
}

// softmax over the k kept logits held one per lane; writes idx / w of token t.
__device__ __forceinline__ void warp_softmax_store(int t, int k, int lane, int e_sel, float l_sel,
                                                   int32_t *idx, float *w, int32_t *counts,
                                                   int *s_idx) {
  const float m = __shfl_sync(0xffffffffu, l_sel, 0);
  const float ev = (lane < k) ? exp_cw(__fsub_rn(l_sel, m)) : 0.0f;
  float z = __shfl_sync(0xffffffffu, ev, 0);
  for (int s = 1; s < k; ++s) z = fadd(z, __shfl_sync(0xffffffffu, ev, s));
  if (lane < k) {
    idx[(size_t)t * k + lane] = e_sel;
    w[(size_t)t * k + lane] = fdiv(ev, z);
    if (s_idx) s_idx[t * k + lane] = e_sel;
    if (counts) atomicAdd(counts + e_sel, 1);
  }
}

// =====================================================================
// Router for small batches: Q8_0 of x (grid-stride), logits of epc experts
// per CTA from shared-memory copies of their Wr rows and of x (TMA bulk),
// then the last CTA to finish takes top-k + softmax and the batch union.
// Logit order: lane l accumulates h = l, l+32, ... with fmaf, then an xor
// tree 16, 8, 4, 2, 1 -- the router's fixed order.
// =====================================================================
__global__ void __launch_bounds__(128) k_route_decode(RouteArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem);
  int *s_flag = reinterpret_cast<int *>(smem + 16);
  float *sW = reinterpret_cast<float *>(smem + 128);
  float *sX = sW + (size_t)a.epc * a.H;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = a.H;

  const int e0 = blockIdx.x * a.epc;
  const int ne = min(a.epc, a.E - e0);
  // start the copies of the first tile before the quantisation work below
  auto issue = [&](int t0) {
    const int nt = min(a.tt, a.T - t0);
    const uint32_t xb = (uint32_t)nt * H * 4u;
    const uint32_t wb = (t0 == 0) ? (uint32_t)ne * H * 4u : 0u;
    mbar_arrive_expect_tx(bar, xb + wb);
    if (wb) bulk_g2s(sW, a.Wr + (size_t)e0 * H, wb, bar);
    bulk_g2s(sX, a.x + (size_t)t0 * H, xb, bar);
  };
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
    issue(0);
  }
  if (a.do_quant) {
    const int64_t nblk = (int64_t)a.T * (H / 32);
    for (int64_t b = (int64_t)blockIdx.x * 4 + warp; b < nblk; b += (int64_t)gridDim.x * 4) {
      const float v = a.x[b * 32 + lane];
      const float d = fdiv(warp_max(fabsf(v)), 127.0f);
      a.xq[b * 32 + lane] = (int8_t)q8_code(v, d);
      if (lane == 0) a.xd[b] = d;
    }
  }
  __syncthreads();
  int phase = 0;
  for (int t0 = 0; t0 < a.T; t0 += a.tt, ++phase) {
    const int nt = min(a.tt, a.T - t0);
    if (tid == 0 && t0 > 0) issue(t0);
    const bool ok = __syncthreads_and(mbar_wait(bar, phase & 1, a.status, kDetRouteBar));
    if (!ok) return;
    for (int p = warp; p < ne * nt; p += 4) {
      const int ei = p / nt, ti = p % nt;
      const float *wv = sW + (size_t)ei * H;
      const float *xv = sX + (size_t)ti * H;
      float acc = 0.0f;
#pragma unroll 8
      for (int i = lane; i < H; i += 32) acc = ffma(xv[i], wv[i], acc);
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) acc = fadd(acc, __shfl_xor_sync(0xffffffffu, acc, off));
      if (lane == 0) a.logits[(size_t)(t0 + ti) * a.E + e0 + ei] = acc;
    }
    __syncthreads();
  }
  if (a.done == nullptr) return;

  // ---- the last CTA to arrive does top-k and the batch union
  __threadfence();
  __syncthreads();
  if (tid == 0) *s_flag = (atomicAdd(a.done, 1u) == gridDim.x - 1) ? 1 : 0;
  __syncthreads();
  if (!*s_flag) return;
  __threadfence();
  int *s_idx = reinterpret_cast<int *>(sW);               // [T*k]
  int *s_work = s_idx + kDecodeTMax * kMaxK;              // bucket scratch
  for (int t = warp; t < a.T; t += 4) {
    int e_sel;
    float l_sel;
    warp_topk(a.logits + (size_t)t * a.E, a.E, a.k, lane, e_sel, l_sel);
    warp_softmax_store(t, a.k, lane, e_sel, l_sel, a.idx, a.w, a.route_counts, s_idx);
  }
  __syncthreads();
  if (warp != 0) return;
  if (a.do_bucket)
    bucket_warp(a.E, a.k, a.T, s_idx, s_work, a.cnt, a.off, a.uni, a.n_uni, a.perm, a.pos,
                a.pair_tok);
  if (lane == 0) *a.done = 0u;
}

size_t route_smem_bytes(int H, int epc, int tt) {
  size_t fl = (size_t)(epc + tt) * H * 4;
  size_t need_tail = (size_t)(kDecodeTMax * kMaxK + 3 * MOE_MAX_E + 64) * 4;
  return 128 + (fl > need_tail ? fl : need_tail);
}

cudaError_t launch_route_decode(const RouteArgs &a, cudaStream_t s) {
  const size_t smem = route_smem_bytes(a.H, a.epc, a.tt);
  cudaError_t err = cudaFuncSetAttribute(k_route_decode, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
  if (err != cudaSuccess) return err;
  const int grid = (a.E + a.epc - 1) / a.epc;
  k_route_decode<<<grid, 128, smem, s>>>(a);
  return cudaGetLastError();
}

// =====================================================================
// Standalone top-k (warp per token) and bucket (one CTA) kernels.
// =====================================================================
__global__ void __launch_bounds__(256) k_topk(const float *logits, int T, int E, int k, int32_t *idx,
                                             float *w, int32_t *counts) {
  const int lane = threadIdx.x & 31;
  const int t = (int)(((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  if (t >= T) return;
  int e_sel;
  float l_sel;
  warp_topk(logits + (size_t)t * E, E, k, lane, e_sel, l_sel);
  warp_softmax_store(t, k, lane, e_sel, l_sel, idx, w, counts, nullptr);
}

cudaError_t launch_topk(const float *logits, int T, int E, int k, int32_t *idx, float *w,
                        int32_t *counts, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  k_topk<<<(T + 7) / 8, 256, 0, s>>>(logits, T, E, k, idx, w, counts);
  return cudaGetLastError();
}

__global__ void __launch_bounds__(1024) k_bucket(BucketArgs a) {
  extern __shared__ __align__(16) int s_work[];
  bucket_block(a.E, a.k, a.T, a.idx, s_work, a.cnt, a.off, a.uni, a.n_uni, a.perm, a.pos,
               a.pair_tok);
}

cudaError_t launch_bucket(const BucketArgs &a, cudaStream_t s) {
  const size_t smem = (size_t)(3 * a.E + 64) * 4;
  k_bucket<<<1, 1024, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace moe
