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

namespace {
inline size_t al128(size_t v) { return align_up(v, 128); }
}  // namespace

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

  if (a.do_quant) {
    const int64_t nblk = (int64_t)a.T * (H / 32);
    for (int64_t b = (int64_t)blockIdx.x * 4 + warp; b < nblk; b += (int64_t)gridDim.x * 4) {
      const float v = a.x[b * 32 + lane];
      const float d = fdiv(warp_max(fabsf(v)), 127.0f);
      a.xq[b * 32 + lane] = (int8_t)q8_code(v, d);
      if (lane == 0) a.xd[b] = d;
    }
  }

  const int e0 = blockIdx.x * a.epc;
  const int ne = min(a.epc, a.E - e0);
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  int phase = 0;
  for (int t0 = 0; t0 < a.T; t0 += a.tt, ++phase) {
    const int nt = min(a.tt, a.T - t0);
    if (tid == 0) {
      const uint32_t xb = (uint32_t)nt * H * 4u;
      const uint32_t wb = (t0 == 0) ? (uint32_t)ne * H * 4u : 0u;
      mbar_arrive_expect_tx(bar, xb + wb);
      if (wb) bulk_g2s(sW, a.Wr + (size_t)e0 * H, wb, bar);
      bulk_g2s(sX, a.x + (size_t)t0 * H, xb, bar);
    }
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
  if (a.do_bucket)
    bucket_block(a.E, a.k, a.T, s_idx, s_work, a.cnt, a.off, a.uni, a.n_uni, a.perm, a.pos,
                 a.pair_tok);
  if (tid == 0) *a.done = 0u;
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

// =====================================================================
// Decode gate/up: h = SiLU(Wg x) * (Wu x), requantised to Q8_0 per 32 rows.
//
// Work unit = (union slot, 32-row block of I); slot 0 is the shared expert,
// slot u >= 1 is uni[u-1].  Units are split evenly over the persistent CTAs.
// A unit is 8 stages of 4 gate rows + 4 up rows (packed nibbles + fp16
// scales, 4H + H/4 bytes at H=6144: 26,112 B), each stage one TMA
// transaction group.  Consumer warp w takes row (w & 3) of matrix (w >> 2);
// lane c owns the chunk of CSZ consecutive 64-groups [c*CSZ, c*CSZ+CSZ) --
// the chunk split of the fixed dot order -- and the 32 chunk sums are added
// left to right by one lane per token.
// =====================================================================
struct GuPlan {
  size_t red, gu, xd, qs, xq, stg, total;
  uint32_t sb;
  int chp;
};

__host__ __device__ inline size_t al128d(size_t v) { return (v + 127) / 128 * 128; }

__host__ __device__ inline GuPlan gu_plan(int H, int T, int ns, int csz) {
  GuPlan p;
  p.chp = csz * 64 + 16;
  p.sb = 4u * (uint32_t)H + (uint32_t)H / 4u;
  size_t o = al128d((size_t)16 * ns);
  p.red = o;
  o += al128d((size_t)8 * T * 33 * 4);
  p.gu = o;
  o += al128d((size_t)T * 64 * 4);
  p.xd = o;
  o += al128d((size_t)T * (H / 32) * 4);
  p.qs = o;
  o += al128d((size_t)T * (H / 32) * 4);
  p.xq = o;
  o += al128d((size_t)T * 32 * p.chp);
  p.stg = o;
  o += (size_t)ns * p.sb;
  p.total = o;
  return p;
}

template <int CSZ>
__global__ void __launch_bounds__(288, 1) k_gateup_decode(GateUpArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int H = a.H, I = a.I, T = a.T, NS = a.nstage;
  const int G = H / 64, HB = H / 32;
  const int nch = (G + CSZ - 1) / CSZ;
  const GuPlan pl = gu_plan(H, T, NS, CSZ);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem);
  uint64_t *empty = full + NS;
  float *red = reinterpret_cast<float *>(smem + pl.red);
  float *gu = reinterpret_cast<float *>(smem + pl.gu);
  float *xd_s = reinterpret_cast<float *>(smem + pl.xd);
  int *qs_s = reinterpret_cast<int *>(smem + pl.qs);
  unsigned char *xq_s = smem + pl.xq;
  unsigned char *stg = smem + pl.stg;
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    s_abort = 0;
    for (int s = 0; s < NS; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 8);
    }
    fence_barrier_init();
  }
  if (a.use_pdl) pdl_wait();

  // an earlier kernel of this call failed: leave everything untouched
  if (*reinterpret_cast<volatile int32_t *>(a.status) != 0) return;
  const int n_uni = min(max(*a.n_uni, 0), a.E);
  const int rbs = I / 32;  // 32-row blocks per expert
  const int n_units = (n_uni + 1) * rbs;
  const int u_begin = (int)((long long)blockIdx.x * n_units / gridDim.x);
  const int u_end = (int)((long long)(blockIdx.x + 1) * n_units / gridDim.x);
  const int n_stages = (u_end - u_begin) * 8;
  const size_t mg = (size_t)I * H / 2 + (size_t)I * H / 32;

  // blobs this CTA reads must be 16-byte aligned (TMA bulk copies)
  {
    bool bad = false;
    const int sl0 = u_begin / rbs, sl1 = (u_end - 1) / rbs;
    for (int sl = sl0 + tid; sl <= sl1 && u_end > u_begin; sl += blockDim.x) {
      const int e = sl == 0 ? a.E : a.uni[sl - 1];
      bad |= (reinterpret_cast<uintptr_t>(a.table[e]) & 15u) != 0;
    }
    if (__syncthreads_or(bad)) {
      if (tid == 0) set_status(a.status, MOE_ERR_DEVICE, kDetGuAlign);
      return;
    }
  }

  // stage this CTA's copy of the activations: xq in per-lane chunks
  // (padded rows, conflict-free 16-byte reads), block scales and code sums.
  {
    const int pieces = CSZ * 4;  // 16-byte pieces per lane chunk
    for (int i = tid; i < T * 32 * pieces; i += blockDim.x) {
      const int t = i / (32 * pieces), r = i % (32 * pieces), c = r / pieces, j = r % pieces;
      const int col = c * CSZ * 64 + 16 * j;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (col < H) v = *reinterpret_cast<const uint4 *>(a.xq + (size_t)t * H + col);
      *reinterpret_cast<uint4 *>(xq_s + (size_t)(t * 32 + c) * pl.chp + 16 * j) = v;
    }
    for (int i = tid; i < T * HB; i += blockDim.x) {
      xd_s[i] = a.xd[i];
      const uint4 *q4 = reinterpret_cast<const uint4 *>(a.xq + (size_t)i * 32);
      int s = 0;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const uint4 v = q4[j];
        s = __dp4a((int)v.x, 0x01010101, s);
        s = __dp4a((int)v.y, 0x01010101, s);
        s = __dp4a((int)v.z, 0x01010101, s);
        s = __dp4a((int)v.w, 0x01010101, s);
      }
      qs_s[i] = s;
    }
  }
  __syncthreads();

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int issued = 0;
      for (int j = 0; j < n_stages; ++j) {
        const int s = j % NS;
        if (j >= NS && !mbar_wait(empty + s, ((j / NS) - 1) & 1, a.status, kDetGuEmpty)) {
          s_abort = 1;
          break;
        }
        if (*reinterpret_cast<volatile int *>(&s_abort)) break;
        const int unit = u_begin + j / 8, st = j % 8;
        const int slot = unit / rbs, rb = unit % rbs;
        const int e = slot == 0 ? a.E : a.uni[slot - 1];
        const unsigned char *blob = reinterpret_cast<const unsigned char *>(a.table[e]);
        const size_t n0 = (size_t)rb * 32 + (size_t)st * 4;
        unsigned char *dst = stg + (size_t)s * pl.sb;
        mbar_arrive_expect_tx(full + s, pl.sb);
        bulk_g2s_hint(dst, blob + n0 * (H / 2), 2u * H, full + s, pol);
        bulk_g2s_hint(dst + 2 * H, blob + mg + n0 * (H / 2), 2u * H, full + s, pol);
        bulk_g2s_hint(dst + 4 * H, blob + (size_t)I * (H / 2) + n0 * (H / 32), H / 8, full + s, pol);
        bulk_g2s_hint(dst + 4 * H + H / 8, blob + mg + (size_t)I * (H / 2) + n0 * (H / 32), H / 8,
                      full + s, pol);
        issued = j + 1;
      }
      for (int j = (issued > NS ? issued - NS : 0); j < issued; ++j)
        mbar_wait(full + j % NS, (j / NS) & 1, a.status, kDetGuDrain);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int r = warp & 3, mat = warp >> 2;
  const int c0 = lane * CSZ;
  int cur_unit = -1, n_tok = 0, pos_base = 0, my_tok = 0;
  bool bad = false;
  for (int j = 0; j < n_stages; ++j) {
    const int s = j % NS;
    const int unit = u_begin + j / 8, st = j % 8;
    const int slot = unit / rbs, rb = unit % rbs;
    if (unit != cur_unit) {
      cur_unit = unit;
      if (slot == 0) {
        n_tok = T;
        pos_base = T * a.k;
        my_tok = lane;
      } else {
        const int e = a.uni[slot - 1];
        pos_base = a.off[e];
        n_tok = a.off[e + 1] - pos_base;
        my_tok = lane < n_tok ? a.pair_tok[pos_base + lane] : 0;
      }
    }
    if (!bad) bad = *reinterpret_cast<volatile int *>(&s_abort) != 0;
    if (!bad) {
      bad = !mbar_wait(full + s, (j / NS) & 1, a.status, kDetGuFull);
      bad = __any_sync(0xffffffffu, bad);
      if (bad && lane == 0) s_abort = 1;
    }
    if (!bad) {
      const unsigned char *sb = stg + (size_t)s * pl.sb;
      const unsigned char *rowp = sb + (size_t)mat * 2 * H + (size_t)r * (H / 2);
      const __half *scp = reinterpret_cast<const __half *>(sb + 4 * H + mat * (H / 8) + r * (H / 32));
      uint32_t lo[CSZ][8], hi[CSZ][8];
      float sc[CSZ];
#pragma unroll
      for (int gi = 0; gi < CSZ; ++gi) {
        const int g = c0 + gi;
        if (g < G) {
          const uint4 w0 = *reinterpret_cast<const uint4 *>(rowp + 32 * g);
          const uint4 w1 = *reinterpret_cast<const uint4 *>(rowp + 32 * g + 16);
          const uint32_t wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            lo[gi][q] = wv[q] & 0x0F0F0F0Fu;
            hi[gi][q] = (wv[q] >> 4) & 0x0F0F0F0Fu;
          }
          sc[gi] = __half2float(scp[g]);
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q) lo[gi][q] = hi[gi][q] = 0u;
          sc[gi] = 0.0f;
        }
      }
      for (int i = 0; i < n_tok; ++i) {
        const int t = __shfl_sync(0xffffffffu, my_tok, i);
        const unsigned char *xa = xq_s + (size_t)(t * 32 + lane) * pl.chp;
        const float *xdt = xd_s + t * HB;
        const int *qst = qs_s + t * HB;
        float acc = 0.0f;
#pragma unroll
        for (int gi = 0; gi < CSZ; ++gi) {
          const int g = c0 + gi;
          if (g < G) {
            const uint4 a0 = *reinterpret_cast<const uint4 *>(xa + 64 * gi);
            const uint4 a1 = *reinterpret_cast<const uint4 *>(xa + 64 * gi + 16);
            const uint4 a2 = *reinterpret_cast<const uint4 *>(xa + 64 * gi + 32);
            const uint4 a3 = *reinterpret_cast<const uint4 *>(xa + 64 * gi + 48);
            int s0 = -8 * qst[2 * g], s1 = -8 * qst[2 * g + 1];
            s0 = dp4a_us(lo[gi][0], a0.x, s0);
            s0 = dp4a_us(lo[gi][1], a0.y, s0);
            s0 = dp4a_us(lo[gi][2], a0.z, s0);
            s0 = dp4a_us(lo[gi][3], a0.w, s0);
            s0 = dp4a_us(lo[gi][4], a1.x, s0);
            s0 = dp4a_us(lo[gi][5], a1.y, s0);
            s0 = dp4a_us(lo[gi][6], a1.z, s0);
            s0 = dp4a_us(lo[gi][7], a1.w, s0);
            s1 = dp4a_us(hi[gi][0], a2.x, s1);
            s1 = dp4a_us(hi[gi][1], a2.y, s1);
            s1 = dp4a_us(hi[gi][2], a2.z, s1);
            s1 = dp4a_us(hi[gi][3], a2.w, s1);
            s1 = dp4a_us(hi[gi][4], a3.x, s1);
            s1 = dp4a_us(hi[gi][5], a3.y, s1);
            s1 = dp4a_us(hi[gi][6], a3.z, s1);
            s1 = dp4a_us(hi[gi][7], a3.w, s1);
            const float fa = fmul((float)s0, xdt[2 * g]);
            const float fb = ffma((float)s1, xdt[2 * g + 1], fa);
            acc = ffma(sc[gi], fb, acc);
          }
        }
        red[(warp * T + i) * 33 + lane] = acc;
      }
      __syncwarp();
      for (int i = lane; i < n_tok; i += 32) {
        const float *rr = red + (warp * T + i) * 33;
        float tot = rr[0];
        for (int c = 1; c < nch; ++c) tot = fadd(tot, rr[c]);
        gu[(i * 2 + mat) * 32 + st * 4 + r] = tot;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + s);
    }
    if (st == 7) {
      // unit complete: h = SiLU(g) * u for its 32 rows, Q8_0 per token
      named_sync(1, 256);
      if (!bad) {
        for (int i = warp; i < n_tok; i += 8) {
          const float g = gu[(i * 2 + 0) * 32 + lane];
          const float u = gu[(i * 2 + 1) * 32 + lane];
          const float h = swiglu(g, u);
          const float d = fdiv(warp_max(fabsf(h)), 127.0f);
          const int q = q8_code(h, d);
          const int pos = pos_base + i;
          a.hq[(size_t)pos * I + rb * 32 + lane] = (int8_t)q;
          int qsum = q;
#pragma unroll
          for (int off = 16; off >= 1; off >>= 1) qsum += __shfl_xor_sync(0xffffffffu, qsum, off);
          if (lane == 0) {
            a.hd[(size_t)pos * (I / 32) + rb] = d;
            a.hqs[(size_t)pos * (I / 32) + rb] = qsum;
          }
        }
      }
      named_sync(1, 256);
    }
  }
  if (a.use_pdl) pdl_launch_dependents();
}

size_t gateup_smem_bytes(int H, int T, int nstage) {
  const int csz = (H / 64 + 31) / 32;
  return gu_plan(H, T, nstage, csz).total;
}

int gateup_max_stages(int H, int T) {
  int ns = 8;
  while (ns >= 2 && gateup_smem_bytes(H, T, ns) > (size_t)kMaxSmem) --ns;
  return ns;
}

template <int CSZ>
static cudaError_t launch_gu(const GateUpArgs &a, int grid, size_t smem, cudaStream_t s) {
  cudaError_t err = cudaFuncSetAttribute(k_gateup_decode<CSZ>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(288);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.use_pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k_gateup_decode<CSZ>, a);
}

cudaError_t launch_gateup_decode(const GateUpArgs &a, int grid, size_t smem, cudaStream_t s) {
  const int csz = (a.H / 64 + 31) / 32;
  switch (csz) {
    case 1: return launch_gu<1>(a, grid, smem, s);
    case 2: return launch_gu<2>(a, grid, smem, s);
    case 3: return launch_gu<3>(a, grid, smem, s);
    case 4: return launch_gu<4>(a, grid, smem, s);
    default: return cudaErrorInvalidValue;
  }
}

// =====================================================================
// Decode down projection + combine.
//
// CTA c owns output rows [m0, m1) (balanced, in row groups of rg rows so
// every scale copy is a multiple of 16 bytes) and loops over the union
// slots; one stage = that slot's rows (packed + scales, ~42 x 1088 B at
// H=6144, I=2048).  y per (position, row) stays in shared memory; the
// combine out = y_shared, then fmaf(w_s, y_s, out) in slot order, runs in
// the same CTA at the end (deterministic, no atomics).
// =====================================================================
struct DnPlan {
  size_t red, ysm, stg, total;
  uint32_t sb;
};

__host__ __device__ inline DnPlan dn_plan(int I, int k, int T, int rows_max, int rs, int ns) {
  DnPlan p;
  p.sb = (uint32_t)al128d((size_t)rs * (I / 2) + (size_t)rs * (I / 32));
  size_t o = al128d((size_t)16 * ns);
  p.red = o;
  o += al128d((size_t)8 * T * 33 * 4);
  p.ysm = o;
  o += al128d((size_t)T * (k + 1) * rows_max * 4);
  p.stg = o;
  o += (size_t)ns * p.sb;
  p.total = o;
  return p;
}

constexpr int kDnTokBatch = 4;

template <int CSZ>
__global__ void __launch_bounds__(288, 1) k_down_decode(DownArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int H = a.H, I = a.I, T = a.T, K = a.k, NS = a.nstage;
  const int G = I / 64, IB = I / 32;
  const int nch = (G + CSZ - 1) / CSZ;
  const DnPlan pl = dn_plan(I, K, T, a.rows_max, a.rs, NS);
  const int RS = a.rs;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem);
  uint64_t *empty = full + NS;
  float *red = reinterpret_cast<float *>(smem + pl.red);
  float *ysm = reinterpret_cast<float *>(smem + pl.ysm);
  unsigned char *stg = smem + pl.stg;
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nrg = H / a.rg;
  const int m0 = (int)((long long)blockIdx.x * nrg / gridDim.x) * a.rg;
  const int m1 = (int)((long long)(blockIdx.x + 1) * nrg / gridDim.x) * a.rg;
  const int nrows = m1 - m0;
  const size_t mg = (size_t)I * H / 2 + (size_t)I * H / 32;
  const size_t pk_off = 2 * mg, sc_off = 2 * mg + (size_t)H * (I / 2);
  const int nsub = (nrows + RS - 1) / RS;  // row sub-ranges per union slot
  const size_t sc_in_stage = (size_t)RS * (I / 2);

  if (tid == 0) {
    s_abort = 0;
    for (int s = 0; s < NS; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 8);
    }
    fence_barrier_init();
  }
  if (a.use_pdl) pdl_wait();
  if (*reinterpret_cast<volatile int32_t *>(a.status) != 0) return;
  const int n_uni = min(max(*a.n_uni, 0), a.E);
  const int nslot = n_uni + 1;
  {
    bool bad = false;
    for (int sl = tid; sl < nslot; sl += blockDim.x) {
      const int e = sl == 0 ? a.E : a.uni[sl - 1];
      bad |= (reinterpret_cast<uintptr_t>(a.table[e]) & 15u) != 0;
    }
    if (__syncthreads_or(bad)) {
      if (tid == 0) set_status(a.status, MOE_ERR_DEVICE, kDetDnAlign);
      return;
    }
  }
  if (nrows <= 0) return;

  if (warp == 8) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int issued = 0;
      for (int j = 0; j < nslot * nsub; ++j) {
        const int s = j % NS;
        if (j >= NS && !mbar_wait(empty + s, ((j / NS) - 1) & 1, a.status, kDetDnEmpty)) {
          s_abort = 1;
          break;
        }
        if (*reinterpret_cast<volatile int *>(&s_abort)) break;
        const int slot = j / nsub, r0 = (j % nsub) * RS;
        const int nr = min(RS, nrows - r0);
        const uint32_t bytes_pk = (uint32_t)nr * (I / 2), bytes_sc = (uint32_t)nr * (I / 32);
        const int e = slot == 0 ? a.E : a.uni[slot - 1];
        const unsigned char *blob = reinterpret_cast<const unsigned char *>(a.table[e]);
        unsigned char *dst = stg + (size_t)s * pl.sb;
        mbar_arrive_expect_tx(full + s, bytes_pk + bytes_sc);
        bulk_g2s_hint(dst, blob + pk_off + (size_t)(m0 + r0) * (I / 2), bytes_pk, full + s, pol);
        bulk_g2s_hint(dst + sc_in_stage, blob + sc_off + (size_t)(m0 + r0) * (I / 32), bytes_sc,
                      full + s, pol);
        issued = j + 1;
      }
      for (int j = (issued > NS ? issued - NS : 0); j < issued; ++j)
        mbar_wait(full + j % NS, (j / NS) & 1, a.status, kDetDnDrain);
    }
    return;
  }

  const int c0 = lane * CSZ;
  bool bad = false;
  for (int j = 0; j < nslot * nsub; ++j) {
    const int s = j % NS;
    const int slot = j / nsub, r0 = (j % nsub) * RS;
    const int nr = min(RS, nrows - r0);
    int n_tok, pos_base;
    if (slot == 0) {
      n_tok = T;
      pos_base = T * K;
    } else {
      const int e = a.uni[slot - 1];
      pos_base = a.off[e];
      n_tok = a.off[e + 1] - pos_base;
    }
    if (!bad) bad = *reinterpret_cast<volatile int *>(&s_abort) != 0;
    if (!bad) {
      bad = !mbar_wait(full + s, (j / NS) & 1, a.status, kDetDnFull);
      bad = __any_sync(0xffffffffu, bad);
      if (bad && lane == 0) s_abort = 1;
    }
    if (bad) continue;
    const unsigned char *sb = stg + (size_t)s * pl.sb;
    for (int i0 = 0; i0 < n_tok; i0 += kDnTokBatch) {
      const int nb = min(kDnTokBatch, n_tok - i0);
      // this lane's activation chunk for up to kDnTokBatch positions
      uint32_t av[kDnTokBatch][CSZ][16];
      float dv[kDnTokBatch][CSZ][2];
      int qv[kDnTokBatch][CSZ][2];
#pragma unroll
      for (int b = 0; b < kDnTokBatch; ++b) {
        const int pos = pos_base + (b < nb ? i0 + b : i0);
#pragma unroll
        for (int gi = 0; gi < CSZ; ++gi) {
          const int g = c0 + gi;
          if (b < nb && g < G) {
            const uint4 *src = reinterpret_cast<const uint4 *>(a.hq + (size_t)pos * I + 64 * g);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 v = __ldg(src + q);
              av[b][gi][4 * q + 0] = v.x;
              av[b][gi][4 * q + 1] = v.y;
              av[b][gi][4 * q + 2] = v.z;
              av[b][gi][4 * q + 3] = v.w;
            }
            dv[b][gi][0] = __ldg(a.hd + (size_t)pos * IB + 2 * g);
            dv[b][gi][1] = __ldg(a.hd + (size_t)pos * IB + 2 * g + 1);
            qv[b][gi][0] = __ldg(a.hqs + (size_t)pos * IB + 2 * g);
            qv[b][gi][1] = __ldg(a.hqs + (size_t)pos * IB + 2 * g + 1);
          } else {
#pragma unroll
            for (int q = 0; q < 16; ++q) av[b][gi][q] = 0u;
            dv[b][gi][0] = dv[b][gi][1] = 0.0f;
            qv[b][gi][0] = qv[b][gi][1] = 0;
          }
        }
      }
      for (int ml = warp; ml < nr; ml += 8) {
        const int m = r0 + ml;  // row of this CTA (stage row ml)
        const unsigned char *rowp = sb + (size_t)ml * (I / 2);
        const __half *scp = reinterpret_cast<const __half *>(sb + sc_in_stage + (size_t)ml * (I / 32));
        float acc[kDnTokBatch];
#pragma unroll
        for (int b = 0; b < kDnTokBatch; ++b) acc[b] = 0.0f;
#pragma unroll
        for (int gi = 0; gi < CSZ; ++gi) {
          const int g = c0 + gi;
          if (g < G) {
            const uint4 w0 = *reinterpret_cast<const uint4 *>(rowp + 32 * g);
            const uint4 w1 = *reinterpret_cast<const uint4 *>(rowp + 32 * g + 16);
            const uint32_t wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
            uint32_t lo[8], hi[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              lo[q] = wv[q] & 0x0F0F0F0Fu;
              hi[q] = (wv[q] >> 4) & 0x0F0F0F0Fu;
            }
            const float sc = __half2float(scp[g]);
#pragma unroll
            for (int b = 0; b < kDnTokBatch; ++b) {
              if (b < nb) {
                int s0 = -8 * qv[b][gi][0], s1 = -8 * qv[b][gi][1];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                  s0 = dp4a_us(lo[q], av[b][gi][q], s0);
                  s1 = dp4a_us(hi[q], av[b][gi][8 + q], s1);
                }
                const float fa = fmul((float)s0, dv[b][gi][0]);
                const float fb = ffma((float)s1, dv[b][gi][1], fa);
                acc[b] = ffma(sc, fb, acc[b]);
              }
            }
          }
        }
#pragma unroll
        for (int b = 0; b < kDnTokBatch; ++b)
          if (b < nb) red[(warp * T + b) * 33 + lane] = acc[b];
        __syncwarp();
        if (lane < nb) {
          const float *rr = red + (warp * T + lane) * 33;
          float tot = rr[0];
          for (int c = 1; c < nch; ++c) tot = fadd(tot, rr[c]);
          ysm[(size_t)(pos_base + i0 + lane) * a.rows_max + m] = tot;
        }
        __syncwarp();
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty + s);
  }
  named_sync(1, 256);
  if (*reinterpret_cast<volatile int *>(&s_abort)) return;
  for (int i = tid; i < T * nrows; i += 256) {
    const int t = i / nrows, m = i % nrows;
    float o = ysm[(size_t)(T * K + t) * a.rows_max + m];
    for (int s = 0; s < K; ++s) {
      const int p = a.pos[t * K + s];
      o = ffma(a.w[t * K + s], ysm[(size_t)p * a.rows_max + m], o);
    }
    a.out[(size_t)t * H + m0 + m] = o;
  }
  if (a.use_pdl) pdl_launch_dependents();
}

size_t down_smem_bytes(int H, int I, int k, int T, int rows_max, int rs, int nstage) {
  (void)H;
  return dn_plan(I, k, T, rows_max, rs, nstage).total;
}

int down_max_stages(int H, int I, int k, int T, int rows_max, int rs) {
  int ns = 6;
  while (ns >= 2 && down_smem_bytes(H, I, k, T, rows_max, rs, ns) > (size_t)kMaxSmem) --ns;
  return ns;
}

template <int CSZ>
static cudaError_t launch_dn(const DownArgs &a, int grid, size_t smem, cudaStream_t s) {
  cudaError_t err = cudaFuncSetAttribute(k_down_decode<CSZ>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(288);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.use_pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k_down_decode<CSZ>, a);
}

cudaError_t launch_down_decode(const DownArgs &a, int grid, size_t smem, cudaStream_t s) {
  const int csz = (a.I / 64 + 31) / 32;
  switch (csz) {
    case 1: return launch_dn<1>(a, grid, smem, s);
    case 2: return launch_dn<2>(a, grid, smem, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace moe
