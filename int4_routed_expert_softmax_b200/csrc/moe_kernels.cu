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

#include "moe_route.cuh"

namespace moe {

// =====================================================================
// Q8_0 quantisation: one warp per 32-block (lane = element).
// =====================================================================
__global__ void __launch_bounds__(256) k_quant(QuantArgs a) {
  prof_start(a.prof, 0);
  const int lane = threadIdx.x & 31;
  const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t b = gw; b < a.nblk; b += nw) {
    const float v = a.x[b * 32 + lane];
    const float d = fdiv(warp_max(fabsf(v)), 127.0f);
    const int c = q8_code(v, d);
    a.q[b * 32 + lane] = (int8_t)c;
    if (lane == 0) a.d[b] = d;
  }
}

// =====================================================================
// Host-buffer entry: zero the workspace's control words and copy x from
// device-accessible pinned host memory into the workspace (one pass of 16-byte
// loads across the link), in place of a memset and a separate copy.
// =====================================================================
__global__ void __launch_bounds__(256) k_stage_in(const float4 *x_host, float4 *x_dev, int64_t n4, uint4 *ctrl,
                                                  int ctrl16) {
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < ctrl16; i += blockDim.x) ctrl[i] = make_uint4(0u, 0u, 0u, 0u);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x)
    x_dev[i] = x_host[i];
}

cudaError_t launch_stage_in(const float *x_host, float *x_dev, int64_t n, void *ctrl, size_t ctrl_bytes,
                            cudaStream_t s) {
  const int64_t n4 = n / 4;
  int64_t blocks = (n4 + 255) / 256;
  if (blocks < 1) blocks = 1;
  if (blocks > 148) blocks = 148;
  k_stage_in<<<(unsigned)blocks, 256, 0, s>>>(reinterpret_cast<const float4 *>(x_host), reinterpret_cast<float4 *>(x_dev),
                                              n4, static_cast<uint4 *>(ctrl), (int)(ctrl_bytes / 16));
  return cudaGetLastError();
}

cudaError_t func_attributes(cudaFuncAttributes *fa) { return cudaFuncGetAttributes(fa, k_quant); }

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
// Stable counting sort of the P = T*k (token, slot) pairs by expert, one CTA.
// Writes cnt, off, uni (+ shared slot E), n_uni, perm, pos and pair_tok
// (routed positions, then T shared positions).
// Each warp owns a contiguous segment of pairs.  Pass 1 counts per (warp,
// expert); an exclusive scan over the warps (per expert) and over the experts
// gives every warp its start inside every expert's range; pass 2 places the
// pairs, lanes with equal experts ranked by lane -- pair order is kept inside
// every expert, with no block-wide barrier in either pass.
// s_work: 3E + 64 + (blockDim.x / 32) * E ints of shared memory.
// =====================================================================
__device__ void bucket_block(int E, int k, int T, const int32_t *idx, int *s_work, int32_t *cnt,
                             int32_t *off, int32_t *uni, int32_t *n_uni, int32_t *perm,
                             int32_t *pos, int32_t *pair_tok) {
  const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
  const int nw = nt >> 5;
  const int P = T * k;
  int *s_cnt = s_work;            // [E]
  int *s_off = s_work + E;        // [E]  (exclusive)
  int *s_flag = s_work + 2 * E;   // [E]  union flags, then union ranks
  int *scratch = s_work + 3 * E;  // [64]
  int *s_wc = scratch + 64;       // [nw][E]: per-warp counts, then per-warp cursors
  for (int i = tid; i < nw * E; i += nt) s_wc[i] = 0;
  __syncthreads();
  const int seg = ((P + nw - 1) / nw + 31) & ~31;
  const int p0 = min(P, warp * seg), p1 = min(P, p0 + seg);
  int *wc = s_wc + (size_t)warp * E;
  const unsigned lt = (1u << lane) - 1u;
  for (int c = p0; c < p1; c += 32) {
    const int p = c + lane;
    const bool has = p < p1;
    const int e = has ? idx[p] : -1 - lane;  // distinct dummies never match
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (has && lane == __ffs(peers) - 1) wc[e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  for (int e = tid; e < E; e += nt) {
    int run = 0;
    for (int w = 0; w < nw; ++w) {
      const int c = s_wc[(size_t)w * E + e];
      s_wc[(size_t)w * E + e] = run;
      run += c;
    }
    s_cnt[e] = run;
  }
  __syncthreads();
  block_exclusive_scan(s_cnt, s_off, E, scratch);
  for (int e = tid; e < E; e += nt) {
    cnt[e] = s_cnt[e];
    off[e] = s_off[e];
    s_flag[e] = (s_cnt[e] > 0) ? 1 : 0;  // flags for the union scan
  }
  if (tid == 0) off[E] = P;
  __syncthreads();
  const int nu = block_exclusive_scan(s_flag, s_flag, E, scratch);
  for (int e = tid; e < E; e += nt)
    if (s_cnt[e] > 0) uni[s_flag[e]] = e;
  if (tid == 0) {
    *n_uni = nu;
    uni[nu] = E;  // the shared expert follows the union
  }
  for (int c = p0; c < p1; c += 32) {
    const int p = c + lane;
    const bool has = p < p1;
    const int e = has ? idx[p] : -1 - lane;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (has) {
      const int q = s_off[e] + wc[e] + __popc(peers & lt);
      perm[q] = p;
      if (pos) pos[p] = q;
      if (pair_tok) pair_tok[q] = p / k;
    }
    __syncwarp();
    if (has && lane == __ffs(peers) - 1) wc[e] += __popc(peers);
    __syncwarp();
  }
  if (pair_tok)
    for (int t = tid; t < T; t += nt) pair_tok[P + t] = t;
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

  // the experts kernel that follows may be scheduled now; it waits for this
  // grid's completion (griddepcontrol.wait) before it reads anything
  pdl_launch_dependents();
  prof_start(a.prof, 0);
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
  __syncthreads();
  const int HB = H / 32;
  int phase = 0;
  for (int t0 = 0; t0 < a.T; t0 += a.tt, ++phase) {
    const int nt = min(a.tt, a.T - t0);
    if (tid == 0 && t0 > 0) issue(t0);
    const bool ok = __syncthreads_and(mbar_wait(bar, phase & 1, a.status, kDetRouteBar, a.wait_limit));
    if (!ok) {
      // the copies of this tile may still be in flight: they land in this
      // CTA's shared memory before it exits
      if (tid == 0) mbar_drain(bar, phase & 1, a.status, kDetRouteDrain);
      return;
    }
    const int npair = ne * nt;
    for (int p = warp; p < npair; p += 4) {
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
    if (a.do_quant) {
      // Q8_0 of this tile's x from the staged copy: block b of the tile goes
      // to CTA b mod grid, on the warps after the logit work
      const int nblk = nt * HB;
      int q = (warp - npair % 4 + 4) % 4;  // spread: idle warps first
      for (int b = blockIdx.x + (int)gridDim.x * q; b < nblk; b += (int)gridDim.x * 4) {
        const float v = sX[(size_t)b * 32 + lane];
        const float d = fdiv(warp_max(fabsf(v)), 127.0f);
        const size_t gb = (size_t)t0 * HB + b;
        a.xq[gb * 32 + lane] = (int8_t)q8_code(v, d);
        if (lane == 0) a.xd[gb] = d;
      }
    }
    __syncthreads();
  }
  if (a.done == nullptr) {
    prof_end(a.prof, 0);
    return;
  }

  // ---- the last CTA to arrive does top-k and the batch union.  The ticket is
  // an acquire-release add at GPU scope: after the barrier it publishes this
  // CTA's logits and codes, and the last CTA's add sees everyone's.
  __syncthreads();
  if (tid == 0) {
    unsigned int old;
    asm volatile("atom.acq_rel.gpu.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(a.done) : "memory");
    *s_flag = (old == gridDim.x - 1) ? 1 : 0;
  }
  __syncthreads();
  if (!*s_flag) return;
  int *s_idx = reinterpret_cast<int *>(sW);               // [T*k]
  int *s_work = s_idx + kDecodeTMax * kMaxK;              // bucket scratch
  uint32_t *s_tk = reinterpret_cast<uint32_t *>(s_work + 3 * MOE_MAX_E + 64);  // [4][128]
  for (int t = warp; t < a.T; t += 4) {
    int e_sel;
    float l_sel;
    warp_topk(a.logits + (size_t)t * a.E, a.E, a.k, lane, e_sel, l_sel, s_tk + warp * 128);
    warp_softmax_store(t, a.k, lane, e_sel, l_sel, a.idx, a.w, a.route_counts, s_idx);
  }
  __syncthreads();
  if (a.do_bucket && a.T * a.k <= 32) bucket_small_counts(a.E, a.T * a.k, s_idx, a.cnt, a.off, warp, 4);
  if (warp != 0) return;
  if (a.do_bucket) {
    if (a.T * a.k <= 32)
      bucket_small(a.E, a.k, a.T, s_idx, a.cnt, a.off, a.uni, a.n_uni, a.perm, a.pos, a.pair_tok);
    else
      bucket_warp(a.E, a.k, a.T, s_idx, s_work, a.cnt, a.off, a.uni, a.n_uni, a.perm, a.pos,
                  a.pair_tok);
    if (a.own != nullptr) {
      // the union slots this call computes, in slot order: the shared expert
      // (slot 0) if with_shared, then the union's experts in [e_lo, e_hi)
      __syncwarp();
      const int nu = *a.n_uni;
      int base = 0;
      for (int s0 = 0; s0 <= nu; s0 += 32) {
        const int sl = s0 + lane;
        bool f = false;
        if (sl <= nu) {
          if (sl == 0) {
            f = a.with_shared != 0;
          } else {
            const int e = a.uni[sl - 1];
            f = e >= a.e_lo && e < a.e_hi;
          }
        }
        const unsigned m = __ballot_sync(0xffffffffu, f);
        if (f) a.own[base + __popc(m & ((1u << lane) - 1u))] = sl;
        base += __popc(m);
      }
      if (lane == 0) *a.n_own = base;
    }
    if (a.mail != nullptr) {
      // post the union to the host's mailbox (mapped pinned memory): the
      // entries and the size first, then the sequence number the host waits on
      __syncwarp();
      const int nu = *a.n_uni;
      for (int i = lane; i < nu; i += 32) a.mail[kMailUni + i] = a.uni[i];
      if (lane == 0) a.mail[kMailN] = nu;
      __threadfence_system();
      __syncwarp();
      if (lane == 0) *reinterpret_cast<volatile int32_t *>(a.mail + kMailSeq) = a.mail_seq;
    }
  }
  if (lane == 0) *a.done = 0u;
  prof_end(a.prof, 0);
}

size_t route_smem_bytes(int H, int epc, int tt) {
  size_t fl = (size_t)(epc + tt) * H * 4;
  size_t need_tail = (size_t)(kDecodeTMax * kMaxK + 3 * MOE_MAX_E + 64 + 4 * 128) * 4;
  return 128 + (fl > need_tail ? fl : need_tail);
}

cudaError_t launch_route_decode(const RouteArgs &a, cudaStream_t s) {
  const size_t smem = route_smem_bytes(a.H, a.epc, a.tt);
  static int smem_set[64] = {0};
  cudaError_t err = ensure_smem(k_route_decode, smem, smem_set);
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
  __shared__ uint32_t s_tk[8][128];
  const int lane = threadIdx.x & 31;
  const int t = (int)(((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  if (t >= T) return;
  int e_sel;
  float l_sel;
  warp_topk(logits + (size_t)t * E, E, k, lane, e_sel, l_sel, s_tk[threadIdx.x >> 5]);
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
  const size_t smem = (size_t)(3 * a.E + 64 + 32 * a.E) * 4;
  static int smem_set[64] = {0};
  cudaError_t err = ensure_smem(k_bucket, smem, smem_set);
  if (err != cudaSuccess) return err;
  k_bucket<<<1, 1024, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace moe
