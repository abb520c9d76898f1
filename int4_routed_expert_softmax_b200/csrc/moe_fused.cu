// moe_fused.cu -- the whole routed-expert MoE layer for one token (decode) in
// one cooperative kernel: Q8_0 of x, router logits, top-k + softmax, the union,
// gate/up + SwiGLU + Q8_0 of h, down, and the weighted combine with the shared
// expert.
//
// The layer's parts, by page and section: the router over 256 experts and the
// shared expert (tantan.ink, 它的核心判断), the batch union read once
// (tantan.ink, 几个关键工程动作), int4 gs64 weights (tantan.ink, 我看到的几个坑)
// against Q8_0-style activations (alphamatch.ai, 優化整數核心).
//
// Why one kernel.  At one token the expert bytes -- (k + 1) blobs of 20 MB at
// the GLM shape -- are the whole cost, and a chain of kernels spends a large
// part of the layer between them: a serial routing tail on one CTA while every
// other SM idles, then the down projection's ramp after the gate/up kernel's
// tail.  Here every CTA (one per SM, all resident: cooperative launch) takes
// part in every phase and the weight stream never stops:
//
//   1. routing: each CTA stages x and its 1-2 router rows (TMA bulk copies),
//      writes their logits in the router's fixed order and quantises x for its
//      own use; its producer warp meanwhile pulls a slice of the shared
//      expert's blob into L2 (the shared expert does not depend on routing);
//   2. a grid-wide arrival count (release/acquire, bounded wait); then every
//      CTA computes the same top-k, softmax and union from the logits in L2
//      (one warp, a few hundred instructions) -- no single-CTA tail;
//   3. one ring of TMA stages streams, per CTA, its gate/up units -- (union
//      slot, 32 rows of I), dealt round-robin so that the slots complete in
//      order -- then its down rows of every slot; each unit's SwiGLU and Q8_0
//      epilogue publishes the unit (release add on the slot's counter), and a
//      down stage waits (acquire, bounded) until its slot's h is complete;
//   4. the combine of the CTA's output rows: y_shared, then fmaf(w_s, y_s) in
//      slot order -- no atomics, the same order as the three-kernel path.
//
// Every per-row dot, every epilogue and the combine are the three-kernel decode
// path's own code and order (moe_decode.cuh), so the two paths agree bit for
// bit.  Every wait is bounded; a wait that runs out records MOE_ERR_TIMEOUT
// and a detail code, the roles leave their loops, and the producer drains the
// copies it issued before the CTA exits.
#include "moe_decode.cuh"
#include "moe_route.cuh"

namespace moe {

namespace {

constexpr int kFuR = 8;                  // gate/up rows per matrix per stage
constexpr int kFuNW = 8;                 // consumer warps (warp 8 = producer)
constexpr int kFuSPU = 32 / kFuR;        // stages per 32-row unit
constexpr int kFuRPW = 2 * kFuR / kFuNW; // rows per warp per gate/up stage
constexpr int kFuPWR = kFuSPU * kFuRPW;  // rows per warp per unit
constexpr int kFuNCT = kFuNW * 32;       // consumer threads
constexpr int kFuWarps = kFuNW + 2;      // + the producer warp and the epilogue warp
constexpr int kFuTMax = kDecodeTMax;     // tokens of one launch
// the red buffer (kFuNW x >= kFuPWR rows of 33 words) doubles as the batch
// record's bucketing scratch (2 E words)
static_assert(kFuNW * kFuPWR * 33 >= 2 * MOE_MAX_E, "bucketing scratch");
constexpr int kFuThreads = kFuWarps * 32;
// named barriers (0 is __syncthreads): the consumers' end, and per unit parity
// the hand-off of the g and u sums to the epilogue warp and the buffer's return
constexpr int kBarEnd = 1, kBarGuFull = 2, kBarGuFree = 4;

struct FuPlan {
  size_t bars, misc, tab, red, gu, ysm, xd, qs, xq, stg, total;
  uint32_t sb;    // bytes of one ring stage
  int chp;        // bytes of one lane's activation chunk
  int rw;         // red rows per warp
};

__host__ __device__ inline uint32_t fu_gu_stage(int H) { return (uint32_t)(2 * kFuR) * (uint32_t)(H / 2 + H / 32); }
__host__ __device__ inline uint32_t fu_dn_row(int I) { return (uint32_t)(I / 2 + I / 32); }
// A down stage: rs rows of packed weights, their scales, then the slot's h
// (Q8_0 codes [I], block scales [I/32] fp32, code sums [I/32] int32).
__host__ __device__ inline uint32_t fu_dn_h(int I) { return (uint32_t)(I + 2 * (I / 32) * 4); }
__host__ __device__ inline uint32_t fu_dn_stage(int I, int rs) { return (uint32_t)rs * fu_dn_row(I) + fu_dn_h(I); }

__host__ __device__ inline FuPlan fu_plan(int H, int I, int E, int k, int rows_max, int rs, int ns) {
  FuPlan p;
  const int csz = (H / 64 + 31) / 32;
  p.chp = csz * 64;
  const uint32_t sg = fu_gu_stage(H), sd = (uint32_t)al128d(fu_dn_stage(I, rs));
  p.sb = (uint32_t)al128d(sg > sd ? sg : sd);
  p.rw = kFuPWR > (rs + kFuNW - 1) / kFuNW ? kFuPWR : (rs + kFuNW - 1) / kFuNW;
  // the ring first, on the allocation's 1024-byte boundary
  size_t o = 0;
  p.stg = o;
  o += (size_t)ns * p.sb;
  p.bars = o;
  o += al128d((size_t)16 * (2 * ns + 2));
  p.misc = o;
  o += al128d((size_t)4 * (8 + kFuTMax + 6 * kFuTMax * (k + 1)) + (size_t)8 * kFuTMax * (k + 1));
  p.red = o;
  o += al128d((size_t)kFuNW * p.rw * 33 * 4);
  p.gu = o;
  o += al128d((size_t)2 * 64 * 4);
  p.ysm = o;
  o += al128d((size_t)(k + 1) * rows_max * 4);
  p.xd = o;
  o += al128d((size_t)(H / 32) * 4);
  p.qs = o;
  o += al128d((size_t)(H / 32) * 4);
  p.xq = o;
  o += al128d((size_t)32 * p.chp);
  p.total = o;
  return p;
}

// Plan of the one-token kernel (k_decode_fused1): the expert table in shared
// memory and one token's tables.
__host__ __device__ inline FuPlan fu1_plan(int H, int I, int E, int k, int rows_max, int rs, int ns) {
  FuPlan p;
  const int csz = (H / 64 + 31) / 32;
  p.chp = csz * 64;
  const uint32_t sg = fu_gu_stage(H), sd = (uint32_t)al128d(fu_dn_stage(I, rs));
  p.sb = (uint32_t)al128d(sg > sd ? sg : sd);
  p.rw = kFuPWR > (rs + kFuNW - 1) / kFuNW ? kFuPWR : (rs + kFuNW - 1) / kFuNW;
  size_t o = 0;
  p.bars = o;
  o += al128d((size_t)16 * (2 * ns + 2));
  p.misc = o;
  o += al128d((size_t)4 * (8 + 6 * (kMaxK + 1)));
  p.tab = o;
  o += al128d((size_t)8 * (E + 1));
  p.red = o;
  o += al128d((size_t)kFuNW * p.rw * 33 * 4);
  p.gu = o;
  o += al128d((size_t)2 * 64 * 4);
  p.ysm = o;
  o += al128d((size_t)(k + 1) * rows_max * 4);
  p.xd = o;
  o += al128d((size_t)(H / 32) * 4);
  p.qs = o;
  o += al128d((size_t)(H / 32) * 4);
  p.xq = o;
  o += al128d((size_t)32 * p.chp);
  p.stg = o;
  o += (size_t)ns * p.sb;
  p.total = o;
  return p;
}

__device__ __forceinline__ void red_release_add(int32_t *p, int32_t v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void red_release_add_u32(unsigned int *p, unsigned int v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int32_t ld_acquire(const int32_t *p) {
  int32_t v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ unsigned int ld_acquire_u32(const unsigned int *p) {
  unsigned int v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long *p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_u64(unsigned long long *p, unsigned long long v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ void st_relaxed_u64(unsigned long long *p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// The call's control words start at zero without a memset launched before
// the kernel.  CTA 0 zeroes the first `nctl` of them (and the status word on a
// call's first launch) as it starts, then publishes the call's sequence number
// in the ready word; every other CTA waits for that number before it arrives
// at the grid barrier, its first use of a control word.  (A status that one of
// them sets before CTA 0's zeroing can be lost, but such a CTA never arrives,
// so CTA 0's own barrier wait runs out and reports.)  CTA 0 puts the ready word
// back to 0 once every CTA has arrived (so has seen it), or when it leaves
// before the barrier, so that a replay of the same launch (a CUDA graph: the
// same sequence number) waits for its own zeroing again.
// ctrl_zero: every thread of CTA 0, after the barrier init.
__device__ __forceinline__ void ctrl_zero(const FusedArgs &a, int nctl) {
  const int tid = threadIdx.x;
  for (int i = tid; i < nctl; i += blockDim.x)
    if (i != kCtrlReady && i != kCtrlReady + 1) a.ctrl[i] = 0;
  if (a.fresh && tid < 4) a.status[tid] = 0;
  __syncthreads();
  if (tid == 0) st_release_u64(a.ready, a.seq);  // after the CTA's zeroing (bar.sync, then release)
}

// Thread 0 of any CTA before its arrival: false if the wait ran out.
__device__ __forceinline__ bool ctrl_ready(const FusedArgs &a, long long lim) {
  if (blockIdx.x == 0 || ld_acquire_u64(a.ready) == a.seq) return true;
  const long long t0 = clock64();
  while (ld_acquire_u64(a.ready) != a.seq) {
    if (clock64() - t0 > lim) {
      set_status(a.status, MOE_ERR_TIMEOUT, kDetFuReady);
      return false;
    }
    __nanosleep(32);
  }
  return true;
}

// CTA 0, thread 0: the ready word back to 0.
__device__ __forceinline__ void ctrl_close(const FusedArgs &a) {
  if (blockIdx.x == 0 && threadIdx.x == 0) st_relaxed_u64(a.ready, 0ull);
}

// Waits (bounded by `limit` SM clocks) until the counter at p reaches `target`.
__device__ __forceinline__ bool wait_count(const int32_t *p, int32_t target, long long limit) {
  if (ld_acquire(p) >= target) return true;
  const long long t0 = clock64();
  while (ld_acquire(p) < target) {
    if (clock64() - t0 > limit) return false;
    __nanosleep(64);
  }
  return true;
}

}  // namespace

// FMT: the expert weight format, kFmtInt4 (int4 gs64, fp16 group scales) or
// kFmtMxfp4 (E2M1 codes, E8M0 exponent per 32-block); both hold K/2 code
// bytes and K/32 scale bytes per row, so the stream is the same.
// A batch of 2 <= a.ntok <= kFuTMax tokens (one token: k_decode_fused1).
template <int CSZG, int CSZD, int FMT>
__global__ void __launch_bounds__(kFuThreads, 1) k_decode_fused(FusedArgs a) {
  constexpr int R = kFuR, NW = kFuNW, SPU = kFuSPU, RPW = kFuRPW, PWR = kFuPWR, NCT = kFuNCT;
  constexpr int PROD = NW, EPI = NW + 1;  // warp roles after routing
  extern __shared__ __align__(1024) unsigned char smem[];
  const int H = a.H, I = a.I, E = a.E, K = a.k, NS = a.nstage;
  const int GG = H / 64, HB = H / 32, GD = I / 64, IB = I / 32;
  const int nchg = (GG + CSZG - 1) / CSZG, nchd = (GD + CSZD - 1) / CSZD;
  const FuPlan pl = fu_plan(H, I, E, K, a.rows_max, a.rs, NS);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + pl.bars);
  uint64_t *empty = full + NS;
  uint64_t *rbar = empty + NS;
  int *misc = reinterpret_cast<int *>(smem + pl.misc);
  volatile int *s_abort = misc;
  // per token t of this launch (stride SW = k + 1, or k):
  const int NT = a.ntok;
  const int SW = K + 1;
  int *t_nsl = misc + 8;                           // [NT] slots computed
  int *t_uni = t_nsl + kFuTMax;                    // [NT][k + 1] slot -> expert (slot 0 = shared)
  int *t_ppos = t_uni + kFuTMax * SW;              // [NT][k + 1] pair s -> slot - 1
  int *t_idx = t_ppos + kFuTMax * SW;              // [NT * k] selected experts in pair order
  float *t_w = reinterpret_cast<float *>(t_idx + kFuTMax * SW);  // [NT * k] softmax weights
  int *t_own = t_idx + 2 * kFuTMax * SW;           // [NT][k + 1] the slots computed, in order
  int *t_bpos = t_own + kFuTMax * SW;              // [NT][k + 1] slot -> row of hq / hd / hqs
  const unsigned char **t_blob =                   // [NT][k + 1] slot -> expert blob (8-byte aligned)
      reinterpret_cast<const unsigned char **>(misc + ((8 + kFuTMax + 6 * kFuTMax * SW + 1) & ~1));
  float *red = reinterpret_cast<float *>(smem + pl.red);
  float *gu = reinterpret_cast<float *>(smem + pl.gu);
  float *ysm = reinterpret_cast<float *>(smem + pl.ysm);
  float *xd_s = reinterpret_cast<float *>(smem + pl.xd);
  int *qs_s = reinterpret_cast<int *>(smem + pl.qs);
  unsigned char *xq_s = smem + pl.xq;
  unsigned char *stg = smem + pl.stg;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = (int)gridDim.x;
  const long long lim = a.wait_limit;
  if (tid == 0) {
    *s_abort = 0;
    for (int s = 0; s < NS; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, NW);
    }
    mbar_init(rbar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  prof_start(a.prof, 0);

  // ---------------------------------------------------------------- routing
  // this CTA's router rows [e0, e1) and the tokens' x rows, staged in the
  // (still idle) ring: the x rows in chunks of as many tokens as the ring
  // holds after the router rows (every token at once for small batches)
  const int e0 = (int)((long long)blockIdx.x * E / G), e1 = (int)((long long)(blockIdx.x + 1) * E / G);
  const int nr = e1 - e0;
  float *rw = reinterpret_cast<float *>(stg);
  float *rx = rw + (size_t)nr * H;
  const int xcap = (int)(((size_t)NS * pl.sb - (size_t)nr * H * 4) / ((size_t)H * 4));  // >= 1 (fused_plan)
  if (tid == 0) {
    const int nx = NT < xcap ? NT : xcap;
    mbar_arrive_expect_tx(rbar, (uint32_t)(nr + nx) * (uint32_t)H * 4u);
    if (nr > 0) bulk_g2s(rw, a.Wr + (size_t)e0 * H, (uint32_t)nr * (uint32_t)H * 4u, rbar);
    bulk_g2s(rx, a.x, (uint32_t)nx * (uint32_t)H * 4u, rbar);
  }
  if (blockIdx.x == 0) ctrl_zero(a, NT * kCtrlWords);
  const int nlp = nr * NT;  // (row, token) pairs of logits
  for (int c0 = 0, ph = 0; c0 < NT; c0 += xcap, ph ^= 1) {
    const int nx = NT - c0 < xcap ? NT - c0 : xcap;
    const bool ok = mbar_wait(rbar, (uint32_t)ph, a.status, kDetFuRoute, lim);
    if (!__syncthreads_and(ok)) {
      if (tid == 0) mbar_drain(rbar, (uint32_t)ph, a.status, kDetFuRouteDrain);  // the copies land before exit
      ctrl_close(a);
      return;
    }
    if (c0 == 0 && warp == PROD && lane == 0 && a.with_shared) {
      // a slice of the shared expert's blob into L2 while the grid routes
      // (after this CTA's routing data, which it must not delay)
      const unsigned char *sh = static_cast<const unsigned char *>(a.table[E]);
      const size_t bytes = 2 * ((size_t)I * (H / 2) + (size_t)I * (H / 64) * 2) +
                           ((size_t)H * (I / 2) + (size_t)H * (I / 64) * 2);
      const size_t slice = ((bytes + G - 1) / G + 15) / 16 * 16;
      const size_t b0 = slice * blockIdx.x;
      if ((reinterpret_cast<uintptr_t>(sh) & 15u) == 0 && b0 < bytes) {
        const size_t n = bytes - b0 < slice ? bytes - b0 : slice;
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(sh + b0), "r"((uint32_t)n) : "memory");
      }
    }
    // logits of this CTA's rows for the chunk's tokens, the router's fixed
    // order: lane l sums h = l, l + 32, ... with fmaf, then an xor tree 16,
    // 8, 4, 2, 1 (the producer and epilogue warps take rows too)
    for (int p = warp; p < nr * nx; p += kFuWarps) {
      const int r = p / nx, tc = p - r * nx;
      const float *wv = rw + (size_t)r * H;
      const float *xv = rx + (size_t)tc * H;
      float acc = 0.0f;
#pragma unroll 8
      for (int i = lane; i < H; i += 32) acc = ffma(xv[i], wv[i], acc);
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) acc = fadd(acc, __shfl_xor_sync(0xffffffffu, acc, off));
      if (lane == 0) a.logits[(size_t)(c0 + tc) * E + e0 + r] = acc;
    }
    if (c0 + xcap < NT) {
      // the next chunk of x rows, once every warp is done with this one
      __syncthreads();
      if (tid == 0) {
        const int nn = NT - c0 - xcap < xcap ? NT - c0 - xcap : xcap;
        mbar_arrive_expect_tx(rbar, (uint32_t)nn * (uint32_t)H * 4u);
        bulk_g2s(rx, a.x + (size_t)(c0 + xcap) * H, (uint32_t)nn * (uint32_t)H * 4u, rbar);
      }
    }
  }
  // Q8_0 of x: this CTA's share of the batch's blocks, into the workspace
  // (every CTA reads the codes back after the grid barrier); one warp per block
  {
    const int NB = NT * HB;
    const int c_last = ((NT - 1) / xcap) * xcap;  // first token of the staged chunk
    const int b0 = (int)((long long)blockIdx.x * NB / G), b1 = (int)((long long)(blockIdx.x + 1) * NB / G);
    const int qw = (warp - nlp % kFuWarps + kFuWarps) % kFuWarps;  // the warps after the logit rows first
    for (int b = b0 + qw; b < b1; b += kFuWarps) {
      const int t = b / HB, bb = b - t * HB;
      // the last chunk's x rows are still staged; earlier ones come from L2
      const float v = t >= c_last ? rx[(size_t)(t - c_last) * H + bb * 32 + lane]
                                  : __ldg(a.x + (size_t)t * H + bb * 32 + lane);
      // the maximum of non-negative floats is the maximum of their bit patterns
      const float d = fdiv(__uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(v)))), 127.0f);
      a.xq[(size_t)t * H + bb * 32 + lane] = (int8_t)q8_code(v, d);
      if (lane == 0) a.xd[(size_t)t * HB + bb] = d;
    }
  }
  // grid-wide: every CTA's logits and codes are written before any CTA reads
  // them (the barrier orders this CTA's writes before thread 0's release)
  __syncthreads();
  if (tid == 0) {
    if (!ctrl_ready(a, lim)) {
      *s_abort = 1;
    } else {
      red_release_add_u32(a.arrivals, 1u);
      if (ld_acquire_u32(a.arrivals) < (unsigned)G) {
        const long long t0 = clock64();
        while (ld_acquire_u32(a.arrivals) < (unsigned)G) {
          if (clock64() - t0 > lim) {
            set_status(a.status, MOE_ERR_TIMEOUT, kDetFuGrid);
            *s_abort = 1;
            break;
          }
          __nanosleep(32);
        }
      }
    }
    ctrl_close(a);  // every CTA has arrived, so has seen the ready word (or the wait ran out)
  }
  __syncthreads();
  if (*s_abort) return;  // nothing in flight: the staging copies have landed

  // the Q8_0 codes of a token (every CTA's share, from L2) into this CTA's
  // activation chunks, with the block scales and code sums; threads
  // [first, first + nthr)
  auto load_token = [&](int t, int first, int nthr) {
    const int8_t *xq_t = a.xq + (size_t)t * H;
    const float *xd_t = a.xd + (size_t)t * HB;
    for (int b = tid - first; b < HB; b += nthr) {
      const uint4 *src = reinterpret_cast<const uint4 *>(xq_t + (size_t)b * 32);
      const uint4 q0 = __ldcg(src), q1 = __ldcg(src + 1);
      int sum = 0;
      sum = __dp4a((int)q0.x, 0x01010101, sum);
      sum = __dp4a((int)q0.y, 0x01010101, sum);
      sum = __dp4a((int)q0.z, 0x01010101, sum);
      sum = __dp4a((int)q0.w, 0x01010101, sum);
      sum = __dp4a((int)q1.x, 0x01010101, sum);
      sum = __dp4a((int)q1.y, 0x01010101, sum);
      sum = __dp4a((int)q1.z, 0x01010101, sum);
      sum = __dp4a((int)q1.w, 0x01010101, sum);
      const int h = b * 32, g = h >> 6, c = g / CSZG;
      uint4 *dst = reinterpret_cast<uint4 *>(xq_s + (size_t)c * pl.chp + (size_t)(g - c * CSZG) * 64 + (h & 63));
      dst[0] = q0;
      dst[1] = q1;
      xd_s[b] = __ldcg(xd_t + b);
      qs_s[b] = sum;
    }
  };
  if (warp != 0) load_token(0, 32, kFuThreads - 32);

  // top-k and softmax of every token (one warp per token) -- the same in
  // every CTA; CTA 0 counts the routes
  for (int t = warp; t < NT; t += kFuWarps) {
    int e_sel;
    float l_sel;
    warp_topk(a.logits + (size_t)t * E, E, K, lane, e_sel, l_sel, reinterpret_cast<uint32_t *>(red) + warp * 128);
    warp_softmax_store(t, K, lane, e_sel, l_sel, t_idx, t_w, blockIdx.x == 0 ? a.route_counts : nullptr, nullptr);
  }
  __syncthreads();  // every token's top-k before the tables
  // each token's union (its k experts in ascending order: pair s at slot
  // 1 + rank(e_s), the shared expert at slot 0), the rows its h codes take in
  // the batch's pair order (the counting sort of the T k pairs by expert), and
  // the slots this call computes (expert parallelism: the shared expert on one
  // rank, the routed experts in [e_lo, e_hi); by default all of them)
  for (int t = warp; t < NT; t += kFuWarps) {
    int *su = t_uni + t * SW, *sp = t_ppos + t * SW, *so = t_own + t * SW, *sbp = t_bpos + t * SW;
    const int *si = t_idx + t * K;
    if (lane < K) {
      const int e = si[lane], me = t * K + lane;
      int rank = 0;
      for (int q = 0; q < K; ++q) rank += si[q] < e ? 1 : 0;
      int bpos = 0;
      for (int q = 0; q < NT * K; ++q) {
        const int eq = t_idx[q];
        bpos += (eq < e || (eq == e && q < me)) ? 1 : 0;
      }
      su[1 + rank] = e;
      sp[lane] = rank;
      sbp[1 + rank] = bpos;
      t_blob[t * SW + 1 + rank] = static_cast<const unsigned char *>(a.table[e]);
    }
    if (lane == 0) {
      su[0] = E;
      sbp[0] = NT * K + t;
      t_blob[t * SW] = static_cast<const unsigned char *>(a.table[E]);
    }
    __syncwarp();
    if (lane == 0) {
      int n = 0;
      if (a.with_shared) so[n++] = 0;
      for (int i = 1; i <= K; ++i)
        if (su[i] >= a.e_lo && su[i] < a.e_hi) so[n++] = i;
      t_nsl[t] = n;
    }
  }
  __syncthreads();
  prof_end(a.prof, 0);
  prof_start(a.prof, 1);

  const int rbs = I / 32;     // 32-row units per expert
  // token t's units (slot, 32-row block) are dealt round-robin from CTA r_t,
  // r_t = the units of the tokens before it, mod G, so the CTAs stay balanced
  // over the launch; this CTA's first unit of token t is u0, then u0 + G, ...
  auto units_of = [&](int t, int r, int &u0) -> int {
    const int nu = t_nsl[t] * rbs;
    u0 = (int)blockIdx.x - r;
    if (u0 < 0) u0 += G;
    return u0 < nu ? (nu - 1 - u0) / G + 1 : 0;
  };
  int units_all = 0;  // this CTA's units over the launch
  {
    int r = 0;
    for (int t = 0; t < NT; ++t) {
      int u0;
      units_all += units_of(t, r, u0);
      r = (r + t_nsl[t] * rbs) % G;
    }
  }
  const int nrg = H / a.rg;
  const int m0 = (int)((long long)blockIdx.x * nrg / G) * a.rg;
  const int m1 = (int)((long long)(blockIdx.x + 1) * nrg / G) * a.rg;
  const int nrows = m1 - m0;
  const int RS = a.rs;
  const int nsub = (nrows + RS - 1) / RS;
  const size_t mg = (size_t)I * H / 2 + (size_t)I * H / 32;  // bytes of the gate (= up) matrix

  // every blob this grid reads must be 16-byte aligned (TMA bulk copies)
  {
    bool bad = false;
    for (int i = tid; i < NT * SW; i += kFuThreads) {
      const int t = i / SW, sl = i % SW;
      if (sl < t_nsl[t]) bad |= (reinterpret_cast<uintptr_t>(t_blob[t * SW + t_own[t * SW + sl]]) & 15u) != 0;
    }
    if (__syncthreads_or(bad)) {
      if (tid == 0) set_status(a.status, MOE_ERR_DEVICE, kDetFuAlign);
      return;
    }
  }

  if (warp == PROD) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      const uint32_t pk = (uint32_t)R * (H / 2), sk = (uint32_t)R * (H / 32);
      const uint32_t hoff = (uint32_t)RS * fu_dn_row(I), hq_b = (uint32_t)I, hd_b = (uint32_t)IB * 4u;
      int s = 0, issued = 0, r = 0;
      uint32_t ph = 0;
      bool stop = false;
      for (int t = 0; t < NT && !stop; ++t) {
        const int *so = t_own + t * SW, *sbp = t_bpos + t * SW;
        const unsigned char *const *tb = t_blob + t * SW;
        const int32_t *sdone = a.slot_done + (size_t)t * kCtrlWords;
        int u0;
        const int mu = units_of(t, r, u0);
        r = (r + t_nsl[t] * rbs) % G;
        const int n_gu = mu * SPU, n_dn = nrows > 0 ? t_nsl[t] * nsub : 0;
        int seen = -1;  // the last slot found published
        int bslot = -1;
        const unsigned char *blob = nullptr;
        for (int j = 0; j < n_gu + n_dn; ++j) {
          if (issued >= NS && !mbar_wait(empty + s, ph ^ 1u, a.status, kDetFuEmpty, lim)) {
            *s_abort = 1;
            stop = true;
            break;
          }
          if (*s_abort) {
            stop = true;
            break;
          }
          unsigned char *dst = stg + (size_t)s * pl.sb;
          if (j < n_gu) {
            const int u = u0 + G * (j / SPU), st = j % SPU;
            const int slot = so[u / rbs], rb = u % rbs;
            if (slot != bslot) {
              bslot = slot;
              blob = tb[slot];
            }
            const size_t n0 = (size_t)rb * 32 + (size_t)st * R;
            mbar_arrive_expect_tx(full + s, 2 * (pk + sk));
            bulk_g2s_hint(dst, blob + n0 * (H / 2), pk, full + s, pol);
            bulk_g2s_hint(dst + pk, blob + mg + n0 * (H / 2), pk, full + s, pol);
            bulk_g2s_hint(dst + 2 * pk, blob + (size_t)I * (H / 2) + n0 * (H / 32), sk, full + s, pol);
            bulk_g2s_hint(dst + 2 * pk + sk, blob + mg + (size_t)I * (H / 2) + n0 * (H / 32), sk, full + s, pol);
          } else {
            const int jd = j - n_gu, slot = so[jd / nsub], r0 = (jd % nsub) * RS;
            const int nr_ = min(RS, nrows - r0);
            if (slot != bslot) {
              bslot = slot;
              blob = tb[slot];
            }
            const uint32_t bp = (uint32_t)nr_ * (I / 2), bs = (uint32_t)nr_ * (I / 32);
            if (slot != seen) {
              // every gate/up unit of the slot published its h codes (acquire);
              // then the copy engine may read them (proxy fence)
              if (!wait_count(sdone + slot, rbs, lim)) {
                set_status(a.status, MOE_ERR_TIMEOUT, kDetFuSlot);
                *s_abort = 1;
                stop = true;
                break;
              }
              asm volatile("fence.proxy.async.global;" ::: "memory");
              seen = slot;
            }
            const int hrow = sbp[slot];
            mbar_arrive_expect_tx(full + s, bp + bs + hq_b + 2 * hd_b);
            bulk_g2s_hint(dst, blob + 2 * mg + (size_t)(m0 + r0) * (I / 2), bp, full + s, pol);
            bulk_g2s_hint(dst + (size_t)RS * (I / 2), blob + 2 * mg + (size_t)H * (I / 2) + (size_t)(m0 + r0) * (I / 32),
                          bs, full + s, pol);
            bulk_g2s(dst + hoff, a.hq + (size_t)hrow * I, hq_b, full + s);
            bulk_g2s(dst + hoff + hq_b, a.hd + (size_t)hrow * IB, hd_b, full + s);
            bulk_g2s(dst + hoff + hq_b + hd_b, a.hqs + (size_t)hrow * IB, hd_b, full + s);
          }
          ++issued;
          if (++s == NS) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      for (int j = (issued > NS ? issued - NS : 0); j < issued; ++j)
        mbar_drain(full + j % NS, (uint32_t)(j / NS) & 1u, a.status, kDetFuDrain);
    }
    return;
  }

  if (warp == EPI) {
    // ---------------------------------------------------------------- epilogue
    // per gate/up unit of this CTA (tokens in order): wait for the consumers'
    // g and u sums (two buffers by unit parity), free the buffer, form h =
    // SiLU(g) * u and its Q8_0 block, store them and count the unit on its
    // slot (release), so that the consumers never wait on this work
    int cu = 0, r = 0;
    for (int t = 0; t < NT; ++t) {
      const int *so = t_own + t * SW, *sbp = t_bpos + t * SW;
      int32_t *sdone = a.slot_done + (size_t)t * kCtrlWords;
      int u0;
      const int mu = units_of(t, r, u0);
      r = (r + t_nsl[t] * rbs) % G;
      for (int c = 0; c < mu; ++c, ++cu) {
        const int par = cu & 1;
        named_sync(kBarGuFull + par, NCT + 32);
        const float *gb = gu + par * 64;
        const float g = gb[lane], uv = gb[32 + lane];
        if (cu + 2 < units_all) named_arrive(kBarGuFree + par, NCT + 32);
        if (__any_sync(0xffffffffu, *s_abort != 0)) continue;  // one decision per warp
        const int u = u0 + G * c;
        const int slot = so[u / rbs], rb = u % rbs;
        const int hrow = sbp[slot];
        const float h = swiglu(g, uv);
        const float d = fdiv(warp_max(fabsf(h)), 127.0f);
        const int q = q8_code(h, d);
        a.hq[(size_t)hrow * I + rb * 32 + lane] = (int8_t)q;
        const int qsum = __reduce_add_sync(0xffffffffu, q);
        if (lane == 0) {
          a.hd[(size_t)hrow * IB + rb] = d;
          a.hqs[(size_t)hrow * IB + rb] = qsum;
        }
        __syncwarp();
        if (lane == 0) red_release_add(sdone + slot, 1);
      }
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  // Tokens in order: gate/up units, down rows, then (after every consumer
  // warp is done with the token) the combine of this CTA's output rows.  On an
  // abort the warps run through the remaining hand-offs without waiting on
  // stages, so the epilogue warp's named barriers always find them.
  float *redw = red + (size_t)warp * pl.rw * 33;
  bool bad = false;
  int s = 0, cu = 0, r = 0;
  uint32_t ph = 0;
  int row_m[RPW], row_r[RPW];
#pragma unroll
  for (int q = 0; q < RPW; ++q) {
    const int jr = warp + NW * q;
    row_m[q] = jr / R;
    row_r[q] = jr % R;
  }
  const int cg0 = lane * CSZG, cd0 = lane * CSZD;
  const size_t hoff = (size_t)RS * fu_dn_row(I);
  for (int t = 0; t < NT; ++t) {
    const int *so = t_own + t * SW;
    const int nsl = t_nsl[t];
    int u0;
    const int mu = units_of(t, r, u0);
    r = (r + nsl * rbs) % G;
    const int n_gu = mu * SPU, n_dn = nrows > 0 ? nsl * nsub : 0;
    if (t > 0) {
      // the next token's codes into the activation chunks, once every
      // consumer is done with the last token (its combine included)
      named_sync(kBarEnd, NCT);
      load_token(t, 0, NCT);
      named_sync(kBarEnd, NCT);
    }
    {
      // gate/up: this CTA's units of the token; the lane's activation chunk
      // stays in registers for the token's gate/up phase
      uint32_t act1[CSZG][16];
      float d1[CSZG][2];
      int z1[CSZG][2];
      load_act<CSZG>(xq_s + (size_t)lane * pl.chp, xd_s, qs_s, cg0, GG, act1, d1, z1);
      for (int j = 0; j < n_gu; ++j) {
        const int st = j % SPU;
        if (!bad) bad = __any_sync(0xffffffffu, *s_abort != 0);  // one decision per warp
        if (!bad) {
          bad = !mbar_wait(full + s, ph, a.status, kDetFuFull, lim);
          bad = __any_sync(0xffffffffu, bad);
          if (bad && lane == 0) *s_abort = 1;
        }
        if (!bad) {
          const unsigned char *sb = stg + (size_t)s * pl.sb;
          uint32_t wv[RPW][CSZG][8];
          float sc[RPW][CSZG];
          uint32_t ex[RPW][CSZG];
#pragma unroll
          for (int q = 0; q < RPW; ++q) {
            const unsigned char *rowp = sb + (size_t)row_m[q] * R * (H / 2) + (size_t)row_r[q] * (H / 2);
            const unsigned char *scp = sb + (size_t)R * H + (size_t)row_m[q] * R * (H / 32) + (size_t)row_r[q] * (H / 32);
            if constexpr (FMT == kFmtMxfp4)
              load_row_mx<CSZG>(rowp, scp, cg0, GG, wv[q], ex[q]);
            else
              load_row<CSZG>(rowp, reinterpret_cast<const __half *>(scp), cg0, GG, wv[q], sc[q]);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(empty + s);  // the stage's rows are in registers
#pragma unroll
          for (int q = 0; q < RPW; ++q) {
            if constexpr (FMT == kFmtMxfp4)
              redw[(st * RPW + q) * 33 + lane] = chunk_dot_mx<CSZG>(wv[q], ex[q], act1, d1, cg0, GG);
            else
              redw[(st * RPW + q) * 33 + lane] = chunk_dot<CSZG>(wv[q], sc[q], act1, d1, z1, cg0, GG);
          }
        }
        if (st == SPU - 1) {
          // unit complete: this warp's g and u row sums into the unit's buffer
          // (once the epilogue warp has read the unit two before), then handed on
          const int par = cu & 1;
          if (cu >= 2) named_sync(kBarGuFree + par, NCT + 32);
          if (!bad) {
            __syncwarp();
            if (lane < PWR) {
              const int sq = lane / RPW, q = lane % RPW;
              const int jr = warp + NW * q;
              gu[par * 64 + (jr / R) * 32 + sq * R + jr % R] = chunk_sum(redw + lane * 33, nchg);
            }
          }
          named_arrive(kBarGuFull + par, NCT + 32);
          ++cu;
        }
        if (++s == NS) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
    if (t == NT - 1 && mu > 0) prof_end(a.prof, 1);
    if (t == 0 && n_dn > 0) prof_start(a.prof, 2);
    // down: this CTA's output rows of every slot of the token, shared expert
    // first; each stage brings the slot's h codes with the weights (the
    // producer issues it once the slot's units are all published)
    for (int jd = 0; jd < n_dn; ++jd) {
      const int slot = so[jd / nsub], sub = jd % nsub;
      const int r0 = sub * RS, nr_ = min(RS, nrows - r0);
      const int pos_base = slot == 0 ? K : slot - 1;
      if (!bad) bad = __any_sync(0xffffffffu, *s_abort != 0);  // one decision per warp
      if (!bad) {
        bad = !mbar_wait(full + s, ph, a.status, kDetFuFull, lim);
        bad = __any_sync(0xffffffffu, bad);
        if (bad && lane == 0) *s_abort = 1;
      }
      if (!bad) {
        const unsigned char *sb = stg + (size_t)s * pl.sb;
        uint32_t av[CSZD][16];
        float dv[CSZD][2];
        int zv[CSZD][2];
        load_act<CSZD>(sb + hoff + 64 * cd0, reinterpret_cast<const float *>(sb + hoff + I),
                       reinterpret_cast<const int *>(sb + hoff + I + (size_t)IB * 4), cd0, GD, av, dv, zv);
        const int ra = warp * nr_ / NW, rz = (warp + 1) * nr_ / NW;  // this warp's rows of the stage
        for (int ml = ra; ml < rz; ++ml) {
          uint32_t wv[CSZD][8];
          const unsigned char *rowp = sb + (size_t)ml * (I / 2);
          const unsigned char *scp = sb + (size_t)RS * (I / 2) + (size_t)ml * (I / 32);
          if constexpr (FMT == kFmtMxfp4) {
            uint32_t ex[CSZD];
            load_row_mx<CSZD>(rowp, scp, cd0, GD, wv, ex);
            redw[(ml - ra) * 33 + lane] = chunk_dot_mx<CSZD>(wv, ex, av, dv, cd0, GD);
          } else {
            float sc[CSZD];
            load_row<CSZD>(rowp, reinterpret_cast<const __half *>(scp), cd0, GD, wv, sc);
            redw[(ml - ra) * 33 + lane] = chunk_dot<CSZD>(wv, sc, av, dv, zv, cd0, GD);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + s);
        if (lane < rz - ra) ysm[(size_t)pos_base * a.rows_max + r0 + ra + lane] = chunk_sum(redw + lane * 33, nchd);
        __syncwarp();
      }
      if (++s == NS) {
        s = 0;
        ph ^= 1u;
      }
    }
    named_sync(kBarEnd, NCT);
    if (!*s_abort) {
      // combine, in the layer's order: shared expert, then the pairs by weight
      const int *si = t_idx + t * K, *sp = t_ppos + t * SW;
      const float *sw = t_w + t * K;
      for (int i = tid; i < nrows; i += NCT) {
        float o = a.with_shared ? ysm[(size_t)K * a.rows_max + i] : 0.0f;
        for (int q = 0; q < K; ++q)
          if (si[q] >= a.e_lo && si[q] < a.e_hi) o = ffma(sw[q], ysm[(size_t)sp[q] * a.rows_max + i], o);
        a.out[(size_t)t * H + m0 + i] = o;
      }
    }
  }
  if (*s_abort) return;
  if (blockIdx.x == 0 && warp == 0) {
    // the routing record of the workspace, as the routing kernel writes it
    // (read by no one in this kernel: written last)
    for (int i = lane; i < NT * K; i += 32) {
      a.idx[i] = t_idx[i];
      a.w[i] = t_w[i];
    }
    __syncwarp();
    if (NT * K <= 32) {
      bucket_small_counts(E, NT * K, t_idx, a.cnt, a.off, 0, 1);
      bucket_small(E, K, NT, t_idx, a.cnt, a.off, a.uni, a.n_uni, a.perm, a.pos, a.pair_tok);
    } else {
      bucket_warp(E, K, NT, t_idx, reinterpret_cast<int *>(red), a.cnt, a.off, a.uni, a.n_uni, a.perm, a.pos,
                  a.pair_tok);
    }
  }
  prof_end(a.prof, 2);
}

// The layer for one token (decode at T = 1): the same phases as the batch
// kernel above with the token loops, the per-token tables and the batch
// bucketing left out, and the expert table copied to shared memory while the
// routing data lands -- kept as its own kernel because the one-token call is
// the most frequent and this form measured 3 us faster per call than the
// batch kernel run with one token.
template <int CSZG, int CSZD, int FMT>
__global__ void __launch_bounds__(kFuThreads, 1) k_decode_fused1(FusedArgs a) {
  constexpr int R = kFuR, NW = kFuNW, SPU = kFuSPU, RPW = kFuRPW, PWR = kFuPWR, NCT = kFuNCT;
  constexpr int PROD = NW, EPI = NW + 1;  // warp roles after routing
  extern __shared__ __align__(128) unsigned char smem[];
  const int H = a.H, I = a.I, E = a.E, K = a.k, NS = a.nstage;
  const int GG = H / 64, HB = H / 32, GD = I / 64, IB = I / 32;
  const int nchg = (GG + CSZG - 1) / CSZG, nchd = (GD + CSZD - 1) / CSZD;
  const FuPlan pl = fu1_plan(H, I, E, K, a.rows_max, a.rs, NS);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + pl.bars);
  uint64_t *empty = full + NS;
  uint64_t *rbar = empty + NS;
  int *misc = reinterpret_cast<int *>(smem + pl.misc);
  volatile int *s_abort = misc;
  int *s_uni = misc + 8;                          // [k + 1] slot -> expert (slot 0 = shared)
  int *s_ppos = s_uni + (kMaxK + 1);              // [k] pair s -> position
  int *s_idx = s_ppos + (kMaxK + 1);              // [k] selected experts in slot order
  float *s_w = reinterpret_cast<float *>(s_idx + (kMaxK + 1));  // [k] softmax weights
  int *s_own = s_idx + 2 * (kMaxK + 1);           // [k + 1] the slots this call computes
  int *s_bpos = s_own + (kMaxK + 1);              // [k + 1] slot -> row of hq / hd / hqs
  const unsigned char **s_tab = reinterpret_cast<const unsigned char **>(smem + pl.tab);  // [E + 1]
  float *red = reinterpret_cast<float *>(smem + pl.red);
  float *gu = reinterpret_cast<float *>(smem + pl.gu);
  float *ysm = reinterpret_cast<float *>(smem + pl.ysm);
  float *xd_s = reinterpret_cast<float *>(smem + pl.xd);
  int *qs_s = reinterpret_cast<int *>(smem + pl.qs);
  unsigned char *xq_s = smem + pl.xq;
  unsigned char *stg = smem + pl.stg;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = (int)gridDim.x;
  const long long lim = a.wait_limit;
  if (tid == 0) {
    *s_abort = 0;
    for (int s = 0; s < NS; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, NW);
    }
    mbar_init(rbar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  prof_start(a.prof, 0);

  // ---------------------------------------------------------------- routing
  // this CTA's router rows [e0, e1) and x, staged in the (still idle) ring
  const int e0 = (int)((long long)blockIdx.x * E / G), e1 = (int)((long long)(blockIdx.x + 1) * E / G);
  const int nr = e1 - e0;
  float *rx = reinterpret_cast<float *>(stg);
  float *rw = rx + H;
  if (tid == 0) {
    mbar_arrive_expect_tx(rbar, (uint32_t)(1 + nr) * (uint32_t)H * 4u);
    bulk_g2s(rx, a.x, (uint32_t)H * 4u, rbar);
    if (nr > 0) bulk_g2s(rw, a.Wr + (size_t)e0 * H, (uint32_t)nr * (uint32_t)H * 4u, rbar);
  }
  // the expert table, for the stream that follows the union
  for (int e = tid; e <= E; e += kFuThreads) s_tab[e] = static_cast<const unsigned char *>(a.table[e]);
  if (blockIdx.x == 0) ctrl_zero(a, kCtrlWords);
  const bool ok = mbar_wait(rbar, 0, a.status, kDetFuRoute, lim);
  if (!__syncthreads_and(ok)) {
    if (tid == 0) mbar_drain(rbar, 0, a.status, kDetFuRouteDrain);  // the copies land before exit
    ctrl_close(a);
    return;
  }
  if (warp == PROD && lane == 0 && a.with_shared) {
    // a slice of the shared expert's blob into L2 while the grid routes (after
    // this CTA's routing data, which it must not delay)
    const unsigned char *sh = s_tab[E];
    const size_t bytes = 2 * ((size_t)I * (H / 2) + (size_t)I * (H / 64) * 2) +
                         ((size_t)H * (I / 2) + (size_t)H * (I / 64) * 2);
    const size_t slice = ((bytes + G - 1) / G + 15) / 16 * 16;
    const size_t b0 = slice * blockIdx.x;
    if ((reinterpret_cast<uintptr_t>(sh) & 15u) == 0 && b0 < bytes) {
      const size_t n = bytes - b0 < slice ? bytes - b0 : slice;
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(sh + b0), "r"((uint32_t)n) : "memory");
    }
  }
  // logits of this CTA's rows, the router's fixed order: lane l sums
  // h = l, l + 32, ... with fmaf, then an xor tree 16, 8, 4, 2, 1 (the
  // producer and epilogue warps take rows too)
  for (int r = warp; r < nr; r += kFuWarps) {
    const float *wv = rw + (size_t)r * H;
    float acc = 0.0f;
#pragma unroll 8
    for (int i = lane; i < H; i += 32) acc = ffma(rx[i], wv[i], acc);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) acc = fadd(acc, __shfl_xor_sync(0xffffffffu, acc, off));
    if (lane == 0) a.logits[e0 + r] = acc;
  }
  // Q8_0 of x: this CTA's share of the blocks, into the workspace (every CTA
  // reads all the codes back after the grid barrier); one warp per block
  {
    const int b0 = (int)((long long)blockIdx.x * HB / G), b1 = (int)((long long)(blockIdx.x + 1) * HB / G);
    const int qw = (warp - nr % kFuWarps + kFuWarps) % kFuWarps;  // the warps after the logit rows first
    for (int b = b0 + qw; b < b1; b += kFuWarps) {
      const float v = rx[b * 32 + lane];
      // the maximum of non-negative floats is the maximum of their bit patterns
      const float d = fdiv(__uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(v)))), 127.0f);
      a.xq[b * 32 + lane] = (int8_t)q8_code(v, d);
      if (lane == 0) a.xd[b] = d;
    }
  }
  // grid-wide: every CTA's logits are written before any CTA reads them (the
  // barrier orders this CTA's writes before thread 0's release)
  __syncthreads();
  if (tid == 0) {
    if (!ctrl_ready(a, lim)) {
      *s_abort = 1;
    } else {
      red_release_add_u32(a.arrivals, 1u);
      if (ld_acquire_u32(a.arrivals) < (unsigned)G) {
        const long long t0 = clock64();
        while (ld_acquire_u32(a.arrivals) < (unsigned)G) {
          if (clock64() - t0 > lim) {
            set_status(a.status, MOE_ERR_TIMEOUT, kDetFuGrid);
            *s_abort = 1;
            break;
          }
          __nanosleep(32);
        }
      }
    }
    ctrl_close(a);  // every CTA has arrived, so has seen the ready word (or the wait ran out)
  }
  __syncthreads();
  if (*s_abort) return;  // nothing in flight: the staging copies have landed

  if (warp != 0) {
    // the Q8_0 codes of x (every CTA's share, from L2) into this CTA's
    // activation chunks, with the block scales and code sums
    for (int b = tid - 32; b < HB; b += kFuThreads - 32) {
      const uint4 *src = reinterpret_cast<const uint4 *>(a.xq + (size_t)b * 32);
      const uint4 q0 = __ldcg(src), q1 = __ldcg(src + 1);
      int sum = 0;
      sum = __dp4a((int)q0.x, 0x01010101, sum);
      sum = __dp4a((int)q0.y, 0x01010101, sum);
      sum = __dp4a((int)q0.z, 0x01010101, sum);
      sum = __dp4a((int)q0.w, 0x01010101, sum);
      sum = __dp4a((int)q1.x, 0x01010101, sum);
      sum = __dp4a((int)q1.y, 0x01010101, sum);
      sum = __dp4a((int)q1.z, 0x01010101, sum);
      sum = __dp4a((int)q1.w, 0x01010101, sum);
      const int h = b * 32, g = h >> 6, c = g / CSZG;
      uint4 *dst = reinterpret_cast<uint4 *>(xq_s + (size_t)c * pl.chp + (size_t)(g - c * CSZG) * 64 + (h & 63));
      dst[0] = q0;
      dst[1] = q1;
      xd_s[b] = __ldcg(a.xd + b);
      qs_s[b] = sum;
    }
  }

  // top-k, softmax and the union -- the same in every CTA
  if (warp == 0) {
    int e_sel;
    float l_sel;
    warp_topk(a.logits, E, K, lane, e_sel, l_sel, reinterpret_cast<uint32_t *>(red));
    warp_softmax_store(0, K, lane, e_sel, l_sel, s_idx, s_w, blockIdx.x == 0 ? a.route_counts : nullptr,
                       nullptr);
    __syncwarp();
    // one token: the union is the k selected experts in ascending order;
    // pair s sits at position rank(e_s), the shared expert's pair at k
    if (lane < K) {
      int rank = 0;
      for (int q = 0; q < K; ++q) rank += s_idx[q] < e_sel ? 1 : 0;
      s_uni[1 + rank] = e_sel;
      s_ppos[lane] = rank;
      s_bpos[1 + rank] = rank;
    }
    if (lane == 0) {
      s_uni[0] = E;
      s_bpos[0] = K;
    }
    __syncwarp();
    // the slots this call computes (expert parallelism: the shared expert on
    // one rank, the routed experts in [e_lo, e_hi); by default all of them)
    if (lane == 0) {
      int n = 0;
      if (a.with_shared) s_own[n++] = 0;
      for (int i = 1; i <= K; ++i)
        if (s_uni[i] >= a.e_lo && s_uni[i] < a.e_hi) s_own[n++] = i;
      misc[1] = n;
    }
  }
  __syncthreads();
  prof_end(a.prof, 0);
  prof_start(a.prof, 1);

  const int nslot = misc[1];  // slots this call computes
  const int rbs = I / 32;     // 32-row units per expert
  const int n_units = nslot * rbs;
  const int my_units = (int)blockIdx.x < n_units ? (n_units - 1 - (int)blockIdx.x) / G + 1 : 0;
  const int n_gu = my_units * SPU;
  const int nrg = H / a.rg;
  const int m0 = (int)((long long)blockIdx.x * nrg / G) * a.rg;
  const int m1 = (int)((long long)(blockIdx.x + 1) * nrg / G) * a.rg;
  const int nrows = m1 - m0;
  const int RS = a.rs;
  const int nsub = (nrows + RS - 1) / RS;
  const int n_dn = nrows > 0 ? nslot * nsub : 0;
  const int n_st = n_gu + n_dn;
  const size_t mg = (size_t)I * H / 2 + (size_t)I * H / 32;  // bytes of the gate (= up) matrix

  // every blob this grid reads must be 16-byte aligned (TMA bulk copies)
  {
    bool bad = false;
    for (int sl = tid; sl < nslot; sl += kFuThreads)
      bad |= (reinterpret_cast<uintptr_t>(s_tab[s_uni[s_own[sl]]]) & 15u) != 0;
    if (__syncthreads_or(bad)) {
      if (tid == 0) set_status(a.status, MOE_ERR_DEVICE, kDetFuAlign);
      return;
    }
  }

  if (warp == PROD) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      const uint32_t pk = (uint32_t)R * (H / 2), sk = (uint32_t)R * (H / 32);
      const uint32_t hoff = (uint32_t)RS * fu_dn_row(I), hq_b = (uint32_t)I, hd_b = (uint32_t)IB * 4u;
      int s = 0, issued = 0, seen = -1;  // seen: the last slot found published
      uint32_t ph = 0;
      for (int j = 0; j < n_st; ++j) {
        if (j >= NS && !mbar_wait(empty + s, ph ^ 1u, a.status, kDetFuEmpty, lim)) {
          *s_abort = 1;
          break;
        }
        if (*s_abort) break;
        unsigned char *dst = stg + (size_t)s * pl.sb;
        if (j < n_gu) {
          const int u = (int)blockIdx.x + G * (j / SPU), st = j % SPU;
          const int slot = s_own[u / rbs], rb = u % rbs;
          const unsigned char *blob = s_tab[s_uni[slot]];
          const size_t n0 = (size_t)rb * 32 + (size_t)st * R;
          mbar_arrive_expect_tx(full + s, 2 * (pk + sk));
          bulk_g2s_hint(dst, blob + n0 * (H / 2), pk, full + s, pol);
          bulk_g2s_hint(dst + pk, blob + mg + n0 * (H / 2), pk, full + s, pol);
          bulk_g2s_hint(dst + 2 * pk, blob + (size_t)I * (H / 2) + n0 * (H / 32), sk, full + s, pol);
          bulk_g2s_hint(dst + 2 * pk + sk, blob + mg + (size_t)I * (H / 2) + n0 * (H / 32), sk, full + s, pol);
        } else {
          const int jd = j - n_gu, slot = s_own[jd / nsub], r0 = (jd % nsub) * RS;
          const int nr_ = min(RS, nrows - r0);
          const unsigned char *blob = s_tab[s_uni[slot]];
          const uint32_t bp = (uint32_t)nr_ * (I / 2), bs = (uint32_t)nr_ * (I / 32);
          if (slot != seen) {
            // every gate/up unit of the slot published its h codes (acquire);
            // then the copy engine may read them (proxy fence)
            if (!wait_count(a.slot_done + slot, rbs, lim)) {
              set_status(a.status, MOE_ERR_TIMEOUT, kDetFuSlot);
              *s_abort = 1;
              break;
            }
            asm volatile("fence.proxy.async.global;" ::: "memory");
            seen = slot;
          }
          const int hrow = s_bpos[slot];
          mbar_arrive_expect_tx(full + s, bp + bs + hq_b + 2 * hd_b);
          bulk_g2s_hint(dst, blob + 2 * mg + (size_t)(m0 + r0) * (I / 2), bp, full + s, pol);
          bulk_g2s_hint(dst + (size_t)RS * (I / 2), blob + 2 * mg + (size_t)H * (I / 2) + (size_t)(m0 + r0) * (I / 32),
                        bs, full + s, pol);
          bulk_g2s(dst + hoff, a.hq + (size_t)hrow * I, hq_b, full + s);
          bulk_g2s(dst + hoff + hq_b, a.hd + (size_t)hrow * IB, hd_b, full + s);
          bulk_g2s(dst + hoff + hq_b + hd_b, a.hqs + (size_t)hrow * IB, hd_b, full + s);
        }
        issued = j + 1;
        if (++s == NS) {
          s = 0;
          ph ^= 1u;
        }
      }
      for (int j = (issued > NS ? issued - NS : 0); j < issued; ++j)
        mbar_drain(full + j % NS, (uint32_t)(j / NS) & 1u, a.status, kDetFuDrain);
    }
    return;
  }

  if (warp == EPI) {
    // ---------------------------------------------------------------- epilogue
    // per gate/up unit of this CTA: wait for the consumers' g and u sums (two
    // buffers by unit parity), free the buffer, form h = SiLU(g) * u and its
    // Q8_0 block, store them and count the unit on its slot (release), so that
    // the consumers never wait on this work
    for (int cu = 0; cu < my_units; ++cu) {
      const int par = cu & 1;
      named_sync(kBarGuFull + par, NCT + 32);
      const float *gb = gu + par * 64;
      const float g = gb[lane], uv = gb[32 + lane];
      if (cu + 2 < my_units) named_arrive(kBarGuFree + par, NCT + 32);
      if (__any_sync(0xffffffffu, *s_abort != 0)) continue;  // one decision per warp
      const int u = (int)blockIdx.x + G * cu;
      const int slot = s_own[u / rbs], rb = u % rbs;
      const int hrow = s_bpos[slot];
      const float h = swiglu(g, uv);
      const float d = fdiv(warp_max(fabsf(h)), 127.0f);
      const int q = q8_code(h, d);
      a.hq[(size_t)hrow * I + rb * 32 + lane] = (int8_t)q;
      const int qsum = __reduce_add_sync(0xffffffffu, q);
      if (lane == 0) {
        a.hd[(size_t)hrow * IB + rb] = d;
        a.hqs[(size_t)hrow * IB + rb] = qsum;
      }
      __syncwarp();
      if (lane == 0) red_release_add(a.slot_done + slot, 1);
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  float *redw = red + (size_t)warp * pl.rw * 33;
  bool bad = false;
  int s = 0;
  uint32_t ph = 0;
  {
    // gate/up: this CTA's units in round-robin order; one token, so the
    // lane's activation chunk stays in registers for the whole phase
    const int c0 = lane * CSZG;
    uint32_t act1[CSZG][16];
    float d1[CSZG][2];
    int z1[CSZG][2];
    load_act<CSZG>(xq_s + (size_t)lane * pl.chp, xd_s, qs_s, c0, GG, act1, d1, z1);
    int row_m[RPW], row_r[RPW];
#pragma unroll
    for (int q = 0; q < RPW; ++q) {
      const int jr = warp + NW * q;
      row_m[q] = jr / R;
      row_r[q] = jr % R;
    }
    for (int j = 0; j < n_gu; ++j) {
      const int cu = j / SPU, st = j % SPU;
      if (!bad) bad = __any_sync(0xffffffffu, *s_abort != 0);  // one decision per warp
      if (!bad) {
        bad = !mbar_wait(full + s, ph, a.status, kDetFuFull, lim);
        bad = __any_sync(0xffffffffu, bad);
        if (bad && lane == 0) *s_abort = 1;
      }
      if (!bad) {
        const unsigned char *sb = stg + (size_t)s * pl.sb;
        uint32_t wv[RPW][CSZG][8];
        float sc[RPW][CSZG];
        uint32_t ex[RPW][CSZG];
#pragma unroll
        for (int q = 0; q < RPW; ++q) {
          const unsigned char *rowp = sb + (size_t)row_m[q] * R * (H / 2) + (size_t)row_r[q] * (H / 2);
          const unsigned char *scp = sb + (size_t)R * H + (size_t)row_m[q] * R * (H / 32) + (size_t)row_r[q] * (H / 32);
          if constexpr (FMT == kFmtMxfp4)
            load_row_mx<CSZG>(rowp, scp, c0, GG, wv[q], ex[q]);
          else
            load_row<CSZG>(rowp, reinterpret_cast<const __half *>(scp), c0, GG, wv[q], sc[q]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + s);  // the stage's rows are in registers
#pragma unroll
        for (int q = 0; q < RPW; ++q) {
          if constexpr (FMT == kFmtMxfp4)
            redw[(st * RPW + q) * 33 + lane] = chunk_dot_mx<CSZG>(wv[q], ex[q], act1, d1, c0, GG);
          else
            redw[(st * RPW + q) * 33 + lane] = chunk_dot<CSZG>(wv[q], sc[q], act1, d1, z1, c0, GG);
        }
      }
      if (st == SPU - 1) {
        // unit complete: this warp's g and u row sums into the unit's buffer
        // (once the epilogue warp has read the unit two before), then handed on
        const int par = cu & 1;
        if (cu >= 2) named_sync(kBarGuFree + par, NCT + 32);
        if (!bad) {
          __syncwarp();
          if (lane < PWR) {
            const int sq = lane / RPW, q = lane % RPW;
            const int jr = warp + NW * q;
            gu[par * 64 + (jr / R) * 32 + sq * R + jr % R] = chunk_sum(redw + lane * 33, nchg);
          }
        }
        named_arrive(kBarGuFull + par, NCT + 32);
      }
      if (++s == NS) {
        s = 0;
        ph ^= 1u;
      }
    }
  }
  if (n_gu > 0) prof_end(a.prof, 1);
  if (n_dn > 0) prof_start(a.prof, 2);
  {
    // down: this CTA's output rows of every slot, shared expert first; each
    // stage brings the slot's h codes with the weights (the producer issues it
    // once the slot's units are all published)
    const int c0 = lane * CSZD;
    const size_t hoff = (size_t)RS * fu_dn_row(I);
    for (int jd = 0; jd < n_dn; ++jd) {
      const int slot = s_own[jd / nsub], sub = jd % nsub;
      const int r0 = sub * RS, nr_ = min(RS, nrows - r0);
      const int pos_base = slot == 0 ? K : slot - 1;
      if (!bad) bad = __any_sync(0xffffffffu, *s_abort != 0);  // one decision per warp
      if (!bad) {
        bad = !mbar_wait(full + s, ph, a.status, kDetFuFull, lim);
        bad = __any_sync(0xffffffffu, bad);
        if (bad && lane == 0) *s_abort = 1;
      }
      if (!bad) {
        const unsigned char *sb = stg + (size_t)s * pl.sb;
        uint32_t av[CSZD][16];
        float dv[CSZD][2];
        int zv[CSZD][2];
        load_act<CSZD>(sb + hoff + 64 * c0, reinterpret_cast<const float *>(sb + hoff + I),
                       reinterpret_cast<const int *>(sb + hoff + I + (size_t)IB * 4), c0, GD, av, dv, zv);
        const int ra = warp * nr_ / NW, rz = (warp + 1) * nr_ / NW;  // this warp's rows of the stage
        for (int ml = ra; ml < rz; ++ml) {
          uint32_t wv[CSZD][8];
          const unsigned char *rowp = sb + (size_t)ml * (I / 2);
          const unsigned char *scp = sb + (size_t)RS * (I / 2) + (size_t)ml * (I / 32);
          if constexpr (FMT == kFmtMxfp4) {
            uint32_t ex[CSZD];
            load_row_mx<CSZD>(rowp, scp, c0, GD, wv, ex);
            redw[(ml - ra) * 33 + lane] = chunk_dot_mx<CSZD>(wv, ex, av, dv, c0, GD);
          } else {
            float sc[CSZD];
            load_row<CSZD>(rowp, reinterpret_cast<const __half *>(scp), c0, GD, wv, sc);
            redw[(ml - ra) * 33 + lane] = chunk_dot<CSZD>(wv, sc, av, dv, zv, c0, GD);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + s);
        if (lane < rz - ra) ysm[(size_t)pos_base * a.rows_max + r0 + ra + lane] = chunk_sum(redw + lane * 33, nchd);
        __syncwarp();
      }
      if (++s == NS) {
        s = 0;
        ph ^= 1u;
      }
    }
  }
  named_sync(kBarEnd, NCT);
  if (*s_abort) return;
  // combine, in the layer's order: shared expert, then the slots by weight
  for (int i = tid; i < nrows; i += NCT) {
    float o = a.with_shared ? ysm[(size_t)K * a.rows_max + i] : 0.0f;
    for (int q = 0; q < K; ++q)
      if (s_idx[q] >= a.e_lo && s_idx[q] < a.e_hi) o = ffma(s_w[q], ysm[(size_t)s_ppos[q] * a.rows_max + i], o);
    a.out[m0 + i] = o;
  }
  if (blockIdx.x == 0 && warp == 0) {
    // the routing record of the workspace, as the routing kernel writes it
    // (read by no one in this kernel: written last)
    if (lane < K) {
      a.idx[lane] = s_idx[lane];
      a.w[lane] = s_w[lane];
    }
    __syncwarp();
    bucket_small_counts(E, K, s_idx, a.cnt, a.off, 0, 1);
    bucket_small(E, K, 1, s_idx, a.cnt, a.off, a.uni, a.n_uni, a.perm, a.pos, a.pair_tok);
  }
  prof_end(a.prof, 2);
}

// Plan of the fused kernel for a grid of `grid` CTAs: ring stages, down row
// split and shared memory; false if the layer's shape does not fit it (the
// three-kernel decode path then runs).
bool fused_plan(int H, int I, int E, int k, int grid, FusedArgs *a, size_t *smem) {
  const int cszg = (H / 64 + 31) / 32, cszd = (I / 64 + 31) / 32;
  if (cszg < 1 || cszg > 4 || cszd < 1 || cszd > 2 || grid < 1 || k > kMaxK) return false;
  // down rows: groups of rg rows whose scale bytes are a multiple of 16
  int g = I / 32, b = 16;
  while (b) {
    const int t = g % b;
    g = b;
    b = t;
  }
  const int rg = 16 / g;
  const int nrg = H / rg;
  const int rows_max = ((nrg + grid - 1) / grid) * rg;
  const uint32_t sg = fu_gu_stage(H);
  int rs = rows_max;
  while (rs > rg && fu_dn_stage(I, rs) > sg) rs -= rg;
  const int rpc = (E + grid - 1) / grid;  // router rows per CTA
  for (int ns = 4; ns >= 3; --ns) {
    const FuPlan p = fu_plan(H, I, E, k, rows_max, rs, ns), p1 = fu1_plan(H, I, E, k, rows_max, rs, ns);
    if (p.total > (size_t)(227 * 1024) || p1.total > (size_t)(227 * 1024)) continue;
    if ((size_t)(1 + rpc) * H * 4 > (size_t)ns * p.sb) continue;
    a->nstage = ns;
    a->rows_max = rows_max;
    a->rg = rg;
    a->rs = rs;
    *smem = p.total;
    return true;
  }
  return false;
}

// Launch: one token -> k_decode_fused1, a batch -> k_decode_fused, each with
// its own shared-memory plan (from the stage count and down split in a).
template <int CSZG, int CSZD, int FMT>
static cudaError_t launch_fu(const FusedArgs &a, int grid, size_t smem_unused, cudaStream_t s) {
  (void)smem_unused;
  const bool one = a.ntok <= 1;
  const size_t smem = one ? fu1_plan(a.H, a.I, a.E, a.k, a.rows_max, a.rs, a.nstage).total
                          : fu_plan(a.H, a.I, a.E, a.k, a.rows_max, a.rs, a.nstage).total;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kFuThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (one) {
    static int smem_set[64] = {0};
    const cudaError_t err = ensure_smem(k_decode_fused1<CSZG, CSZD, FMT>, smem, smem_set);
    if (err != cudaSuccess) return err;
    return cudaLaunchKernelEx(&cfg, k_decode_fused1<CSZG, CSZD, FMT>, a);
  }
  static int smem_set[64] = {0};
  const cudaError_t err = ensure_smem(k_decode_fused<CSZG, CSZD, FMT>, smem, smem_set);
  if (err != cudaSuccess) return err;
  return cudaLaunchKernelEx(&cfg, k_decode_fused<CSZG, CSZD, FMT>, a);
}

template <typename Kern>
static int ctas_of(Kern k, size_t smem, int (&smem_set)[64]) {
  if (ensure_smem(k, smem, smem_set) != cudaSuccess) return 0;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, kFuThreads, smem) != cudaSuccess) return 0;
  return n;
}

// CTAs per SM that both kernels (one token, a batch) reach with their plans
template <int CSZG, int CSZD, int FMT>
static int ctas_fu(const FusedArgs &a) {
  static int set1[64] = {0}, setb[64] = {0};
  const int n1 = ctas_of(k_decode_fused1<CSZG, CSZD, FMT>,
                         fu1_plan(a.H, a.I, a.E, a.k, a.rows_max, a.rs, a.nstage).total, set1);
  const int nb = ctas_of(k_decode_fused<CSZG, CSZD, FMT>,
                         fu_plan(a.H, a.I, a.E, a.k, a.rows_max, a.rs, a.nstage).total, setb);
  return n1 < nb ? n1 : nb;
}

#define MOE_FU_CASES(FN, F, ...)                                           \
  case 11: return FN<1, 1, F>(__VA_ARGS__);                                \
  case 12: return FN<1, 2, F>(__VA_ARGS__);                                \
  case 21: return FN<2, 1, F>(__VA_ARGS__);                                \
  case 22: return FN<2, 2, F>(__VA_ARGS__);                                \
  case 31: return FN<3, 1, F>(__VA_ARGS__);                                \
  case 32: return FN<3, 2, F>(__VA_ARGS__);                                \
  case 41: return FN<4, 1, F>(__VA_ARGS__);                                \
  case 42: return FN<4, 2, F>(__VA_ARGS__);
#define MOE_FU_DISPATCH(FN, ...)                                           \
  {                                                                        \
    const int key = (a.H / 64 + 31) / 32 * 10 + (a.I / 64 + 31) / 32;     \
    if (a.fmt == kFmtMxfp4) {                                              \
      switch (key) { MOE_FU_CASES(FN, kFmtMxfp4, __VA_ARGS__) default: break; } \
    } else {                                                               \
      switch (key) { MOE_FU_CASES(FN, kFmtInt4, __VA_ARGS__) default: break; }  \
    }                                                                      \
  }

cudaError_t launch_decode_fused(const FusedArgs &a, int grid, size_t smem, cudaStream_t s) {
  MOE_FU_DISPATCH(launch_fu, a, grid, smem, s)
  return cudaErrorInvalidValue;
}

int fused_ctas_per_sm(const FusedArgs &a, size_t smem) {
  (void)smem;
  MOE_FU_DISPATCH(ctas_fu, a)
  return 0;
}

}  // namespace moe
