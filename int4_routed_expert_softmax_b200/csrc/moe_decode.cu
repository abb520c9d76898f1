// moe_decode.cu -- decode (GEMV) expert kernels of the routed-expert MoE layer.
//
//   k_gateup_decode: h = SiLU(W_gate x) * (W_up x) for every (union expert,
//                    token) pair, requantised to Q8_0 per 32 rows of I.
//   k_down_decode:   y = W_down Q8_0(h) per pair, then the combine
//                    out[t] = y_shared, out = fmaf(w_s, y_s, out) in slot order.
//
// int4 gs64 weights (colibri, tantan.ink, 我看到的几个坑) against Q8_0-style int8
// activations (Colibri, alphamatch.ai, 優化整數核心); the expert union of the
// batch is read once per call (tantan.ink, 几个关键工程动作, Batch union).
//
// B200 design.  Both kernels are persistent, one CTA of 8 consumer warps +
// 1 producer warp per SM.  The producer streams weight rows through a ring of
// shared-memory stages with TMA bulk copies (cp.async.bulk, completion counted
// on an mbarrier per stage, L2 evict-first), so the bytes in flight per SM
// (3-4 stages of 45-52 KB) cover the HBM latency.  Consumers copy a stage's
// rows to registers, release the stage at once, then unpack nibbles with one
// LOP3 per word (low nibbles masked as values 0..15, high nibbles masked in
// place as 16x their value) and run dp4a (unsigned x signed bytes) per
// 32-block; the offset-binary bias and the 16x are folded into the integer
// accumulator's start value, so each block sum is exact.  Tile shapes are
// compile-time and every ring / unit index advances incrementally: the
// per-stage bookkeeping is a handful of instructions.
//
// Fixed order of the fp32 part (this kernel's own, so every call gives the
// same bits): per 64-group a = S0*d0, b = fma(S1, d1, a), chunk acc =
// fma(s_g, b, acc); lane c owns the chunk of CSZ consecutive groups; the 32
// chunk sums are added left to right (one lane per row after a transpose in
// shared memory).  The definition sums the groups in plain ascending order;
// the two orders differ by a few units in the last place of each sum, so a
// Q8_0 code of h can differ by one where h lies that close to a rounding
// boundary, and the outputs agree within the layer's float tolerance.
#include "moe_decode.cuh"

namespace moe {

// ===========================================================================
// gate/up
// ===========================================================================
struct GuPlan {
  size_t red, gu, xd, qs, xq, stg, total;
  uint32_t sb;
  int chp;
};

__host__ __device__ inline GuPlan gu_plan(int H, int T, int R, int ns, int csz) {
  GuPlan p;
  p.chp = csz * 64 + 16;
  p.sb = (uint32_t)((size_t)R * H + (size_t)R * H / 16);
  size_t o = al128d((size_t)16 * ns);
  p.red = o;
  o += al128d((size_t)8 * (2 * T > 8 ? 2 * T : 8) * 33 * 4);
  p.gu = o;
  o += al128d((size_t)(T == 1 ? 2 : T) * 64 * 4);  // one token: two buffers (unit parity)
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

// Work unit = (union slot, 32-row block of I); slot 0 is the shared expert,
// slot u >= 1 is uni[u-1]; units are split evenly over the CTAs.  A stage is
// R gate rows + R up rows (packed nibbles + fp16 scales).  NW consumer warps
// (warp NW is the producer); consumer warp w owns rows w, w + NW, ... of the
// stage's 2R rows (NW = 8, R = 8: gate row w and up row w; NW = 16: one row).
template <int CSZ, bool ONE, int R, int NW>
__global__ void __launch_bounds__(NW * 32 + 32, 1) k_gateup_decode(GateUpArgs a) {
  static_assert(NW == 8 || (ONE && NW == 16 && R == 8), "16 consumer warps: one token, 8-row stages");
  constexpr int SPU = 32 / R;         // stages per 32-row unit
  constexpr int RPW = 2 * R / NW;     // rows per warp per stage
  constexpr int PWR = SPU * RPW;      // rows per warp per unit
  constexpr int NCT = NW * 32;        // consumer threads
  extern __shared__ __align__(128) unsigned char smem[];
  const int H = a.H, I = a.I, T = a.T, NS = a.nstage;
  const int G = H / 64, HB = H / 32;
  const int nch = (G + CSZ - 1) / CSZ;
  const GuPlan pl = gu_plan(H, T, R, NS, CSZ);
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
      mbar_init(empty + s, NW);
    }
    fence_barrier_init();
  }
  if (a.use_pdl) {
    pdl_wait();
    // the down kernel may be scheduled from here on (as SMs free up); this
    // grid's own routing inputs are complete, which is all it reads early
    pdl_launch_dependents();
  }
  // an earlier kernel of this call failed: leave everything untouched (one
  // decision for the whole CTA, so that no named barrier below misses a warp)
  if (__syncthreads_or(*reinterpret_cast<volatile int32_t *>(a.status) != 0)) return;
  prof_start(a.prof, 1);
  const int n_slots = min(max(*a.n_own, 0), a.E + 1);  // the union slots this call computes
  const int rbs = I / 32;  // 32-row units per expert
  const int n_units = n_slots * rbs;
  const int u_begin = (int)((long long)blockIdx.x * n_units / gridDim.x);
  const int u_end = (int)((long long)(blockIdx.x + 1) * n_units / gridDim.x);
  const int n_stages = (u_end - u_begin) * SPU;
  const size_t mg = (size_t)I * H / 2 + (size_t)I * H / 32;

  // blobs this CTA reads must be 16-byte aligned (TMA bulk copies)
  {
    bool bad = false;
    const int sl0 = u_begin / rbs, sl1 = (u_end - 1) / rbs;
    for (int sl = sl0 + tid; sl <= sl1 && u_end > u_begin; sl += blockDim.x) {
      const int so = a.own[sl];
      const int e = so == 0 ? a.E : a.uni[so - 1];
      bad |= (reinterpret_cast<uintptr_t>(a.table[e]) & 15u) != 0;
    }
    if (__syncthreads_or(bad)) {
      if (tid == 0) set_status(a.status, MOE_ERR_DEVICE, kDetGuAlign);
      return;
    }
  }

  // activations (consumer warps only; the producer starts streaming weights
  // at once): xq in per-lane chunks (padded rows), block scales, code sums
  if (warp != NW) {
    const int pieces = CSZ * 4;
    for (int i = tid; i < T * 32 * pieces; i += NCT) {
      const int t = i / (32 * pieces), r = i % (32 * pieces), c = r / pieces, j = r % pieces;
      const int col = c * CSZ * 64 + 16 * j;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (col < H) v = *reinterpret_cast<const uint4 *>(a.xq + (size_t)t * H + col);
      *reinterpret_cast<uint4 *>(xq_s + (size_t)(t * 32 + c) * pl.chp + 16 * j) = v;
    }
    for (int i = tid; i < T * HB; i += NCT) {
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
    named_sync(1, NCT);
  }

  if (warp == NW) {
    // -------------------------------------------------------------- producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      const uint32_t pk = (uint32_t)R * (H / 2), sk = (uint32_t)R * (H / 32);
      int s = 0, issued = 0;
      uint32_t ph = 0;
      int slot = u_begin / rbs, rb = u_begin % rbs, st = 0;
      const unsigned char *blob = nullptr;
      int blob_slot = -1;
      for (int j = 0; j < n_stages; ++j) {
        if (j >= NS && !mbar_wait(empty + s, ph ^ 1u, a.status, kDetGuEmpty, a.wait_limit)) {
          s_abort = 1;
          break;
        }
        if (*reinterpret_cast<volatile int *>(&s_abort)) break;
        if (slot != blob_slot) {
          blob_slot = slot;
          const int so = a.own[slot];
          blob = reinterpret_cast<const unsigned char *>(a.table[so == 0 ? a.E : a.uni[so - 1]]);
        }
        const size_t n0 = (size_t)rb * 32 + (size_t)st * R;
        unsigned char *dst = stg + (size_t)s * pl.sb;
        mbar_arrive_expect_tx(full + s, 2 * (pk + sk));
        bulk_g2s_hint(dst, blob + n0 * (H / 2), pk, full + s, pol);
        bulk_g2s_hint(dst + pk, blob + mg + n0 * (H / 2), pk, full + s, pol);
        bulk_g2s_hint(dst + 2 * pk, blob + (size_t)I * (H / 2) + n0 * (H / 32), sk, full + s, pol);
        bulk_g2s_hint(dst + 2 * pk + sk, blob + mg + (size_t)I * (H / 2) + n0 * (H / 32), sk,
                      full + s, pol);
        issued = j + 1;
        if (++s == NS) {
          s = 0;
          ph ^= 1u;
        }
        if (++st == SPU) {
          st = 0;
          if (++rb == rbs) {
            rb = 0;
            ++slot;
          }
        }
      }
      for (int j = (issued > NS ? issued - NS : 0); j < issued; ++j)
        mbar_drain(full + j % NS, (j / NS) & 1, a.status, kDetGuDrain);
    }
    return;
  }

  if (!ONE) {
    // ------------------------------------------------------ consumers, batch
    // unit by unit: a slot with one token (most routed slots of a small
    // batch) keeps that token's activation chunk in registers for the unit and
    // sums each row's chunks once per unit, as the single-token kernel does;
    // a slot with several tokens runs them per stage against the rows in
    // registers.  Each unit ends with every consumer warp at a named barrier
    // (h = SiLU(g) * u and its Q8_0 per token), so all warps work on the same
    // unit and share the red and gu buffers by unit.
    const int c0 = lane * CSZ;
    int row_m[RPW], row_r[RPW];
#pragma unroll
    for (int q = 0; q < RPW; ++q) {
      const int jr = warp + NW * q;
      row_m[q] = jr / R;
      row_r[q] = jr % R;
    }
    float *redw = red + (size_t)warp * (2 * T > 8 ? 2 * T : 8) * 33;
    int slot = u_begin / rbs, rb = u_begin % rbs, s = 0;
    uint32_t ph = 0;
    bool bad = false;
    for (int u = u_begin; u < u_end; ++u) {
      int n_tok, pos_base, my_tok;
      const int so = a.own[slot];
      if (so == 0) {
        n_tok = T;
        pos_base = T * a.k;
        my_tok = lane;
      } else {
        const int e = a.uni[so - 1];
        pos_base = a.off[e];
        n_tok = a.off[e + 1] - pos_base;
        my_tok = lane < n_tok ? a.pair_tok[pos_base + lane] : 0;
      }
      if (n_tok == 1) {
        const int t = __shfl_sync(0xffffffffu, my_tok, 0);
        uint32_t act1[CSZ][16];
        float d1[CSZ][2];
        int z1[CSZ][2];
        load_act<CSZ>(xq_s + (size_t)(t * 32 + lane) * pl.chp, xd_s + t * HB, qs_s + t * HB, c0, G, act1, d1, z1);
        for (int st = 0; st < SPU; ++st) {
          if (!bad) bad = __any_sync(0xffffffffu, *reinterpret_cast<volatile int *>(&s_abort) != 0);
          if (!bad) {
            bad = !mbar_wait(full + s, ph, a.status, kDetGuFull, a.wait_limit);
            bad = __any_sync(0xffffffffu, bad);
            if (bad && lane == 0) s_abort = 1;
          }
          if (!bad) {
            const unsigned char *sb = stg + (size_t)s * pl.sb;
            uint32_t wv[RPW][CSZ][8];
            float sc[RPW][CSZ];
#pragma unroll
            for (int q = 0; q < RPW; ++q)
              load_row<CSZ>(sb + (size_t)row_m[q] * R * (H / 2) + (size_t)row_r[q] * (H / 2),
                            reinterpret_cast<const __half *>(sb + (size_t)R * H + (size_t)row_m[q] * R * (H / 32) +
                                                             (size_t)row_r[q] * (H / 32)),
                            c0, G, wv[q], sc[q]);
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + s);  // the stage's rows are in registers
#pragma unroll
            for (int q = 0; q < RPW; ++q)
              redw[(st * RPW + q) * 33 + lane] = chunk_dot<CSZ>(wv[q], sc[q], act1, d1, z1, c0, G);
          }
          if (++s == NS) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!bad) {
          // the warp's PWR rows of the unit: one chunk sum each
          __syncwarp();
          if (lane < PWR) {
            const int sq = lane / RPW, q = lane % RPW;
            const int jr = warp + NW * q;
            gu[(jr / R) * 32 + sq * R + jr % R] = chunk_sum(redw + lane * 33, nch);
          }
        }
      } else {
        for (int st = 0; st < SPU; ++st) {
          if (!bad) bad = __any_sync(0xffffffffu, *reinterpret_cast<volatile int *>(&s_abort) != 0);
          if (!bad) {
            bad = !mbar_wait(full + s, ph, a.status, kDetGuFull, a.wait_limit);
            bad = __any_sync(0xffffffffu, bad);
            if (bad && lane == 0) s_abort = 1;
          }
          if (!bad) {
            const unsigned char *sb = stg + (size_t)s * pl.sb;
            uint32_t wv[RPW][CSZ][8];
            float sc[RPW][CSZ];
#pragma unroll
            for (int q = 0; q < RPW; ++q)
              load_row<CSZ>(sb + (size_t)row_m[q] * R * (H / 2) + (size_t)row_r[q] * (H / 2),
                            reinterpret_cast<const __half *>(sb + (size_t)R * H + (size_t)row_m[q] * R * (H / 32) +
                                                             (size_t)row_r[q] * (H / 32)),
                            c0, G, wv[q], sc[q]);
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + s);  // the stage's rows are in registers
            for (int i = 0; i < n_tok; ++i) {
              const int t = __shfl_sync(0xffffffffu, my_tok, i);
              uint32_t act[CSZ][16];
              float dd[CSZ][2];
              int zz[CSZ][2];
              load_act<CSZ>(xq_s + (size_t)(t * 32 + lane) * pl.chp, xd_s + t * HB, qs_s + t * HB, c0, G,
                            act, dd, zz);
#pragma unroll
              for (int q = 0; q < RPW; ++q)
                redw[(q * T + i) * 33 + lane] = chunk_dot<CSZ>(wv[q], sc[q], act, dd, zz, c0, G);
            }
            __syncwarp();
            if (lane < RPW * n_tok) {
              const int q = lane / n_tok, i = lane % n_tok;
              const int jr = warp + NW * q;
              gu[(i * 2 + jr / R) * 32 + st * R + jr % R] = chunk_sum(redw + (q * T + i) * 33, nch);
            }
            __syncwarp();
          }
          if (++s == NS) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      // unit complete: h = SiLU(g) * u for its 32 rows, Q8_0 per token
      named_sync(1, NCT);
      if (!bad) {
        for (int i = warp; i < n_tok; i += NW) {
          const float g = gu[(i * 2 + 0) * 32 + lane];
          const float uv = gu[(i * 2 + 1) * 32 + lane];
          const float h = swiglu(g, uv);
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
      named_sync(1, NCT);
      if (++rb == rbs) {
        rb = 0;
        ++slot;
      }
    }
    prof_end(a.prof, 1);
    return;
  }

  // ------------------------------------------------------ consumers, one token
  const int c0 = lane * CSZ;
  // this lane's activation chunk stays in registers
  uint32_t act1[CSZ][16];
  float d1[CSZ][2];
  int z1[CSZ][2];
  load_act<CSZ>(xq_s + (size_t)lane * pl.chp, xd_s, qs_s, c0, G, act1, d1, z1);
  // this warp's rows of a stage
  int row_m[RPW], row_r[RPW];
#pragma unroll
  for (int q = 0; q < RPW; ++q) {
    const int jr = warp + NW * q;
    row_m[q] = jr / R;
    row_r[q] = jr % R;
  }

  int pos_base = 0;
  int slot = u_begin / rbs, rb = u_begin % rbs, st = 0, s = 0;
  int cu = 0;  // units this CTA has completed
  uint32_t ph = 0;
  bool bad = false;
  for (int j = 0; j < n_stages; ++j) {
    if (st == 0) {  // a new unit: its expert's position
      const int so = a.own[slot];
      pos_base = so == 0 ? a.k : a.off[a.uni[so - 1]];
    }
    if (!bad) bad = __any_sync(0xffffffffu, *reinterpret_cast<volatile int *>(&s_abort) != 0);
    if (!bad) {
      bad = !mbar_wait(full + s, ph, a.status, kDetGuFull, a.wait_limit);
      bad = __any_sync(0xffffffffu, bad);
      if (bad && lane == 0) s_abort = 1;
    }
    if (!bad) {
      const unsigned char *sb = stg + (size_t)s * pl.sb;
      uint32_t wv[RPW][CSZ][8];
      float sc[RPW][CSZ];
#pragma unroll
      for (int q = 0; q < RPW; ++q)
        load_row<CSZ>(sb + (size_t)row_m[q] * R * (H / 2) + (size_t)row_r[q] * (H / 2),
                      reinterpret_cast<const __half *>(sb + (size_t)R * H + (size_t)row_m[q] * R * (H / 32) +
                                                       (size_t)row_r[q] * (H / 32)),
                      c0, G, wv[q], sc[q]);
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + s);  // the stage's rows are in registers
      {
        // chunk values of the warp's PWR rows of the unit, summed once per unit
#pragma unroll
        for (int q = 0; q < RPW; ++q)
          red[(warp * PWR + st * RPW + q) * 33 + lane] = chunk_dot<CSZ>(wv[q], sc[q], act1, d1, z1, c0, G);
        if (st == SPU - 1) {
          __syncwarp();
          if (lane < PWR) {
            const int sq = lane / RPW, q = lane % RPW;
            const int jr = warp + NW * q;
            gu[(cu & 1) * 64 + (jr / R) * 32 + sq * R + jr % R] = chunk_sum(red + (warp * PWR + lane) * 33, nch);
          }
          __syncwarp();
        }
      }
    }
    if (st == SPU - 1) {
      // unit complete: one warp (rotating with the unit) waits for the
      // others' g and u sums and forms h = SiLU(g) * u and its Q8_0 block;
      // the rest arrive and go on to the next unit.  The sums sit in one of
      // two buffers and barriers by unit parity: the ring of NS < 2 units of
      // stages keeps every warp within one unit of the slowest, so a buffer
      // is rewritten only after its reader is done with it.
      const int par = cu & 1;
      __threadfence_block();
      if (cu % NW == warp) {
        named_sync(2 + par, NCT);
        if (!bad) {
          const float *gb = gu + par * 64;
          const float h = swiglu(gb[lane], gb[32 + lane]);
          const float d = fdiv(warp_max(fabsf(h)), 127.0f);
          const int q = q8_code(h, d);
          a.hq[(size_t)pos_base * I + rb * 32 + lane] = (int8_t)q;
          int qsum = q;
#pragma unroll
          for (int off = 16; off >= 1; off >>= 1) qsum += __shfl_xor_sync(0xffffffffu, qsum, off);
          if (lane == 0) {
            a.hd[(size_t)pos_base * (I / 32) + rb] = d;
            a.hqs[(size_t)pos_base * (I / 32) + rb] = qsum;
          }
        }
      } else {
        named_arrive(2 + par, NCT);
      }
      ++cu;
    }
    if (++s == NS) {
      s = 0;
      ph ^= 1u;
    }
    if (++st == SPU) {
      st = 0;
      if (++rb == rbs) {
        rb = 0;
        ++slot;
      }
    }
  }
  named_sync(1, NCT);  // the end stamp follows the last unit's epilogue
  prof_end(a.prof, 1);
}

static int gu_csz(int H) { return (H / 64 + 31) / 32; }

size_t gateup_smem_bytes(int H, int T, int R, int nstage) {
  return gu_plan(H, T, R, nstage, gu_csz(H)).total;
}

// Rows per matrix per stage and stage count: 8 rows (two per warp) when three
// or more stages of that size fit, else 4.  At most 6 stages: fewer than the
// 2 x 32 / R stages of two units, which the single-token epilogue hand-off
// relies on.
void gateup_plan(int H, int T, int *R, int *nstage) {
  for (int r = 8; r >= 4; r -= 4) {
    int ns = 8;
    while (ns >= 2 && gateup_smem_bytes(H, T, r, ns) > (size_t)kMaxSmem) --ns;
    if (ns >= 3 || r == 4) {
      *R = r;
      *nstage = ns > 6 ? 6 : ns;
      return;
    }
  }
}

template <int CSZ, bool ONE, int R, int NW = 8>
static cudaError_t launch_gu(const GateUpArgs &a, int grid, size_t smem, cudaStream_t s) {
  static int smem_set[64] = {0};
  cudaError_t err = ensure_smem(k_gateup_decode<CSZ, ONE, R, NW>, smem, smem_set);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(NW * 32 + 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.use_pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k_gateup_decode<CSZ, ONE, R, NW>, a);
}

template <int CSZ>
static cudaError_t launch_gu_csz(const GateUpArgs &a, int grid, size_t smem, cudaStream_t s) {
  const bool one = a.T == 1;
  // 8 consumer warps.  The consumers, not the copies, bound this kernel (the
  // producer waits for a free stage over half its time), but 16 consumer
  // warps (NW = 16) measured slower: 17 warps per CTA cap the registers at 96
  // and the hot loop spills (36.8 us against 27.5 us per launch).
  if (a.rpm == 8)
    return one ? launch_gu<CSZ, true, 8>(a, grid, smem, s) : launch_gu<CSZ, false, 8>(a, grid, smem, s);
  return one ? launch_gu<CSZ, true, 4>(a, grid, smem, s) : launch_gu<CSZ, false, 4>(a, grid, smem, s);
}

cudaError_t launch_gateup_decode(const GateUpArgs &a, int grid, size_t smem, cudaStream_t s) {
  if (a.rpm != 4 && a.rpm != 8) return cudaErrorInvalidValue;
  switch (gu_csz(a.H)) {
    case 1: return launch_gu_csz<1>(a, grid, smem, s);
    case 2: return launch_gu_csz<2>(a, grid, smem, s);
    case 3: return launch_gu_csz<3>(a, grid, smem, s);
    case 4: return launch_gu_csz<4>(a, grid, smem, s);
    default: return cudaErrorInvalidValue;
  }
}

// ===========================================================================
// down + combine
//
// CTA c owns output rows [m0, m1) (balanced, in row groups of rg rows so every
// scale copy is a multiple of 16 bytes) and loops over the union slots; one
// stage = that slot's rows (or a sub-range of RS rows when the whole range
// does not fit three stages).  y per (position, row) stays in shared memory;
// the combine out = y_shared, then fmaf(w_s, y_s, out) in slot order, runs in
// the same CTA at the end (deterministic, no atomics).
// ===========================================================================
constexpr int kDnTokBatch = 4;

struct DnPlan {
  size_t red, ysm, act, stg, total;
  uint32_t sb;
};

// Bytes of the per-position activations (codes, scales, code sums) when they
// are small enough to keep in shared memory for the whole kernel, else 0.
__host__ __device__ inline size_t dn_act_bytes(int I, int k, int T) {
  const size_t P = (size_t)T * (k + 1);
  const size_t b = P * I + 2 * P * (I / 32) * 4;
  return b <= 48 * 1024 ? b : 0;
}

__host__ __device__ inline DnPlan dn_plan(int I, int k, int T, int rows_max, int rs, int ns) {
  DnPlan p;
  p.sb = (uint32_t)al128d((size_t)rs * (I / 2) + (size_t)rs * (I / 32));
  size_t o = al128d((size_t)16 * ns + 16);
  p.red = o;
  o += al128d((size_t)8 * 32 * 33 * 4);
  p.ysm = o;
  o += al128d((size_t)T * (k + 1) * rows_max * 4);
  p.act = o;
  o += al128d(dn_act_bytes(I, k, T));
  p.stg = o;
  o += (size_t)ns * p.sb;
  p.total = o;
  return p;
}

template <int CSZ, bool ONE>
__global__ void __launch_bounds__(288, 1) k_down_decode(DownArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int H = a.H, I = a.I, T = a.T, K = a.k, NS = a.nstage, RS = a.rs;
  const int G = I / 64, IB = I / 32;
  const int nch = (G + CSZ - 1) / CSZ;
  const DnPlan pl = dn_plan(I, K, T, a.rows_max, RS, NS);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem);
  uint64_t *empty = full + NS;
  uint64_t *actbar = empty + NS;
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
    mbar_init(actbar, 1);
    fence_barrier_init();
  }
  // The union comes from the routing kernel, which completed before the gate/up
  // kernel passed its own dependency wait; this grid is scheduled only after
  // that point, so the union and the expert table are read before this grid's
  // wait, and the first ring of weight copies overlaps the gate/up kernel's
  // tail.  The h codes (the gate/up kernel's output) are read after it.
  prof_start(a.prof, 2);
  if (__syncthreads_or(*reinterpret_cast<volatile int32_t *>(a.status) != 0)) return;
  const int nslot = min(max(*a.n_own, 0), a.E + 1);  // the union slots this call computes
  {
    bool bad = false;
    for (int sl = tid; sl < nslot; sl += blockDim.x) {
      const int so = a.own[sl];
      const int e = so == 0 ? a.E : a.uni[so - 1];
      bad |= (reinterpret_cast<uintptr_t>(a.table[e]) & 15u) != 0;
    }
    if (__syncthreads_or(bad)) {
      if (tid == 0) set_status(a.status, MOE_ERR_DEVICE, kDetDnAlign);
      return;
    }
  }
  if (nrows <= 0) return;

  // small batches: the h codes, scales and code sums of every position come
  // into shared memory once (one TMA transaction) instead of per stage
  const int P = T * (K + 1);
  unsigned char *act_s = smem + pl.act;
  const unsigned char *hq_b = a.preload ? act_s : reinterpret_cast<const unsigned char *>(a.hq);
  const float *hd_b = a.preload ? reinterpret_cast<const float *>(act_s + (size_t)P * I) : a.hd;
  const int *hqs_b =
      a.preload ? reinterpret_cast<const int *>(act_s + (size_t)P * I + (size_t)P * IB * 4) : a.hqs;
  const int n_st = nslot * nsub;

  if (warp == 8) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int s = 0, issued = 0, slot = 0, sub = 0;
      uint32_t ph = 0;
      bool waited = !a.use_pdl, failed = false;
      for (int j = 0; j < n_st; ++j) {
        if (j == NS && !waited) {
          // the ring is full: wait for the gate/up kernel, then its outputs
          pdl_wait();
          waited = true;
          if (*reinterpret_cast<volatile int32_t *>(a.status) != 0) {
            failed = true;
            s_abort = 1;
            break;
          }
          if (a.preload) {
            const uint32_t bq = (uint32_t)P * I, bd = (uint32_t)P * IB * 4;
            mbar_arrive_expect_tx(actbar, bq + 2 * bd);
            bulk_g2s(act_s, a.hq, bq, actbar);
            bulk_g2s(act_s + bq, a.hd, bd, actbar);
            bulk_g2s(act_s + bq + bd, a.hqs, bd, actbar);
          }
        }
        if (j >= NS && !mbar_wait(empty + s, ph ^ 1u, a.status, kDetDnEmpty, a.wait_limit)) {
          s_abort = 1;
          break;
        }
        if (*reinterpret_cast<volatile int *>(&s_abort)) break;
        const int r0 = sub * RS;
        const int nr = min(RS, nrows - r0);
        const uint32_t bytes_pk = (uint32_t)nr * (I / 2), bytes_sc = (uint32_t)nr * (I / 32);
        const int so = a.own[slot];
        const unsigned char *blob = reinterpret_cast<const unsigned char *>(a.table[so == 0 ? a.E : a.uni[so - 1]]);
        unsigned char *dst = stg + (size_t)s * pl.sb;
        mbar_arrive_expect_tx(full + s, bytes_pk + bytes_sc);
        bulk_g2s_hint(dst, blob + pk_off + (size_t)(m0 + r0) * (I / 2), bytes_pk, full + s, pol);
        bulk_g2s_hint(dst + sc_in_stage, blob + sc_off + (size_t)(m0 + r0) * (I / 32), bytes_sc,
                      full + s, pol);
        issued = j + 1;
        if (++s == NS) {
          s = 0;
          ph ^= 1u;
        }
        if (++sub == nsub) {
          sub = 0;
          ++slot;
        }
      }
      if (!waited && !failed) {
        // fewer stages than ring slots
        pdl_wait();
        waited = true;
        if (*reinterpret_cast<volatile int32_t *>(a.status) != 0) {
          failed = true;
          s_abort = 1;
        } else if (a.preload) {
          const uint32_t bq = (uint32_t)P * I, bd = (uint32_t)P * IB * 4;
          mbar_arrive_expect_tx(actbar, bq + 2 * bd);
          bulk_g2s(act_s, a.hq, bq, actbar);
          bulk_g2s(act_s + bq, a.hd, bd, actbar);
          bulk_g2s(act_s + bq + bd, a.hqs, bd, actbar);
        }
      }
      for (int j = (issued > NS ? issued - NS : 0); j < issued; ++j)
        mbar_drain(full + j % NS, (j / NS) & 1, a.status, kDetDnDrain);
      if (a.preload && waited && !failed) mbar_drain(actbar, 0, a.status, kDetDnDrain);
    }
    return;
  }
  // consumers: the gate/up kernel's outputs are read only after its completion.
  // A failure seen here skips the work but not the final named barrier.
  if (a.use_pdl) pdl_wait();
  bool bad = __any_sync(0xffffffffu, *reinterpret_cast<volatile int32_t *>(a.status) != 0);
  if (bad && lane == 0) s_abort = 1;

  const int c0 = lane * CSZ;
  float *redw = red + warp * 32 * 33;
  if (a.preload && !bad) {
    bad = !mbar_wait(actbar, 0, a.status, kDetDnFull, a.wait_limit);
    bad = __any_sync(0xffffffffu, bad);
    if (bad && lane == 0) s_abort = 1;
  }
  int s = 0, slot = 0, sub = 0;
  uint32_t ph = 0;
  for (int j = 0; j < n_st; ++j) {
    const int r0 = sub * RS;
    const int nr = min(RS, nrows - r0);
    int n_tok, pos_base;
    const int so = a.own[slot];
    if (so == 0) {
      n_tok = T;
      pos_base = T * K;
    } else {
      const int e = a.uni[so - 1];
      pos_base = a.off[e];
      n_tok = a.off[e + 1] - pos_base;
    }
    if (!bad) bad = __any_sync(0xffffffffu, *reinterpret_cast<volatile int *>(&s_abort) != 0);
    if (!bad) {
      bad = !mbar_wait(full + s, ph, a.status, kDetDnFull, a.wait_limit);
      bad = __any_sync(0xffffffffu, bad);
      if (bad && lane == 0) s_abort = 1;
    }
    if (!bad) {
      const unsigned char *sb = stg + (size_t)s * pl.sb;
      // this warp's rows of the stage: a contiguous block
      const int rpw = (nr + 7) >> 3;
      const int ra = min(nr, warp * rpw), rz = min(nr, ra + rpw);
      if (ONE || n_tok == 1) {
        // one pair in the slot: activation chunk in registers for the stage
        uint32_t av[CSZ][16];
        float dv[CSZ][2];
        int zv[CSZ][2];
        load_act<CSZ>(hq_b + (size_t)pos_base * I + 64 * c0, hd_b + (size_t)pos_base * IB,
                      hqs_b + (size_t)pos_base * IB, c0, G, av, dv, zv);
        for (int ml = ra; ml < rz; ++ml) {
          uint32_t wv[CSZ][8];
          float sc[CSZ];
          load_row<CSZ>(sb + (size_t)ml * (I / 2),
                        reinterpret_cast<const __half *>(sb + sc_in_stage + (size_t)ml * (I / 32)), c0,
                        G, wv, sc);
          redw[(ml - ra) * 33 + lane] = chunk_dot<CSZ>(wv, sc, av, dv, zv, c0, G);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty + s);
        if (lane < rz - ra)
          ysm[(size_t)pos_base * a.rows_max + r0 + ra + lane] = chunk_sum(redw + lane * 33, nch);
        __syncwarp();
      } else {
        for (int i0 = 0; i0 < n_tok; i0 += kDnTokBatch) {
          const int nb = min(kDnTokBatch, n_tok - i0);
          uint32_t av[kDnTokBatch][CSZ][16];
          float dv[kDnTokBatch][CSZ][2];
          int zv[kDnTokBatch][CSZ][2];
#pragma unroll
          for (int b = 0; b < kDnTokBatch; ++b) {
            const int pos = pos_base + (b < nb ? i0 + b : i0);
            load_act<CSZ>(hq_b + (size_t)pos * I + 64 * c0, hd_b + (size_t)pos * IB,
                          hqs_b + (size_t)pos * IB, c0, G, av[b], dv[b], zv[b]);
          }
          const bool last_batch = i0 + kDnTokBatch >= n_tok;
          // rows in passes so that (row, token) pairs fit the 32 lanes of the sum
          const int ppass = 32 / nb;
          for (int p0 = ra; p0 < rz; p0 += ppass) {
            const int p1 = min(rz, p0 + ppass);
            for (int ml = p0; ml < p1; ++ml) {
              uint32_t wv[CSZ][8];
              float sc[CSZ];
              load_row<CSZ>(sb + (size_t)ml * (I / 2),
                            reinterpret_cast<const __half *>(sb + sc_in_stage + (size_t)ml * (I / 32)),
                            c0, G, wv, sc);
#pragma unroll
              for (int b = 0; b < kDnTokBatch; ++b)
                if (b < nb)
                  redw[((ml - p0) * nb + b) * 33 + lane] = chunk_dot<CSZ>(wv, sc, av[b], dv[b], zv[b], c0, G);
            }
            if (last_batch && p1 == rz) {
              __syncwarp();
              if (lane == 0) mbar_arrive(empty + s);  // every row of this warp is read
            }
            __syncwarp();
            if (lane < (p1 - p0) * nb) {
              const int ml = p0 + lane / nb, b = lane % nb;
              ysm[(size_t)(pos_base + i0 + b) * a.rows_max + r0 + ml] = chunk_sum(redw + lane * 33, nch);
            }
            __syncwarp();
          }
          if (last_batch && ra >= rz) {
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + s);  // this warp had no rows
          }
        }
      }
    }
    if (++s == NS) {
      s = 0;
      ph ^= 1u;
    }
    if (++sub == nsub) {
      sub = 0;
      ++slot;
    }
  }
  named_sync(1, 256);
  if (*reinterpret_cast<volatile int *>(&s_abort)) return;
  for (int i = tid; i < T * nrows; i += 256) {
    const int t = i / nrows, m = i % nrows;
    float o = a.with_shared ? ysm[(size_t)(T * K + t) * a.rows_max + m] : 0.0f;
    for (int q = 0; q < K; ++q) {
      const int e = a.idx[t * K + q];
      if (e < a.e_lo || e >= a.e_hi) continue;  // another rank's expert
      const int p = a.pos[t * K + q];
      o = ffma(a.w[t * K + q], ysm[(size_t)p * a.rows_max + m], o);
    }
    a.out[(size_t)t * H + m0 + m] = o;
  }
  prof_end(a.prof, 2);
  if (a.use_pdl) pdl_launch_dependents();
}

size_t down_smem_bytes(int H, int I, int k, int T, int rows_max, int rs, int nstage) {
  (void)H;
  return dn_plan(I, k, T, rows_max, rs, nstage).total;
}

int down_preload(int I, int k, int T) { return dn_act_bytes(I, k, T) > 0 ? 1 : 0; }

int down_max_stages(int H, int I, int k, int T, int rows_max, int rs) {
  int ns = 6;
  while (ns >= 2 && down_smem_bytes(H, I, k, T, rows_max, rs, ns) > (size_t)kMaxSmem) --ns;
  return ns;
}

template <int CSZ, bool ONE>
static cudaError_t launch_dn(const DownArgs &a, int grid, size_t smem, cudaStream_t s) {
  static int smem_set[64] = {0};
  cudaError_t err = ensure_smem(k_down_decode<CSZ, ONE>, smem, smem_set);
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
  return cudaLaunchKernelEx(&cfg, k_down_decode<CSZ, ONE>, a);
}

cudaError_t launch_down_decode(const DownArgs &a, int grid, size_t smem, cudaStream_t s) {
  const int csz = (a.I / 64 + 31) / 32;
  const bool one = a.T == 1;
  switch (csz) {
    case 1: return one ? launch_dn<1, true>(a, grid, smem, s) : launch_dn<1, false>(a, grid, smem, s);
    case 2: return one ? launch_dn<2, true>(a, grid, smem, s) : launch_dn<2, false>(a, grid, smem, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace moe
