// moe_prefill.cu -- prefill path of the routed-expert MoE layer: one pass over
// the union of the experts a long batch selects (batched expert unions: the
// colibri deep review page, technology table, row I/O 即引擎; batch union:
// tantan.ink page, section 几个关键工程动作).  That a GPU prefill GEMM sums in
// another order than the byte-identical decode path is noted on the tantan.ink
// page, section 我看到的几个坑 (Metal prefill precision); here the decode path
// keeps the fixed order and this path stays within the layer's tolerance.
//
//   k_router_tiled : router logits for many tokens, in the router's fixed
//                    fp32 order (32 strided fmaf chains per logit, xor tree).
//   k_gemm_pf      : grouped GEMM over the expert union on the 5th-generation
//                    tensor cores.  mode 0 = gate/up + SwiGLU + Q8_0 of h,
//                    mode 1 = down into per-pair rows y.
//   k_combine      : out = y_shared + sum_s w_s * y_s, slot order.
//
// The GEMM tile is 128 weight rows (MMA M) by up to 128 token rows of one
// expert (MMA N, a multiple of 16), so an expert with few tokens wastes at most
// 15 columns.  K advances one 64-group per pipeline stage.
//
// Exact block sums on fp16 tensor cores.  The int4 weights (-8..7) and the
// Q8_0 activation codes (-127..127) are small integers, exact in fp16, and
// every product and every 32-element block sum (|sum| <= 32512) is exact in
// the fp32 accumulator.  So tcgen05.mma kind::f16 yields, per 32-block b, the
// exact integer S_b as an fp32 value in TMEM.  The epilogue then applies the
// scales, three fp32 operations per output and 64-group:
//     acc += s_g * (S_0 * d_0 + S_1 * d_1)
// (kind::i8 would return int32 sums and need two more fp32 operations per
// output to convert them; the epilogue's fp32 rate, not the MMA rate, bounds
// this kernel.)  The weights are expanded nibble -> fp16 in shared memory by
// the producer warps: bytes 0x64 0x0u form the half 1024 + u, one packed fp16
// subtraction of 1032 gives u - 8.
//
// Warp roles (13 warps): 0-3 producers (cp.async of packed weights, activation
// rows gathered by token, scales; nibble expansion), 4 MMA issuer (one thread)
// and TMEM owner, 5-12 epilogue (two warps per TMEM lane quarter).  Every wait
// is bounded; a wait that runs out records MOE_ERR_TIMEOUT in the status word
// and every role leaves its loop.
#include <cuda_fp16.h>

#include "moe_device.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// tcgen05 / TMEM / cp.async wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, fp16 x fp16 -> fp32, issued by one thread.
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// The mbarrier receives one arrival once every MMA this thread issued so far is complete.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// cp.async with zero fill: src_bytes = 0 writes zeros and reads nothing.
__device__ __forceinline__ void cp_async16(void *dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Shared-memory operand descriptor, K-major without swizzle: core matrices of
// 8 rows x 16 bytes; the two 16-byte K halves of a 32-byte row slice are 128
// bytes apart (leading offset), consecutive 8-row groups 256 bytes apart
// (stride offset); descriptor version 1 (bit 46).
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)(128u >> 4) << 16;
  d |= (uint64_t)(256u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  return d;
}
// Descriptor of a K-major operand with 128-byte swizzle (rows of 128 bytes,
// 8-row atoms 1024 bytes apart) as a 2D TMA copy with SWIZZLE_128B writes it;
// a K slice of 32 bytes starts 32 bytes further into the row.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

// TMA: one box of a 2D tensor (64 fp16 from column x, rows y ..) into shared
// memory; completion counted on `bar`.  x * 2 bytes is a multiple of 16.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Byte offset of byte kb (0..31) of row `row` in a no-swizzle 32-byte-wide slice.
__host__ __device__ __forceinline__ uint32_t il_off(int row, int kb) {
  return (uint32_t)((row >> 3) * 256 + (kb >> 4) * 128 + (row & 7) * 16 + (kb & 15));
}
// Instruction descriptor: fp32 accumulator, fp16 A and B, both K-major, M = 128.
__device__ __forceinline__ uint32_t pf_idesc(int n) {
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

// Four offset-binary nibbles (one per byte, 0..15) -> four fp16 values u - 8.
__device__ __forceinline__ void nib4_to_f16(uint32_t n, uint32_t &lo, uint32_t &hi) {
  const uint32_t a = __byte_perm(n, 0x64646464u, 0x4140);  // halves 1024 + u0, 1024 + u1
  const uint32_t b = __byte_perm(n, 0x64646464u, 0x4342);  // halves 1024 + u2, 1024 + u3
  const __half2 c = __halves2half2(__ushort_as_half((unsigned short)0x6408), __ushort_as_half((unsigned short)0x6408));
  __half2 ha = *reinterpret_cast<const __half2 *>(&a);
  __half2 hb = *reinterpret_cast<const __half2 *>(&b);
  ha = __hsub2(ha, c);
  hb = __hsub2(hb, c);
  lo = *reinterpret_cast<const uint32_t *>(&ha);
  hi = *reinterpret_cast<const uint32_t *>(&hb);
}


// ===========================================================================
// grouped GEMM
//
// 9 warps per CTA, one CTA per SM, persistent over the CTA's stages (stage =
// one 64-group of one tile; tiles blockIdx.x, + gridDim.x, ...; a tile has an
// even number of stages).
//   copy warp (lane 0): TMA copies of the packed weights (tensor maps built
//     per expert on the device), of the activation rows and of their block
//     scales, as far ahead as the rings allow;
//   MMA warp (lane 0): the 4 MMAs of each stage.
//   8 worker warps, each at its own pace: expand stage i's nibbles to fp16
//     (A buffer i & 1), then apply the scales of stage i-1 to the TMEM block
//     sums and write a tile's outputs after its last group.
// Every hand-off is an mbarrier; every wait is bounded.
// ===========================================================================
constexpr int kPfWorkers = 256;
constexpr int kPfThreads = kPfWorkers + 64;
constexpr int kPfTmaWarp = 8;                // issues the TMA copies
constexpr int kPfMmaWarp = 9;                // issues the MMAs
constexpr int kPfLR = 8, kPfRR = kPfLR + 1;  // packed-weight TMA: stages ahead, ring slots
constexpr int kPfLB = 4, kPfRB = kPfLB + 2;  // activation TMA: stages ahead, ring slots
constexpr int kPfRD = 4;                     // block-scale ring slots (one per stage pair)
constexpr uint32_t kPfTmemCols = 512;        // 2 buffers x 2 blocks x 128 columns
constexpr int kUxPitch = 129;                // up-projection exchange rows (floats), odd: no bank conflicts

constexpr uint32_t kABytes = 16384;   // 4 K-slices x [128 rows x 32 B] fp16 weights, no swizzle
constexpr uint32_t kBBytes = 16384;   // [N rows][128 B] fp16 activations, 128-byte swizzle (N <= 128)
constexpr uint32_t kRawBytes = 4096;  // [128 rows][32 B] packed weights of a group
constexpr uint32_t kDBytes = 2048;    // [N rows][4] fp32 block scales of a stage pair

struct PfLayout {
  uint32_t tile_pre, a, b, raw, d, ux, total;
};
__host__ __device__ inline PfLayout pf_layout(int E) {
  PfLayout L;
  L.tile_pre = 576;
  L.a = (uint32_t)((L.tile_pre + 4 * (E + 2) + 1023) / 1024 * 1024);
  L.b = L.a + 2 * kABytes;
  L.raw = L.b + (uint32_t)kPfRB * kBBytes;
  L.d = L.raw + (uint32_t)kPfRR * kRawBytes;
  L.ux = L.d + (uint32_t)kPfRD * kDBytes;
  L.total = L.ux + 64u * kUxPitch * 4u;
  return L;
}

struct PfTile {
  int e;     // table index (E = the shared expert)
  int wt;    // weight tile
  int p0;    // first pair position of the token tile
  int nval;  // valid token rows
  int n;     // MMA N (nval rounded up to 16)
};

// Tile t -> (slot, weight tile, token tile).  Slot 0 is the shared expert
// (positions T*k ..), slot u >= 1 the union's expert uni[u-1]; inside a slot the
// token tile runs fastest, so CTAs working on neighbouring tiles read the same
// weight rows (one HBM read, the rest from L2).
__device__ __forceinline__ PfTile pf_tile(int t, const int *tile_pre, int nslot, const PfArgs &a) {
  int lo = 0, hi = nslot - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tile_pre[mid] <= t) lo = mid; else hi = mid - 1;
  }
  PfTile r;
  int p0, n;
  if (lo == 0) {
    r.e = a.E;
    p0 = a.T * a.k;
    n = a.T;
  } else {
    r.e = a.uni[lo - 1];
    p0 = a.off[r.e];
    n = a.off[r.e + 1] - p0;
  }
  const int ntt = (n + 127) >> 7;
  const int q = t - tile_pre[lo];
  r.wt = q / ntt;
  const int tt = q - r.wt * ntt;
  r.p0 = p0 + tt * 128;
  r.nval = min(128, n - tt * 128);
  r.n = (r.nval + 15) & ~15;
  return r;
}

// A position in the CTA's stage sequence.
struct PfCur {
  int t, g;
  PfTile tl;
};

__device__ __forceinline__ void tmap_acquire(const CUtensorMap *m) {
  asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;" ::"l"(m) : "memory");
}

template <int MODE>
__global__ void __maxnreg__(160) k_gemm_pf(const PfArgs a, const __grid_constant__ CUtensorMap bmap,
                                           const __grid_constant__ CUtensorMap dmap) {
  // 10 warps: one SM sub-partition holds 3 of them, so at most 16K / 96 = 170 registers.
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = a.H, I = a.I;
  const int K = MODE == 0 ? H : I;
  const int G = K / 64;
  const int NWT = MODE == 0 ? I / 64 : H / 128;
  const PfLayout L = pf_layout(a.E);
  uint64_t *rawfull = reinterpret_cast<uint64_t *>(smem);  // [RR] packed weights landed (TMA bytes)
  uint64_t *rawfree = rawfull + kPfRR;                      // [RR] expanded (8 worker warps)
  uint64_t *bfull = rawfree + kPfRR;                        // [RB] activation rows landed (TMA bytes)
  uint64_t *bfree = bfull + kPfRB;                          // [RB] read by the MMAs (commit)
  uint64_t *aready = bfree + kPfRB;                         // [2]  A buffer written (8 worker warps)
  uint64_t *accf = aready + 2;                              // [2]  accumulators written (commit)
  uint64_t *tfree = accf + 2;                               // [2]  accumulators read (8 worker warps)
  uint64_t *dfull = tfree + 2;                              // [RD] block scales landed (TMA bytes)
  uint64_t *dfree = dfull + kPfRD;                          // [RD] read (8 worker warps)
  uint64_t *uxw = dfree + kPfRD;                            // up rows handed over (8 worker warps)
  uint64_t *uxr = uxw + 1;                                  // up rows consumed (8 worker warps)
  uint64_t *drain = uxr + 1;                                // teardown
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + 512);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + 516);
  int *s_ntiles = reinterpret_cast<int *>(smem + 520);
  int *tile_pre = reinterpret_cast<int *>(smem + L.tile_pre);
  unsigned char *abuf = smem + L.a;
  unsigned char *bbuf = smem + L.b;
  unsigned char *raw = smem + L.raw;
  unsigned char *dsm = smem + L.d;
  float *ux = reinterpret_cast<float *>(smem + L.ux);

  if (*reinterpret_cast<volatile int32_t *>(a.status) != 0) return;
  const int n_uni = min(max(*a.n_uni, 0), a.E);
  const int nslot = n_uni + 1;

  if (tid == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kPfRR; ++s) {
      mbar_init(rawfull + s, 1);
      mbar_init(rawfree + s, 8);
    }
    for (int s = 0; s < kPfRB; ++s) {
      mbar_init(bfull + s, 1);
      mbar_init(bfree + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(aready + b, 8);
      mbar_init(accf + b, 1);
      mbar_init(tfree + b, 8);
    }
    for (int s = 0; s < kPfRD; ++s) {
      mbar_init(dfull + s, 1);
      mbar_init(dfree + s, 8);
    }
    mbar_init(uxw, 8);
    mbar_init(uxr, 8);
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    // tiles per slot, exclusive prefix over the slots
    int run = 0;
    for (int s0 = 0; s0 < nslot; s0 += 32) {
      const int s = s0 + lane;
      int nt = 0;
      if (s < nslot) {
        int n;
        if (s == 0) {
          n = a.T;
        } else {
          const int e = a.uni[s - 1];
          n = a.off[e + 1] - a.off[e];
        }
        nt = ((max(n, 0) + 127) >> 7) * NWT;
      }
      int incl = nt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (s < nslot) tile_pre[s] = run + incl - nt;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      tile_pre[nslot] = run;
      *s_ntiles = run;
    }
    tmem_alloc(tmem_slot, kPfTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_tiles = *s_ntiles;
  const int my_tiles = blockIdx.x < (unsigned)n_tiles ? (n_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int S = my_tiles * G;  // stages of this CTA

  auto cur_begin = [&](PfCur &c) {
    c.t = blockIdx.x;
    c.g = 0;
    if (c.t < n_tiles) c.tl = pf_tile(c.t, tile_pre, nslot, a);
  };
  auto cur_next = [&](PfCur &c) {
    if (++c.g == G) {
      c.g = 0;
      c.t += gridDim.x;
      if (c.t < n_tiles) c.tl = pf_tile(c.t, tile_pre, nslot, a);
    }
  };

  if (warp == kPfTmaWarp) {
    // ================================================================ copies
    if (lane == 0) {
      bool bad = false;
      PfCur cr;
      cur_begin(cr);
      int rtile = -1, issued = 0;
      const CUtensorMap *m0 = nullptr, *m1 = nullptr;
      asm volatile("prefetch.tensormap [%0];" ::"l"(&bmap) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(&dmap) : "memory");
      for (int j = 0; j < S && !bad; ++j, cur_next(cr)) {
        // packed weights of stage j
        const int s = j % kPfRR;
        if (j >= kPfRR && !mbar_wait(rawfree + s, (uint32_t)(j / kPfRR - 1) & 1u, a.status, kDetPfEmpty)) {
          bad = true;
          break;
        }
        if (cr.t != rtile) {
          rtile = cr.t;
          const CUtensorMap *em = a.maps + (size_t)cr.tl.e * 3;
          m0 = MODE == 0 ? em : em + 2;
          m1 = em + 1;
          tmap_acquire(m0);
          if (MODE == 0) tmap_acquire(m1);
        }
        unsigned char *dst = raw + (size_t)s * kRawBytes;
        mbar_arrive_expect_tx(rawfull + s, kRawBytes);
        if (MODE == 0) {
          tma_load_2d(dst, m0, cr.g * 32, cr.tl.wt * 64, rawfull + s);
          tma_load_2d(dst + 64 * 32, m1, cr.g * 32, cr.tl.wt * 64, rawfull + s);
        } else {
          tma_load_2d(dst, m0, cr.g * 32, cr.tl.wt * 128, rawfull + s);
        }
        // activation rows of stage j
        const int sb = j % kPfRB;
        if (j >= kPfRB && !mbar_wait(bfree + sb, (uint32_t)(j / kPfRB - 1) & 1u, a.status, kDetPfEmpty)) {
          bad = true;
          break;
        }
        unsigned char *db = bbuf + (size_t)sb * kBBytes;
        mbar_arrive_expect_tx(bfull + sb, (uint32_t)cr.tl.n * 128u);
        for (int i = 0; i < cr.tl.n / (int)kPfBoxRows; ++i)
          tma_load_2d(db + i * (int)kPfBoxRows * 128, &bmap, cr.g * 64, cr.tl.p0 + i * (int)kPfBoxRows, bfull + sb);
        if ((j & 1) == 0) {
          // block scales of groups g, g+1: [N rows][4 floats], 4-float boxes from column 2g
          const int jp = j >> 1, ds = jp % kPfRD;
          if (jp >= kPfRD && !mbar_wait(dfree + ds, (uint32_t)(jp / kPfRD - 1) & 1u, a.status, kDetPfEmpty)) {
            bad = true;
            break;
          }
          unsigned char *dd = dsm + (size_t)ds * kDBytes;
          mbar_arrive_expect_tx(dfull + ds, (uint32_t)cr.tl.n * 16u);
          for (int i = 0; i < cr.tl.n / (int)kPfBoxRows; ++i)
            tma_load_2d(dd + i * (int)kPfBoxRows * 16, &dmap, cr.g * 2, cr.tl.p0 + i * (int)kPfBoxRows, dfull + ds);
        }
        issued = j + 1;
        if (*abort_flag) bad = true;
      }
      if (bad) *abort_flag = 1;
      // teardown: copies issued but not yet landed (only after a failure can
      // some never have been waited for)
      for (int j = max(0, issued - kPfRR); j < issued; ++j)
        mbar_wait(rawfull + j % kPfRR, (uint32_t)(j / kPfRR) & 1u, a.status, kDetPfDrain);
      for (int j = max(0, issued - kPfRB); j < issued; ++j)
        mbar_wait(bfull + j % kPfRB, (uint32_t)(j / kPfRB) & 1u, a.status, kDetPfDrain);
      for (int jp = max(0, (issued + 1) / 2 - kPfRD); jp < (issued + 1) / 2; ++jp)
        mbar_wait(dfull + jp % kPfRD, (uint32_t)(jp / kPfRD) & 1u, a.status, kDetPfDrain);
    }
    __syncwarp();
  } else if (warp == kPfMmaWarp) {
    // ================================================================ MMAs
    if (lane == 0) {
      bool bad = false;
      PfCur cm;
      cur_begin(cm);
      uint64_t adesc[2][4], bdesc[kPfRB][4];
#pragma unroll
      for (int b = 0; b < 2; ++b)
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) adesc[b][k4] = umma_desc(smem_u32(abuf + (size_t)b * kABytes) + k4 * 4096);
#pragma unroll
      for (int r = 0; r < kPfRB; ++r)
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4)
          bdesc[r][k4] = umma_desc_sw128(smem_u32(bbuf + (size_t)r * kBBytes) + (uint32_t)(k4 * 32));
      int done = 0;
      for (int j = 0; j < S && !bad; ++j, cur_next(cm)) {
        const int buf = j & 1, sb = j % kPfRB;
        if (!mbar_wait(aready + buf, (uint32_t)(j >> 1) & 1u, a.status, kDetPfFull) ||
            !mbar_wait(bfull + sb, (uint32_t)(j / kPfRB) & 1u, a.status, kDetPfFull) ||
            (j >= 2 && !mbar_wait(tfree + buf, (uint32_t)((j >> 1) - 1) & 1u, a.status, kDetPfAccFree)) ||
            *abort_flag) {
          bad = true;
          break;
        }
        tc_fence_after();
        const uint32_t idesc = pf_idesc(cm.tl.n);
        const uint32_t d = tmem + (uint32_t)(buf * 256);
        uint64_t bd[4];
#pragma unroll
        for (int r = 0; r < kPfRB; ++r)
          if (r == sb)
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) bd[k4] = bdesc[r][k4];
#pragma unroll
        for (int b = 0; b < 2; ++b)
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            const int k4 = 2 * b + ks;
            umma_f16(d + (uint32_t)(b * 128), buf ? adesc[1][k4] : adesc[0][k4], bd[k4], idesc, (uint32_t)ks);
          }
        umma_commit(accf + buf);
        umma_commit(bfree + sb);
        done = j + 1;
      }
      if (bad) *abort_flag = 1;
      if (done > 0) {
        umma_commit(drain);
        mbar_wait(drain, 0, a.status, kDetPfDrain);
      }
    }
    __syncwarp();
  } else {
    // ================================================================ workers
    bool bad = false;
    const size_t mg = (size_t)I * (size_t)(H / 2) + (size_t)I * (size_t)(H / 64) * 2;  // bytes of gate (= up)
    const int crow = tid & 127, chalf = tid >> 7;  // expansion: row, 16-byte half of its 32 packed bytes
    const int q = warp & 3, half = warp >> 2;      // epilogue: TMEM lane quarter, 16-column chunks half, +2, ..
    const int row = q * 32 + lane;
    const uint32_t tq = tmem + ((uint32_t)(q * 32) << 16);
    // weight scales of this thread's row: 4 bytes (groups g, g+1) per stage
    // pair, loaded one pair ahead
    auto scale_row = [&](const PfTile &tl) -> const uint32_t * {
      const unsigned char *blob = static_cast<const unsigned char *>(a.table[tl.e]);
      if (MODE == 0) {
        const size_t base = row < 64 ? 0 : mg;
        const size_t r = (size_t)tl.wt * 64 + (row & 63);
        return reinterpret_cast<const uint32_t *>(blob + base + (size_t)I * (size_t)(H / 2) + r * (size_t)(H / 64) * 2);
      }
      const size_t r = (size_t)tl.wt * 128 + row;
      return reinterpret_cast<const uint32_t *>(blob + 2 * mg + (size_t)H * (size_t)(I / 2) + r * (size_t)(I / 64) * 2);
    };
    PfCur cw;
    cur_begin(cw);
    uint32_t w_next = 0, w_cur = 0;
    if (S > 0) w_next = __ldg(scale_row(cw.tl) + (cw.g >> 1));
    PfCur ce;
    cur_begin(ce);
    float2 acc[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = make_float2(0.0f, 0.0f);
    int tcount = 0;

    for (int i = 0; i <= S && !bad; ++i) {
      // expansion of stage i: row crow, bytes 16 chalf ..: K-slices chalf (low
      // nibbles) and 2 + chalf (high nibbles)
      if (i < S) {
        if (!__all_sync(0xffffffffu, mbar_wait(rawfull + i % kPfRR, (uint32_t)(i / kPfRR) & 1u, a.status, kDetPfFull))) {
          bad = true;
          break;
        }
        const uint4 src = *reinterpret_cast<const uint4 *>(raw + (size_t)(i % kPfRR) * kRawBytes + crow * 32 + chalf * 16);
        unsigned char *ab = abuf + (size_t)(i & 1) * kABytes;
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
          const int sh = hi * 4;
          uint32_t h[8];
          nib4_to_f16((src.x >> sh) & 0x0F0F0F0Fu, h[0], h[1]);
          nib4_to_f16((src.y >> sh) & 0x0F0F0F0Fu, h[2], h[3]);
          nib4_to_f16((src.z >> sh) & 0x0F0F0F0Fu, h[4], h[5]);
          nib4_to_f16((src.w >> sh) & 0x0F0F0F0Fu, h[6], h[7]);
          unsigned char *dst = ab + (2 * hi + chalf) * 4096;
          *reinterpret_cast<uint4 *>(dst + il_off(crow, 0)) = make_uint4(h[0], h[1], h[2], h[3]);
          *reinterpret_cast<uint4 *>(dst + il_off(crow, 16)) = make_uint4(h[4], h[5], h[6], h[7]);
        }
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(aready + (i & 1));
          mbar_arrive(rawfree + i % kPfRR);
        }
      }
      if (i == 0) continue;
      // scales of stage j = i-1
      const int j = i - 1, buf = j & 1, jp = j >> 1, ds = jp % kPfRD;
      if ((j & 1) == 0) {
        w_cur = w_next;
        cur_next(cw);
        cur_next(cw);
        if (cw.t < n_tiles) w_next = __ldg(scale_row(cw.tl) + (cw.g >> 1));
      }
      if (!__all_sync(0xffffffffu, mbar_wait(accf + buf, (uint32_t)(j >> 1) & 1u, a.status, kDetPfAccFull) &&
                                       mbar_wait(dfull + ds, (uint32_t)(jp / kPfRD) & 1u, a.status, kDetPfFull))) {
        bad = true;
        break;
      }
      tc_fence_after();
      const int nch = ce.tl.n >> 4;
      const float sg = __half2float(__ushort_as_half((unsigned short)((ce.g & 1) ? (w_cur >> 16) : (w_cur & 0xFFFFu))));
      const float2 sg2 = make_float2(sg, sg);
      const float *dp = reinterpret_cast<const float *>(dsm + (size_t)ds * kDBytes) + 2 * (ce.g & 1);  // [col][4]
#pragma unroll
      for (int ci = 0; ci < 4; ++ci) {
        const int c = half + 2 * ci;
        if (c < nch) {
          float2 dv[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) dv[k] = *reinterpret_cast<const float2 *>(dp + (c * 16 + k) * 4);
          uint32_t v0[16], v1[16];
          tmem_ld16(tq + (uint32_t)(buf * 256 + c * 16), v0);
          tmem_ld16(tq + (uint32_t)(buf * 256 + 128 + c * 16), v1);
          tmem_ld_wait();
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const float2 dap = make_float2(dv[2 * jj].x, dv[2 * jj + 1].x);
            const float2 dbp = make_float2(dv[2 * jj].y, dv[2 * jj + 1].y);
            const float2 s0 = make_float2(__uint_as_float(v0[2 * jj]), __uint_as_float(v0[2 * jj + 1]));
            const float2 s1 = make_float2(__uint_as_float(v1[2 * jj]), __uint_as_float(v1[2 * jj + 1]));
            const float2 fb = __ffma2_rn(s1, dbp, __fmul2_rn(s0, dap));
            acc[ci][jj] = __ffma2_rn(sg2, fb, acc[ci][jj]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(tfree + buf);
        if (j & 1) mbar_arrive(dfree + ds);
      }
      if (ce.g == G - 1) {
        // the tile's outputs
        const PfTile tl = ce.tl;
        if (MODE == 1) {
          float *yc = a.y + (size_t)tl.p0 * H + (size_t)tl.wt * 128 + row;
#pragma unroll
          for (int ci = 0; ci < 4; ++ci) {
            const int c = half + 2 * ci;
            if (c < nch) {
#pragma unroll
              for (int jj = 0; jj < 8; ++jj) {
                const int col = c * 16 + 2 * jj;
                if (col < tl.nval) yc[(size_t)col * H] = acc[ci][jj].x;
                if (col + 1 < tl.nval) yc[(size_t)(col + 1) * H] = acc[ci][jj].y;
              }
            }
          }
        } else {
          // Rows 64..127 hold u of rows 0..63 (g): hand u over, then SwiGLU and
          // Q8_0 of h along I (one 32-block = one warp's lanes), per token.
          if (q >= 2) {
            if (tcount > 0 &&
                !__all_sync(0xffffffffu, mbar_wait(uxr, (uint32_t)(tcount - 1) & 1u, a.status, kDetPfFull))) {
              bad = true;
              break;
            }
#pragma unroll
            for (int ci = 0; ci < 4; ++ci) {
              const int c = half + 2 * ci;
              if (c < nch) {
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                  ux[(row - 64) * kUxPitch + c * 16 + 2 * jj] = acc[ci][jj].x;
                  ux[(row - 64) * kUxPitch + c * 16 + 2 * jj + 1] = acc[ci][jj].y;
                }
              }
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(uxw);
          if (!__all_sync(0xffffffffu, mbar_wait(uxw, (uint32_t)tcount & 1u, a.status, kDetPfFull))) {
            bad = true;
            break;
          }
          if (q < 2) {
            // h = SiLU(g) * u and its Q8_0 codes in fast fp32 (this path is held
            // to the layer's tolerance, not to the fixed-order bits)
            const int ii = tl.wt * 64 + row;  // row of I
            __half *hh = static_cast<__half *>(a.hh);
#pragma unroll
            for (int ci = 0; ci < 4; ++ci) {
              const int c = half + 2 * ci;
              if (c < nch) {
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                  const int col = c * 16 + jj;
                  const float gv = (jj & 1) ? acc[ci][jj >> 1].y : acc[ci][jj >> 1].x;
                  const float h = __fdividef(gv, 1.0f + __expf(-gv)) * ux[row * kUxPitch + col];
                  const float amax = warp_max(fabsf(h));
                  const float d = amax * (1.0f / 127.0f);
                  const float inv = amax > 0.0f ? __fdividef(127.0f, amax) : 0.0f;
                  const int qv = (int)fminf(fmaxf(rintf(h * inv), -127.0f), 127.0f);
                  if (col < tl.nval) {
                    const size_t p = (size_t)(tl.p0 + col);
                    a.hq[p * I + ii] = (int8_t)qv;
                    hh[p * I + ii] = __int2half_rn(qv);
                    if (lane == 0) a.hd[p * (I / 32) + ii / 32] = d;
                  }
                }
              }
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(uxr);
          ++tcount;
        }
#pragma unroll
        for (int ci = 0; ci < 4; ++ci)
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) acc[ci][jj] = make_float2(0.0f, 0.0f);
      }
      cur_next(ce);
      if (*abort_flag) bad = true;
    }
    if (bad) *abort_flag = 1;
  }
  // teardown: every copy and MMA of this CTA has completed (see the control warp)
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kPfTmemCols);
  }
}

// Tensor maps of the packed weights of the union's experts and the shared
// expert, [E+1][gate, up, down], from host-encoded templates (the global
// address patched per expert).  A blob that is not 16-byte aligned sets
// MOE_ERR_DEVICE and gets no maps.
__global__ void __launch_bounds__(32) k_make_maps(const PfArgs a, const __grid_constant__ CUtensorMap tgu,
                                                 const __grid_constant__ CUtensorMap tdn, CUtensorMap *maps) {
  const int e = blockIdx.x;
  if (e < a.E && a.off[e + 1] == a.off[e]) return;  // not in the union
  const unsigned char *blob = static_cast<const unsigned char *>(a.table[e]);
  if ((reinterpret_cast<uintptr_t>(blob) & 15) != 0) {
    if (threadIdx.x == 0) set_status(a.status, MOE_ERR_DEVICE, kDetPfAlign);
    return;
  }
  const size_t mg = (size_t)a.I * (size_t)(a.H / 2) + (size_t)a.I * (size_t)(a.H / 64) * 2;
  CUtensorMap *em = maps + (size_t)e * 3;
  const uint32_t *sgu = reinterpret_cast<const uint32_t *>(&tgu);
  const uint32_t *sdn = reinterpret_cast<const uint32_t *>(&tdn);
  const int m = threadIdx.x >> 5;  // one warp: 32 words per map, three maps in turn
  (void)m;
  for (int mi = 0; mi < 3; ++mi) {
    uint32_t *dst = reinterpret_cast<uint32_t *>(em + mi);
    dst[threadIdx.x] = (mi == 2 ? sdn : sgu)[threadIdx.x];
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    for (int mi = 0; mi < 3; ++mi) {
      const unsigned char *base = blob + (size_t)mi * mg;
      asm volatile("tensormap.replace.tile.global_address.global.b1024.b64 [%0], %1;" ::"l"(em + mi), "l"(base)
                   : "memory");
    }
    asm volatile("fence.proxy.tensormap::generic.release.gpu;" ::: "memory");
  }
}

size_t pf_smem_bytes(int E) { return pf_layout(E).total; }

cudaError_t launch_make_maps(const PfArgs &a, const CUtensorMap &tgu, const CUtensorMap &tdn, cudaStream_t s) {
  k_make_maps<<<a.E + 1, 32, 0, s>>>(a, tgu, tdn, const_cast<CUtensorMap *>(a.maps));
  return cudaGetLastError();
}

cudaError_t launch_gemm_pf(const PfArgs &a, const CUtensorMap &bmap, const CUtensorMap &dmap, int grid, cudaStream_t s) {
  const size_t smem = pf_layout(a.E).total;
  if (smem > (size_t)kMaxSmem) return cudaErrorInvalidConfiguration;
  cudaError_t err;
  if (a.mode == 0) {
    static int smem_set0[64] = {0};
    err = ensure_smem(k_gemm_pf<0>, smem, smem_set0);
    if (err != cudaSuccess) return err;
    k_gemm_pf<0><<<grid, kPfThreads, smem, s>>>(a, bmap, dmap);
  } else {
    static int smem_set1[64] = {0};
    err = ensure_smem(k_gemm_pf<1>, smem, smem_set1);
    if (err != cudaSuccess) return err;
    k_gemm_pf<1><<<grid, kPfThreads, smem, s>>>(a, bmap, dmap);
  }
  return cudaGetLastError();
}

// ===========================================================================
// Router logits for long batches in the router's fixed order: logit(t, e) is
// the xor-tree sum over 32 chains, chain l = fmaf over h = 32 i + l with i
// ascending.  A CTA holds 16 tokens x 32 experts; a warp keeps 8 x 8 logits,
// lane l owning chain l of each.  x and Wr come through shared memory in K
// chunks of 512.
// ===========================================================================
constexpr int kRtTok = 16, kRtExp = 32, kRtKC = 512;

__global__ void __launch_bounds__(256) k_router_tiled(const RouterTiledArgs a) {
  extern __shared__ __align__(16) float rsm[];
  float *xs = rsm;                    // [kRtTok][kRtKC]
  float *wsm = rsm + kRtTok * kRtKC;  // [kRtExp][kRtKC]
  const int H = a.H, E = a.E, T = a.T;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kRtTok, e0 = blockIdx.y * kRtExp;
  const int tw = (warp & 1) * 8, ew = (warp >> 1) * 8;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;
  for (int k0 = 0; k0 < H; k0 += kRtKC) {
    const int kc = min(kRtKC, H - k0);  // a multiple of 128
    const int kc4 = kc / 4;
    __syncthreads();
    for (int i = threadIdx.x; i < kRtTok * kc4; i += 256) {
      const int r = i / kc4, c = i - r * kc4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (t0 + r < T) v = __ldg(reinterpret_cast<const float4 *>(a.x + (size_t)(t0 + r) * H + k0) + c);
      reinterpret_cast<float4 *>(xs + r * kRtKC)[c] = v;
    }
    for (int i = threadIdx.x; i < kRtExp * kc4; i += 256) {
      const int r = i / kc4, c = i - r * kc4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (e0 + r < E) v = __ldg(reinterpret_cast<const float4 *>(a.Wr + (size_t)(e0 + r) * H + k0) + c);
      reinterpret_cast<float4 *>(wsm + r * kRtKC)[c] = v;
    }
    __syncthreads();
    for (int k = lane; k < kc; k += 32) {
      float xv[8], wv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) xv[i] = xs[(tw + i) * kRtKC + k];
#pragma unroll
      for (int j = 0; j < 8; ++j) wv[j] = wsm[(ew + j) * kRtKC + k];
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = ffma(xv[i], wv[j], acc[i][j]);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float v = acc[i][j];
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) v = fadd(v, __shfl_xor_sync(0xffffffffu, v, off));
      const int t = t0 + tw + i, e = e0 + ew + j;
      if (lane == 0 && t < T && e < E) a.logits[(size_t)t * E + e] = v;
    }
}

cudaError_t launch_router_tiled(const RouterTiledArgs &a, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  const size_t smem = (size_t)(kRtTok + kRtExp) * kRtKC * 4;
  static int smem_set[64] = {0};
  cudaError_t err = ensure_smem(k_router_tiled, smem, smem_set);
  if (err != cudaSuccess) return err;
  const dim3 grid((unsigned)((a.T + kRtTok - 1) / kRtTok), (unsigned)((a.E + kRtExp - 1) / kRtExp));
  k_router_tiled<<<grid, 256, smem, s>>>(a);
  return cudaGetLastError();
}

// ===========================================================================
// x's fp16 codes in pair order: xg[p] = xh[pair_tok[p]] (the gate/up GEMM's
// activation rows, copied by TMA boxes of consecutive rows).
// ===========================================================================
__global__ void __launch_bounds__(256) k_gather_rows(const GatherRowsArgs a) {
  const int64_t P = (int64_t)a.T * (a.k + 1);
  const int w = a.H / 8;  // 16-byte units per row
  const int64_t n = P * w;
  const uint4 *src = static_cast<const uint4 *>(a.xh);
  uint4 *dst = static_cast<uint4 *>(a.xg);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t p = i / w, c = i - p * w;
    dst[i] = src[(int64_t)a.pair_tok[p] * w + c];
  }
}

cudaError_t launch_gather_rows(const GatherRowsArgs &a, cudaStream_t s) {
  const int64_t n = (int64_t)a.T * (a.k + 1) * (a.H / 8);
  if (n == 0) return cudaSuccess;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  k_gather_rows<<<(unsigned)blocks, 256, 0, s>>>(a);
  return cudaGetLastError();
}

// ===========================================================================
// x's Q8_0 block scales in pair order (rows of H/32): the gate/up GEMM copies
// a tile's scales of two groups as 4-float boxes.
// ===========================================================================
__global__ void __launch_bounds__(256) k_gather_scales(const GatherScaleArgs a) {
  const int64_t P = (int64_t)a.T * (a.k + 1);
  const int64_t n = P * a.nb;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t p = i / a.nb, b = i - p * a.nb;
    a.xdp[i] = a.xd[(int64_t)a.pair_tok[p] * a.nb + b];
  }
}

cudaError_t launch_gather_scales(const GatherScaleArgs &a, cudaStream_t s) {
  const int64_t n = (int64_t)a.T * (a.k + 1) * a.nb;
  if (n == 0) return cudaSuccess;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 148 * 8) blocks = 148 * 8;
  k_gather_scales<<<(unsigned)blocks, 256, 0, s>>>(a);
  return cudaGetLastError();
}

// ===========================================================================
// Combine: out[t] = y[shared(t)], then out = fmaf(w[t,s], y[pos(t,s)], out) for
// s = 0..k-1 -- the layer's combine order.
// ===========================================================================
__global__ void __launch_bounds__(256) k_combine(const CombineArgs a) {
  const int H4 = a.H / 4;
  const int64_t n = (int64_t)a.T * H4;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int t = (int)(i / H4), c = (int)(i - (int64_t)t * H4);
    float4 o = reinterpret_cast<const float4 *>(a.y + ((size_t)a.T * a.k + t) * a.H)[c];
    for (int s = 0; s < a.k; ++s) {
      const float w = a.w[(size_t)t * a.k + s];
      const float4 v = reinterpret_cast<const float4 *>(a.y + (size_t)a.pos[(size_t)t * a.k + s] * a.H)[c];
      o.x = ffma(w, v.x, o.x);
      o.y = ffma(w, v.y, o.y);
      o.z = ffma(w, v.z, o.z);
      o.w = ffma(w, v.w, o.w);
    }
    reinterpret_cast<float4 *>(a.out + (size_t)t * a.H)[c] = o;
  }
}

cudaError_t launch_combine(const CombineArgs &a, cudaStream_t s) {
  const int64_t n = (int64_t)a.T * (a.H / 4);
  if (n == 0) return cudaSuccess;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 148 * 8) blocks = 148 * 8;
  k_combine<<<(unsigned)blocks, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace moe
