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
// Byte offset of byte kb (0..31) of row `row` in such a 32-byte-wide slice.
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

// Bounded wait by every lane of a warp; the verdict is made warp-uniform.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, int32_t *status, int32_t detail,
                                          volatile int *abort_flag) {
  const bool ok = mbar_wait(bar, parity, status, detail) && !*abort_flag;
  return __all_sync(0xffffffffu, ok);
}

// ===========================================================================
// grouped GEMM
// ===========================================================================
constexpr int kPfNS = 5;          // pipeline stages (one 64-group each)
constexpr int kPfLag = 3;         // stages of copies in flight ahead of the nibble expansion
constexpr int kPfWarps = 13;
constexpr int kPfThreads = kPfWarps * 32;
constexpr int kPfMmaWarp = 4;
constexpr int kPfEpi0 = 5;
constexpr uint32_t kPfTmemCols = 512;  // 2 buffers x 2 blocks x 128 columns
constexpr int kUxPitch = 129;          // up-projection exchange rows (floats), odd: no bank conflicts

// stage slot layout (bytes)
constexpr uint32_t kSlotA = 0;         // 4 K-slices x [128 rows x 32 B] fp16 weights
constexpr uint32_t kSlotB = 16384;     // 4 K-slices x [N rows x 32 B] fp16 activations (N <= 128)
constexpr uint32_t kSlotRaw = 32768;   // [128 rows][32 B] packed weights of the group
constexpr uint32_t kSlotD = 36864;     // [2 blocks][128] fp32 activation block scales
constexpr uint32_t kSlotW = 37888;     // [128] u32: the fp16 weight scales of groups g & ~1, g | 1
constexpr uint32_t kSlotBytes = 38400;

struct PfLayout {
  uint32_t stage, ux, total;
};
__host__ __device__ inline PfLayout pf_layout(int E) {
  PfLayout L;
  L.stage = (uint32_t)((256 + 4 * (E + 2) + 1023) / 1024 * 1024);
  L.ux = L.stage + (uint32_t)kPfNS * kSlotBytes;
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

template <int MODE>
__global__ void __launch_bounds__(kPfThreads, 1) k_gemm_pf(const PfArgs a) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = a.H, I = a.I;
  const int K = MODE == 0 ? H : I;
  const int G = K / 64;
  const int NWT = MODE == 0 ? I / 64 : H / 128;
  const PfLayout L = pf_layout(a.E);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem);  // [NS] producers: stage written (128 arrivals)
  uint64_t *empty = full + kPfNS;                       // [NS] MMA commit + 8 epilogue warps
  uint64_t *accf = empty + kPfNS;                       // [2]  accumulator buffer written (MMA commit)
  uint64_t *acce = accf + 2;                            // [2]  accumulator buffer read (8 epilogue warps)
  uint64_t *drain = acce + 2;                           // MMA drain before teardown
  uint64_t *uxw = drain + 1;                            // up rows handed over (8 epilogue warps)
  uint64_t *uxr = uxw + 1;                              // up rows consumed (8 epilogue warps)
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + 192);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + 196);
  int *s_ntiles = reinterpret_cast<int *>(smem + 200);
  int *tile_pre = reinterpret_cast<int *>(smem + 256);
  unsigned char *stage = smem + L.stage;
  float *ux = reinterpret_cast<float *>(smem + L.ux);

  if (*reinterpret_cast<volatile int32_t *>(a.status) != 0) return;
  const int n_uni = min(max(*a.n_uni, 0), a.E);
  const int nslot = n_uni + 1;

  if (tid == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kPfNS; ++s) {
      mbar_init(full + s, 128);
      mbar_init(empty + s, 9);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf + b, 1);
      mbar_init(acce + b, 8);
    }
    mbar_init(drain, 1);
    mbar_init(uxw, 8);
    mbar_init(uxr, 8);
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
  }
  if (warp == kPfMmaWarp) {
    tmem_alloc(tmem_slot, kPfTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_tiles = *s_ntiles;
  const size_t mg = (size_t)I * (size_t)(H / 2) + (size_t)I * (size_t)(H / 64) * 2;  // bytes of gate (= up)

  if (warp < kPfMmaWarp) {
    // ---------------------------------------------------------------- producers
    const int pt = tid;  // weight row of the tile this thread copies and expands
    int st = 0, cv = 0;
    bool bad = false;
    auto expand = [&](int cs) {
      unsigned char *sl = stage + (size_t)(cs % kPfNS) * kSlotBytes;
      const uint4 q0 = *reinterpret_cast<const uint4 *>(sl + kSlotRaw + pt * 32);
      const uint4 q1 = *reinterpret_cast<const uint4 *>(sl + kSlotRaw + pt * 32 + 16);
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) {
        // K-slice k4 holds group elements 16*k4 .. 16*k4+15: low nibbles of
        // bytes 0..15 / 16..31, then high nibbles of the same bytes.
        const uint4 src = (k4 & 1) ? q1 : q0;
        const int sh = (k4 >> 1) * 4;
        uint32_t h[8];
        nib4_to_f16((src.x >> sh) & 0x0F0F0F0Fu, h[0], h[1]);
        nib4_to_f16((src.y >> sh) & 0x0F0F0F0Fu, h[2], h[3]);
        nib4_to_f16((src.z >> sh) & 0x0F0F0F0Fu, h[4], h[5]);
        nib4_to_f16((src.w >> sh) & 0x0F0F0F0Fu, h[6], h[7]);
        unsigned char *dst = sl + kSlotA + k4 * 4096;
        *reinterpret_cast<uint4 *>(dst + il_off(pt, 0)) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4 *>(dst + il_off(pt, 16)) = make_uint4(h[4], h[5], h[6], h[7]);
      }
      fence_proxy_async();
      mbar_arrive(full + cs % kPfNS);
    };
    for (int t = blockIdx.x; t < n_tiles && !bad; t += gridDim.x) {
      const PfTile tl = pf_tile(t, tile_pre, nslot, a);
      const unsigned char *blob = static_cast<const unsigned char *>(a.table[tl.e]);
      if ((reinterpret_cast<uintptr_t>(blob) & 15) != 0) {
        set_status(a.status, MOE_ERR_DEVICE, kDetPfAlign);
        *abort_flag = 1;
        bad = true;
        break;
      }
      const unsigned char *wrow, *srow;
      if (MODE == 0) {
        const size_t base = pt < 64 ? 0 : mg;
        const size_t row = (size_t)tl.wt * 64 + (pt & 63);
        wrow = blob + base + row * (size_t)(H / 2);
        srow = blob + base + (size_t)I * (size_t)(H / 2) + row * (size_t)(H / 64) * 2;
      } else {
        const size_t base = 2 * mg;
        const size_t row = (size_t)tl.wt * 128 + pt;
        wrow = blob + base + row * (size_t)(I / 2);
        srow = blob + base + (size_t)H * (size_t)(I / 2) + row * (size_t)(I / 64) * 2;
      }
      const __half *bsrc = static_cast<const __half *>(a.bsrc);
      for (int g = 0; g < G; ++g) {
        const int s = st % kPfNS;
        const uint32_t u = (uint32_t)(st / kPfNS);
        if (u > 0 && !mbar_wait(empty + s, (u - 1) & 1u, a.status, kDetPfEmpty)) bad = true;
        if (bad || *abort_flag) {
          *abort_flag = 1;
          bad = true;
          break;
        }
        unsigned char *sl = stage + (size_t)s * kSlotBytes;
        cp_async16(sl + kSlotRaw + pt * 32, wrow + g * 32, 16);
        cp_async16(sl + kSlotRaw + pt * 32 + 16, wrow + g * 32 + 16, 16);
        cp_async4(sl + kSlotW + pt * 4, srow + (g & ~1) * 2, 4);
        for (int ch = pt; ch < tl.n * 8; ch += 128) {
          const int r = ch >> 3, cc = ch & 7;
          const bool ok = r < tl.nval;
          const size_t brow = ok ? (MODE == 0 ? (size_t)a.pair_tok[tl.p0 + r] : (size_t)(tl.p0 + r)) : 0;
          cp_async16(sl + kSlotB + (cc >> 1) * (tl.n * 32) + il_off(r, (cc & 1) * 16),
                     bsrc + brow * (size_t)K + g * 64 + cc * 8, ok ? 16u : 0u);
        }
        for (int r = pt; r < tl.n; r += 128) {
          const bool ok = r < tl.nval;
          const size_t brow = ok ? (MODE == 0 ? (size_t)a.pair_tok[tl.p0 + r] : (size_t)(tl.p0 + r)) : 0;
          const float *src = a.bscale + brow * (size_t)(K / 32) + 2 * g;
          float *dd = reinterpret_cast<float *>(sl + kSlotD);
          cp_async4(dd + r, src, ok ? 4u : 0u);
          cp_async4(dd + 128 + r, src + 1, ok ? 4u : 0u);
        }
        cp_async_commit();
        ++st;
        if (st - cv > kPfLag) {
          cp_async_wait<kPfLag>();
          expand(cv++);
        }
      }
    }
    cp_async_wait_all();
    while (!bad && cv < st) expand(cv++);
  } else if (warp == kPfMmaWarp) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int st = 0;
      bool bad = false;
      for (int t = blockIdx.x; t < n_tiles && !bad; t += gridDim.x) {
        const PfTile tl = pf_tile(t, tile_pre, nslot, a);
        const uint32_t idesc = pf_idesc(tl.n);
        for (int g = 0; g < G; ++g, ++st) {
          const int s = st % kPfNS, buf = st & 1;
          const uint32_t u = (uint32_t)(st / kPfNS), nu = (uint32_t)(st >> 1);
          if (!mbar_wait(full + s, u & 1u, a.status, kDetPfFull) ||
              !mbar_wait(acce + buf, (nu & 1u) ^ 1u, a.status, kDetPfAccFree) || *abort_flag) {
            *abort_flag = 1;
            bad = true;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(stage + (size_t)s * kSlotBytes + kSlotA);
          const uint32_t sb = smem_u32(stage + (size_t)s * kSlotBytes + kSlotB);
#pragma unroll
          for (int b = 0; b < 2; ++b)
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
              const int k4 = 2 * b + ks;
              umma_f16(tmem + (uint32_t)(buf * 256 + b * 128), umma_desc(sa + k4 * 4096),
                       umma_desc(sb + (uint32_t)(k4 * tl.n * 32)), idesc, (uint32_t)ks);
            }
          umma_commit(accf + buf);
          umma_commit(empty + s);
        }
      }
      if (st > 0) {  // wait for the MMAs still in flight before TMEM is released
        umma_commit(drain);
        mbar_wait(drain, 0, a.status, kDetPfDrain);
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    const int ew = warp - kPfEpi0;
    const int q = warp & 3;      // TMEM lane quarter this warp may access
    const int half = ew >> 2;    // its 16-column chunks: half, half + 2, ...
    const int row = q * 32 + lane;
    const uint32_t tq = tmem + ((uint32_t)(q * 32) << 16);
    int st = 0, tcount = 0;
    bool bad = false;
    for (int t = blockIdx.x; t < n_tiles && !bad; t += gridDim.x, ++tcount) {
      const PfTile tl = pf_tile(t, tile_pre, nslot, a);
      const int nch = tl.n >> 4;
      float2 acc[4][8];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = make_float2(0.0f, 0.0f);
      for (int g = 0; g < G; ++g, ++st) {
        const int s = st % kPfNS, buf = st & 1;
        const uint32_t u = (uint32_t)(st / kPfNS), nu = (uint32_t)(st >> 1);
        if (!warp_wait(full + s, u & 1u, a.status, kDetPfFull, abort_flag) ||
            !warp_wait(accf + buf, nu & 1u, a.status, kDetPfAccFull, abort_flag)) {
          if (lane == 0) *abort_flag = 1;
          bad = true;
          break;
        }
        tc_fence_after();
        const unsigned char *sl = stage + (size_t)s * kSlotBytes;
        const uint32_t wsv = *reinterpret_cast<const uint32_t *>(sl + kSlotW + row * 4);
        const float sg = __half2float(__ushort_as_half((unsigned short)((g & 1) ? (wsv >> 16) : (wsv & 0xFFFFu))));
        const float2 sg2 = make_float2(sg, sg);
        const float *d0p = reinterpret_cast<const float *>(sl + kSlotD);
        const float *d1p = d0p + 128;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int c = half + 2 * i;
          if (c < nch) {
            uint32_t v0[16], v1[16];
            tmem_ld16(tq + (uint32_t)(buf * 256 + c * 16), v0);
            tmem_ld16(tq + (uint32_t)(buf * 256 + 128 + c * 16), v1);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float2 da = *reinterpret_cast<const float2 *>(d0p + c * 16 + 2 * j);
              const float2 db = *reinterpret_cast<const float2 *>(d1p + c * 16 + 2 * j);
              const float2 s0 = make_float2(__uint_as_float(v0[2 * j]), __uint_as_float(v0[2 * j + 1]));
              const float2 s1 = make_float2(__uint_as_float(v1[2 * j]), __uint_as_float(v1[2 * j + 1]));
              const float2 fb = __ffma2_rn(s1, db, __fmul2_rn(s0, da));
              acc[i][j] = __ffma2_rn(sg2, fb, acc[i][j]);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(acce + buf);
          mbar_arrive(empty + s);
        }
      }
      if (bad) break;
      if (MODE == 1) {
        float *yc = a.y + (size_t)tl.p0 * H + (size_t)tl.wt * 128 + row;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int c = half + 2 * i;
          if (c < nch) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int col = c * 16 + 2 * j;
              if (col < tl.nval) yc[(size_t)col * H] = acc[i][j].x;
              if (col + 1 < tl.nval) yc[(size_t)(col + 1) * H] = acc[i][j].y;
            }
          }
        }
      } else {
        // Rows 64..127 hold u of rows 0..63 (g): hand u over, then SwiGLU and
        // Q8_0 of h along I (one 32-block = one warp's lanes), per token.
        if (q >= 2) {
          if (tcount > 0 && !warp_wait(uxr, (uint32_t)(tcount - 1) & 1u, a.status, kDetPfFull, abort_flag)) {
            if (lane == 0) *abort_flag = 1;
            bad = true;
            break;
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int c = half + 2 * i;
            if (c < nch) {
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                ux[(row - 64) * kUxPitch + c * 16 + 2 * j] = acc[i][j].x;
                ux[(row - 64) * kUxPitch + c * 16 + 2 * j + 1] = acc[i][j].y;
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(uxw);
        if (!warp_wait(uxw, (uint32_t)tcount & 1u, a.status, kDetPfFull, abort_flag)) {
          if (lane == 0) *abort_flag = 1;
          bad = true;
          break;
        }
        if (q < 2) {
          const int ii = tl.wt * 64 + row;  // row of I
          __half *hh = static_cast<__half *>(a.hh);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int c = half + 2 * i;
            if (c < nch) {
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const int col = c * 16 + j;
                const float gv = (j & 1) ? acc[i][j >> 1].y : acc[i][j >> 1].x;
                const float h = swiglu(gv, ux[row * kUxPitch + col]);
                const float d = fdiv(warp_max(fabsf(h)), 127.0f);
                const int qv = q8_code(h, d);
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
      }
    }
  }
  // every role has left its loop; every wait above is bounded
  tc_fence_before();
  __syncthreads();
  if (warp == kPfMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kPfTmemCols);
  }
}

size_t pf_smem_bytes(int E) { return pf_layout(E).total; }

cudaError_t launch_gemm_pf(const PfArgs &a, int grid, cudaStream_t s) {
  const size_t smem = pf_layout(a.E).total;
  if (smem > (size_t)kMaxSmem) return cudaErrorInvalidConfiguration;
  cudaError_t err;
  if (a.mode == 0) {
    err = cudaFuncSetAttribute(k_gemm_pf<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    k_gemm_pf<0><<<grid, kPfThreads, smem, s>>>(a);
  } else {
    err = cudaFuncSetAttribute(k_gemm_pf<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    k_gemm_pf<1><<<grid, kPfThreads, smem, s>>>(a);
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
  cudaError_t err = cudaFuncSetAttribute(k_router_tiled, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const dim3 grid((unsigned)((a.T + kRtTok - 1) / kRtTok), (unsigned)((a.E + kRtExp - 1) / kRtExp));
  k_router_tiled<<<grid, 256, smem, s>>>(a);
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
