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
// The GEMM tile is two blocks of 128 weight rows (MMA M = 128 each; for
// gate/up the gate and the up rows of the same 128 intermediate rows) by up to
// 96 token rows of one expert (MMA N, a multiple of 16), so an expert with few
// tokens wastes at most 15 columns.  K advances one 64-group per pipeline
// stage.
//
// Operands.  The int4 weights (-8..7) are exact in fp16; the expansion warps
// turn nibbles into fp16 in tensor memory (bytes 0x64 0x0u form the half
// 1024 + u, one packed fp16 subtraction of 1032 gives u - 8).  The activations
// enter as the dequantised Q8_0 values x^ = q d split into two fp16 numbers,
// hi = fp16(x^) and lo = fp16(x^ - hi), together 22 significant bits.  Per
// K16 slice two tcgen05.mma kind::f16 (hi, then lo) accumulate into one fp32
// TMEM accumulator, so the activation block scales never reach the epilogue:
// per output and 64-group it does one fp32 FMA with the weight scale,
//     acc += s_g * C_g.
// (The exact alternative -- integer codes, one accumulator per 32-block,
// acc += s_g * (S_0 d_0 + S_1 d_1) -- costs three fp32 operations and two TMEM
// reads per output and group, more than the tensor cores' time for the same
// group.)  The down GEMM takes h the same way: the gate/up epilogue writes
// h's Q8_0 codes and scales and the hi/lo split of their product.
//
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
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&v)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

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
// One CTA per SM, persistent over its tiles (blockIdx.x, + gridDim.x, ...);
// a tile is G pipeline stages, one 64-group of K each.  A tile is two blocks
// of 128 weight rows (gate/up: the gate rows and the up rows of the same 128
// intermediate rows; down: 256 consecutive output rows) against up to 96
// token rows of one expert.  23 warps (at most 88 registers per thread):
//   0-15  epilogue: TMEM lane quarter warp & 3, columns 24 * (warp >> 2) ..
//         of both blocks; per stage acc += s_g * C_g in fp32 registers --
//         every group's accumulator is read out, so that no tensor-core
//         accumulation runs longer than one group (the tensor cores' fp32
//         sums lose about 2^-25 relative per accumulation step, which over a
//         whole K of 6144 would flip Q8_0 codes of h); after a tile's last
//         group its outputs (gate/up: SwiGLU and Q8_0 of h in the thread that
//         holds g and u);
//   16-19 expansion: packed nibbles of stage i -> fp16 A operands in tensor
//         memory (thread = weight row = TMEM lane, both blocks);
//   20    weight copies (lane 0): TMA of the packed weights (tensor maps built
//         per expert on the device), as far ahead as the ring allows;
//   21    activation copies (lane 0): TMA of the hi/lo token rows;
//   22    MMAs (lane 0): per block and K16 slice hi then lo, A from tensor
//         memory, B from shared memory;
//   23    idle (completes the last warpgroup for setmaxnreg).
// Launched at 80 registers per thread and split with setmaxnreg: the four
// epilogue warpgroups take 96, the other two give theirs down to 48
// (4 x 128 x 96 + 2 x 128 x 48 = 61440 = 768 x 80; the host checks the
// launch count).
// Shared memory then carries only the activation rows and the packed weights,
// which keeps its bandwidth below the tensor cores' need.  Every hand-off is
// an mbarrier; every wait is bounded.
// ===========================================================================
constexpr int kPfEpiWarps = 16;              // epilogue warps 0..15
constexpr int kPfExpWarp0 = 16;              // expansion warps 16..19
constexpr int kPfRawWarp = 20;
constexpr int kPfActWarp = 21;
constexpr int kPfMmaWarp = 22;
constexpr int kPfThreads = 24 * 32;
constexpr int kPfRegsLaunch = 80;            // registers per thread at launch (checked on the host)
constexpr int kPfRegsEpi = 96;               // epilogue warpgroups after setmaxnreg.inc
constexpr int kPfRegsOther = 48;             // the other two after setmaxnreg.dec
static_assert(4 * 128 * kPfRegsEpi + 2 * 128 * kPfRegsOther <= kPfThreads * kPfRegsLaunch,
              "register split exceeds the launch's registers");
constexpr int kPfTileN = 96;                 // token rows per tile (MMA N <= 96)
constexpr int kPfNA = 2;                     // A operand buffers (tensor memory, 64 columns each)
constexpr int kPfNT = 2;                     // accumulator buffers (tensor memory, 192 columns each)
constexpr int kPfRB = 4;                     // activation ring slots
constexpr int kPfRR = 7;                     // packed-weight ring slots
// Stage j's MMAs complete on mdone[j % MD] (one commit per stage).  Its
// waiters -- the epilogue for stage j, the activation copies for j - RB, the
// expansion for j - NA -- each wait for a stage that the barrier cannot have
// passed: its next completion, stage j + MD, needs work from that waiter first
// (MD >= RB, NA and NT).
constexpr int kPfMD = 4;
constexpr uint32_t kPfTmemCols = 512;
constexpr uint32_t kPfAccCols = 192;         // per buffer: block 0 at +0, block 1 at +96
constexpr uint32_t kPfACol0 = kPfNT * kPfAccCols;  // A buffers from column 384: block b, slice k at +32 b + 8 k
constexpr int kPfEpiCols = 24;
static_assert(kPfMD >= kPfRB && kPfMD >= kPfNA && kPfMD >= kPfNT, "stage-done ring too short");               // token columns per epilogue thread (4 column quarters)

constexpr uint32_t kBHalf = (uint32_t)kPfTileN * 128;  // [96 rows][128 B] fp16, 128-byte swizzle (hi or lo)
constexpr uint32_t kBBytes = 2 * kBHalf;
constexpr uint32_t kRawBlk = 4096;    // [128 rows][32 B] packed weights of a group, one block
constexpr uint32_t kRawBytes = 2 * kRawBlk;

struct PfLayout {
  uint32_t tile_pre, b, raw, total;
};
__host__ __device__ inline PfLayout pf_layout(int E) {
  PfLayout L;
  L.tile_pre = 1024;
  L.b = (uint32_t)((L.tile_pre + 4 * (E + 2) + 1023) / 1024 * 1024);
  L.raw = L.b + (uint32_t)kPfRB * kBBytes;
  L.total = L.raw + (uint32_t)kPfRR * kRawBytes;
  return L;
}

struct PfTile {
  int e;     // table index (E = the shared expert)
  int wt;    // weight tile
  int nblk;  // 128-row weight blocks in the tile (down: 1 for the last tile when H % 256 = 128)
  int p0;    // first pair position of the token tile
  int nval;  // valid token rows
  int n;     // MMA N (nval rounded up to 16)
};

// Tile t -> (slot, weight tile, token tile).  Slot 0 is the shared expert
// (positions T*k ..), slot u >= 1 the union's expert uni[u-1]; inside a slot the
// token tile runs fastest, so CTAs working on neighbouring tiles read the same
// weight rows (one HBM read, the rest from L2).
template <int MODE>
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
  const int ntt = (n + kPfTileN - 1) / kPfTileN;
  const int q = t - tile_pre[lo];
  r.wt = q / ntt;
  const int tt = q - r.wt * ntt;
  r.nblk = (MODE == 1 && 256 * r.wt + 128 >= a.H) ? 1 : 2;
  r.p0 = p0 + tt * kPfTileN;
  r.nval = min(kPfTileN, n - tt * kPfTileN);
  r.n = (r.nval + 15) & ~15;
  return r;
}

// A position in the CTA's stage sequence.
template <int MODE>
struct PfCur {
  int t, g;
  PfTile tl;
};

__device__ __forceinline__ void tmap_acquire(const CUtensorMap *m) {
  asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;" ::"l"(m) : "memory");
}

// All lanes of the warp wait on `bar` (bounded); false when it ran out.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, int32_t *status, int32_t det,
                                          long long limit) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, status, det, limit));
}

// D[tmem] (+)= A[tmem] * B[smem]^T, fp16 x fp16 -> fp32, issued by one thread.
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 16 consecutive TMEM columns of this warp's 32 lanes from registers.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

template <int MODE>
__global__ void __launch_bounds__(kPfThreads, 1) k_gemm_pf(const PfArgs a, const __grid_constant__ CUtensorMap bmap) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = a.H, I = a.I;
  const int K = MODE == 0 ? H : I;
  const int G = K / 64;
  const int NWT = MODE == 0 ? I / 128 : (H + 255) / 256;
  const PfLayout L = pf_layout(a.E);
  uint64_t *rawfull = reinterpret_cast<uint64_t *>(smem);  // [RR] packed weights landed (TMA bytes)
  uint64_t *rawfree = rawfull + kPfRR;                      // [RR] expanded (4 expansion warps)
  uint64_t *bfull = rawfree + kPfRR;                        // [RB] activation rows landed (TMA bytes)
  uint64_t *aready = bfull + kPfRB;                         // [NA] A operands written (4 expansion warps)
  uint64_t *mdone = aready + kPfNA;                         // [MD] the stage's MMAs complete (one commit)
  uint64_t *tfree = mdone + kPfMD;                          // [NT] accumulators read (16 epilogue warps)
  uint64_t *drain = tfree + kPfNT;                          // teardown
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + 512);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + 516);
  int *s_ntiles = reinterpret_cast<int *>(smem + 520);
  int *tile_pre = reinterpret_cast<int *>(smem + L.tile_pre);
  unsigned char *bbuf = smem + L.b;
  unsigned char *raw = smem + L.raw;

  prof_start(a.prof, MODE + 1);
  // one decision for the whole CTA: no barrier below may miss a thread
  if (__syncthreads_or(*reinterpret_cast<volatile int32_t *>(a.status) != 0)) return;
  const int n_uni = min(max(*a.n_uni, 0), a.E);
  const int nslot = n_uni + 1;

  if (tid == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kPfRR; ++s) {
      mbar_init(rawfull + s, 1);
      mbar_init(rawfree + s, 4);
    }
    for (int s = 0; s < kPfRB; ++s) mbar_init(bfull + s, 1);
    for (int s = 0; s < kPfNA; ++s) mbar_init(aready + s, 4);
    for (int s = 0; s < kPfMD; ++s) mbar_init(mdone + s, 1);
    for (int s = 0; s < kPfNT; ++s) mbar_init(tfree + s, kPfEpiWarps);
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
        nt = ((max(n, 0) + kPfTileN - 1) / kPfTileN) * NWT;
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

  auto cur_begin = [&](PfCur<MODE> &c) {
    c.t = blockIdx.x;
    c.g = 0;
    if (c.t < n_tiles) c.tl = pf_tile<MODE>(c.t, tile_pre, nslot, a);
  };
  auto cur_next = [&](PfCur<MODE> &c) {
    if (++c.g == G) {
      c.g = 0;
      c.t += gridDim.x;
      if (c.t < n_tiles) c.tl = pf_tile<MODE>(c.t, tile_pre, nslot, a);
    }
  };

  if (warp >= kPfRawWarp) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kPfRegsOther));
  if (warp == kPfRawWarp) {
    // ======================================================= weight copies
    if (lane == 0) {
      bool bad = false;
      PfCur<MODE> cr;
      cur_begin(cr);
      int rtile = -1, issued = 0;
      const CUtensorMap *m0 = nullptr, *m1 = nullptr;
      for (int j = 0; j < S && !bad; ++j, cur_next(cr)) {
        const int s = j % kPfRR;
        if (j >= kPfRR && !mbar_wait(rawfree + s, (uint32_t)(j / kPfRR - 1) & 1u, a.status, kDetPfEmpty, a.wait_limit)) {
          bad = true;
          break;
        }
        if (cr.t != rtile) {
          rtile = cr.t;
          const CUtensorMap *em = a.maps + (size_t)cr.tl.e * 3;
          m0 = MODE == 0 ? em : em + 2;
          m1 = MODE == 0 ? em + 1 : em + 2;
          tmap_acquire(m0);
          if (MODE == 0) tmap_acquire(m1);
        }
        unsigned char *dst = raw + (size_t)s * kRawBytes;
        const int nb = cr.tl.nblk;
        mbar_arrive_expect_tx(rawfull + s, (uint32_t)nb * kRawBlk);
        if (MODE == 0) {
          tma_load_2d(dst, m0, cr.g * 32, cr.tl.wt * 128, rawfull + s);
          tma_load_2d(dst + kRawBlk, m1, cr.g * 32, cr.tl.wt * 128, rawfull + s);
        } else {
          tma_load_2d(dst, m0, cr.g * 32, cr.tl.wt * 256, rawfull + s);
          if (nb == 2) tma_load_2d(dst + kRawBlk, m1, cr.g * 32, cr.tl.wt * 256 + 128, rawfull + s);
        }
        issued = j + 1;
        if (*abort_flag) bad = true;
      }
      if (bad) *abort_flag = 1;
      // teardown: copies issued but not yet landed
      for (int j = max(0, issued - kPfRR); j < issued; ++j)
        mbar_drain(rawfull + j % kPfRR, (uint32_t)(j / kPfRR) & 1u, a.status, kDetPfDrain);
    }
    __syncwarp();
  } else if (warp == kPfActWarp) {
    // =================================================== activation copies
    if (lane == 0) {
      bool bad = false;
      PfCur<MODE> cb;
      cur_begin(cb);
      int issued = 0;
      asm volatile("prefetch.tensormap [%0];" ::"l"(&bmap) : "memory");
      for (int j = 0; j < S && !bad; ++j, cur_next(cb)) {
        // hi/lo rows of stage j: boxes of kPfBoxRows rows; rows past the
        // tile's own land in unused B rows, rows past the array read zero
        const int sb = j % kPfRB, jp = j - kPfRB;  // jp: the stage that used this slot last
        if (j >= kPfRB &&
            !mbar_wait(mdone + jp % kPfMD, (uint32_t)(jp / kPfMD) & 1u, a.status, kDetPfEmpty, a.wait_limit)) {
          bad = true;
          break;
        }
        unsigned char *db = bbuf + (size_t)sb * kBBytes;
        const int nbox = (cb.tl.n + (int)kPfBoxRows - 1) / (int)kPfBoxRows;
        mbar_arrive_expect_tx(bfull + sb, (uint32_t)nbox * kPfBoxRows * 256u);
        for (int i = 0; i < nbox; ++i) {
          const int y = cb.tl.p0 + i * (int)kPfBoxRows;
          tma_load_2d(db + i * (int)kPfBoxRows * 128, &bmap, cb.g * 128, y, bfull + sb);
          tma_load_2d(db + kBHalf + i * (int)kPfBoxRows * 128, &bmap, cb.g * 128 + 64, y, bfull + sb);
        }
        issued = j + 1;
        if (*abort_flag) bad = true;
      }
      if (bad) *abort_flag = 1;
      for (int j = max(0, issued - kPfRB); j < issued; ++j)
        mbar_drain(bfull + j % kPfRB, (uint32_t)(j / kPfRB) & 1u, a.status, kDetPfDrain);
    }
    __syncwarp();
  } else if (warp == kPfMmaWarp) {
    // ================================================================ MMAs
    if (lane == 0) {
      bool bad = false;
      PfCur<MODE> cm;
      cur_begin(cm);
      // descriptors advance by (byte offset >> 4) in their start-address field
      const uint64_t b0 = umma_desc_sw128(smem_u32(bbuf));
      int done = 0;
      for (int j = 0; j < S && !bad; ++j, cur_next(cm)) {
        const int na = j % kPfNA, sb = j % kPfRB, tb = j % kPfNT;
        if (!mbar_wait(aready + na, (uint32_t)(j / kPfNA) & 1u, a.status, kDetPfFull, a.wait_limit) ||
            !mbar_wait(bfull + sb, (uint32_t)(j / kPfRB) & 1u, a.status, kDetPfFull, a.wait_limit) ||
            (j >= kPfNT && !mbar_wait(tfree + tb, (uint32_t)(j / kPfNT - 1) & 1u, a.status, kDetPfAccFree, a.wait_limit)) ||
            *abort_flag) {
          bad = true;
          break;
        }
        tc_fence_after();
        const uint32_t idesc = pf_idesc(cm.tl.n);
        const uint64_t bd = b0 + (uint64_t)((sb * kBBytes) >> 4);
        for (int blk = 0; blk < cm.tl.nblk; ++blk) {
          const uint32_t d = tmem + (uint32_t)(tb * kPfAccCols + kPfTileN * blk);
          const uint32_t at = tmem + kPfACol0 + (uint32_t)(na * 64 + 32 * blk);
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            umma_f16_ts(d, at + 8 * k4, bd + (uint64_t)((k4 * 32) >> 4), idesc, (uint32_t)(k4 > 0));
            umma_f16_ts(d, at + 8 * k4, bd + (uint64_t)((kBHalf + k4 * 32) >> 4), idesc, 1u);
          }
        }
        umma_commit(mdone + j % kPfMD);
        done = j + 1;
      }
      if (bad) *abort_flag = 1;
      if (done > 0) {
        umma_commit(drain);
        mbar_drain(drain, 0, a.status, kDetPfDrain);
      }
    }
    __syncwarp();
  }
  } else if (warp >= kPfExpWarp0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kPfRegsOther));
    // ================================================================ expansion
    bool bad = false;
    const int q = warp - kPfExpWarp0;   // TMEM lane quarter
    const int r = q * 32 + lane;        // weight row of both blocks = TMEM lane
    const uint32_t tl_a = tmem + ((uint32_t)(q * 32) << 16) + kPfACol0;
    PfCur<MODE> cx;
    cur_begin(cx);
    for (int i = 0; i < S && !bad; ++i, cur_next(cx)) {
      const int ra = i % kPfRR, na = i % kPfNA;
      if (!warp_wait(rawfull + ra, (uint32_t)(i / kPfRR) & 1u, a.status, kDetPfFull, a.wait_limit) ||
          (i >= kPfNA && !warp_wait(mdone + (i - kPfNA) % kPfMD, (uint32_t)((i - kPfNA) / kPfMD) & 1u, a.status,
                                    kDetPfFull, a.wait_limit))) {
        bad = true;
        break;
      }
      tc_fence_after();
      for (int blk = 0; blk < cx.tl.nblk; ++blk) {
        const uint4 *src = reinterpret_cast<const uint4 *>(raw + (size_t)ra * kRawBytes + blk * kRawBlk + r * 32);
        const uint4 s0 = src[0], s1 = src[1];
        // byte j: low nibble = element j, high nibble = element j + 32; column
        // 8 k + c of the block holds elements 16 k + 2 c (low half), + 1
#pragma unroll
        for (int hk = 0; hk < 2; ++hk) {  // K16 slices 2 hk, 2 hk + 1: the low / high nibbles
          uint32_t v[16];
#pragma unroll
          for (int k2 = 0; k2 < 2; ++k2) {
            const uint4 w = k2 ? s1 : s0;
            const int sh = hk * 4;
            nib4_to_f16((w.x >> sh) & 0x0F0F0F0Fu, v[8 * k2 + 0], v[8 * k2 + 1]);
            nib4_to_f16((w.y >> sh) & 0x0F0F0F0Fu, v[8 * k2 + 2], v[8 * k2 + 3]);
            nib4_to_f16((w.z >> sh) & 0x0F0F0F0Fu, v[8 * k2 + 4], v[8 * k2 + 5]);
            nib4_to_f16((w.w >> sh) & 0x0F0F0F0Fu, v[8 * k2 + 6], v[8 * k2 + 7]);
          }
          tmem_st16(tl_a + (uint32_t)(na * 64 + 32 * blk + 16 * hk), v);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(aready + na);
        mbar_arrive(rawfree + ra);
      }
      if (__any_sync(0xffffffffu, *abort_flag != 0)) bad = true;  // one decision per warp
    }
    if (bad) *abort_flag = 1;
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kPfRegsEpi));
    // ================================================================ epilogue
    bool bad = false;
    const size_t mg = (size_t)I * (size_t)(H / 2) + (size_t)I * (size_t)(H / 64) * 2;  // bytes of gate (= up)
    const int q = warp & 3, cq = warp >> 2;  // TMEM lane quarter, 24-column quarter
    const int row = q * 32 + lane;
    const int col0 = cq * kPfEpiCols;
    const uint32_t tq = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)col0;
    // weight scales of this thread's rows of both blocks (fp16 per group), as
    // a row pointer per tile taken one tile ahead (block 1's row lies a fixed
    // distance after block 0's); 4 bytes (groups g, g + 1) each per stage
    // pair, loaded one pair ahead
    const size_t blk1 = MODE == 0 ? mg / 4 : (size_t)128 * (I / 64) / 2;  // in 4-byte words
    auto scale_row = [&](const PfTile &tl) -> const uint32_t * {
      const unsigned char *blob = static_cast<const unsigned char *>(a.table[tl.e]);
      const unsigned char *p;
      if (MODE == 0) {
        const size_t rr = (size_t)tl.wt * 128 + row;
        p = blob + (size_t)I * (size_t)(H / 2) + rr * (size_t)(H / 64) * 2;
      } else {
        const size_t rr = (size_t)tl.wt * 256 + row;
        p = blob + 2 * mg + (size_t)H * (size_t)(I / 2) + rr * (size_t)(I / 64) * 2;
      }
      return reinterpret_cast<const uint32_t *>(p);
    };
    PfCur<MODE> ce;
    cur_begin(ce);
    // this tile's scale row and the next tile's, each with its block count
    const uint32_t *sr = nullptr, *sn = nullptr;
    int nbn = 0;
    auto next_rows = [&](int t) {
      sn = nullptr;
      if (t < n_tiles) {
        const PfTile nt = pf_tile<MODE>(t, tile_pre, nslot, a);
        sn = scale_row(nt);
        nbn = nt.nblk;
      }
    };
    uint32_t w0n = 0, w1n = 0;  // scales of the next stage pair
    if (S > 0) {
      sr = scale_row(ce.tl);
      w0n = __ldg(sr);
      if (ce.tl.nblk == 2) w1n = __ldg(sr + blk1);
      next_rows(ce.t + (int)gridDim.x);
    }
    uint32_t w0c = 0, w1c = 0;
    float acc0[kPfEpiCols], acc1[kPfEpiCols];
#pragma unroll
    for (int i = 0; i < kPfEpiCols; ++i) acc0[i] = acc1[i] = 0.0f;

    for (int j = 0; j < S && !bad; ++j) {
      const int tb = j % kPfNT;
      if ((ce.g & 1) == 0) {
        w0c = w0n;
        w1c = w1n;
        // the pair after this one: in this tile, or the first of the next
        if (ce.g + 2 < G) {
          w0n = __ldg(sr + ((ce.g + 2) >> 1));
          if (ce.tl.nblk == 2) w1n = __ldg(sr + blk1 + ((ce.g + 2) >> 1));
        } else if (sn != nullptr) {
          w0n = __ldg(sn);
          if (nbn == 2) w1n = __ldg(sn + blk1);
        }
      }
      if (!warp_wait(mdone + j % kPfMD, (uint32_t)(j / kPfMD) & 1u, a.status, kDetPfAccFull, a.wait_limit)) {
        bad = true;
        break;
      }
      tc_fence_after();
      if (col0 < ce.tl.n) {
        const int sh = (ce.g & 1) * 16;
        const float s0 = __half2float(__ushort_as_half((unsigned short)(w0c >> sh)));
        const float s1 = __half2float(__ushort_as_half((unsigned short)(w1c >> sh)));
        // eight columns at a time (48 accumulators stay live in registers)
#pragma unroll
        for (int c8 = 0; c8 < kPfEpiCols; c8 += 8) {
          uint32_t v8[8];
          tmem_ld8(tq + (uint32_t)(tb * kPfAccCols + c8), v8);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 8; ++k) acc0[c8 + k] = ffma(s0, __uint_as_float(v8[k]), acc0[c8 + k]);
        }
#pragma unroll
        for (int c8 = 0; c8 < kPfEpiCols; c8 += 8) {
          uint32_t v8[8];
          tmem_ld8(tq + (uint32_t)(tb * kPfAccCols + kPfTileN + c8), v8);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 8; ++k) acc1[c8 + k] = ffma(s1, __uint_as_float(v8[k]), acc1[c8 + k]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tfree + tb);
      if (ce.g == G - 1 && col0 < ce.tl.nval) {
        // the tile's outputs; this thread holds columns col0 .. col0 + 23 of both blocks
        const PfTile tl = ce.tl;
        const int ncol = min(kPfEpiCols, tl.nval - col0);
        if (MODE == 1) {
          float *yc = a.y + (size_t)(tl.p0 + col0) * H + (size_t)tl.wt * 256 + row;
#pragma unroll
          for (int k = 0; k < kPfEpiCols; ++k) {
            if (k < ncol) {
              yc[(size_t)k * H] = acc0[k];
              if (tl.nblk == 2) yc[(size_t)k * H + 128] = acc1[k];
            }
          }
        } else {
          // h = SiLU(g) * u, its Q8_0 codes along I (one 32-block of I = one
          // warp's lanes) and the hi/lo split of the dequantised h for the down
          // GEMM, in fast fp32 (this path is held to the layer's tolerance, not
          // to the fixed-order bits)
          const int ii = tl.wt * 128 + row;  // row of I
          __half *hs = static_cast<__half *>(a.hs);
          const size_t hcol = (size_t)(ii >> 6) * 128 + (ii & 63);
#pragma unroll
          for (int k = 0; k < kPfEpiCols; ++k) {
            const float gv = acc0[k];
            const float h = __fdividef(gv, 1.0f + __expf(-gv)) * acc1[k];
            const float amax = warp_max(fabsf(h));
            const float d = amax * (1.0f / 127.0f);
            const float inv = amax > 0.0f ? __fdividef(127.0f, amax) : 0.0f;
            const int qv = (int)fminf(fmaxf(rintf(h * inv), -127.0f), 127.0f);
            if (k < ncol) {
              const size_t p = (size_t)(tl.p0 + col0 + k);
              a.hq[p * I + ii] = (int8_t)qv;
              if (lane == 0) a.hd[p * (I / 32) + ii / 32] = d;
              const float hv = (float)qv * d;
              const __half hi = __float2half_rn(hv);
              const __half lo = __float2half_rn(hv - __half2float(hi));
              hs[p * (size_t)(2 * I) + hcol] = hi;
              hs[p * (size_t)(2 * I) + hcol + 64] = lo;
            }
          }
        }
      }
      if (ce.g == G - 1) {
#pragma unroll
        for (int k = 0; k < kPfEpiCols; ++k) acc0[k] = acc1[k] = 0.0f;
        // the next tile's scale rows become current; look up the one after
        sr = sn;
        next_rows(ce.t + 2 * (int)gridDim.x);
      }
      cur_next(ce);
      if (__any_sync(0xffffffffu, *abort_flag != 0)) bad = true;  // one decision per warp
    }
    if (bad) *abort_flag = 1;
  }
  // teardown: every copy and MMA of this CTA has completed (see the MMA warp)
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kPfTmemCols);
  }
  prof_end(a.prof, MODE + 1);
}

// Tensor maps of the packed weights of the union's experts and the shared
// expert, [E+1][gate, up, down], from host-encoded templates (the global
// address patched per expert).  A blob that is not 16-byte aligned sets
// MOE_ERR_DEVICE and gets no maps.
__global__ void __launch_bounds__(32) k_make_maps(const PfArgs a, const __grid_constant__ CUtensorMap tgu,
                                                 const __grid_constant__ CUtensorMap tdn, CUtensorMap *maps) {
  const int e = blockIdx.x;
  prof_end(a.prof, 0);
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

// The register split of k_gemm_pf assumes the launch's count: a build that
// gave the kernel fewer registers would leave setmaxnreg.inc waiting.
template <int MODE>
cudaError_t pf_regs_ok() {
  static int ok = 0;  // 1 checked, -1 refused
  if (ok == 0) {
    cudaFuncAttributes fa{};
    const cudaError_t err = cudaFuncGetAttributes(&fa, k_gemm_pf<MODE>);
    if (err != cudaSuccess) return err;
    ok = fa.numRegs == kPfRegsLaunch ? 1 : -1;
  }
  return ok == 1 ? cudaSuccess : cudaErrorInvalidConfiguration;
}

cudaError_t launch_gemm_pf(const PfArgs &a, const CUtensorMap &bmap, int grid, cudaStream_t s) {
  const size_t smem = pf_layout(a.E).total;
  if (smem > (size_t)kMaxSmem) return cudaErrorInvalidConfiguration;
  cudaError_t err = a.mode == 0 ? pf_regs_ok<0>() : pf_regs_ok<1>();
  if (err != cudaSuccess) return err;
  if (a.mode == 0) {
    static int smem_set0[64] = {0};
    err = ensure_smem(k_gemm_pf<0>, smem, smem_set0);
    if (err != cudaSuccess) return err;
    k_gemm_pf<0><<<grid, kPfThreads, smem, s>>>(a, bmap);
  } else {
    static int smem_set1[64] = {0};
    err = ensure_smem(k_gemm_pf<1>, smem, smem_set1);
    if (err != cudaSuccess) return err;
    k_gemm_pf<1><<<grid, kPfThreads, smem, s>>>(a, bmap);
  }
  return cudaGetLastError();
}

// ===========================================================================
// Router logits for long batches in the router's fixed order: logit(t, e) is
// the xor-tree sum over 32 chains, chain l = fmaf over h = 32 i + l with i
// ascending.  A CTA holds 16 tokens x 32 experts; a warp keeps 8 x 8 logits,
// lane l owning chain l of each.  x and Wr come through shared memory in K
// chunks of 256, copied asynchronously one chunk ahead (two buffers).
// ===========================================================================
constexpr int kRtTok = 16, kRtExp = 32, kRtKC = 256;
constexpr int kRtBuf = (kRtTok + kRtExp) * kRtKC;  // floats per K-chunk buffer

// 16-byte asynchronous global -> shared copy; src_bytes = 0 writes zeros.
__device__ __forceinline__ void cp_async16z(void *dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}

__global__ void __launch_bounds__(256) k_router_tiled(const RouterTiledArgs a) {
  extern __shared__ __align__(16) float rsm[];  // 2 x {x [kRtTok][kRtKC], Wr [kRtExp][kRtKC]}
  const int H = a.H, E = a.E, T = a.T;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t0 = blockIdx.x * kRtTok, e0 = blockIdx.y * kRtExp;
  const int tw = (warp & 1) * 8, ew = (warp >> 1) * 8;
  // K-chunk copies run one chunk ahead of the arithmetic (two buffers)
  auto load = [&](int k0, int b) {
    const int kc4 = min(kRtKC, H - k0) / 4;
    float *xs = rsm + b * kRtBuf, *wsm = xs + kRtTok * kRtKC;
    for (int i = tid; i < kRtTok * kc4; i += 256) {
      const int r = i / kc4, c = i - r * kc4;
      const bool ok = t0 + r < T;
      cp_async16z(xs + r * kRtKC + 4 * c, ok ? a.x + (size_t)(t0 + r) * H + k0 + 4 * c : a.x, ok ? 16u : 0u);
    }
    for (int i = tid; i < kRtExp * kc4; i += 256) {
      const int r = i / kc4, c = i - r * kc4;
      const bool ok = e0 + r < E;
      cp_async16z(wsm + r * kRtKC + 4 * c, ok ? a.Wr + (size_t)(e0 + r) * H + k0 + 4 * c : a.Wr, ok ? 16u : 0u);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;
  const int nch = (H + kRtKC - 1) / kRtKC;
  load(0, 0);
  for (int ci = 0; ci < nch; ++ci) {
    if (ci + 1 < nch) {
      load((ci + 1) * kRtKC, (ci + 1) & 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    const int kc = min(kRtKC, H - ci * kRtKC);  // a multiple of 128
    const float *xs = rsm + (ci & 1) * kRtBuf, *wsm = xs + kRtTok * kRtKC;
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
    __syncthreads();  // the buffer is refilled by the next iteration's copies
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
  const size_t smem = (size_t)2 * kRtBuf * 4;
  static int smem_set[64] = {0};
  cudaError_t err = ensure_smem(k_router_tiled, smem, smem_set);
  if (err != cudaSuccess) return err;
  const dim3 grid((unsigned)((a.T + kRtTok - 1) / kRtTok), (unsigned)((a.E + kRtExp - 1) / kRtExp));
  k_router_tiled<<<grid, 256, smem, s>>>(a);
  return cudaGetLastError();
}

// ===========================================================================
// The gate/up GEMM's activation rows in pair order, as an fp16 hi/lo split of
// the Q8_0-dequantised x: for p and h, x^ = q[t][h] * d[t][h / 32] (t =
// pair_tok[p]), hi = fp16(x^), lo = fp16(x^ - hi); row p of xg holds, per
// 64-group g, hi of the group's 64 elements at 128 g and lo at 128 g + 64.
// A thread writes 8 elements (16 bytes of hi, 16 of lo).
// ===========================================================================
__global__ void __launch_bounds__(256) k_gather_rows(const GatherRowsArgs a) {
  const int64_t P = (int64_t)a.T * (a.k + 1);
  const int w = a.H / 8;  // 8-element units per row
  const int64_t n = P * w;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t p = i / w;
    const int h = (int)(i - p * w) * 8;
    const int64_t t = a.pair_tok[p];
    const uint2 qv = *reinterpret_cast<const uint2 *>(a.xq + t * a.H + h);
    const float d = a.xd[t * (a.H / 32) + h / 32];
    const int8_t *qb = reinterpret_cast<const int8_t *>(&qv);
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const float x0 = (float)qb[2 * m] * d, x1 = (float)qb[2 * m + 1] * d;
      const __half h0 = __float2half_rn(x0), h1 = __float2half_rn(x1);
      const __half l0 = __float2half_rn(x0 - __half2float(h0)), l1 = __float2half_rn(x1 - __half2float(h1));
      hi[m] = (uint32_t)__half_as_ushort(h0) | ((uint32_t)__half_as_ushort(h1) << 16);
      lo[m] = (uint32_t)__half_as_ushort(l0) | ((uint32_t)__half_as_ushort(l1) << 16);
    }
    __half *row = static_cast<__half *>(a.xg) + p * (2 * (int64_t)a.H) + (h >> 6) * 128 + (h & 63);
    *reinterpret_cast<uint4 *>(row) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4 *>(row + 64) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
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
  prof_end(a.prof, 2);
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
