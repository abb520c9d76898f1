// moe_internal.h -- definitions shared by the libmoe host code and kernels:
// workspace layout, kernel argument blocks, launcher declarations.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/moe.h"

namespace moe {

constexpr long long kWaitLimitCycles = 2000000000LL;  // ~1 s at 1.9 GHz: default wait limit, and every drain's
constexpr int kMaxK = 32;                              // kernels keep <= 32 slots per token
constexpr int kDecodeTMax = MOE_DECODE_T_MAX;
constexpr int kMaxSmem = 227 * 1024 - 1024;            // dynamic shared memory per CTA (sm_100 opt-in limit, minus static)
constexpr int kPfMaxCtas = 256;                        // prefill GEMM grid bound (one CTA per SM)
constexpr int kProfSlots = 1024;                       // per-call profiling records kept per device
constexpr int kProfWords = 8;                          // per record: 4 phases x (~first start, last end) in ns
// Control words of the workspace, zero at the start of every call: [0] the
// routing kernel's arrival ticket, [1] the fused kernel's routing arrivals,
// [kCtrlReady, +1] the fused kernel's 64-bit ready word, [kCtrlSlot0 + s]
// gate/up units completed for union slot s (fused kernel).  The memset before
// the other paths' launches zeroes them; the fused kernel zeroes its own (CTA 0,
// then the call's sequence number in the ready word).
constexpr int kCtrlReady = 2;
constexpr int kCtrlSlot0 = 4;
// Control words per token of a decode batch (token t's block at kCtrlWords t;
// the fused kernel's per-token launches each use their own block).
constexpr int kCtrlWords = kCtrlSlot0 + kMaxK + 1;
// Expert weight formats of the decode kernels.
constexpr int kFmtInt4 = 0;   // int4 gs64, fp16 group scales
constexpr int kFmtMxfp4 = 1;  // E2M1 codes, one E8M0 exponent per 32-block

// Device-side error details (status[1]) -- which wait or check failed.
enum Detail : int32_t {
  kDetRouteBar = 1,
  kDetRouteDrain = 2,
  kDetGuFull = 10,
  kDetGuEmpty = 11,
  kDetGuDrain = 12,
  kDetGuAlign = 13,
  kDetDnFull = 20,
  kDetDnEmpty = 21,
  kDetDnDrain = 22,
  kDetDnAlign = 23,
  kDetPfAlign = 30,
  kDetPfFull = 31,
  kDetPfEmpty = 32,
  kDetPfAccFull = 33,
  kDetPfAccFree = 34,
  kDetPfDrain = 35,
  kDetFuRoute = 40,
  kDetFuRouteDrain = 41,
  kDetFuGrid = 42,
  kDetFuFull = 43,
  kDetFuEmpty = 44,
  kDetFuDrain = 45,
  kDetFuSlot = 46,
  kDetFuAlign = 47,
  kDetFuReady = 48,
};

// The wait limit kernels launched now take for their work waits (set by
// moe_set_wait_limit; kWaitLimitCycles by default).
long long wait_limit_cycles();

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Raises a kernel's dynamic shared-memory limit once per device (the call
// costs host time on every launch otherwise).  `cache` is the kernel's own
// per-device record; concurrent first calls both set the same value.
template <typename K>
inline cudaError_t ensure_smem(K kernel, size_t smem, int (&cache)[64]) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if ((int)smem <= cache[dev]) return cudaSuccess;
  err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err == cudaSuccess) cache[dev] = (int)smem;
  return err;
}

inline size_t matrix_bytes(int N, int K) {
  return (size_t)N * (size_t)(K / 2) + (size_t)N * (size_t)(K / 64) * 2;
}
inline size_t expert_bytes(int H, int I) { return 2 * matrix_bytes(I, H) + matrix_bytes(H, I); }

// Byte offsets of the workspace segments for batches of up to T tokens.  The
// prefill segments (xg, hs, y, maps) are sized only when `prefill` is set.
struct WsLayout {
  size_t status, ctrl, xin, yout, xq, xd, logits, idx, w, cnt, off, uni, n_uni, own, n_own, perm, pos,
      pair_tok, hq, hqs, hd, xg, hs, y, maps, total;
};

inline WsLayout ws_layout(const moe_dims &d, int T, bool prefill = false) {
  WsLayout L{};
  const size_t P = (size_t)T * (size_t)(d.k + 1);
  size_t o = 0;
  auto seg = [&](size_t bytes) {
    size_t at = o;
    o = align_up(o + (bytes ? bytes : 1), 256);
    return at;
  };
  L.status = seg(16);
  L.ctrl = seg((size_t)kCtrlWords * 4 * (size_t)(T < 1 ? 1 : (T < kDecodeTMax ? T : kDecodeTMax)));
  L.xin = seg((size_t)T * d.H * 4);
  L.yout = seg((size_t)T * d.H * 4);
  L.xq = seg((size_t)T * d.H);
  L.xd = seg((size_t)T * (d.H / 32) * 4);
  L.logits = seg((size_t)T * d.E * 4);
  L.idx = seg((size_t)T * d.k * 4);
  L.w = seg((size_t)T * d.k * 4);
  L.cnt = seg((size_t)d.E * 4);
  L.off = seg((size_t)(d.E + 1) * 4);
  L.uni = seg((size_t)(d.E + 1) * 4);
  L.n_uni = seg(16);
  L.own = seg((size_t)(d.E + 1) * 4);  // the union slots a call computes (expert parallelism)
  L.n_own = seg(16);
  L.perm = seg((size_t)T * d.k * 4);
  L.pos = seg((size_t)T * d.k * 4);
  L.pair_tok = seg(P * 4);
  L.hq = seg(P * d.I);
  L.hqs = seg(P * (d.I / 32) * 4);
  L.hd = seg(P * (d.I / 32) * 4);
  const size_t Pp = prefill ? P : 0;
  L.xg = seg(Pp * d.H * 4);  // fp16 hi/lo split of x^, [P][2H]
  L.hs = seg(Pp * d.I * 4);  // fp16 hi/lo split of h^, [P][2I]
  L.y = seg(Pp * d.H * 4);
  L.maps = seg(prefill ? (size_t)(d.E + 1) * 3 * 128 : 0);
  L.total = o;
  return L;
}

struct QuantArgs {
  const float *x;
  int8_t *q;
  float *d;
  int64_t nblk;
  unsigned long long *prof;  // profiling record or null (phase 0 start)
};

struct RouteArgs {
  int H, E, k, T;
  const float *x, *Wr;
  int8_t *xq;
  float *xd, *logits, *w;
  int32_t *idx, *route_counts;
  int32_t *cnt, *off, *uni, *n_uni, *perm, *pos, *pair_tok;
  int32_t *own, *n_own;     // owned slot list (null: not written)
  int e_lo, e_hi, with_shared;
  int32_t *mail;            // mapped pinned host mailbox [2 + E] or null: [0] seq, [1] n_uni, [2..] union
  int32_t mail_seq;
  unsigned int *done;
  int32_t *status;
  int do_quant;
  int do_bucket;
  int epc;  // experts per CTA
  int tt;   // tokens per x tile
  unsigned long long *prof;  // profiling record or null (phase 0)
  long long wait_limit;  // SM clocks a work wait may take (wait_limit_cycles())
};

struct BucketArgs {
  int E, k, T;
  const int32_t *idx;
  int32_t *cnt, *off, *uni, *n_uni, *perm, *pos, *pair_tok;
};

struct GateUpArgs {
  int H, I, E, k, T;
  const void *const *table;
  const int32_t *uni, *n_uni, *off, *pair_tok;
  const int32_t *own, *n_own;  // the slots to compute: 0 = shared expert, s >= 1 = uni[s - 1]
  const int8_t *xq;
  const float *xd;
  int8_t *hq;
  int32_t *hqs;
  float *hd;
  int32_t *status;
  int nstage;
  int rpm;  // weight rows per matrix per stage (4 or 8)
  int use_pdl;
  unsigned long long *prof;  // profiling record or null (phase 1)
  long long wait_limit;  // SM clocks a work wait may take (wait_limit_cycles())
};

struct DownArgs {
  int H, I, E, k, T;
  const void *const *table;
  const int32_t *uni, *n_uni, *off, *pos;
  const int32_t *own, *n_own;  // the slots to compute: 0 = shared expert, s >= 1 = uni[s - 1]
  const int32_t *idx;          // the combine adds the pairs whose expert is in [e_lo, e_hi)
  int e_lo, e_hi, with_shared;
  const float *w;
  const int8_t *hq;
  const int32_t *hqs;
  const float *hd;
  float *out;
  int32_t *status;
  int nstage;
  int rg;        // row granularity (scale bytes of a row group are a multiple of 16)
  int rows_max;  // most output rows any CTA owns
  int rs;        // rows per stage (a multiple of rg)
  int preload;   // per-position activations kept in shared memory (small batches)
  int use_pdl;
  unsigned long long *prof;  // profiling record or null (phase 2)
  long long wait_limit;  // SM clocks a work wait may take (wait_limit_cycles())
};

// Prefill grouped GEMM over the expert union (moe_prefill.cu).  mode 0: gate/up
// of every (slot, token) pair with SwiGLU and Q8_0 of h; mode 1: down into y.
struct PfArgs {
  int mode, H, I, E, k, T;
  const void *const *table;
  const int32_t *uni, *n_uni, *off, *pair_tok;
  int8_t *hq;           // mode 0 outputs in pair order: Q8_0 codes of h [P][I],
  float *hd;            //   their block scales [P][I/32],
  void *hs;             //   and the fp16 hi/lo split of h^ = q d [P][2I] (mode 1's B rows)
  float *y;             // mode 1 output [P][H]
  const CUtensorMap *maps;  // [E+1][gate, up, down] tensor maps of the packed weights (device)
  int32_t *status;
  unsigned long long *prof;  // profiling record or null (phase mode + 1; k_make_maps ends phase 0)
  long long wait_limit;  // SM clocks a work wait may take (wait_limit_cycles())
};

// The gate/up GEMM's activation rows in pair order: xg[p] = fp16 hi/lo split of
// the dequantised Q8_0 codes of token pair_tok[p] ([P][2H], per 64-group 64 hi
// then 64 lo).
struct GatherRowsArgs {
  int H, T, k;
  const int8_t *xq;
  const float *xd;
  const int32_t *pair_tok;
  void *xg;
};

struct RouterTiledArgs {
  int H, E, T;
  const float *x, *Wr;
  float *logits;
};

// The whole batch-1 decode layer in one cooperative kernel (moe_fused.cu).
struct FusedArgs {
  int H, I, E, k;
  const float *x, *Wr;
  const void *const *table;
  float *out;
  int8_t *xq;
  float *xd, *logits, *w;
  int32_t *idx, *route_counts;
  int32_t *cnt, *off, *uni, *n_uni, *perm, *pos, *pair_tok;
  int8_t *hq;
  int32_t *hqs;
  float *hd;
  int32_t *status;
  unsigned int *arrivals;  // routing arrivals of the grid (zeroed per call by CTA 0)
  int32_t *slot_done;      // [k + 1] gate/up units completed per union slot (zeroed per call by CTA 0)
  int32_t *ctrl;           // the control words (arrivals and slot_done point into them)
  unsigned long long *ready;  // ctrl + kCtrlReady: the call's sequence number once CTA 0 has zeroed
  unsigned long long seq;     // this call's sequence number (never 0)
  int fresh;               // the first launch of a call: CTA 0 zeroes the status word too
  int nstage;              // ring stages
  int rows_max;            // down: most output rows a CTA owns
  int rg;                  // down: row granularity (scale bytes of rg rows: a multiple of 16)
  int rs;                  // down: rows per stage (a multiple of rg)
  int e_lo, e_hi;          // routed experts this call computes (expert parallelism)
  int with_shared;         // and the shared expert
  int fmt;                 // kFmtInt4 or kFmtMxfp4
  // tokens of the launch (1 .. kDecodeTMax): x, xq, xd, logits [ntok] rows,
  // idx, w [ntok][k], out [ntok][H]; token t's gate/up counters at
  // slot_done + kCtrlWords t; the record (cnt .. pair_tok) covers the batch
  int ntok;
  long long wait_limit;
  unsigned long long *prof;
};

struct CombineArgs {
  int H, k, T;
  const float *y, *w;
  const int32_t *pos;
  float *out;
  unsigned long long *prof;  // profiling record or null (phase 2 end)
};

// Offsets of the union mailbox (mapped pinned host memory the routing kernel
// writes for the tiered cache): sequence number, union size, union.
constexpr int kMailSeq = 0, kMailN = 1, kMailUni = 2;

// moe_layer_route that also posts the union to a mailbox (moe_api.cu):
// mail = device address of mapped pinned host memory [2 + E], seq = the value
// the host waits for in mail[kMailSeq]; profile = take a profiling record.
int route_to_mailbox(const moe_dims *dims, int32_t T, const float *x, const float *Wr, void *ws, size_t ws_bytes,
                     int32_t *route_counts_opt, int32_t *mail, int32_t seq, bool profile, cudaStream_t s);

// Launchers (moe_kernels.cu).  Return cudaSuccess or the launch error.
cudaError_t launch_quant(const QuantArgs &a, cudaStream_t s);
// Attributes of one of the library's kernels (binaryVersion: the SM the
// loaded code was built for).
cudaError_t func_attributes(cudaFuncAttributes *fa);
// Zero ctrl_bytes (a multiple of 16) at ctrl and copy n floats (a multiple of 4)
// from device-accessible host memory to x_dev.
cudaError_t launch_stage_in(const float *x_host, float *x_dev, int64_t n, void *ctrl, size_t ctrl_bytes,
                            cudaStream_t s);
cudaError_t launch_route_decode(const RouteArgs &a, cudaStream_t s);
cudaError_t launch_bucket(const BucketArgs &a, cudaStream_t s);
cudaError_t launch_topk(const float *logits, int T, int E, int k, int32_t *idx, float *w,
                        int32_t *counts, cudaStream_t s);
cudaError_t launch_gateup_decode(const GateUpArgs &a, int grid, size_t smem, cudaStream_t s);
cudaError_t launch_down_decode(const DownArgs &a, int grid, size_t smem, cudaStream_t s);

// Fused batch-1 decode (moe_fused.cu): plan (false if the shape does not fit
// one CTA per SM) and launch (cooperative: every CTA resident at once).
bool fused_plan(int H, int I, int E, int k, int grid, FusedArgs *a, size_t *smem);
cudaError_t launch_decode_fused(const FusedArgs &a, int grid, size_t smem, cudaStream_t s);
// CTAs of the fused kernel that fit on one SM with `smem` bytes (0 if none).
int fused_ctas_per_sm(const FusedArgs &a, size_t smem);

cudaError_t launch_gemm_pf(const PfArgs &a, const CUtensorMap &bmap, int grid, cudaStream_t s);
// 2D tensor map over a row-major fp16 matrix [rows][cols] for TMA copies of
// boxes of 64 columns x box_rows rows with 128-byte swizzle (moe_tma.cpp).
cudaError_t make_f16_map(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows);
// Template for the packed-weight maps: a uint8 matrix [rows][cols] (cols = K/2),
// boxes of 32 bytes x box_rows rows, no swizzle (moe_tma.cpp).
cudaError_t make_u8_map(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows);
cudaError_t launch_make_maps(const PfArgs &a, const CUtensorMap &tgu, const CUtensorMap &tdn, cudaStream_t s);
constexpr uint32_t kPfBoxRows = 32;  // rows per activation TMA box of the prefill GEMM
cudaError_t launch_router_tiled(const RouterTiledArgs &a, cudaStream_t s);
cudaError_t launch_combine(const CombineArgs &a, cudaStream_t s);
cudaError_t launch_gather_rows(const GatherRowsArgs &a, cudaStream_t s);
size_t pf_smem_bytes(int E);

// Shared-memory plans (host side, moe_kernels.cu).
size_t route_smem_bytes(int H, int epc, int tt);
size_t gateup_smem_bytes(int H, int T, int R, int nstage);
void gateup_plan(int H, int T, int *R, int *nstage);
size_t down_smem_bytes(int H, int I, int k, int T, int rows_max, int rs, int nstage);
int down_max_stages(int H, int I, int k, int T, int rows_max, int rs);
int down_preload(int I, int k, int T);

}  // namespace moe
