// moe_api.cu -- the C ABI of libmoe (declared in include/moe.h): argument
// checks, workspace carving and the launch sequence of the layer.
#include <atomic>
#include <chrono>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "moe_internal.h"

namespace moe {

// Wait limit of the kernels' work waits (moe_set_wait_limit), process-wide.
static std::atomic<long long> g_wait_limit{kWaitLimitCycles};
long long wait_limit_cycles() { return g_wait_limit.load(std::memory_order_relaxed); }

namespace {

constexpr int kMaxDevices = 64;
int g_sms[kMaxDevices] = {0};
std::mutex g_mu;

int device_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_sms[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    g_sms[dev] = n;
  }
  return g_sms[dev];
}

// Sequence numbers of fused-kernel launches: unique within the process and
// never 0 (the ready word's idle value).  The start is drawn from the clock so
// that a workspace holding another process's last number does not match.
unsigned long long next_call_seq() {
  static std::atomic<unsigned long long> seq{
      (unsigned long long)std::chrono::steady_clock::now().time_since_epoch().count() * 0x9E3779B97F4A7C15ull};
  unsigned long long v = seq.fetch_add(1, std::memory_order_relaxed);
  while (v == 0) v = seq.fetch_add(1, std::memory_order_relaxed);
  return v;
}

bool dims_shape_ok(const moe_dims &d) {
  return d.H > 0 && d.I > 0 && d.H % 128 == 0 && d.I % 128 == 0 && d.H <= 8192 && d.I <= 4096 &&
         d.E >= 1 && d.E <= MOE_MAX_E && d.k >= 1 && d.k <= d.E && d.k <= kMaxK;
}

// ---- optional per-call kernel timing (moe_profile_enable).  Each profiled
// call owns one zeroed record of a per-device ring; its kernels stamp their
// phases there with %globaltimer, so nothing is added to the stream between
// them.  The ring is zeroed at enable and after every read.  The state is
// process-wide; g_prof_mu serialises every access to it across host threads.
std::mutex g_prof_mu;
bool g_prof = false;
unsigned long long *g_prof_buf[kMaxDevices] = {};
int g_prof_n[kMaxDevices] = {};
unsigned long long *g_prof_cur[kMaxDevices] = {};

int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}

// A fresh record for the next call on the current device, or null when
// profiling is off or the ring is full (the call then goes unrecorded).
unsigned long long *prof_next() {
  std::lock_guard<std::mutex> lock(g_prof_mu);
  if (!g_prof) return nullptr;
  const int dev = current_device();
  if (dev < 0) return nullptr;
  if (g_prof_buf[dev] == nullptr || g_prof_n[dev] >= kProfSlots) {
    g_prof_cur[dev] = nullptr;  // the experts half of this call goes unrecorded too
    return nullptr;
  }
  g_prof_cur[dev] = g_prof_buf[dev] + (size_t)(g_prof_n[dev]++) * kProfWords;
  return g_prof_cur[dev];
}

// The record of the most recent routing call (the experts half of a split layer).
unsigned long long *prof_current() {
  std::lock_guard<std::mutex> lock(g_prof_mu);
  if (!g_prof) return nullptr;
  const int dev = current_device();
  return dev < 0 ? nullptr : g_prof_cur[dev];
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return MOE_OK;
  std::fprintf(stderr, "libmoe: CUDA error %d (%s)\n", (int)e, cudaGetErrorString(e));
  return MOE_ERR_CUDA;
}

template <typename T>
T *at(void *ws, size_t off) {
  return reinterpret_cast<T *>(static_cast<unsigned char *>(ws) + off);
}

// Routing half of the decode path on Tc <= kDecodeTMax tokens: Q8_0 of x,
// logits, top-k + softmax, batch union.  Per-token arrays (xq, xd, logits,
// idx, w) are at token offset t0 of the layout L; pair arrays are chunk-local.
struct ChunkPtrs {
  int8_t *xq;
  float *xd, *logits, *w;
  int32_t *idx, *cnt, *off, *uni, *n_uni, *own, *n_own, *perm, *pos, *pair_tok, *hqs, *status;
  int8_t *hq;
  float *hd;
  unsigned int *done;
};

ChunkPtrs chunk_ptrs(const moe_dims &d, int t0, const WsLayout &L, void *ws) {
  const size_t H = d.H, E = d.E, K = d.k;
  ChunkPtrs p{};
  p.xq = at<int8_t>(ws, L.xq) + (size_t)t0 * H;
  p.xd = at<float>(ws, L.xd) + (size_t)t0 * (H / 32);
  p.logits = at<float>(ws, L.logits) + (size_t)t0 * E;
  p.idx = at<int32_t>(ws, L.idx) + (size_t)t0 * K;
  p.w = at<float>(ws, L.w) + (size_t)t0 * K;
  p.cnt = at<int32_t>(ws, L.cnt);
  p.off = at<int32_t>(ws, L.off);
  p.uni = at<int32_t>(ws, L.uni);
  p.n_uni = at<int32_t>(ws, L.n_uni);
  p.own = at<int32_t>(ws, L.own);
  p.n_own = at<int32_t>(ws, L.n_own);
  p.perm = at<int32_t>(ws, L.perm);
  p.pos = at<int32_t>(ws, L.pos);
  p.pair_tok = at<int32_t>(ws, L.pair_tok);
  p.hq = at<int8_t>(ws, L.hq);
  p.hqs = at<int32_t>(ws, L.hqs);
  p.hd = at<float>(ws, L.hd);
  p.status = at<int32_t>(ws, L.status);
  p.done = at<unsigned int>(ws, L.ctrl);
  return p;
}

// The routed experts [lo, hi) and the shared expert (if shared) that a call
// computes: all of them, except on one rank of an expert-parallel layer.
struct Owned {
  int lo, hi, shared;
};
Owned all_owned(const moe_dims &d) { return Owned{0, d.E, 1}; }

int route_chunk(const moe_dims &d, int t0, int Tc, const WsLayout &L, const float *x,
                const float *Wr, void *ws, int32_t *counts, unsigned long long *prof,
                const Owned &ow, cudaStream_t s, int32_t *mail = nullptr, int32_t mail_seq = 0) {
  const ChunkPtrs p = chunk_ptrs(d, t0, L, ws);
  RouteArgs ra{};
  ra.H = d.H;
  ra.E = d.E;
  ra.k = d.k;
  ra.T = Tc;
  ra.x = x + (size_t)t0 * d.H;
  ra.Wr = Wr;
  ra.xq = p.xq;
  ra.xd = p.xd;
  ra.logits = p.logits;
  ra.idx = p.idx;
  ra.w = p.w;
  ra.route_counts = counts;
  ra.cnt = p.cnt;
  ra.off = p.off;
  ra.uni = p.uni;
  ra.n_uni = p.n_uni;
  ra.perm = p.perm;
  ra.pos = p.pos;
  ra.pair_tok = p.pair_tok;
  ra.own = p.own;
  ra.n_own = p.n_own;
  ra.mail = mail;
  ra.mail_seq = mail_seq;
  ra.e_lo = ow.lo;
  ra.e_hi = ow.hi;
  ra.with_shared = ow.shared;
  ra.done = p.done;
  ra.status = p.status;
  ra.do_quant = 1;
  ra.do_bucket = 1;
  ra.epc = 2;
  ra.tt = Tc < 2 ? Tc : 2;
  ra.prof = prof;
  ra.wait_limit = wait_limit_cycles();
  cudaError_t err = launch_route_decode(ra, s);
  if (err != cudaSuccess) return cuda_status(err);
  return MOE_OK;
}

int experts_chunk(const moe_dims &d, int t0, int Tc, const WsLayout &L, const void *const *table,
                  float *out, void *ws, unsigned long long *prof, const Owned &ow, cudaStream_t s) {
  const int sms = device_sms();
  if (sms <= 0) return MOE_ERR_CUDA;
  const ChunkPtrs p = chunk_ptrs(d, t0, L, ws);
  GateUpArgs ga{};
  ga.H = d.H;
  ga.I = d.I;
  ga.E = d.E;
  ga.k = d.k;
  ga.T = Tc;
  ga.table = table;
  ga.uni = p.uni;
  ga.n_uni = p.n_uni;
  ga.off = p.off;
  ga.pair_tok = p.pair_tok;
  ga.own = p.own;
  ga.n_own = p.n_own;
  ga.xq = p.xq;
  ga.xd = p.xd;
  ga.hq = p.hq;
  ga.hqs = p.hqs;
  ga.hd = p.hd;
  ga.status = p.status;
  gateup_plan(d.H, Tc, &ga.rpm, &ga.nstage);
  ga.use_pdl = 1;
  ga.prof = prof;
  ga.wait_limit = wait_limit_cycles();
  if (ga.nstage < 2) return MOE_ERR_SHAPE;
  cudaError_t err =
      launch_gateup_decode(ga, sms, gateup_smem_bytes(d.H, Tc, ga.rpm, ga.nstage), s);
  if (err != cudaSuccess) return cuda_status(err);

  DownArgs da{};
  da.H = d.H;
  da.I = d.I;
  da.E = d.E;
  da.k = d.k;
  da.T = Tc;
  da.table = table;
  da.uni = p.uni;
  da.n_uni = p.n_uni;
  da.off = p.off;
  da.pos = p.pos;
  da.own = p.own;
  da.n_own = p.n_own;
  da.idx = p.idx;
  da.e_lo = ow.lo;
  da.e_hi = ow.hi;
  da.with_shared = ow.shared;
  da.w = p.w;
  da.hq = p.hq;
  da.hqs = p.hqs;
  da.hd = p.hd;
  da.out = out + (size_t)t0 * d.H;
  da.status = p.status;
  // row groups: the fp16 scales of rg rows span a multiple of 16 bytes
  int g = d.I / 32, b = 16;
  while (b) {
    const int t = g % b;
    g = b;
    b = t;
  }
  da.rg = 16 / g;
  const int nrg = d.H / da.rg;
  const int grid = nrg < sms ? nrg : sms;
  da.rows_max = ((nrg + grid - 1) / grid) * da.rg;
  // rows per stage: the CTA's whole range if three stages fit, else halves
  da.rs = da.rows_max;
  while (da.rs > da.rg && down_max_stages(d.H, d.I, d.k, Tc, da.rows_max, da.rs) < 3)
    da.rs = ((da.rs / 2 + da.rg - 1) / da.rg) * da.rg;
  da.nstage = down_max_stages(d.H, d.I, d.k, Tc, da.rows_max, da.rs);
  da.use_pdl = 1;
  da.prof = prof;
  da.wait_limit = wait_limit_cycles();
  da.preload = down_preload(d.I, d.k, Tc);
  if (da.nstage < 2) return MOE_ERR_SHAPE;
  err = launch_down_decode(
      da, grid, down_smem_bytes(d.H, d.I, d.k, Tc, da.rows_max, da.rs, da.nstage), s);
  if (err != cudaSuccess) return cuda_status(err);
  return MOE_OK;
}

// The fused batch-1 kernel (moe_fused.cu) when the layer's shape fits it:
// kFusedNA when it does not (the three-kernel path then runs), else a status.
constexpr int kFusedNA = 1;

// Whether the fused kernel runs this layer's one-token calls on the current
// device (its shape fits one CTA per SM, cooperative launch available); fills
// its plan.  Asked once per device and shape.
bool fused_usable(const moe_dims &d, int fmt, FusedArgs *fa, size_t *smem, int *grid) {
  const int sms = device_sms();
  if (sms <= 0) return false;
  *fa = FusedArgs{};
  if (!fused_plan(d.H, d.I, d.E, d.k, sms, fa, smem)) return false;
  fa->H = d.H;
  fa->I = d.I;
  fa->E = d.E;
  fa->k = d.k;
  fa->fmt = fmt;
  *grid = sms;
  static std::mutex mu;
  static int known[kMaxDevices][2] = {};
  static moe_dims key[kMaxDevices][2];
  static bool fits[kMaxDevices][2] = {};
  const int dev = current_device();
  if (dev < 0 || fmt < 0 || fmt > 1) return false;
  std::lock_guard<std::mutex> lock(mu);
  moe_dims &kd = key[dev][fmt];
  if (!known[dev][fmt] || kd.H != d.H || kd.I != d.I || kd.E != d.E || kd.k != d.k) {
    int coop = 0;
    if (cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess) coop = 0;
    fits[dev][fmt] = coop && fused_ctas_per_sm(*fa, *smem) >= 1;
    cudaGetLastError();
    known[dev][fmt] = 1;
    kd = d;
  }
  return fits[dev][fmt];
}

// One launch of the fused kernel: the whole layer for T <= kDecodeTMax
// tokens (their routing, the experts of each token streamed one token after
// the other, the combine), in the workspace rows of layout L.
int fused_forward(const moe_dims &d, const WsLayout &L, const float *x, const float *Wr,
                  const void *const *table, float *out, void *ws, int32_t *counts,
                  unsigned long long *prof, const Owned &ow, cudaStream_t s, int fmt = kFmtInt4,
                  int T = 1, bool fresh = true) {
  FusedArgs fa{};
  size_t smem = 0;
  int sms = 0;
  if (!fused_usable(d, fmt, &fa, &smem, &sms)) return kFusedNA;
  const ChunkPtrs p = chunk_ptrs(d, 0, L, ws);
  fa.x = x;
  fa.Wr = Wr;
  fa.table = table;
  fa.out = out;
  fa.xq = p.xq;
  fa.xd = p.xd;
  fa.logits = p.logits;
  fa.w = p.w;
  fa.idx = p.idx;
  fa.route_counts = counts;
  fa.cnt = p.cnt;
  fa.off = p.off;
  fa.uni = p.uni;
  fa.n_uni = p.n_uni;
  fa.perm = p.perm;
  fa.pos = p.pos;
  fa.pair_tok = p.pair_tok;
  fa.hq = p.hq;
  fa.hqs = p.hqs;
  fa.hd = p.hd;
  fa.status = p.status;
  // no memset: the kernel zeroes its control words (and, on a call's first
  // launch, the status word) itself
  fa.ctrl = at<int32_t>(ws, L.ctrl);
  fa.arrivals = reinterpret_cast<unsigned int *>(fa.ctrl + 1);
  fa.slot_done = fa.ctrl + kCtrlSlot0;
  fa.ready = reinterpret_cast<unsigned long long *>(fa.ctrl + kCtrlReady);
  fa.seq = next_call_seq();
  fa.fresh = fresh ? 1 : 0;
  fa.e_lo = ow.lo;
  fa.e_hi = ow.hi;
  fa.with_shared = ow.shared;
  fa.wait_limit = wait_limit_cycles();
  fa.prof = prof;
  fa.ntok = T;
  return cuda_status(launch_decode_fused(fa, sms, smem, s));
}

// The fused kernel runs this shape and weight format on the current device.
bool fused_fits(const moe_dims &d, int fmt) {
  FusedArgs fa{};
  size_t smem = 0;
  int grid = 0;
  return fused_usable(d, fmt, &fa, &smem, &grid);
}

bool use_prefill(int T, int path) {
  return path == MOE_PATH_PREFILL || (path == MOE_PATH_AUTO && T > kDecodeTMax);
}

// The prefill path on all T tokens at once: Q8_0 of x (int8 and fp16 codes),
// router logits, top-k + softmax, bucketing, grouped GEMM gate/up, grouped GEMM
// down, combine.
int prefill_forward(const moe_dims &d, int T, const float *x, const float *Wr,
                    const void *const *table, float *out, void *ws, const WsLayout &L,
                    int32_t *counts, cudaStream_t s) {
  const int sms = device_sms();
  if (sms <= 0) return MOE_ERR_CUDA;
  int8_t *xq = at<int8_t>(ws, L.xq);
  float *xd = at<float>(ws, L.xd);
  float *logits = at<float>(ws, L.logits);
  int32_t *idx = at<int32_t>(ws, L.idx);
  float *w = at<float>(ws, L.w);
  int32_t *status = at<int32_t>(ws, L.status);
  unsigned long long *prof = prof_next();
  QuantArgs qa{x, xq, xd, (int64_t)T * (d.H / 32), prof};
  cudaError_t err = launch_quant(qa, s);
  if (err != cudaSuccess) return cuda_status(err);
  RouterTiledArgs ra{d.H, d.E, T, x, Wr, logits};
  err = launch_router_tiled(ra, s);
  if (err != cudaSuccess) return cuda_status(err);
  err = launch_topk(logits, T, d.E, d.k, idx, w, counts, s);
  if (err != cudaSuccess) return cuda_status(err);
  BucketArgs ba{};
  ba.E = d.E;
  ba.k = d.k;
  ba.T = T;
  ba.idx = idx;
  ba.cnt = at<int32_t>(ws, L.cnt);
  ba.off = at<int32_t>(ws, L.off);
  ba.uni = at<int32_t>(ws, L.uni);
  ba.n_uni = at<int32_t>(ws, L.n_uni);
  ba.perm = at<int32_t>(ws, L.perm);
  ba.pos = at<int32_t>(ws, L.pos);
  ba.pair_tok = at<int32_t>(ws, L.pair_tok);
  err = launch_bucket(ba, s);
  if (err != cudaSuccess) return cuda_status(err);
  GatherRowsArgs gr{d.H, T, d.k, xq, xd, ba.pair_tok, at<void>(ws, L.xg)};
  err = launch_gather_rows(gr, s);
  if (err != cudaSuccess) return cuda_status(err);

  PfArgs pa{};
  pa.mode = 0;
  pa.H = d.H;
  pa.I = d.I;
  pa.E = d.E;
  pa.k = d.k;
  pa.T = T;
  pa.table = table;
  pa.uni = ba.uni;
  pa.n_uni = ba.n_uni;
  pa.off = ba.off;
  pa.pair_tok = ba.pair_tok;
  pa.hq = at<int8_t>(ws, L.hq);
  pa.hd = at<float>(ws, L.hd);
  pa.hs = at<void>(ws, L.hs);
  pa.y = at<float>(ws, L.y);
  pa.status = status;
  pa.prof = prof;
  pa.wait_limit = wait_limit_cycles();
  const size_t P = (size_t)T * (size_t)(d.k + 1);
  pa.maps = at<CUtensorMap>(ws, L.maps);
  CUtensorMap map_x, map_h, tmpl_gu, tmpl_dn;
  err = make_f16_map(&map_x, gr.xg, (uint64_t)P, 2 * (uint64_t)d.H, kPfBoxRows);
  if (err == cudaSuccess) err = make_f16_map(&map_h, pa.hs, (uint64_t)P, 2 * (uint64_t)d.I, kPfBoxRows);
  // the templates' address is replaced per expert on the device
  if (err == cudaSuccess) err = make_u8_map(&tmpl_gu, pa.maps, (uint64_t)d.I, (uint64_t)d.H / 2, 128);
  if (err == cudaSuccess) err = make_u8_map(&tmpl_dn, pa.maps, (uint64_t)d.H, (uint64_t)d.I / 2, 128);
  if (err != cudaSuccess) return cuda_status(err);
  err = launch_make_maps(pa, tmpl_gu, tmpl_dn, s);
  if (err != cudaSuccess) return cuda_status(err);
  const int grid = sms < kPfMaxCtas ? sms : kPfMaxCtas;
  err = launch_gemm_pf(pa, map_x, grid, s);
  if (err != cudaSuccess) return cuda_status(err);
  pa.mode = 1;
  err = launch_gemm_pf(pa, map_h, grid, s);
  if (err != cudaSuccess) return cuda_status(err);
  CombineArgs ca{d.H, d.k, T, pa.y, w, ba.pos, out, prof};
  err = launch_combine(ca, s);
  if (err != cudaSuccess) return cuda_status(err);
  return MOE_OK;
}

// The device address of pinned host memory the current device can use, or
// null (pageable or unknown memory, or no mapping).
const void *host_device_view(const void *p) {
  cudaPointerAttributes at{};
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();  // clear the sticky-free error of an unknown pointer
    return nullptr;
  }
  if (at.type != cudaMemoryTypeHost || at.devicePointer == nullptr) return nullptr;
  return at.devicePointer;
}

}  // namespace

int route_to_mailbox(const moe_dims *dims, int32_t T, const float *x, const float *Wr, void *ws, size_t ws_bytes,
                     int32_t *route_counts_opt, int32_t *mail, int32_t seq, bool profile, cudaStream_t s) {
  int rc = moe_check_dims(dims);
  if (rc != MOE_OK) return rc;
  if (T < 1 || T > kDecodeTMax || !x || !Wr || !ws || !mail) return MOE_ERR_BAD_ARG;
  if (!aligned(x, 16) || !aligned(Wr, 16)) return MOE_ERR_BAD_ARG;
  if (!aligned(ws, 256)) return MOE_ERR_WORKSPACE;
  const WsLayout L = ws_layout(*dims, T);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  cudaError_t err = cudaMemsetAsync(ws, 0, L.xin, s);
  if (err != cudaSuccess) return cuda_status(err);
  return route_chunk(*dims, 0, T, L, x, Wr, ws, route_counts_opt, profile ? prof_next() : nullptr,
                     all_owned(*dims), s, mail, seq);
}

}  // namespace moe

using namespace moe;

extern "C" {

const char *moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_BAD_ARG: return "bad argument";
    case MOE_ERR_SHAPE: return "unsupported shape";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_WORKSPACE: return "workspace too small or misaligned";
    case MOE_ERR_CACHE_FULL: return "expert cache full";
    case MOE_ERR_NOT_RESIDENT: return "expert not resident";
    case MOE_ERR_TIMEOUT: return "device wait timed out";
    case MOE_ERR_DEVICE: return "device-side check failed";
    case MOE_ERR_ALLOC: return "allocation failed";
    case MOE_ERR_IO: return "file missing, unreadable or corrupt";
    default: return "unknown status";
  }
}

int moe_check_dims(const moe_dims *dims) {
  if (dims == nullptr) return MOE_ERR_BAD_ARG;
  return dims_shape_ok(*dims) ? MOE_OK : MOE_ERR_SHAPE;
}

size_t moe_expert_bytes(const moe_dims *dims) {
  if (moe_check_dims(dims) != MOE_OK) return 0;
  return expert_bytes(dims->H, dims->I);
}

size_t moe_workspace_bytes(const moe_dims *dims, int32_t T_max) {
  return moe_workspace_bytes_path(dims, T_max, MOE_PATH_AUTO);
}

size_t moe_workspace_bytes_path(const moe_dims *dims, int32_t T_max, int32_t path) {
  if (moe_check_dims(dims) != MOE_OK || T_max < 0) return 0;
  if (path < MOE_PATH_AUTO || path > MOE_PATH_PREFILL) return 0;
  return ws_layout(*dims, T_max, use_prefill(T_max, path)).total;
}

int moe_workspace_view(const moe_dims *dims, int32_t T, void *ws, moe_ws_view *v) {
  if (moe_check_dims(dims) != MOE_OK) return MOE_ERR_SHAPE;
  if (ws == nullptr || v == nullptr || T < 0) return MOE_ERR_BAD_ARG;
  // every field of the view lies before the prefill-only segments of the
  // layout, so the decode layout gives the same offsets on either path
  const WsLayout L = ws_layout(*dims, T);
  v->status = at<int32_t>(ws, L.status);
  v->xq = at<int8_t>(ws, L.xq);
  v->xd = at<float>(ws, L.xd);
  v->logits = at<float>(ws, L.logits);
  v->idx = at<int32_t>(ws, L.idx);
  v->w = at<float>(ws, L.w);
  v->cnt = at<int32_t>(ws, L.cnt);
  v->off = at<int32_t>(ws, L.off);
  v->uni = at<int32_t>(ws, L.uni);
  v->n_uni = at<int32_t>(ws, L.n_uni);
  v->perm = at<int32_t>(ws, L.perm);
  v->pos = at<int32_t>(ws, L.pos);
  v->pair_tok = at<int32_t>(ws, L.pair_tok);
  v->hq = at<int8_t>(ws, L.hq);
  v->hd = at<float>(ws, L.hd);
  v->T_max = T;
  return MOE_OK;
}

int64_t moe_set_wait_limit(int64_t cycles) {
  const long long v = cycles > 0 ? (long long)cycles : kWaitLimitCycles;
  return (int64_t)g_wait_limit.exchange(v);
}

int moe_device_binary_version(void) {
  cudaFuncAttributes fa{};
  const cudaError_t e = func_attributes(&fa);
  if (e != cudaSuccess) return cuda_status(e);
  return fa.binaryVersion;
}

int moe_layer_launches(const moe_dims *dims, int32_t T, int32_t path) {
  int rc = moe_check_dims(dims);
  if (rc != MOE_OK) return rc;
  if (T < 0 || path < MOE_PATH_AUTO || path > MOE_PATH_PREFILL) return MOE_ERR_BAD_ARG;
  if (T == 0) return 0;
  if (use_prefill(T, path)) return 9;  // quant, router, top-k, bucket, gather, maps, 2 GEMMs, combine
  if (T == 1 || (path == MOE_PATH_AUTO && T <= kDecodeTMax)) {
    FusedArgs fa{};
    size_t smem = 0;
    int grid = 0;
    // one fused launch for the whole layer
    if (fused_usable(*dims, kFmtInt4, &fa, &smem, &grid)) return 1;
  }
  return 3 * ((T + kDecodeTMax - 1) / kDecodeTMax);
}

int moe_device_sms(void) {
  const int n = device_sms();
  return n > 0 ? n : MOE_ERR_CUDA;
}

int moe_profile_enable(int on) {
  std::lock_guard<std::mutex> lock(g_prof_mu);
  if (on) {
    const int dev = current_device();
    if (dev < 0) return MOE_ERR_CUDA;
    const size_t bytes = (size_t)kProfSlots * kProfWords * sizeof(unsigned long long);
    if (g_prof_buf[dev] == nullptr) {
      cudaError_t e = cudaMalloc(&g_prof_buf[dev], bytes);
      if (e != cudaSuccess) {
        g_prof_buf[dev] = nullptr;
        return cuda_status(e);
      }
    }
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemset(g_prof_buf[dev], 0, bytes);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_status(e);
    g_prof_n[dev] = 0;
    g_prof_cur[dev] = nullptr;
  }
  g_prof = on != 0;
  return MOE_OK;
}

int moe_profile_read(float *ms, int max_calls) {
  if (ms == nullptr || max_calls < 0) return MOE_ERR_BAD_ARG;
  std::lock_guard<std::mutex> lock(g_prof_mu);
  const int dev = current_device();
  if (dev < 0) return MOE_ERR_CUDA;
  if (g_prof_buf[dev] == nullptr) return 0;
  const int n = g_prof_n[dev];
  const size_t bytes = (size_t)kProfSlots * kProfWords * sizeof(unsigned long long);
  static thread_local unsigned long long rec[kProfSlots * kProfWords];
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess && n > 0)
    e = cudaMemcpy(rec, g_prof_buf[dev], (size_t)n * kProfWords * sizeof(unsigned long long),
                   cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(g_prof_buf[dev], 0, bytes);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_status(e);
  g_prof_n[dev] = 0;
  g_prof_cur[dev] = nullptr;
  const int w = n < max_calls ? n : max_calls;
  for (int c = 0; c < w; ++c) {
    const unsigned long long *r = rec + (size_t)c * kProfWords;
    unsigned long long first = ~0ull, last = 0;
    for (int k = 0; k < 3; ++k) {
      const unsigned long long st = ~r[2 * k], en = r[2 * k + 1];
      const bool ok = r[2 * k] != 0 && en != 0 && en >= st;
      ms[(size_t)c * 4 + k] = ok ? (float)((double)(en - st) * 1e-6) : 0.0f;
      if (ok) {
        first = st < first ? st : first;
        last = en > last ? en : last;
      }
    }
    ms[(size_t)c * 4 + 3] = last > 0 ? (float)((double)(last - first) * 1e-6) : 0.0f;
  }
  return w;
}

int moe_quant_q8_0(const float *x, int64_t rows, int32_t cols, int8_t *q, float *d, void *stream) {
  if (rows < 0 || cols <= 0 || cols % 32 != 0) return MOE_ERR_SHAPE;
  if (rows == 0) return MOE_OK;
  if (!x || !q || !d) return MOE_ERR_BAD_ARG;
  QuantArgs a{x, q, d, rows * (int64_t)(cols / 32), nullptr};
  return cuda_status(launch_quant(a, static_cast<cudaStream_t>(stream)));
}

int moe_router_topk(const moe_dims *dims, int32_t T, const float *x, const float *Wr, int32_t *idx,
                    float *w, float *logits, int32_t *route_counts_opt, void *stream) {
  int rc = moe_check_dims(dims);
  if (rc != MOE_OK) return rc;
  if (T < 0) return MOE_ERR_BAD_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !Wr || !idx || !w || !logits) return MOE_ERR_BAD_ARG;
  if (!aligned(x, 16) || !aligned(Wr, 16)) return MOE_ERR_BAD_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  RouteArgs ra{};
  ra.H = dims->H;
  ra.E = dims->E;
  ra.k = dims->k;
  ra.T = T;
  ra.x = x;
  ra.Wr = Wr;
  ra.logits = logits;
  ra.epc = 2;
  ra.tt = T < 2 ? T : 2;
  ra.done = nullptr;
  ra.status = nullptr;
  ra.wait_limit = wait_limit_cycles();
  cudaError_t err = launch_route_decode(ra, s);
  if (err != cudaSuccess) return cuda_status(err);
  return cuda_status(launch_topk(logits, T, dims->E, dims->k, idx, w, route_counts_opt, s));
}

int moe_bucket(const moe_dims *dims, int32_t T, const int32_t *idx, int32_t *cnt, int32_t *off,
               int32_t *uni, int32_t *n_uni, int32_t *perm, void *stream) {
  int rc = moe_check_dims(dims);
  if (rc != MOE_OK) return rc;
  if (T < 0) return MOE_ERR_BAD_ARG;
  if (!cnt || !off || !uni || !n_uni || (T > 0 && (!idx || !perm))) return MOE_ERR_BAD_ARG;
  BucketArgs a{};
  a.E = dims->E;
  a.k = dims->k;
  a.T = T;
  a.idx = idx;
  a.cnt = cnt;
  a.off = off;
  a.uni = uni;
  a.n_uni = n_uni;
  a.perm = perm;
  a.pos = nullptr;
  a.pair_tok = nullptr;
  return cuda_status(launch_bucket(a, static_cast<cudaStream_t>(stream)));
}

// The layer after argument checks; `zeroed`: the caller has already zeroed the
// status word and the router's arrival counter for this call.
static int forward_checked(const moe_dims &d, int32_t T, const float *x, const float *Wr, const void *const *expert_table,
                    float *out, void *ws, int32_t *route_counts_opt, bool pf, const WsLayout &L, bool zeroed,
                    cudaStream_t s, const Owned &ow, bool auto_path = true) {
  int rc = MOE_OK;
  const moe_dims *dims = &d;
  // One token, or a small batch on the auto path: one fused launch streams
  // the tokens' experts one token after the other.  At these sizes the batch
  // union is nearly the sum of the tokens' selections, so per-token streaming
  // costs few extra bytes and runs at the fused kernel's rate.  The kernel
  // zeroes its own control words and status word: no memset before it.
  if (!pf && (T == 1 || (auto_path && T <= kDecodeTMax)) && fused_fits(d, kFmtInt4))
  {
    rc = fused_forward(d, L, x, Wr, expert_table, out, ws, route_counts_opt, prof_next(), ow, s, kFmtInt4, T);
    return rc == kFusedNA ? MOE_ERR_SHAPE : rc;
  }
  if (!zeroed) {
    // status word and the router's arrival counter start at zero on every call
    cudaError_t err = cudaMemsetAsync(ws, 0, L.xin, s);
    if (err != cudaSuccess) return cuda_status(err);
  }
  if (pf) return prefill_forward(*dims, T, x, Wr, expert_table, out, ws, L, route_counts_opt, s);
  unsigned long long *prof = prof_next();
  for (int t0 = 0; t0 < T; t0 += kDecodeTMax) {
    const int Tc = (T - t0) < kDecodeTMax ? (T - t0) : kDecodeTMax;
    rc = route_chunk(*dims, t0, Tc, L, x, Wr, ws, route_counts_opt, prof, ow, s);
    if (rc != MOE_OK) return rc;
    rc = experts_chunk(*dims, t0, Tc, L, expert_table, out, ws, prof, ow, s);
    if (rc != MOE_OK) return rc;
  }
  return MOE_OK;
}

int moe_layer_forward(const moe_dims *dims, int32_t T, const float *x, const float *Wr,
                      const void *const *expert_table, float *out, void *ws, size_t ws_bytes,
                      int32_t *route_counts_opt, int32_t path, void *stream) {
  int rc = moe_check_dims(dims);
  if (rc != MOE_OK) return rc;
  if (T < 0 || path < MOE_PATH_AUTO || path > MOE_PATH_PREFILL) return MOE_ERR_BAD_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !Wr || !expert_table || !out || !ws) return MOE_ERR_BAD_ARG;
  if (!aligned(x, 16) || !aligned(Wr, 16) || !aligned(out, 16)) return MOE_ERR_BAD_ARG;
  if (!aligned(ws, 256)) return MOE_ERR_WORKSPACE;
  const bool pf = use_prefill(T, path);
  const WsLayout L = ws_layout(*dims, T, pf);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  return forward_checked(*dims, T, x, Wr, expert_table, out, ws, route_counts_opt, pf, L, false,
                         static_cast<cudaStream_t>(stream), all_owned(*dims), path == MOE_PATH_AUTO);
}

int moe_layer_forward_mxfp4(const moe_dims *dims, int32_t T, const float *x, const float *Wr,
                            const void *const *expert_table, float *out, void *ws, size_t ws_bytes,
                            int32_t *route_counts_opt, void *stream) {
  int rc = moe_check_dims(dims);
  if (rc != MOE_OK) return rc;
  if (T < 0) return MOE_ERR_BAD_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !Wr || !expert_table || !out || !ws) return MOE_ERR_BAD_ARG;
  if (!aligned(x, 16) || !aligned(Wr, 16) || !aligned(out, 16)) return MOE_ERR_BAD_ARG;
  if (!aligned(ws, 256)) return MOE_ERR_WORKSPACE;
  const WsLayout L = ws_layout(*dims, T, false);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  if (!fused_fits(*dims, kFmtMxfp4)) return MOE_ERR_SHAPE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned long long *prof = prof_next();
  if (T == 1 || T > kDecodeTMax) {
    // token by token with the kernel's own routing; every launch zeroes its
    // control words, the first one the status word too (a later launch
    // keeps an earlier one's error)
    for (int t = 0; t < T; ++t) {
      // token t in the per-token rows of the workspace; the pair rows are reused
      WsLayout Lt = L;
      Lt.xq += (size_t)t * dims->H;
      Lt.xd += (size_t)t * (dims->H / 32) * 4;
      Lt.logits += (size_t)t * dims->E * 4;
      Lt.idx += (size_t)t * dims->k * 4;
      Lt.w += (size_t)t * dims->k * 4;
      rc = fused_forward(*dims, Lt, x + (size_t)t * dims->H, Wr, expert_table, out + (size_t)t * dims->H, ws,
                         route_counts_opt, t == 0 ? prof : nullptr, all_owned(*dims), s, kFmtMxfp4, 1, t == 0);
      if (rc != MOE_OK) return rc == kFusedNA ? MOE_ERR_SHAPE : rc;
    }
    return MOE_OK;
  }
  rc = fused_forward(*dims, L, x, Wr, expert_table, out, ws, route_counts_opt, prof, all_owned(*dims), s, kFmtMxfp4,
                     T);
  return rc == kFusedNA ? MOE_ERR_SHAPE : rc;
}

int moe_layer_forward_ep(const moe_dims *dims, int32_t T, const float *x, const float *Wr,
                         const void *const *expert_table, float *out, void *ws, size_t ws_bytes,
                         int32_t *route_counts_opt, int32_t expert_lo, int32_t expert_hi,
                         int32_t with_shared, void *stream) {
  int rc = moe_check_dims(dims);
  if (rc != MOE_OK) return rc;
  if (T < 0 || expert_lo < 0 || expert_hi < expert_lo || expert_hi > dims->E) return MOE_ERR_BAD_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !Wr || !expert_table || !out || !ws) return MOE_ERR_BAD_ARG;
  if (!aligned(x, 16) || !aligned(Wr, 16) || !aligned(out, 16)) return MOE_ERR_BAD_ARG;
  if (!aligned(ws, 256)) return MOE_ERR_WORKSPACE;
  const WsLayout L = ws_layout(*dims, T, false);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  return forward_checked(*dims, T, x, Wr, expert_table, out, ws, route_counts_opt, false, L, false,
                         static_cast<cudaStream_t>(stream),
                         Owned{expert_lo, expert_hi, with_shared ? 1 : 0});
}

int moe_layer_route(const moe_dims *dims, int32_t T, const float *x, const float *Wr, void *ws,
                    size_t ws_bytes, int32_t *route_counts_opt, void *stream) {
  int rc = moe_check_dims(dims);
  if (rc != MOE_OK) return rc;
  if (T < 0 || T > kDecodeTMax) return MOE_ERR_BAD_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !Wr || !ws) return MOE_ERR_BAD_ARG;
  if (!aligned(x, 16) || !aligned(Wr, 16)) return MOE_ERR_BAD_ARG;
  if (!aligned(ws, 256)) return MOE_ERR_WORKSPACE;
  const WsLayout L = ws_layout(*dims, T);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t err = cudaMemsetAsync(ws, 0, L.xin, s);
  if (err != cudaSuccess) return cuda_status(err);
  return route_chunk(*dims, 0, T, L, x, Wr, ws, route_counts_opt, prof_next(), all_owned(*dims), s);
}

int moe_read_union(const moe_dims *dims, int32_t T, void *ws, int32_t *host_uni, int32_t *host_n,
                   void *stream) {
  int rc = moe_check_dims(dims);
  if (rc != MOE_OK) return rc;
  if (T < 0 || !ws || !host_uni || !host_n) return MOE_ERR_BAD_ARG;
  const WsLayout L = ws_layout(*dims, T);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t st[2] = {0, 0};
  cudaError_t err = cudaMemcpyAsync(host_n, at<int32_t>(ws, L.n_uni), 4, cudaMemcpyDeviceToHost, s);
  if (err == cudaSuccess)
    err = cudaMemcpyAsync(host_uni, at<int32_t>(ws, L.uni), (size_t)dims->E * 4,
                          cudaMemcpyDeviceToHost, s);
  if (err == cudaSuccess)
    err = cudaMemcpyAsync(st, at<int32_t>(ws, L.status), 8, cudaMemcpyDeviceToHost, s);
  if (err == cudaSuccess) err = cudaStreamSynchronize(s);
  if (err != cudaSuccess) return cuda_status(err);
  if (st[0] != 0) return st[0];
  if (*host_n < 0 || *host_n > dims->E) return MOE_ERR_DEVICE;
  return MOE_OK;
}

int moe_layer_experts(const moe_dims *dims, int32_t T, const void *const *expert_table, float *out,
                      void *ws, size_t ws_bytes, void *stream) {
  int rc = moe_check_dims(dims);
  if (rc != MOE_OK) return rc;
  if (T < 0 || T > kDecodeTMax) return MOE_ERR_BAD_ARG;
  if (T == 0) return MOE_OK;
  if (!expert_table || !out || !ws) return MOE_ERR_BAD_ARG;
  if (!aligned(out, 16)) return MOE_ERR_BAD_ARG;
  if (!aligned(ws, 256)) return MOE_ERR_WORKSPACE;
  const WsLayout L = ws_layout(*dims, T);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  return experts_chunk(*dims, 0, T, L, expert_table, out, ws, prof_current(), all_owned(*dims),
                       static_cast<cudaStream_t>(stream));
}

int moe_layer_forward_host(const moe_dims *dims, int32_t T, const float *x_host, const float *Wr,
                           const void *const *expert_table, float *out_host, void *ws,
                           size_t ws_bytes, int32_t *route_counts_opt, int32_t path, void *stream) {
  int rc = moe_check_dims(dims);
  if (rc != MOE_OK) return rc;
  if (T < 0) return MOE_ERR_BAD_ARG;
  if (T == 0) return MOE_OK;
  if (!x_host || !out_host || !ws) return MOE_ERR_BAD_ARG;
  if (!aligned(ws, 256)) return MOE_ERR_WORKSPACE;
  if (path < MOE_PATH_AUTO || path > MOE_PATH_PREFILL) return MOE_ERR_BAD_ARG;
  const WsLayout L = ws_layout(*dims, T, use_prefill(T, path));
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  if (!Wr || !expert_table || !aligned(Wr, 16)) return MOE_ERR_BAD_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float *xd = at<float>(ws, L.xin);
  float *yd = at<float>(ws, L.yout);
  const bool pf = use_prefill(T, path);
  const size_t bytes = (size_t)T * dims->H * sizeof(float);
  // Pinned host buffers the device can address: x comes across in the kernel
  // that also zeroes the control words, and the decode path's down kernel
  // writes out straight into host memory -- no separate copies.  Anything else
  // (pageable memory, the prefill path's out) goes through cudaMemcpyAsync.
  const float *x_dev_view = static_cast<const float *>(host_device_view(x_host));
  float *out_dev_view = pf ? nullptr : static_cast<float *>(const_cast<void *>(host_device_view(out_host)));
  cudaError_t err;
  if (x_dev_view != nullptr && aligned(x_dev_view, 16)) {
    err = launch_stage_in(x_dev_view, xd, (int64_t)T * dims->H, ws, L.xin, s);
  } else {
    err = cudaMemcpyAsync(xd, x_host, bytes, cudaMemcpyHostToDevice, s);
    if (err == cudaSuccess) err = cudaMemsetAsync(ws, 0, L.xin, s);
  }
  if (err != cudaSuccess) return cuda_status(err);
  float *out_target = (out_dev_view != nullptr && aligned(out_dev_view, 16)) ? out_dev_view : yd;
  rc = forward_checked(*dims, T, xd, Wr, expert_table, out_target, ws, route_counts_opt, pf, L, true, s,
                       all_owned(*dims), path == MOE_PATH_AUTO);
  if (rc != MOE_OK) return rc;
  if (out_target == out_dev_view) return MOE_OK;
  return cuda_status(cudaMemcpyAsync(out_host, yd, bytes, cudaMemcpyDeviceToHost, s));
}

}  // extern "C"
