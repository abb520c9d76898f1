/*
 * moe.h -- C ABI of libmoe: the routed-expert MoE layer (softmax top-k router,
 * batch union, int4 gs64 x Q8_0 SwiGLU experts, shared expert, weighted
 * combine) on NVIDIA B200 (sm_100a).
 *
 * What the layer is, by page and section of the sources:
 *  - MoE layer with 256 routed experts per layer plus shared experts kept in
 *    the resident dense part; only the routed experts are streamed:
 *    "colibrì：把 744B 模型当数据流流到 25GB 的笔记本上跑" (tantan.ink),
 *    section 它的核心判断.
 *  - int4 weights with one scale per group of 64 ("gs64 group-scaled"): same
 *    page, section 我看到的几个坑.
 *  - int8 activations in 32-wide blocks with one scale per block ("Q8_0
 *    style") and an integer dot kernel: "Colibri：革命性 AI 引擎" (alphamatch.ai),
 *    section 優化整數核心.
 *  - batch union (each selected expert read once per batch) and gate/up/down
 *    stored next to each other: tantan.ink page, section 几个关键工程动作.
 *  - per-layer LRU cache, learned pins from route counts, one-layer-ahead
 *    prefetch: same section, and "colibri deep review" (ai-tools-nav), the
 *    "权重 JIT" row of its technique table.
 *
 * Conventions (every entry point):
 *  - Returns MOE_OK (0) or a negative MOE_ERR_* code.  Argument and shape
 *    errors are detected on the host before anything is enqueued.
 *  - Tensor pointers are DEVICE pointers owned by the caller unless the
 *    parameter says "host".  The library never frees caller memory.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls are asynchronous on that stream.
 *  - Device-side failures (a bounded wait that ran out, a misaligned expert
 *    pointer) are written to the status word of the workspace (see
 *    moe_workspace_view); kernels never trap.
 *  - Not thread-safe for concurrent calls sharing one workspace.
 *
 * Data layouts (row-major, little-endian):
 *  - Expert blob: gate [I][H] | up [I][H] | down [H][I], each matrix
 *    [N][K] stored as N*K/2 packed bytes then N*K/64 fp16 scales.
 *    Group g of row n = bytes [32g, 32g+32) of the row; byte j holds element
 *    64g+j in its low nibble and element 64g+32+j in its high nibble; a
 *    nibble u encodes w = u - 8 in [-8, 7]; dequantised weight = w * scale.
 *    Blob pointers must be 16-byte aligned.
 *  - Q8_0 vectors: int8 codes [n] and fp32 scales [n/32]; d = amax/127,
 *    q = round-half-even(x/d), all-zero codes when d == 0.
 *  - Shapes: H % 128 == 0, I % 128 == 0, H <= 8192, I <= 4096,
 *    1 <= k <= min(E, 32), E <= 1024.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_GROUP 64 /* int4 weights per fp16 scale */
#define MOE_BLOCK 32 /* int8 activations per fp32 scale */
#define MOE_MAX_E 1024
#define MOE_DECODE_T_MAX 16 /* largest batch the decode kernels take in one call */

enum moe_status {
  MOE_OK = 0,
  MOE_ERR_BAD_ARG = -1,     /* NULL pointer, negative size, bad enum */
  MOE_ERR_SHAPE = -2,       /* dims outside the accepted shapes */
  MOE_ERR_CUDA = -3,        /* a CUDA runtime call failed */
  MOE_ERR_WORKSPACE = -4,   /* workspace too small or misaligned */
  MOE_ERR_CACHE_FULL = -5,  /* every cache slot is pinned or in use */
  MOE_ERR_NOT_RESIDENT = -6,/* expert not in the cache */
  MOE_ERR_TIMEOUT = -7,     /* a device-side bounded wait ran out */
  MOE_ERR_DEVICE = -8,      /* device-side check failed (see status word) */
  MOE_ERR_ALLOC = -9,       /* host or device allocation failed */
  MOE_ERR_IO = -10          /* a file is missing, unreadable or corrupt */
};

typedef struct moe_dims {
  int32_t H; /* hidden size */
  int32_t I; /* SwiGLU intermediate size of every expert (routed and shared) */
  int32_t E; /* routed experts */
  int32_t k; /* experts kept per token */
} moe_dims;

enum moe_path {
  MOE_PATH_AUTO = 0,    /* decode kernels for T <= MOE_DECODE_T_MAX, else prefill */
  MOE_PATH_DECODE = 1,  /* union GEMV kernels, T in chunks of MOE_DECODE_T_MAX */
  MOE_PATH_PREFILL = 2  /* grouped GEMM over the expert union */
};

/* Human-readable name of a status code (static string). */
const char *moe_status_string(int status);

/* MOE_OK if the dims are accepted, else MOE_ERR_SHAPE / MOE_ERR_BAD_ARG. */
int moe_check_dims(const moe_dims *dims);

/* Bytes of one expert blob: 3*H*I/2 + 3*H*I/32 (20,054,016 for H=6144,
 * I=2048).  0 if the dims are not accepted. */
size_t moe_expert_bytes(const moe_dims *dims);

/* Device workspace needed by moe_layer_forward for batches of up to T_max
 * tokens on the path MOE_PATH_AUTO picks for T_max (256-byte aligned
 * segments).  0 if the dims are not accepted. */
size_t moe_workspace_bytes(const moe_dims *dims, int32_t T_max);

/* Same for an explicit path: MOE_PATH_PREFILL needs the prefill segments (the
 * fp16 hi/lo activation rows and the per-pair down rows, about
 * T*(k+1)*(2H+I)*4 bytes) for any T; MOE_PATH_DECODE never does. */
size_t moe_workspace_bytes_path(const moe_dims *dims, int32_t T_max, int32_t path);

/* Q8_0 quantisation of rows x T x cols fp32 (cols % 32 == 0):
 * q [rows][cols] int8, d [rows][cols/32] fp32.  Bit-exact definition above.
 * (Q8_0-style activations: alphamatch.ai page, section 優化整數核心.) */
int moe_quant_q8_0(const float *x, int64_t rows, int32_t cols, int8_t *q, float *d,
                   void *stream);

/* Router: logits[t][e] = x[t] . Wr[e] in the library's fixed fp32 order
 * (32 strided fmaf chains, xor tree), then top-k per token (ties to the lower
 * expert index, listed by descending logit) and the softmax over the k kept
 * logits.  x [T][H] fp32, Wr [E][H] fp32 (both 16-byte aligned), idx [T][k]
 * int32, w [T][k] fp32, logits [T][E] fp32 (written; also the scratch the
 * top-k reads), route_counts_opt [E] int32 or NULL
 * (incremented by one per selection: the route-count record behind learned
 * pins, tantan.ink page section 几个关键工程动作). */
int moe_router_topk(const moe_dims *dims, int32_t T, const float *x, const float *Wr,
                    int32_t *idx, float *w, float *logits, int32_t *route_counts_opt,
                    void *stream);

/* Batch union (tantan.ink page, section 几个关键工程动作): counting sort of the
 * T*k (token, slot) pairs by expert.  idx [T][k] int32 ->
 *   cnt [E]      pairs per expert
 *   off [E+1]    exclusive prefix sum, off[E] = T*k
 *   uni [E]      experts with cnt > 0, ascending (first *n_uni entries)
 *   n_uni [1]    union size
 *   perm [T*k]   pair ids t*k+s grouped by expert, ascending inside a group.
 * All outputs are bit-exact (one correct answer). */
int moe_bucket(const moe_dims *dims, int32_t T, const int32_t *idx, int32_t *cnt,
               int32_t *off, int32_t *uni, int32_t *n_uni, int32_t *perm, void *stream);

/* The whole layer on T tokens.
 * Both paths: the Q8_0 codes of x, the router logits (canonical fixed fp32
 * order), the top-k indices and the union (cnt, off, uni, perm) are bit-exact;
 * the softmax weights agree with the definition within a few units in the
 * last place (CUDA's expf); the outputs are within the layer's float
 * tolerance of the definition (relative L2 <= 1e-4, max-abs <= 2e-3 rms), a
 * Q8_0 code of SiLU(g)*u differing by one where h lies within rounding of a
 * code boundary.  Each path is deterministic: the same call gives the same
 * bits.
 * Decode path (T <= MOE_DECODE_T_MAX under MOE_PATH_AUTO): one cooperative
 * kernel (one CTA per SM) routes the batch and streams each token's experts in
 * turn -- routing, gate/up, down and combine, the expert sums in the kernels'
 * own fixed fp32 order -- when the shape fits it.  That kernel zeroes its own
 * control words (nothing else is enqueued), so the call can be captured in a
 * CUDA graph and replayed; make one call with the same dims on the device
 * before capturing (it sets the kernels' attributes).  MOE_PATH_DECODE at 2 or
 * more tokens (and a shape the cooperative kernel does not fit) runs three
 * kernels per 16 tokens over the batch union instead (routing, gate/up, down +
 * combine), each union expert's bytes streamed once; one token takes the
 * cooperative kernel on either path.  Both give the same bits.
 * Prefill path: router GEMM, top-k, bucketing, then a grouped GEMM over the
 * union on the tensor cores (the int4 weights, exact in fp16, times an fp16
 * hi + lo split of the dequantised Q8_0 activations, 22 significant bits;
 * fp32 accumulation; weight scales applied per group) and the combine.  (Batched expert unions: colibri deep review
 * page, technology table, row I/O 即引擎; prefill GEMM order: tantan.ink
 * page, section 我看到的几个坑.)
 * Arguments:
 *   x [T][H] fp32 (the normalised hidden state; no residual, no norm here),
 *   Wr [E][H] fp32,
 *   expert_table: DEVICE array of E+1 device pointers to expert blobs;
 *                 entry E is the shared expert (weight 1),
 *   out [T][H] fp32 = shared(x) + sum_s w[t,s] * expert_{idx[t,s]}(x),
 *   ws / ws_bytes: device workspace of at least moe_workspace_bytes_path(dims,
 *                  T, path),
 *                  256-byte aligned; holds every intermediate (see view),
 *   route_counts_opt [E] int32 or NULL (incremented per selection),
 *   path: enum moe_path.
 * Every step runs in the library's kernels; nothing is synchronised with the
 * host.  Device-side failures (a bounded wait that ran out, a misaligned
 * blob) are written to the workspace status word (see moe_ws_view), which
 * every call resets first: read it after a call and before the next. */
int moe_layer_forward(const moe_dims *dims, int32_t T, const float *x, const float *Wr,
                      const void *const *expert_table, float *out, void *ws, size_t ws_bytes,
                      int32_t *route_counts_opt, int32_t path, void *stream);

/* Same as moe_layer_forward with x_host [T][H] and out_host [T][H] in HOST
 * memory.  Pinned memory the device can address (cudaHostAlloc /
 * cudaMallocHost, or registered and mapped) moves without separate copies: a
 * staging kernel reads x across the link into the workspace while it zeroes
 * the control words, and on the decode path the down kernel stores out
 * straight into out_host.  Other memory (pageable) goes through
 * cudaMemcpyAsync before and after the layer; so does out on the prefill path.
 * Everything is enqueued on `stream`; the call returns after enqueueing
 * (synchronise the stream before reading out_host). */
int moe_layer_forward_host(const moe_dims *dims, int32_t T, const float *x_host,
                           const float *Wr, const void *const *expert_table, float *out_host,
                           void *ws, size_t ws_bytes, int32_t *route_counts_opt, int32_t path,
                           void *stream);

/* moe_layer_forward without a caller workspace.  (No counterpart in the
 * source pages: this is an interface convenience of this library.)
 * For callers that cannot call cudaMalloc -- code that runs inside a host
 * which owns and budgets all device memory, or latency-critical paths that
 * must not allocate once they are running -- the workspace lives in the
 * library itself: one statically allocated device array of
 * MOE_STATIC_WS_BYTES (4 MiB) per GPU that loads the library, held until the
 * process exits.  Arguments as moe_layer_forward.  The call allocates
 * nothing.  Its first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current and keeps it for later
 * calls; make that first call before capturing any stream into a graph, and
 * do not reset the device's context (cudaDeviceReset) between calls, which
 * would leave the kept address stale.  Batches whose workspace
 * (moe_workspace_bytes) exceeds MOE_STATIC_WS_BYTES are refused with
 * MOE_ERR_WORKSPACE and a message on stderr (for H=6144, I=2048, E=256,
 * k=8 every T <= 16 fits).  All calls share the one array and each call
 * leaves its intermediates there (the call resets what must start at zero);
 * calls whose work overlaps on the GPU, e.g. on two streams at once, race on
 * it and give wrong results. */
#define MOE_STATIC_WS_BYTES (4u << 20)
int moe_layer_forward_static(const moe_dims *dims, int32_t T, const float *x, const float *Wr,
                             const void *const *expert_table, float *out, int32_t *route_counts_opt,
                             int32_t path, void *stream);

/* The layer with MXFP4 expert blobs: the format in which the Kimi K3
 * family's experts ship, QAT-trained and streamed without conversion (colibri
 * deep review page, model-family table, Kimi K3 row).  Each blob is
 * gate [I][H] | up [I][H] | down [H][I]; a matrix [N][K] is N*K/2 bytes of
 * E2M1 codes (two consecutive elements per byte, the lower-indexed one in the
 * low nibble; sign bit, two exponent bits of bias 1, one mantissa bit) then
 * N*K/32 E8M0 exponent bytes, one per 32-block of a row (weight =
 * e2m1 * 2^(E - 127), E = 255 outside the contract): the same byte count as
 * int4 gs64.  Activations stay Q8_0, so every block sum is exact in integers
 * (2 * e2m1 is an integer).  Decode path only, in the fused kernel: up to
 * MOE_DECODE_T_MAX tokens in one launch (the workspace holds the batch's
 * routing record); larger batches token by token (the record then holds the
 * last token's).  MOE_ERR_SHAPE if the shape does not fit the fused kernel.  Other arguments as
 * moe_layer_forward (workspace: moe_workspace_bytes_path(dims, T,
 * MOE_PATH_DECODE)). */
int moe_layer_forward_mxfp4(const moe_dims *dims, int32_t T, const float *x, const float *Wr,
                            const void *const *expert_table, float *out, void *ws, size_t ws_bytes,
                            int32_t *route_counts_opt, void *stream);

/* One rank's share of the layer under expert parallelism (GPU form of the
 * pages' cluster mode, where the routed-expert FFNs run on workers: colibri
 * deep review page, its local-cluster section).  Routing (Q8_0 of x, logits,
 * top-k, softmax, union) covers every expert, as in moe_layer_forward, and
 * writes the same workspace record; then only the union experts e with
 * expert_lo <= e < expert_hi, and the shared expert if with_shared != 0, run
 * their FFNs, and
 *   out[t] = [with_shared: shared(x_t)] + sum over s with expert_lo <= idx[t,s] < expert_hi
 *            of w[t,s] * expert_{idx[t,s]}(x_t),
 * in the same order as moe_layer_forward (the terms of other ranks left out).
 * Summing every rank's out over a partition of [0, E) with the shared expert
 * on one rank (an all-reduce) gives the layer's output within its float
 * tolerance.  expert_table entries outside the range (and entry E when
 * !with_shared) are never read and may be NULL.  Always the decode path
 * (up to MOE_DECODE_T_MAX tokens in the fused kernel, larger batches in
 * chunks of MOE_DECODE_T_MAX on the union kernels).
 * MOE_ERR_BAD_ARG unless 0 <= expert_lo <= expert_hi <= E.  Other arguments
 * as moe_layer_forward; workspace: moe_workspace_bytes_path(dims, T,
 * MOE_PATH_DECODE). */
int moe_layer_forward_ep(const moe_dims *dims, int32_t T, const float *x, const float *Wr,
                         const void *const *expert_table, float *out, void *ws, size_t ws_bytes,
                         int32_t *route_counts_opt, int32_t expert_lo, int32_t expert_hi,
                         int32_t with_shared, void *stream);

/* The layer in two halves, for callers that must place the experts between
 * routing and the FFN (the tiered cache below):
 *   moe_layer_route:   Q8_0 of x, router + top-k + softmax, batch union into ws
 *                      (T <= MOE_DECODE_T_MAX);
 *   moe_read_union:    copies the union of that call to host memory
 *                      (synchronises `stream`): host_uni [E], *host_n;
 *   moe_layer_experts: gate/up + SwiGLU + requant and down + combine for the
 *                      routing held in ws; expert_table entries are read only
 *                      for the union experts and the shared expert (E).
 * moe_layer_route + moe_layer_experts == moe_layer_forward, bit for bit. */
int moe_layer_route(const moe_dims *dims, int32_t T, const float *x, const float *Wr, void *ws,
                    size_t ws_bytes, int32_t *route_counts_opt, void *stream);
int moe_read_union(const moe_dims *dims, int32_t T, void *ws, int32_t *host_uni, int32_t *host_n,
                   void *stream);
int moe_layer_experts(const moe_dims *dims, int32_t T, const void *const *expert_table, float *out,
                      void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------
 * HBM expert cache over host memory: the VRAM tier above host RAM
 * ("三层 memory hierarchy", tantan.ink page, section 它的核心判断), with a
 * per-layer LRU, pins learned from route counts and one-layer-ahead
 * prefetch (section 几个关键工程动作; "colibri deep review", 权重 JIT row).
 *
 * The cache owns a pool of expert-sized slots in HBM (allocated once at
 * create), split evenly between the layers; each layer keeps its own LRU
 * order and pin set.  Copies host -> HBM are cudaMemcpyAsync of whole blobs
 * (one blob = gate|up|down, one transfer) on the stream given to the call;
 * a slot is never overwritten before the kernels that last read it are done
 * (an event recorded by expert_cache_release).  Placement changes speed,
 * never results: the tiered output is bitwise the resident output.
 * host_blobs: [n_layers][E+1] host pointers (pinned memory for async copies;
 * entry E of a layer = its shared expert), owned by the caller, alive until
 * destroy.  backend MOE_CACHE_HOST runs the same policy with host memory as
 * the "HBM" pool and memcpy copies (no GPU; for tests of the policy).
 * ------------------------------------------------------------------------ */
typedef struct moe_cache moe_cache;

enum moe_cache_backend { MOE_CACHE_DEVICE = 0, MOE_CACHE_HOST = 1 };

/* fault kinds for expert_cache_inject_fault (host side, never on the GPU) */
enum moe_cache_fault {
  MOE_FAULT_NONE = 0,
  MOE_FAULT_COPY = 1,   /* the next `count` blob copies report an error */
  MOE_FAULT_ALLOC = 2   /* the next create() pool allocation fails (global) */
};

typedef struct moe_cache_stats {
  uint64_t hits;            /* requested experts already resident */
  uint64_t misses;          /* requested experts copied on demand */
  uint64_t prefetches;      /* blobs copied by expert_cache_prefetch */
  uint64_t prefetch_hits;   /* requested experts resident thanks to a prefetch */
  uint64_t evictions;
  uint64_t bytes_h2d;       /* bytes copied host -> pool */
  uint64_t copy_errors;
  int32_t slots;            /* slots in the pool */
  int32_t slots_per_layer;
  int32_t pinned;           /* pinned experts, all layers */
  int32_t resident;         /* resident experts, all layers */
} moe_cache_stats;

int expert_cache_create(const moe_dims *dims, int32_t n_layers, const void *const *host_blobs,
                        size_t hbm_bytes, int32_t backend, moe_cache **out);
void expert_cache_destroy(moe_cache *cache);
/* Pin: make resident (copied on `stream` if needed) and never evict. */
int expert_cache_pin(moe_cache *cache, int32_t layer, const int32_t *experts, int32_t n,
                     void *stream);
int expert_cache_unpin(moe_cache *cache, int32_t layer, const int32_t *experts, int32_t n);
/* Evict (unpinned, resident) experts now; pinned ones are skipped. */
int expert_cache_evict(moe_cache *cache, int32_t layer, const int32_t *experts, int32_t n);
/* Start copies of the listed experts that are not resident on `side_stream`
 * (one-layer-ahead prefetch); returns the number of copies started.  Never
 * evicts pinned experts; gives up (returning what it started) when the
 * layer has no evictable slot. */
int expert_cache_prefetch(moe_cache *cache, int32_t layer, const int32_t *experts, int32_t n,
                          void *side_stream);
/* Make the listed experts (and the shared expert E) resident -- misses are
 * copied on `copy_stream` -- and return in *d_table a device table of E+1
 * blob pointers for the layer (NULL for experts not resident), valid until
 * the next acquire of the same layer.  `compute_stream` is made to wait for
 * every copy the listed experts depend on.  MOE_ERR_CACHE_FULL if the layer
 * cannot hold them all. */
int expert_cache_acquire(moe_cache *cache, int32_t layer, const int32_t *experts, int32_t n,
                         void *copy_stream, void *compute_stream, const void **d_table);
/* Record on `compute_stream` that the kernels reading the layer's last
 * acquired experts have been enqueued (their slots may be reused after). */
int expert_cache_release(moe_cache *cache, int32_t layer, void *compute_stream);
/* Learned pins: unpin the layer, then pin its n_pin most routed experts by
 * the host counts [E] (ties to the lower index). */
int expert_cache_learn_pins(moe_cache *cache, int32_t layer, const int32_t *host_counts,
                            int32_t n_pin, void *stream);
int expert_cache_resident(const moe_cache *cache, int32_t layer, int32_t expert);
int expert_cache_pinned(const moe_cache *cache, int32_t layer, int32_t expert);
int expert_cache_stats(const moe_cache *cache, moe_cache_stats *stats);
/* Host-side fault injection for failure tests (see enum moe_cache_fault);
 * cache may be NULL for MOE_FAULT_ALLOC. */
int expert_cache_inject_fault(moe_cache *cache, int32_t kind, int32_t count);

/* Route-usage record on disk (the learned cache's history across sessions:
 * the engine writes the experts each turn routes to into a usage file and
 * pins the hottest -- tantan.ink page, section 几个关键工程动作; "colibri deep
 * review", 学习缓存 row).  counts: HOST array [n_layers][E] of selection
 * counts (the per-layer route_counts of the layer calls, widened to 64 bits).
 * moe_usage_save writes <path>.tmp and renames it over <path> (a reader never
 * sees a partial record); the file holds a magic tag, the version, n_layers,
 * E, the counts and an FNV-1a 64 hash of them.  moe_usage_load replaces
 * counts (accumulate = 0) or adds the file's counts to them (accumulate = 1);
 * MOE_ERR_SHAPE if the file was written for other n_layers / E, MOE_ERR_IO if
 * it is missing, truncated, longer than its record or fails its hash --
 * counts are left untouched on every error.  Host only; no GPU needed. */
int moe_usage_save(const char *path, int32_t n_layers, int32_t E, const uint64_t *counts);
int moe_usage_load(const char *path, int32_t n_layers, int32_t E, uint64_t *counts,
                   int32_t accumulate);

/* One tiered decode layer (native runtime of the cache):
 * route(x) -> read union -> acquire (misses copied on side_stream, compute
 * waits) -> if Wr_next is given, route the same x with the next layer's
 * router into ws_pred and prefetch that union for layer+1 on side_stream ->
 * experts -> release.  Synchronises with the host once per call (the union
 * read) and once more when predicting.  prefetch_out_opt (host, 2 ints):
 * [0] copies started for layer+1, [1] predicted union size. */
int moe_tiered_layer_forward(moe_cache *cache, int32_t layer, const moe_dims *dims, int32_t T,
                             const float *x, const float *Wr, const float *Wr_next_opt, float *out,
                             void *ws, size_t ws_bytes, void *ws_pred, size_t ws_pred_bytes,
                             int32_t *route_counts_opt, void *compute_stream, void *side_stream,
                             int32_t *prefetch_out_opt);

/* Device pointers to the intermediates a moe_layer_forward call leaves in its
 * workspace (for tests and tools).  Pair positions: the T*k routed pairs in
 * bucket order (position off[e]+i for the i-th pair of expert e), then T
 * shared-expert pairs at positions T*k + t. */
typedef struct moe_ws_view {
  int32_t *status;   /* [4]: [0] = MOE_OK or a device error code, [1] = detail */
  int8_t *xq;        /* [T][H] */
  float *xd;         /* [T][H/32] */
  float *logits;     /* [T][E] */
  int32_t *idx;      /* [T][k] */
  float *w;          /* [T][k] */
  int32_t *cnt;      /* [E] */
  int32_t *off;      /* [E+1] */
  int32_t *uni;      /* [E+1]: union ascending, then E (the shared expert) */
  int32_t *n_uni;    /* [1] */
  int32_t *perm;     /* [T*k] */
  int32_t *pos;      /* [T*k]: position of pair t*k+s */
  int32_t *pair_tok; /* [T*(k+1)]: token of each position */
  int8_t *hq;        /* [T*(k+1)][I] Q8_0 codes of SiLU(g)*u per position */
  float *hd;         /* [T*(k+1)][I/32] */
  int32_t T_max;
} moe_ws_view;

int moe_workspace_view(const moe_dims *dims, int32_t T_max, void *ws, moe_ws_view *view);

/* Wait limit of the kernels' bounded waits, in SM clock cycles, for layer
 * calls enqueued after this call (process-wide); cycles <= 0 restores the
 * default (2e9, about a second).  Returns the previous limit.  Every wait of
 * a kernel for data (an mbarrier phase: a copy landed, a stage freed, an MMA
 * done) gives up after the limit, writes MOE_ERR_TIMEOUT and the wait's
 * detail code to the workspace status word, and ends its role; the copies and
 * MMAs its CTA already issued are still awaited (with the default limit)
 * before the CTA exits, and the kernels after it in the call skip their work.
 * The workspace, the device and later calls stay usable.  A short limit is
 * for failure tests: it makes the waits of a healthy call run out.  (The
 * pages' engine degrades with a warning instead of crashing when a source
 * fails: tantan.ink page, section 我看到的几个坑.) */
int64_t moe_set_wait_limit(int64_t cycles);

/* Binary version (major * 10 + minor, e.g. 100 for sm_100a) of the kernels
 * the current device loaded from this library, or a negative status. */
int moe_device_binary_version(void);

/* Number of this library's kernels one moe_layer_forward call of T tokens on
 * `path` enqueues on the current device, or a negative status: 1 for a
 * decode call of up to MOE_DECODE_T_MAX tokens that the fused kernel runs
 * (nothing else is enqueued), 3 per 16-token chunk on the union kernels and 9
 * on the prefill path (each of those two also enqueues one workspace
 * memset). */
int moe_layer_launches(const moe_dims *dims, int32_t T, int32_t path);

/* Number of streaming multiprocessors the kernels size their grids for
 * (device of the current context), or a negative status. */
int moe_device_sms(void);

/* Per-call kernel timing on the device.  moe_profile_enable(1) allocates (once)
 * and zeroes a library-owned ring of 1024 records on the current device; from
 * then on every moe_layer_forward, and every moe_layer_route with the
 * moe_layer_experts that follows it, takes the next record, and its kernels
 * stamp each phase's first start and last end there with the GPU's global
 * nanosecond timer (thread 0 of every CTA, atomics; no stream events, so the
 * launch sequence and its programmatic dependent launches are unchanged).
 * Calls after the ring is full go unrecorded.  moe_profile_enable(0) stops
 * recording.
 * moe_profile_read(ms, max_calls) synchronizes the device, writes 4 floats
 * (milliseconds) per recorded call, oldest first, into ms[4 * max_calls]:
 *   [0] routing: decode = the routing kernel (Q8_0, logits, top-k, union);
 *       prefill = quantisation through the tensor-map build,
 *   [1] gate/up: decode = from the gate/up kernel's dependency wait to its
 *       last CTA's end; prefill = the gate/up grouped GEMM,
 *   [2] down: decode = the down kernel including its combine, from its first
 *       CTA's start (weight copies overlap the gate/up kernel's tail);
 *       prefill = the down grouped GEMM and the combine kernel,
 *   [3] the call: first start to last end over the three phases,
 * (0 for a phase that was not stamped), then zeroes the ring and starts a new
 * history.  Returns the number of calls written, or a negative status.
 * The profiling state is process-wide; a lock serialises these calls and the
 * record hand-out of concurrent layer calls. */
int moe_profile_enable(int on);
int moe_profile_read(float *ms, int max_calls);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H */
