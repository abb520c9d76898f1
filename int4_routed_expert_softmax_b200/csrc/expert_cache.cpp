// expert_cache.cpp -- HBM expert cache over host memory (the VRAM tier of the
// three-tier weight placement: "三层 memory hierarchy", tantan.ink page,
// section 它的核心判断), with a per-layer LRU, pins learned from route counts
// and one-layer-ahead prefetch (section 几个关键工程动作; "colibri deep
// review", 权重 JIT row).
//
// Pool: one cudaMalloc of n_slots expert-sized slots, split evenly between the
// layers (each layer has its own slots, LRU order and pins).  A blob (gate |
// up | down of one expert) moves host -> slot as ONE cudaMemcpyAsync, the
// engine's "one read per expert" (tantan.ink, 几个关键工程动作).
// Ordering: every copy into a slot first waits for the event recorded by the
// last expert_cache_release of the slot's layer (the kernels that read the
// old contents), and records a per-slot ready event that compute streams wait
// on before reading the slot.
// Backend MOE_CACHE_HOST keeps the policy identical but uses host memory and
// memcpy, so the policy and its failure paths are testable without a GPU.
#include <algorithm>
#include <atomic>
#include <chrono>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <list>
#include <vector>

#include <cuda_runtime.h>

#include "../../include/moe.h"
#include "moe_internal.h"

namespace {

int g_fault_alloc = 0;  // MOE_FAULT_ALLOC: pending allocation failures

struct Layer {
  std::vector<int> slot_of;       // [E+1] slot or -1
  std::vector<char> pinned;       // [E+1]
  std::vector<char> prefetched;   // [E+1] resident through a prefetch, not yet requested
  std::list<int> lru;             // resident experts, front = most recently used
  std::vector<std::list<int>::iterator> where;
  std::vector<int> free_slots;
  std::vector<int> last_slots;    // slots of the last acquire
  const void **h_table = nullptr; // pinned staging table [E+1]
  const void **d_table = nullptr; // device table [E+1]
  cudaEvent_t table_done = nullptr;
  bool table_pending = false;
  bool table_dirty = true;        // residency changed since the device table was uploaded
  cudaEvent_t released = nullptr; // last release of this layer
  bool released_valid = false;
  int n_pinned = 0;
};

}  // namespace

struct moe_cache {
  moe_dims d{};
  int L = 0, E1 = 0;
  size_t blob = 0;
  int backend = MOE_CACHE_DEVICE;
  std::vector<const unsigned char *> host;  // [L*(E+1)]
  unsigned char *pool = nullptr;
  int n_slots = 0, per_layer = 0;
  std::vector<Layer> layers;
  std::vector<cudaEvent_t> slot_ready;
  std::vector<char> slot_ready_valid;
  moe_cache_stats st{};
  int fault_copy = 0;
  // tiered layers: union mailboxes (mapped pinned host memory the routing
  // kernel writes; [0] this layer's union, [1] the predicted one), their
  // sequence counter, and the stream the one-layer-ahead prediction runs on
  int32_t *mbox_host[2] = {nullptr, nullptr};
  int32_t *mbox_dev[2] = {nullptr, nullptr};
  int32_t seq = 0;
  cudaStream_t pred_stream = nullptr;
  cudaEvent_t x_ready = nullptr;
};

namespace {

int cuda_err(cudaError_t e) {
  if (e == cudaSuccess) return MOE_OK;
  std::fprintf(stderr, "libmoe cache: CUDA error %d (%s)\n", (int)e, cudaGetErrorString(e));
  return MOE_ERR_CUDA;
}

bool dev(const moe_cache *c) { return c->backend == MOE_CACHE_DEVICE; }

void touch(Layer &ly, int e) {
  ly.lru.erase(ly.where[e]);
  ly.lru.push_front(e);
  ly.where[e] = ly.lru.begin();
}

void drop(moe_cache *c, Layer &ly, int e) {
  const int slot = ly.slot_of[e];
  ly.lru.erase(ly.where[e]);
  ly.slot_of[e] = -1;
  ly.table_dirty = true;
  ly.prefetched[e] = 0;
  ly.free_slots.push_back(slot);
  c->st.evictions++;
  c->st.resident--;
}

// A free slot of the layer, evicting its least recently used expert that is
// neither pinned nor protected.  -1 when none.
int take_slot(moe_cache *c, Layer &ly, const std::vector<char> &protect) {
  if (ly.free_slots.empty()) {
    for (auto it = ly.lru.rbegin(); it != ly.lru.rend(); ++it) {
      const int e = *it;
      if (!ly.pinned[e] && !protect[e]) {
        drop(c, ly, e);
        break;
      }
    }
  }
  if (ly.free_slots.empty()) return -1;
  const int s = ly.free_slots.back();
  ly.free_slots.pop_back();
  return s;
}

int copy_blob(moe_cache *c, int layer, int e, int slot, cudaStream_t s) {
  if (c->fault_copy > 0) {
    c->fault_copy--;
    c->st.copy_errors++;
    return MOE_ERR_CUDA;
  }
  Layer &ly = c->layers[layer];
  unsigned char *dst = c->pool + (size_t)slot * c->blob;
  const unsigned char *src = c->host[(size_t)layer * c->E1 + e];
  if (dev(c)) {
    if (ly.released_valid) {
      int rc = cuda_err(cudaStreamWaitEvent(s, ly.released, 0));
      if (rc) return rc;
    }
    if (c->slot_ready_valid[slot]) {
      // a copy into this slot may still be in flight, and on another stream
      // (acquire and prefetch take the caller's streams): this one follows it
      int rc = cuda_err(cudaStreamWaitEvent(s, c->slot_ready[slot], 0));
      if (rc) return rc;
    }
    int rc = cuda_err(cudaMemcpyAsync(dst, src, c->blob, cudaMemcpyHostToDevice, s));
    if (rc) {
      c->st.copy_errors++;
      return rc;
    }
    rc = cuda_err(cudaEventRecord(c->slot_ready[slot], s));
    if (rc) return rc;
    c->slot_ready_valid[slot] = 1;
  } else {
    std::memcpy(dst, src, c->blob);
  }
  c->st.bytes_h2d += c->blob;
  return MOE_OK;
}

// Make expert e of the layer resident; returns MOE_OK or an error.
int make_resident(moe_cache *c, int layer, int e, cudaStream_t s, const std::vector<char> &protect) {
  Layer &ly = c->layers[layer];
  if (ly.slot_of[e] >= 0) return MOE_OK;
  const int slot = take_slot(c, ly, protect);
  if (slot < 0) return MOE_ERR_CACHE_FULL;
  const int rc = copy_blob(c, layer, e, slot, s);
  if (rc != MOE_OK) {
    ly.free_slots.push_back(slot);
    return rc;
  }
  ly.slot_of[e] = slot;
  ly.table_dirty = true;
  ly.lru.push_front(e);
  ly.where[e] = ly.lru.begin();
  c->st.resident++;
  return MOE_OK;
}

bool valid_layer(const moe_cache *c, int layer) { return c && layer >= 0 && layer < c->L; }

int check_list(const moe_cache *c, const int32_t *experts, int32_t n, bool allow_shared) {
  if (n < 0 || (n > 0 && experts == nullptr)) return MOE_ERR_BAD_ARG;
  const int lim = allow_shared ? c->E1 : c->E1 - 1;
  for (int i = 0; i < n; ++i)
    if (experts[i] < 0 || experts[i] >= lim) return MOE_ERR_BAD_ARG;
  return MOE_OK;
}

void destroy_all(moe_cache *c) {
  if (!c) return;
  for (auto &ly : c->layers) {
    if (dev(c)) {
      if (ly.table_done) cudaEventDestroy(ly.table_done);
      if (ly.released) cudaEventDestroy(ly.released);
      if (ly.h_table) cudaFreeHost(ly.h_table);
      if (ly.d_table) cudaFree(ly.d_table);
    } else {
      std::free(ly.h_table);
    }
  }
  if (dev(c)) {
    for (auto ev : c->slot_ready)
      if (ev) cudaEventDestroy(ev);
    if (c->pool) cudaFree(c->pool);
    for (int i = 0; i < 2; ++i)
      if (c->mbox_host[i]) cudaFreeHost(c->mbox_host[i]);
    if (c->x_ready) cudaEventDestroy(c->x_ready);
    if (c->pred_stream) cudaStreamDestroy(c->pred_stream);
  } else {
    std::free(c->pool);
  }
  delete c;
}

}  // namespace

extern "C" {

int expert_cache_inject_fault(moe_cache *cache, int32_t kind, int32_t count) {
  if (count < 0) return MOE_ERR_BAD_ARG;
  switch (kind) {
    case MOE_FAULT_NONE:
      g_fault_alloc = 0;
      if (cache) cache->fault_copy = 0;
      return MOE_OK;
    case MOE_FAULT_COPY:
      if (!cache) return MOE_ERR_BAD_ARG;
      cache->fault_copy = count;
      return MOE_OK;
    case MOE_FAULT_ALLOC:
      g_fault_alloc = count;
      return MOE_OK;
    default:
      return MOE_ERR_BAD_ARG;
  }
}

int expert_cache_create(const moe_dims *dims, int32_t n_layers, const void *const *host_blobs,
                        size_t hbm_bytes, int32_t backend, moe_cache **out) {
  if (out == nullptr) return MOE_ERR_BAD_ARG;
  *out = nullptr;
  int rc = moe_check_dims(dims);
  if (rc != MOE_OK) return rc;
  if (n_layers <= 0 || host_blobs == nullptr) return MOE_ERR_BAD_ARG;
  if (backend != MOE_CACHE_DEVICE && backend != MOE_CACHE_HOST) return MOE_ERR_BAD_ARG;
  moe_cache *c = new moe_cache();
  c->d = *dims;
  c->L = n_layers;
  c->E1 = dims->E + 1;
  c->blob = moe::expert_bytes(dims->H, dims->I);
  c->backend = backend;
  c->host.resize((size_t)n_layers * c->E1);
  for (size_t i = 0; i < c->host.size(); ++i) {
    c->host[i] = static_cast<const unsigned char *>(host_blobs[i]);
    if (c->host[i] == nullptr) {
      delete c;
      return MOE_ERR_BAD_ARG;
    }
  }
  c->per_layer = (int)std::min<size_t>(hbm_bytes / c->blob / (size_t)n_layers, (size_t)c->E1);
  if (c->per_layer < 1) {
    delete c;
    return MOE_ERR_CACHE_FULL;
  }
  c->n_slots = c->per_layer * n_layers;
  const size_t pool_bytes = (size_t)c->n_slots * c->blob;
  if (g_fault_alloc > 0) {
    g_fault_alloc--;
    delete c;
    return MOE_ERR_ALLOC;
  }
  if (dev(c)) {
    if (cudaMalloc(&c->pool, pool_bytes) != cudaSuccess) {
      c->pool = nullptr;
      destroy_all(c);
      return MOE_ERR_ALLOC;
    }
    c->slot_ready.assign(c->n_slots, nullptr);
    for (auto &ev : c->slot_ready)
      if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) {
        destroy_all(c);
        return MOE_ERR_CUDA;
      }
    for (int i = 0; i < 2; ++i) {
      void *p = nullptr, *pd = nullptr;
      if (cudaHostAlloc(&p, sizeof(int32_t) * (size_t)(moe::kMailUni + dims->E), cudaHostAllocMapped) !=
              cudaSuccess ||
          cudaHostGetDevicePointer(&pd, p, 0) != cudaSuccess) {
        if (p) cudaFreeHost(p);
        destroy_all(c);
        return MOE_ERR_ALLOC;
      }
      c->mbox_host[i] = static_cast<int32_t *>(p);
      c->mbox_dev[i] = static_cast<int32_t *>(pd);
      std::memset(p, 0, sizeof(int32_t) * (size_t)(moe::kMailUni + dims->E));
    }
    if (cudaStreamCreateWithFlags(&c->pred_stream, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&c->x_ready, cudaEventDisableTiming) != cudaSuccess) {
      destroy_all(c);
      return MOE_ERR_CUDA;
    }
  } else {
    c->pool = static_cast<unsigned char *>(std::malloc(pool_bytes));
    if (!c->pool) {
      destroy_all(c);
      return MOE_ERR_ALLOC;
    }
    c->slot_ready.assign(c->n_slots, nullptr);
  }
  c->slot_ready_valid.assign(c->n_slots, 0);
  c->layers.resize(n_layers);
  for (int l = 0; l < n_layers; ++l) {
    Layer &ly = c->layers[l];
    ly.slot_of.assign(c->E1, -1);
    ly.pinned.assign(c->E1, 0);
    ly.prefetched.assign(c->E1, 0);
    ly.where.resize(c->E1);
    for (int s = c->per_layer - 1; s >= 0; --s) ly.free_slots.push_back(l * c->per_layer + s);
    const size_t tb = sizeof(void *) * (size_t)c->E1;
    if (dev(c)) {
      if (cudaMallocHost(reinterpret_cast<void **>(&ly.h_table), tb) != cudaSuccess ||
          cudaMalloc(reinterpret_cast<void **>(&ly.d_table), tb) != cudaSuccess ||
          cudaEventCreateWithFlags(&ly.table_done, cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&ly.released, cudaEventDisableTiming) != cudaSuccess) {
        destroy_all(c);
        return MOE_ERR_ALLOC;
      }
    } else {
      ly.h_table = static_cast<const void **>(std::malloc(tb));
      if (!ly.h_table) {
        destroy_all(c);
        return MOE_ERR_ALLOC;
      }
      ly.d_table = ly.h_table;
    }
  }
  c->st.slots = c->n_slots;
  c->st.slots_per_layer = c->per_layer;
  *out = c;
  return MOE_OK;
}

void expert_cache_destroy(moe_cache *cache) {
  if (cache && dev(cache)) cudaDeviceSynchronize();
  destroy_all(cache);
}

int expert_cache_pin(moe_cache *c, int32_t layer, const int32_t *experts, int32_t n, void *stream) {
  if (!valid_layer(c, layer)) return MOE_ERR_BAD_ARG;
  int rc = check_list(c, experts, n, true);
  if (rc) return rc;
  Layer &ly = c->layers[layer];
  std::vector<char> protect(c->E1, 0);
  for (int i = 0; i < n; ++i) protect[experts[i]] = 1;
  int new_pins = 0;
  for (int i = 0; i < n; ++i) new_pins += ly.pinned[experts[i]] ? 0 : 1;
  // keep room for a full union of the layer's largest decode batch
  if (ly.n_pinned + new_pins > c->per_layer - (c->d.k + 1)) return MOE_ERR_CACHE_FULL;
  for (int i = 0; i < n; ++i) {
    const int e = experts[i];
    rc = make_resident(c, layer, e, static_cast<cudaStream_t>(stream), protect);
    if (rc != MOE_OK) return rc;
    if (!ly.pinned[e]) {
      ly.pinned[e] = 1;
      ly.n_pinned++;
      c->st.pinned++;
    }
  }
  return MOE_OK;
}

int expert_cache_unpin(moe_cache *c, int32_t layer, const int32_t *experts, int32_t n) {
  if (!valid_layer(c, layer)) return MOE_ERR_BAD_ARG;
  int rc = check_list(c, experts, n, true);
  if (rc) return rc;
  Layer &ly = c->layers[layer];
  for (int i = 0; i < n; ++i) {
    const int e = experts[i];
    if (ly.pinned[e]) {
      ly.pinned[e] = 0;
      ly.n_pinned--;
      c->st.pinned--;
    }
  }
  return MOE_OK;
}

int expert_cache_evict(moe_cache *c, int32_t layer, const int32_t *experts, int32_t n) {
  if (!valid_layer(c, layer)) return MOE_ERR_BAD_ARG;
  int rc = check_list(c, experts, n, true);
  if (rc) return rc;
  Layer &ly = c->layers[layer];
  for (int i = 0; i < n; ++i) {
    const int e = experts[i];
    if (ly.slot_of[e] >= 0 && !ly.pinned[e]) drop(c, ly, e);
  }
  return MOE_OK;
}

int expert_cache_prefetch(moe_cache *c, int32_t layer, const int32_t *experts, int32_t n,
                          void *side_stream) {
  if (!valid_layer(c, layer)) return MOE_ERR_BAD_ARG;
  int rc = check_list(c, experts, n, true);
  if (rc) return rc;
  Layer &ly = c->layers[layer];
  std::vector<char> protect(c->E1, 0);
  for (int i = 0; i < n; ++i) protect[experts[i]] = 1;
  protect[c->E1 - 1] = 1;  // never push out the shared expert for a guess
  int started = 0;
  for (int i = 0; i < n; ++i) {
    const int e = experts[i];
    if (ly.slot_of[e] >= 0) continue;
    rc = make_resident(c, layer, e, static_cast<cudaStream_t>(side_stream), protect);
    if (rc == MOE_ERR_CACHE_FULL) break;
    if (rc != MOE_OK) return rc;
    ly.prefetched[e] = 1;
    c->st.prefetches++;
    started++;
  }
  return started;
}

int expert_cache_acquire(moe_cache *c, int32_t layer, const int32_t *experts, int32_t n,
                         void *copy_stream, void *compute_stream, const void **d_table) {
  if (!valid_layer(c, layer) || d_table == nullptr) return MOE_ERR_BAD_ARG;
  int rc = check_list(c, experts, n, true);
  if (rc) return rc;
  Layer &ly = c->layers[layer];
  cudaStream_t cs = static_cast<cudaStream_t>(copy_stream);
  cudaStream_t ks = static_cast<cudaStream_t>(compute_stream);
  std::vector<int> want;
  std::vector<char> protect(c->E1, 0);
  for (int i = 0; i < n; ++i)
    if (!protect[experts[i]]) {
      protect[experts[i]] = 1;
      want.push_back(experts[i]);
    }
  if (!protect[c->E1 - 1]) {
    protect[c->E1 - 1] = 1;
    want.push_back(c->E1 - 1);
  }
  if ((int)want.size() > c->per_layer) return MOE_ERR_CACHE_FULL;
  for (int e : want) {
    if (ly.slot_of[e] >= 0) {
      if (ly.prefetched[e]) {
        ly.prefetched[e] = 0;
        c->st.prefetch_hits++;
      } else {
        c->st.hits++;
      }
      touch(ly, e);
    } else {
      c->st.misses++;
      rc = make_resident(c, layer, e, cs, protect);
      if (rc != MOE_OK) return rc;
    }
  }
  ly.last_slots.clear();
  for (int e : want) ly.last_slots.push_back(ly.slot_of[e]);
  if (dev(c)) {
    // the compute stream waits for the copies these slots still have in
    // flight; a copy found complete is not waited on again
    for (int s : ly.last_slots)
      if (c->slot_ready_valid[s]) {
        const cudaError_t q = cudaEventQuery(c->slot_ready[s]);
        if (q == cudaSuccess) {
          c->slot_ready_valid[s] = 0;
        } else if (q == cudaErrorNotReady) {
          rc = cuda_err(cudaStreamWaitEvent(ks, c->slot_ready[s], 0));
          if (rc) return rc;
        } else {
          return cuda_err(q);
        }
      }
  }
  if (ly.table_dirty || !dev(c)) {
    // the device table of the layer changes only with its residency
    if (dev(c) && ly.table_pending) {
      rc = cuda_err(cudaEventSynchronize(ly.table_done));
      if (rc) return rc;
      ly.table_pending = false;
    }
    for (int e = 0; e < c->E1; ++e)
      ly.h_table[e] = ly.slot_of[e] >= 0 ? c->pool + (size_t)ly.slot_of[e] * c->blob : nullptr;
    if (dev(c)) {
      rc = cuda_err(cudaMemcpyAsync(ly.d_table, ly.h_table, sizeof(void *) * (size_t)c->E1,
                                    cudaMemcpyHostToDevice, ks));
      if (rc) return rc;
      rc = cuda_err(cudaEventRecord(ly.table_done, ks));
      if (rc) return rc;
      ly.table_pending = true;
    }
    ly.table_dirty = false;
  }
  *d_table = ly.d_table;
  return MOE_OK;
}

int expert_cache_release(moe_cache *c, int32_t layer, void *compute_stream) {
  if (!valid_layer(c, layer)) return MOE_ERR_BAD_ARG;
  Layer &ly = c->layers[layer];
  if (dev(c)) {
    const int rc =
        cuda_err(cudaEventRecord(ly.released, static_cast<cudaStream_t>(compute_stream)));
    if (rc) return rc;
    ly.released_valid = true;
  }
  return MOE_OK;
}

int expert_cache_learn_pins(moe_cache *c, int32_t layer, const int32_t *host_counts, int32_t n_pin,
                            void *stream) {
  if (!valid_layer(c, layer) || host_counts == nullptr || n_pin < 0) return MOE_ERR_BAD_ARG;
  Layer &ly = c->layers[layer];
  const int E = c->E1 - 1;
  std::vector<int> order;
  for (int e = 0; e < E; ++e)
    if (host_counts[e] > 0) order.push_back(e);
  std::stable_sort(order.begin(), order.end(),
                   [&](int a, int b) { return host_counts[a] > host_counts[b]; });
  if ((int)order.size() > n_pin) order.resize(n_pin);
  for (int e = 0; e < c->E1; ++e)
    if (ly.pinned[e]) {
      ly.pinned[e] = 0;
      ly.n_pinned--;
      c->st.pinned--;
    }
  return expert_cache_pin(c, layer, order.data(), (int)order.size(), stream);
}

int expert_cache_resident(const moe_cache *c, int32_t layer, int32_t expert) {
  if (!valid_layer(c, layer) || expert < 0 || expert >= c->E1) return MOE_ERR_BAD_ARG;
  return c->layers[layer].slot_of[expert] >= 0 ? 1 : 0;
}

int expert_cache_pinned(const moe_cache *c, int32_t layer, int32_t expert) {
  if (!valid_layer(c, layer) || expert < 0 || expert >= c->E1) return MOE_ERR_BAD_ARG;
  return c->layers[layer].pinned[expert] ? 1 : 0;
}

int expert_cache_stats(const moe_cache *c, moe_cache_stats *stats) {
  if (!c || !stats) return MOE_ERR_BAD_ARG;
  *stats = c->st;
  return MOE_OK;
}

}  // extern "C"

namespace {

// Waits (host, bounded) until the routing kernel has posted sequence `seq` to
// the mailbox, then copies the union out.  If it never comes, the routing
// failed on the device: the stream is synchronised and its status returned.
int wait_mailbox(const int32_t *mb, int32_t seq, int E, int32_t *uni, int32_t *n, cudaStream_t s, void *ws,
                 const moe_dims *dims, int T) {
  const volatile int32_t *vm = mb;
  const auto t0 = std::chrono::steady_clock::now();
  for (long spin = 0; vm[moe::kMailSeq] != seq; ++spin) {
    if ((spin & 1023) == 0 && std::chrono::steady_clock::now() - t0 > std::chrono::seconds(2)) {
      int32_t h[1];
      int32_t hn = 0;
      const int rc = moe_read_union(dims, T, ws, h, &hn, s);  // synchronises; returns the device status
      return rc != MOE_OK ? rc : MOE_ERR_TIMEOUT;
    }
  }
  std::atomic_thread_fence(std::memory_order_acquire);
  const int nu = vm[moe::kMailN];
  if (nu < 0 || nu > E) return MOE_ERR_DEVICE;
  for (int i = 0; i < nu; ++i) uni[i] = vm[moe::kMailUni + i];
  *n = nu;
  return MOE_OK;
}

}  // namespace

extern "C" int moe_tiered_layer_forward(moe_cache *c, int32_t layer, const moe_dims *dims, int32_t T,
                                        const float *x, const float *Wr, const float *Wr_next_opt,
                                        float *out, void *ws, size_t ws_bytes, void *ws_pred,
                                        size_t ws_pred_bytes, int32_t *route_counts_opt,
                                        void *compute_stream, void *side_stream,
                                        int32_t *prefetch_out_opt) {
  if (!valid_layer(c, layer) || c->backend != MOE_CACHE_DEVICE) return MOE_ERR_BAD_ARG;
  if (dims == nullptr || dims->H != c->d.H || dims->I != c->d.I || dims->E != c->d.E ||
      dims->k != c->d.k)
    return MOE_ERR_SHAPE;
  if (prefetch_out_opt) prefetch_out_opt[0] = prefetch_out_opt[1] = 0;
  cudaStream_t cs = static_cast<cudaStream_t>(compute_stream);
  // routing; the kernel posts the union to the mailbox when it is done
  const int32_t seq = ++c->seq;
  int rc = moe::route_to_mailbox(dims, T, x, Wr, ws, ws_bytes, route_counts_opt, c->mbox_dev[0], seq, true, cs);
  if (rc != MOE_OK) return rc;
  const bool predict = Wr_next_opt != nullptr && ws_pred != nullptr && layer + 1 < c->L;
  int32_t seq_pred = 0;
  if (predict) {
    // one-layer-ahead: the next layer's router on this layer's input, on the
    // cache's own stream (off the layer's critical path)
    seq_pred = ++c->seq;
    if (cudaEventRecord(c->x_ready, cs) != cudaSuccess || cudaStreamWaitEvent(c->pred_stream, c->x_ready, 0) != cudaSuccess)
      return MOE_ERR_CUDA;
    rc = moe::route_to_mailbox(dims, T, x, Wr_next_opt, ws_pred, ws_pred_bytes, nullptr, c->mbox_dev[1], seq_pred,
                               false, c->pred_stream);
    if (rc != MOE_OK) return rc;
  }
  std::vector<int32_t> uni(dims->E), pred(dims->E);
  int32_t n = 0, np = 0;
  rc = wait_mailbox(c->mbox_host[0], seq, dims->E, uni.data(), &n, cs, ws, dims, T);
  if (rc != MOE_OK) return rc;
  const void *table = nullptr;
  rc = expert_cache_acquire(c, layer, uni.data(), n, side_stream, compute_stream, &table);
  if (rc != MOE_OK) return rc;
  rc = moe_layer_experts(dims, T, static_cast<const void *const *>(table), out, ws, ws_bytes, compute_stream);
  if (rc != MOE_OK) return rc;
  rc = expert_cache_release(c, layer, compute_stream);
  if (rc != MOE_OK) return rc;
  if (predict) {
    // the prediction has long been posted: prefetch layer + 1's union
    rc = wait_mailbox(c->mbox_host[1], seq_pred, dims->E, pred.data(), &np, c->pred_stream, ws_pred, dims, T);
    if (rc != MOE_OK) return rc;
    const int started = expert_cache_prefetch(c, layer + 1, pred.data(), np, side_stream);
    if (started < 0) return started;
    if (prefetch_out_opt) {
      prefetch_out_opt[0] = started;
      prefetch_out_opt[1] = np;
    }
  }
  return MOE_OK;
}
