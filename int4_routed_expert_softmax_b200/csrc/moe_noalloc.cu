// moe_noalloc.cu -- moe_layer_forward_static: the layer with a library-owned,
// statically allocated device workspace, for callers that cannot allocate
// device memory themselves.
//
// The workspace is one file-scope __device__ array of kStaticWsBytes (every
// GPU that loads the library holds it until the process exits).  Host code
// cannot use the array's name as a device address, so the first call on each
// device asks the runtime for the address (cudaGetSymbolAddress) with that
// device current and caches it; later calls reuse it (a reset of the
// device's context between calls would leave the cached address stale, which
// the header tells callers not to do).  The call itself allocates nothing: it
// runs the same launch sequence as moe_layer_forward on that workspace.
#include <cstdio>
#include <mutex>

#include "moe_internal.h"

namespace {

constexpr size_t kStaticWsBytes = (size_t)MOE_STATIC_WS_BYTES;

__device__ __align__(256) unsigned char g_static_ws[kStaticWsBytes];

constexpr int kMaxDev = 64;
void *g_ws_addr[kMaxDev] = {nullptr};
std::mutex g_ws_mu;

}  // namespace

extern "C" int moe_layer_forward_static(const moe_dims *dims, int32_t T, const float *x,
                                        const float *Wr, const void *const *expert_table,
                                        float *out, int32_t *route_counts_opt, int32_t path,
                                        void *stream) {
  const int rc = moe_check_dims(dims);
  if (rc != MOE_OK) return rc;
  if (T < 0 || path < MOE_PATH_AUTO || path > MOE_PATH_PREFILL) return MOE_ERR_BAD_ARG;
  const size_t need = moe_workspace_bytes_path(dims, T, path);
  if (need > kStaticWsBytes) {
    std::fprintf(stderr,
                 "libmoe: moe_layer_forward_static needs %zu workspace bytes for T=%d, more than "
                 "its static %zu; use moe_layer_forward with a caller workspace\n",
                 need, (int)T, kStaticWsBytes);
    return MOE_ERR_WORKSPACE;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return MOE_ERR_CUDA;
  void *ws = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_ws_mu);
    if (g_ws_addr[dev] == nullptr) {
      void *p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_static_ws);
      if (e != cudaSuccess || p == nullptr) {
        std::fprintf(stderr, "libmoe: cudaGetSymbolAddress of the static workspace failed: %s\n",
                     cudaGetErrorString(e));
        return MOE_ERR_CUDA;
      }
      g_ws_addr[dev] = p;
    }
    ws = g_ws_addr[dev];
  }
  return moe_layer_forward(dims, T, x, Wr, expert_table, out, ws, kStaticWsBytes, route_counts_opt,
                           path, stream);
}
