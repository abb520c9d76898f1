// usage.cpp -- the route-usage record on disk: per layer and expert, how often
// the router selected it, kept across sessions so that the pins learned from
// it survive a restart.  The engine of "colibrì：把 744B 模型当数据流流到 25GB
// 的笔记本上跑" (tantan.ink) writes the experts each turn routes to into a usage
// file and pins the hottest (section 几个关键工程动作, the learned-cache item);
// "colibri deep review" (ai-tools-nav) describes the same record driving its
// learned cache (technique table, 学习缓存 row).
//
// File layout (little-endian): 8-byte magic "MOEUSAGE", u32 version (1),
// i32 n_layers, i32 E, u32 zero, u64 counts [n_layers][E], u64 FNV-1a 64 hash
// of the counts bytes.  A save writes "<path>.tmp" and renames it over <path>,
// so a reader never sees a partly written record.
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "../../include/moe.h"

namespace {

const char kMagic[8] = {'M', 'O', 'E', 'U', 'S', 'A', 'G', 'E'};
constexpr uint32_t kVersion = 1;

uint64_t fnv1a64(const unsigned char *p, size_t n) {
  uint64_t h = 1469598103934665603ull;
  for (size_t i = 0; i < n; ++i) {
    h ^= p[i];
    h *= 1099511628211ull;
  }
  return h;
}

struct Header {
  char magic[8];
  uint32_t version;
  int32_t n_layers;
  int32_t E;
  uint32_t zero;
};
static_assert(sizeof(Header) == 24, "usage header layout");

bool args_ok(const char *path, int32_t n_layers, int32_t E, const void *counts) {
  return path != nullptr && path[0] != '\0' && n_layers > 0 && E > 0 && E <= MOE_MAX_E &&
         counts != nullptr;
}

}  // namespace

extern "C" int moe_usage_save(const char *path, int32_t n_layers, int32_t E, const uint64_t *counts) {
  if (!args_ok(path, n_layers, E, counts)) return MOE_ERR_BAD_ARG;
  const size_t n = (size_t)n_layers * (size_t)E;
  Header h;
  std::memcpy(h.magic, kMagic, 8);
  h.version = kVersion;
  h.n_layers = n_layers;
  h.E = E;
  h.zero = 0;
  const uint64_t sum = fnv1a64(reinterpret_cast<const unsigned char *>(counts), n * sizeof(uint64_t));
  const std::string tmp = std::string(path) + ".tmp";
  FILE *f = std::fopen(tmp.c_str(), "wb");
  if (f == nullptr) return MOE_ERR_IO;
  bool ok = std::fwrite(&h, sizeof h, 1, f) == 1 && std::fwrite(counts, sizeof(uint64_t), n, f) == n &&
            std::fwrite(&sum, sizeof sum, 1, f) == 1;
  ok = (std::fflush(f) == 0) && ok;
  ok = (std::fclose(f) == 0) && ok;
  if (!ok || std::rename(tmp.c_str(), path) != 0) {
    std::remove(tmp.c_str());
    return MOE_ERR_IO;
  }
  return MOE_OK;
}

extern "C" int moe_usage_load(const char *path, int32_t n_layers, int32_t E, uint64_t *counts,
                              int32_t accumulate) {
  if (!args_ok(path, n_layers, E, counts)) return MOE_ERR_BAD_ARG;
  FILE *f = std::fopen(path, "rb");
  if (f == nullptr) return MOE_ERR_IO;
  Header h;
  const size_t n = (size_t)n_layers * (size_t)E;
  std::vector<uint64_t> buf(n);
  uint64_t sum = 0;
  int rc = MOE_OK;
  if (std::fread(&h, sizeof h, 1, f) != 1 || std::memcmp(h.magic, kMagic, 8) != 0 ||
      h.version != kVersion || h.zero != 0) {
    rc = MOE_ERR_IO;
  } else if (h.n_layers != n_layers || h.E != E) {
    rc = MOE_ERR_SHAPE;
  } else if (std::fread(buf.data(), sizeof(uint64_t), n, f) != n || std::fread(&sum, sizeof sum, 1, f) != 1 ||
             std::fgetc(f) != EOF ||
             fnv1a64(reinterpret_cast<const unsigned char *>(buf.data()), n * sizeof(uint64_t)) != sum) {
    rc = MOE_ERR_IO;
  }
  std::fclose(f);
  if (rc != MOE_OK) return rc;
  for (size_t i = 0; i < n; ++i) counts[i] = accumulate ? counts[i] + buf[i] : buf[i];
  return MOE_OK;
}
