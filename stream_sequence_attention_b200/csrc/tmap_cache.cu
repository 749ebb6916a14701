// Host-side cache of TMA tensor maps keyed by (base pointer, view shape,
// kind): the kernels re-read the same q/k/v/cache buffers call after call,
// so each map is encoded once.  A map depends only on the address and the
// shape it is keyed by, so an entry stays valid even if its buffer is freed
// and another one of the same shape is allocated at the same address.
#include <cstring>
#include <mutex>

#include "hd_launch.h"

namespace hd {

namespace {
constexpr int kSlots = 64;
struct Entry {
  bool used = false;
  TmapKey key;
  CUtensorMap map;
};
Entry g_entries[kSlots];
int g_next = 0;
std::mutex g_mu;

bool same(const TmapKey& a, const TmapKey& b) { return std::memcmp(&a, &b, sizeof(TmapKey)) == 0; }
}  // namespace

bool tmap_cached(const TmapKey& key, CUtensorMap* out, bool (*make)(const TmapKey&, CUtensorMap*)) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    for (int i = 0; i < kSlots; ++i)
      if (g_entries[i].used && same(g_entries[i].key, key)) {
        *out = g_entries[i].map;
        return true;
      }
  }
  if (!make(key, out)) return false;
  std::lock_guard<std::mutex> lk(g_mu);
  Entry& e = g_entries[g_next];
  g_next = (g_next + 1) % kSlots;
  e.used = true;
  e.key = key;
  e.map = *out;
  return true;
}

}  // namespace hd
