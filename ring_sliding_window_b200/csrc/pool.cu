// Token pool for continuous batching: a host-side allocator of contiguous
// cache-slot ranges in one shared K/V pool per layer.
//
// Method ("开源5天Star破万之后：百度Unlimited-OCR的爆火路径复盘", §三, serving
// with a page size of one token): every request owns prefill_len + W slots,
// constant for its whole life, so a request's cache is one range allocated
// when it joins and freed when it leaves.  With a page size of one token the
// allocation unit is a single slot.
//
// Free space is kept as a map base -> length of maximal free ranges (adjacent
// free ranges are always merged), allocated ranges as a map base -> length.
// Allocation is first fit (lowest base whose free range is long enough), so
// the placement is deterministic.  Every entry point takes the pool's mutex.
#include <map>
#include <mutex>
#include <new>

#include "internal.h"

struct rswa_pool {
  int64_t capacity = 0;
  std::map<int64_t, int64_t> free_ranges;  // base -> length, disjoint, non-adjacent
  std::map<int64_t, int64_t> used;         // base -> length
  int64_t free_slots = 0;
  mutable std::mutex mu;
};

extern "C" {

rswa_status rswa_pool_create(int64_t capacity, rswa_pool **out) {
  if (!out) return RSWA_EINVAL;
  *out = nullptr;
  if (capacity < 1 || capacity >= (int64_t(1) << 40)) return RSWA_EINVAL;
  rswa_pool *p = new (std::nothrow) rswa_pool();
  if (!p) return RSWA_ENOMEM;
  p->capacity = capacity;
  p->free_ranges[0] = capacity;
  p->free_slots = capacity;
  *out = p;
  return RSWA_OK;
}

rswa_status rswa_pool_destroy(rswa_pool *p) {
  if (!p) return RSWA_EINVAL;
  delete p;
  return RSWA_OK;
}

rswa_status rswa_pool_alloc(rswa_pool *p, int64_t slots, int64_t *base) {
  if (!p || !base || slots < 1) return RSWA_EINVAL;
  std::lock_guard<std::mutex> lock(p->mu);
  for (auto it = p->free_ranges.begin(); it != p->free_ranges.end(); ++it) {
    if (it->second < slots) continue;
    const int64_t b = it->first, len = it->second;
    p->free_ranges.erase(it);
    if (len > slots) p->free_ranges[b + slots] = len - slots;
    p->used[b] = slots;
    p->free_slots -= slots;
    *base = b;
    return RSWA_OK;
  }
  return RSWA_ENOMEM;
}

rswa_status rswa_pool_free(rswa_pool *p, int64_t base) {
  if (!p) return RSWA_EINVAL;
  std::lock_guard<std::mutex> lock(p->mu);
  auto u = p->used.find(base);
  if (u == p->used.end()) return RSWA_EINVAL;  // not the base of an allocated range
  int64_t b = base, len = u->second;
  p->used.erase(u);
  p->free_slots += len;
  // merge with the free range ending at `base` and the one starting right after
  auto next = p->free_ranges.lower_bound(base);
  if (next != p->free_ranges.end() && next->first == base + len) {
    len += next->second;
    next = p->free_ranges.erase(next);
  }
  if (next != p->free_ranges.begin()) {
    auto prev = std::prev(next);
    if (prev->first + prev->second == base) {
      b = prev->first;
      len += prev->second;
      p->free_ranges.erase(prev);
    }
  }
  p->free_ranges[b] = len;
  return RSWA_OK;
}

rswa_status rswa_pool_stats(const rswa_pool *p, int64_t *free_slots, int64_t *largest_free,
                            int32_t *n_free_ranges, int32_t *n_allocated) {
  if (!p) return RSWA_EINVAL;
  std::lock_guard<std::mutex> lock(p->mu);
  int64_t largest = 0;
  for (const auto &r : p->free_ranges) largest = r.second > largest ? r.second : largest;
  if (free_slots) *free_slots = p->free_slots;
  if (largest_free) *largest_free = largest;
  if (n_free_ranges) *n_free_ranges = (int32_t)p->free_ranges.size();
  if (n_allocated) *n_allocated = (int32_t)p->used.size();
  return RSWA_OK;
}

int64_t rswa_pool_capacity(const rswa_pool *p) { return p ? p->capacity : -1; }

}  // extern "C"
