// Unified page pools for the cache kinds (P1 §3.1.3, "unifying page sizes").
//
// Every cache kind stores one 256-token logical block per physical page; its
// page holds 256 / ratio entries, so its page size is (256 / ratio) x bytes
// per entry. Rather than one pool per kind, the kinds are grouped into a few
// buckets (three on the page), each a pool of pages of one fixed size: the
// grouping is planned once from the page sizes ("static planning"), and
// requests then take pages from their kind's bucket ("dynamic allocation"),
// with no compaction and no migration between pools.
//
// Host code only: the pools hand out page indices; the caller owns the device
// memory behind them and writes the indices into its block tables.
#include <stdint.h>

#include <algorithm>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/v4kv.h"

struct v4kv_page_pools {
  std::vector<uint64_t> bytes;                 // page bytes per bucket
  std::vector<std::vector<int32_t>> free_list; // free page indices per bucket (LIFO)
  std::vector<std::vector<uint8_t>> in_use;    // 1 per allocated page
  std::mutex mu;
};

extern "C" {

uint64_t v4kv_page_bytes(int32_t ratio, int32_t dim, int32_t elem_bits, int32_t scale_bytes) {
  if (ratio <= 0 || 256 % ratio || dim <= 0 || elem_bits <= 0 || scale_bytes < 0) return 0;
  const uint64_t entry = ((uint64_t)dim * (uint64_t)elem_bits + 7) / 8 + (uint64_t)scale_bytes;
  return (uint64_t)(256 / ratio) * entry;
}

v4kv_status v4kv_plan_buckets(int32_t n_kinds, const uint64_t* page_bytes, int32_t max_buckets,
                              int32_t* bucket_of, uint64_t* bucket_bytes, int32_t* n_buckets) {
  if (n_kinds <= 0 || !page_bytes || max_buckets <= 0 || !bucket_of || !bucket_bytes || !n_buckets)
    return V4KV_ERR_INVALID_ARG;
  for (int i = 0; i < n_kinds; ++i)
    if (page_bytes[i] == 0) return V4KV_ERR_INVALID_ARG;
  // distinct sizes, ascending
  std::vector<uint64_t> sizes(page_bytes, page_bytes + n_kinds);
  std::sort(sizes.begin(), sizes.end());
  sizes.erase(std::unique(sizes.begin(), sizes.end()), sizes.end());
  const int n = (int)sizes.size();
  const int k = std::min(n, (int)max_buckets);
  // Split the ascending sizes into k contiguous groups; a group's page size is
  // its largest member. Minimise the largest waste ratio (group page / kind
  // page) over all kinds, then the sum of those ratios, by dynamic
  // programming over (groups used, sizes covered).
  const double inf = 1e300;
  std::vector<std::vector<double>> worst(k + 1, std::vector<double>(n + 1, inf));
  std::vector<std::vector<double>> total(k + 1, std::vector<double>(n + 1, inf));
  std::vector<std::vector<int>> cut(k + 1, std::vector<int>(n + 1, -1));
  worst[0][0] = 1.0;
  total[0][0] = 0.0;
  for (int g = 1; g <= k; ++g) {
    for (int e = 1; e <= n; ++e) {
      for (int s = g - 1; s < e; ++s) {  // group g covers sizes [s, e)
        if (worst[g - 1][s] >= inf) continue;
        const double top = (double)sizes[e - 1];
        double w = worst[g - 1][s], t = total[g - 1][s];
        for (int i = s; i < e; ++i) {
          w = std::max(w, top / (double)sizes[i]);
          t += top / (double)sizes[i];
        }
        if (w < worst[g][e] || (w == worst[g][e] && t < total[g][e])) {
          worst[g][e] = w;
          total[g][e] = t;
          cut[g][e] = s;
        }
      }
    }
  }
  // group boundaries, then each kind's bucket (bucket 0 = the largest pages)
  std::vector<int> group_of_size(n);
  int e = n;
  for (int g = k; g >= 1; --g) {
    const int s = cut[g][e];
    if (s < 0) return V4KV_ERR_INVALID_ARG;
    for (int i = s; i < e; ++i) group_of_size[i] = g - 1;
    bucket_bytes[k - g] = sizes[e - 1];
    e = s;
  }
  for (int i = 0; i < n_kinds; ++i) {
    const int si = (int)(std::lower_bound(sizes.begin(), sizes.end(), page_bytes[i]) - sizes.begin());
    bucket_of[i] = k - 1 - group_of_size[si];
  }
  *n_buckets = k;
  return V4KV_OK;
}

v4kv_status v4kv_page_pools_create(int32_t n_buckets, const uint64_t* bucket_bytes,
                                   const int32_t* pages_per_bucket, v4kv_page_pools** out) {
  if (n_buckets <= 0 || !bucket_bytes || !pages_per_bucket || !out) return V4KV_ERR_INVALID_ARG;
  for (int b = 0; b < n_buckets; ++b)
    if (bucket_bytes[b] == 0 || pages_per_bucket[b] < 0) return V4KV_ERR_INVALID_ARG;
  v4kv_page_pools* p = new (std::nothrow) v4kv_page_pools;
  if (!p) return V4KV_ERR_INVALID_ARG;
  p->bytes.assign(bucket_bytes, bucket_bytes + n_buckets);
  p->free_list.resize(n_buckets);
  p->in_use.resize(n_buckets);
  for (int b = 0; b < n_buckets; ++b) {
    const int n = pages_per_bucket[b];
    p->free_list[b].reserve(n);
    for (int i = n - 1; i >= 0; --i) p->free_list[b].push_back(i);  // page 0 first out
    p->in_use[b].assign(n, 0);
  }
  *out = p;
  return V4KV_OK;
}

void v4kv_page_pools_destroy(v4kv_page_pools* p) { delete p; }

v4kv_status v4kv_page_alloc(v4kv_page_pools* p, int32_t bucket, int32_t n, int32_t* pages_out) {
  if (!p || n < 0 || (n > 0 && !pages_out)) return V4KV_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(p->mu);
  if (bucket < 0 || bucket >= (int)p->free_list.size()) return V4KV_ERR_INVALID_ARG;
  std::vector<int32_t>& fl = p->free_list[bucket];
  if ((size_t)n > fl.size()) return V4KV_ERR_UNSUPPORTED;  // pool exhausted: nothing taken
  for (int i = 0; i < n; ++i) {
    const int32_t pg = fl.back();
    fl.pop_back();
    p->in_use[bucket][pg] = 1;
    pages_out[i] = pg;
  }
  return V4KV_OK;
}

v4kv_status v4kv_page_free(v4kv_page_pools* p, int32_t bucket, int32_t n, const int32_t* pages) {
  if (!p || n < 0 || (n > 0 && !pages)) return V4KV_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(p->mu);
  if (bucket < 0 || bucket >= (int)p->free_list.size()) return V4KV_ERR_INVALID_ARG;
  std::vector<uint8_t>& used = p->in_use[bucket];
  // all or nothing: every page must be allocated and appear once
  for (int i = 0; i < n; ++i) {
    const int32_t pg = pages[i];
    if (pg < 0 || pg >= (int32_t)used.size() || used[pg] != 1) {
      for (int j = 0; j < i; ++j) used[pages[j]] = 1;  // undo the marks made so far
      return V4KV_ERR_INVALID_ARG;
    }
    used[pg] = 2;  // marked for release
  }
  for (int i = 0; i < n; ++i) {
    used[pages[i]] = 0;
    p->free_list[bucket].push_back(pages[i]);
  }
  return V4KV_OK;
}

int64_t v4kv_pages_free(v4kv_page_pools* p, int32_t bucket) {
  if (!p) return -1;
  std::lock_guard<std::mutex> lock(p->mu);
  if (bucket < 0 || bucket >= (int)p->free_list.size()) return -1;
  return (int64_t)p->free_list[bucket].size();
}

}  // extern "C"
