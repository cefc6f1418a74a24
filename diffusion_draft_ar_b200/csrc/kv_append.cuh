// Commit step on sm_100a ("Orthrus: Memory-Efficient Parallel Token Generation
// via Dual-View Diffusion", technical summary §2.3 item 3, commit and truncate
// the cache; agents-report.net commentary, "core design": the accepted tokens'
// KV is appended to the shared cache).
//
// One CTA per sequence copies its accepted rows' K and V (VERIFY view) into the
// slots L_b .. L_b + n_b - 1 of its pages with 16-byte loads and stores, then
// (optionally) advances prefix_lens[b] once every row found its page. The ids of
// the first kMaxAppendPages pages the rows land in are read once into shared
// memory (rows rarely span more than two pages), so the copies carry no
// dependent loads. A row whose page is out of range is skipped and flagged.
#pragma once

#include <cstdint>

#include "orthrus.h"

namespace orthrus {

constexpr int kAppendThreads = 512;
constexpr int kMaxAppendPages = 8;

__global__ void __launch_bounds__(kAppendThreads)
    kv_append_kernel(const uint4* __restrict__ k_block, const uint4* __restrict__ v_block,
                     const int* __restrict__ cu_block, int max_block,
                     const int* __restrict__ accept_len, int* prefix_lens, int update_lens,
                     const int* __restrict__ page_table, int max_pages, int num_pages,
                     uint4* k_cache, uint4* v_cache, int Hkv, int D, int page_size,
                     int* error_flag) {
  __shared__ int sh_page[kMaxAppendPages];
  __shared__ int sh_flags;
  const int b = blockIdx.x;
  const int row0 = cu_block ? cu_block[b] : b * max_block;
  const int Kb = cu_block ? cu_block[b + 1] - row0 : max_block;
  const int L = prefix_lens[b];
  const int n = accept_len[b];
  const int cpr = D / 8;  // 16-byte chunks per head row
  const bool seq_bad = n < 0 || n > Kb || L < 0;
  const long long p_first = seq_bad ? 0 : L / page_size;

  // page id of page index pidx, or -1 (and a flag) when it is out of range
  auto page_of = [&](long long pidx) -> int {
    if (pidx >= max_pages) {
      atomicOr(&sh_flags, ORTHRUS_FLAG_BAD_LENGTH);
      return -1;
    }
    const int page = page_table[static_cast<long long>(b) * max_pages + pidx];
    if (page < 0 || page >= num_pages) {
      atomicOr(&sh_flags, ORTHRUS_FLAG_BAD_PAGE);
      return -1;
    }
    return page;
  };

  if (threadIdx.x == 0) sh_flags = 0;
  __syncthreads();
  if (!seq_bad && n > 0) {
    const long long n_pages = (static_cast<long long>(L) + n - 1) / page_size - p_first + 1;
    if (threadIdx.x < kMaxAppendPages && threadIdx.x < n_pages)
      sh_page[threadIdx.x] = page_of(p_first + threadIdx.x);
  }
  // every thread has read L (and the page ids are in place) from here on
  __syncthreads();
  if (!seq_bad) {
    const int items = n * Hkv * cpr;
    constexpr int U = 4;
    for (int base = threadIdx.x; base < items; base += U * kAppendThreads) {
      uint4 kv[U], vv[U];
      long long dst[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int it = base + u * kAppendThreads;
        dst[u] = -1;
        if (it < items) {
          const int c = it % cpr;
          const int rest = it / cpr;
          const int h = rest % Hkv;
          const int i = rest / Hkv;
          const long long pos = static_cast<long long>(L) + i;
          const long long k = pos / page_size - p_first;
          const int page = k < kMaxAppendPages ? sh_page[k] : page_of(pos / page_size);
          if (page >= 0) {
            const long long slot = pos % page_size;
            dst[u] = ((static_cast<long long>(page) * Hkv + h) * page_size + slot) * cpr + c;
            const long long src = (static_cast<long long>(row0 + i) * Hkv + h) * cpr + c;
            kv[u] = k_block[src];
            vv[u] = v_block[src];
          }
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (dst[u] >= 0) {
          k_cache[dst[u]] = kv[u];
          v_cache[dst[u]] = vv[u];
        }
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const int flags = seq_bad ? ORTHRUS_FLAG_BAD_LENGTH : sh_flags;
    if (flags) {
      if (error_flag) atomicOr(error_flag, flags);
    } else if (update_lens) {
      prefix_lens[b] = L + n;
    }
  }
}

}  // namespace orthrus
