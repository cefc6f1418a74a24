// Commit step on sm_100a ("Orthrus: Memory-Efficient Parallel Token Generation
// via Dual-View Diffusion", technical summary §2.3 item 3, commit and truncate
// the cache; agents-report.net commentary, "core design": the accepted tokens'
// KV is appended to the shared cache).
//
// One CTA per sequence copies its accepted rows' K and V (VERIFY view) into the
// slots L_b .. L_b + n_b - 1 of its pages with 16-byte loads and stores, then
// (optionally) advances prefix_lens[b] once every row found its page.
#pragma once

#include <cstdint>

#include "orthrus.h"

namespace orthrus {

constexpr int kAppendThreads = 256;

__global__ void __launch_bounds__(kAppendThreads)
    kv_append_kernel(const uint4* __restrict__ k_block, const uint4* __restrict__ v_block,
                     const int* __restrict__ cu_block, int max_block,
                     const int* __restrict__ accept_len, int* prefix_lens, int update_lens,
                     const int* __restrict__ page_table, int max_pages, int num_pages,
                     uint4* k_cache, uint4* v_cache, int Hkv, int D, int page_size,
                     int* error_flag) {
  const int b = blockIdx.x;
  const int row0 = cu_block ? cu_block[b] : b * max_block;
  const int Kb = cu_block ? cu_block[b + 1] - row0 : max_block;
  const int L = prefix_lens[b];
  const int n = accept_len[b];
  const int cpr = D / 8;  // 16-byte chunks per head row
  int flags = 0;
  if (n < 0 || n > Kb || L < 0) flags |= ORTHRUS_FLAG_BAD_LENGTH;
  if (!flags) {
    const int items = n * Hkv * cpr;
    for (int it = threadIdx.x; it < items; it += blockDim.x) {
      const int c = it % cpr;
      const int rest = it / cpr;
      const int h = rest % Hkv;
      const int i = rest / Hkv;
      const long long pos = static_cast<long long>(L) + i;
      const long long pidx = pos / page_size;
      if (pidx >= max_pages) {
        flags |= ORTHRUS_FLAG_BAD_LENGTH;
        continue;
      }
      const int page = page_table[static_cast<long long>(b) * max_pages + pidx];
      if (page < 0 || page >= num_pages) {
        flags |= ORTHRUS_FLAG_BAD_PAGE;
        continue;
      }
      const long long slot = pos % page_size;
      const long long dst = ((static_cast<long long>(page) * Hkv + h) * page_size + slot) * cpr + c;
      const long long src = (static_cast<long long>(row0 + i) * Hkv + h) * cpr + c;
      k_cache[dst] = k_block[src];
      v_cache[dst] = v_block[src];
    }
  }
  // every thread has read L before anyone may change it
  const int any = __syncthreads_or(flags);
  if (any) {
    // collect the flag bits of the whole block
    __shared__ int bits;
    if (threadIdx.x == 0) bits = 0;
    __syncthreads();
    if (flags) atomicOr(&bits, flags);
    __syncthreads();
    if (threadIdx.x == 0 && error_flag) atomicOr(error_flag, bits);
  } else if (update_lens && threadIdx.x == 0) {
    prefix_lens[b] = L + n;
  }
}

}  // namespace orthrus
