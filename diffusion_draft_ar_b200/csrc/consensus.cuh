// Greedy consensus on sm_100a ("Orthrus: Memory-Efficient Parallel Token
// Generation via Dual-View Diffusion", technical summary §2.3 item 3: accept a
// drafted token iff it equals the frozen AR view's greedy token, checked left to
// right; at the first divergence commit the synchronised prefix and the AR
// correction token).
//
// Pass 1 (HBM-bound): every (row, vocabulary chunk) CTA streams its slice of
// the fp32 logits with 128-bit non-allocating loads and keeps, per thread, the
// first index of the largest value it has seen (strict >, so NaN never wins and
// -0 == +0). The winners are packed into 64-bit keys ordered by value, then by
// lowest index, and max-reduced with warp shuffles into one key per chunk.
// Pass 2 (tiny): one warp per sequence reduces the chunk keys of its rows,
// compares each row's greedy token with its draft, finds the first mismatch
// with a ballot and writes accept length and next token.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace orthrus {

constexpr int kConsThreads = 256;
constexpr int kConsChunk = 16384;  // logits per CTA in pass 1

// Order-preserving 64-bit key: larger value first, then smaller index.
// NaN counts as -inf and -0 as +0, so equal keys mean equal values.
__device__ __forceinline__ unsigned long long consensus_key(float x, uint32_t idx) {
  uint32_t u = __float_as_uint(x);
  if (x != x) u = 0xff800000u;          // NaN -> -inf
  if (u == 0x80000000u) u = 0u;         // -0 -> +0
  const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (static_cast<unsigned long long>(ord) << 32) | (0xffffffffu - idx);
}

__device__ __forceinline__ uint32_t key_index(unsigned long long key) {
  return 0xffffffffu - static_cast<uint32_t>(key & 0xffffffffull);
}

__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long k) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long other = __shfl_xor_sync(0xffffffffu, k, o);
    k = other > k ? other : k;
  }
  return k;
}

__device__ __forceinline__ float4 ld_nc_f4(const float* p) {
  float4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}

// Keep the first index of the largest value; strict > so ties keep the earlier
// index and NaN never replaces anything.
__device__ __forceinline__ void take(float x, int idx, float& best, int& bidx) {
  if (x > best) {
    best = x;
    bidx = idx;
  }
}

__global__ void __launch_bounds__(kConsThreads)
    consensus_argmax_kernel(const float* __restrict__ logits, long long ld, int V,
                            const int* __restrict__ cu_block, int B, int max_block, int n_chunks,
                            unsigned long long* __restrict__ part) {
  pdl_launch_dependents();  // the finalize pass may start its launch now
  const int r = blockIdx.y;
  const int R = cu_block ? cu_block[B] : B * max_block;
  if (r >= R) return;
  const int c = blockIdx.x;
  const int v0 = c * kConsChunk;
  const int v1 = min(V, v0 + kConsChunk);
  const float* row = logits + static_cast<long long>(r) * ld;
  const int tid = threadIdx.x;

  float best = -__int_as_float(0x7f800000);
  int bidx = -1;  // -1: this thread saw no element
  // scalar head up to a 16-byte boundary
  int head = v0;
  const int mis = static_cast<int>((reinterpret_cast<uintptr_t>(row + v0) & 15u) >> 2);
  if (mis) head = min(v1, v0 + (4 - mis));
  // every thread scans increasing indices, so the first element it sees is its
  // lowest index: use it as the tie-default when nothing beats -inf
  if (v0 + tid < head) {
    bidx = v0 + tid;
    take(row[v0 + tid], v0 + tid, best, bidx);
  }
  const int n4 = (v1 - head) >> 2;
  const float* vrow = row + head;
  int i = tid;
  if (bidx < 0 && i < n4) bidx = head + 4 * i;
  for (; i + 3 * kConsThreads < n4; i += 4 * kConsThreads) {
    float4 x[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) x[u] = ld_nc_f4(vrow + 4 * (i + u * kConsThreads));
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int b = head + 4 * (i + u * kConsThreads);
      take(x[u].x, b, best, bidx);
      take(x[u].y, b + 1, best, bidx);
      take(x[u].z, b + 2, best, bidx);
      take(x[u].w, b + 3, best, bidx);
    }
  }
  for (; i < n4; i += kConsThreads) {
    const float4 x = ld_nc_f4(vrow + 4 * i);
    const int b = head + 4 * i;
    take(x.x, b, best, bidx);
    take(x.y, b + 1, best, bidx);
    take(x.z, b + 2, best, bidx);
    take(x.w, b + 3, best, bidx);
  }
  // scalar tail
  const int tail = head + 4 * n4;
  if (tail + tid < v1) {
    if (bidx < 0) bidx = tail + tid;
    take(row[tail + tid], tail + tid, best, bidx);
  }
  unsigned long long key = (bidx >= 0) ? consensus_key(best, static_cast<uint32_t>(bidx)) : 0ull;
  key = warp_max_u64(key);
  __shared__ unsigned long long red[kConsThreads / 32];
  if ((tid & 31) == 0) red[tid >> 5] = key;
  __syncthreads();
  if (tid < 32) {
    key = tid < kConsThreads / 32 ? red[tid] : 0ull;
    key = warp_max_u64(key);
    if (tid == 0) part[static_cast<long long>(r) * n_chunks + c] = key;
  }
}

// ---------------------------------------------------------------------------
// Temperature > 0 (the pages name temperature settings but fix no sampling
// rule; the rule taken): row r's AR token is the Gumbel-max sample
//   t_r = argmax_v  logits[r, v] / T - ln(-ln u_{r,v})
// of softmax(logits[r] / T), and the drafts are accepted left to right iff
// they equal it, as in the greedy rule (the finalize kernel below). u comes
// from the counter-based generator Philox4x32-10 (Salmon, Moraes, Dror, Shaw,
// "Parallel random numbers: as easy as 1, 2, 3", SC 2011): counter
// (v / 4, r, offset lo, offset hi), key (seed lo, seed hi), word v % 4, and
// u = (top 24 bits + 1/2) / 2^24, in (0, 1).

struct Philox4 {
  uint32_t x, y, z, w;
};

// Philox4x32-10: ten rounds, the key bumped by the Weyl constants between
// rounds (the published definition).
__device__ __forceinline__ Philox4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2,
                                                 uint32_t c3, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int i = 0; i < 10; ++i) {
    if (i > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * c0;  // one wide multiply each
    const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * c2;
    const uint32_t hi0 = static_cast<uint32_t>(p0 >> 32), lo0 = static_cast<uint32_t>(p0);
    const uint32_t hi1 = static_cast<uint32_t>(p1 >> 32), lo1 = static_cast<uint32_t>(p1);
    const uint32_t n0 = hi1 ^ c1 ^ k0;
    const uint32_t n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  return Philox4{c0, c1, c2, c3};
}

// The kernel ranks base-2 scores. With e = -ln u, the Gumbel-max score
// s = x / T - ln e divided by ln 2 is x log2(e) / T - log2(ln 2) - log2(a)
// with a = e / ln 2 = -log2 u; the constant is the same for every entry, so
// r = x * x_scale - log2(a), x_scale = log2(e) / T, has the same argmax.
// noise_log2 returns -log2(a) for u = (k + 1/2) / 2^24, k = word >> 8. a must
// be accurate in relative terms. For u < 15/16, |log2 u| >= 0.09 and the
// hardware base-2 logarithm (absolute error ~2^-22) gives a to ~3e-6. For
// u >= 15/16 (where the largest noise values, the likely winners, come from)
// a is the series of -log2(1 - v) = (v + v^2/2 + v^3/3 + ...) / ln 2 in
// v = 1 - u, which is exact in fp32; seven terms leave a relative error below
// v^7/8 <= 2^-31. The outer logarithm needs only absolute accuracy. Both
// forms are evaluated and one is selected: in nearly every warp some lane
// needs the series, so a branch would run both anyway. Emulated in fp32
// against fp64 over every series k and a million sampled log-branch k, the
// result is within 2e-7 and 8e-7 (base-2 units) of -log2(-log2 u).
__device__ __forceinline__ float noise_log2(uint32_t word) {
  const uint32_t k = word >> 8;
  const float kf = static_cast<float>(k);
  const float v = ((16777216.f - kf) - 0.5f) * 5.9604644775390625e-8f;  // exact: v = m / 2^25
  float q = fmaf(v, 2.060992867e-01f, 2.404491752e-01f);  // 1 / (j ln 2), j = 7, 6
  q = fmaf(v, q, 2.885390222e-01f);                       // j = 5
  q = fmaf(v, q, 3.606737554e-01f);                       // j = 4
  q = fmaf(v, q, 4.808983505e-01f);                       // j = 3
  q = fmaf(v, q, 7.213475108e-01f);                       // j = 2
  q = fmaf(v, q, 1.442695022e+00f);                       // j = 1
  const float a_series = v * q;
  const float u = fmaf(kf, 5.9604644775390625e-8f, 2.98023223876953125e-8f);  // (k + 1/2) 2^-24
  const float a_log = -__log2f(u);
  const float a = (k >= (15u << 20)) ? a_series : a_log;
  return -__log2f(a);
}

// One CTA per (row, 16,384-entry chunk): every thread takes groups of four
// consecutive entries (one Philox call each), keeps the first index of its
// largest score, and the CTA reduces the order-preserving keys as the greedy
// pass does. The chunk start is a multiple of 4, so a group never straddles
// two counters; its logits are one 16-byte load when the row allows. Entries
// past the row end score -inf. A group is compared once, by its largest
// score m (fmaxf drops NaN, so a NaN logit never wins): only when m beats the
// thread's best is the first entry equal to m looked up, which keeps the
// first index of the largest score as a comparison per entry would.
__global__ void __launch_bounds__(kConsThreads)
    consensus_sample_kernel(const float* __restrict__ logits, long long ld, int V,
                            const int* __restrict__ cu_block, int B, int max_block, int n_chunks,
                            unsigned long long* __restrict__ part, float x_scale, uint32_t seed_lo,
                            uint32_t seed_hi, uint32_t off_lo, uint32_t off_hi) {
  pdl_launch_dependents();  // the finalize pass may start its launch now
  const int r = blockIdx.y;
  const int R = cu_block ? cu_block[B] : B * max_block;
  if (r >= R) return;
  const int c = blockIdx.x;
  const int v0 = c * kConsChunk;
  const int v1 = min(V, v0 + kConsChunk);
  const float* row = logits + static_cast<long long>(r) * ld;
  const bool vec = ((reinterpret_cast<uintptr_t>(row) & 15u) == 0);
  const float NEG_INF = -__int_as_float(0x7f800000);
  float best = NEG_INF;
  int bidx = -1;
  const int g0 = v0 >> 2, g1 = (v1 + 3) >> 2;
  for (int g = g0 + static_cast<int>(threadIdx.x); g < g1; g += kConsThreads) {
    const int v = g << 2;
    float x[4];
    if (vec && v + 3 < v1) {
      const float4 q = ld_nc_f4(row + v);
      x[0] = q.x, x[1] = q.y, x[2] = q.z, x[3] = q.w;
    } else {
#pragma unroll
      for (int k = 0; k < 4; ++k) x[k] = (v + k < v1) ? row[v + k] : NEG_INF;
    }
    const Philox4 w = philox4x32_10(static_cast<uint32_t>(g), static_cast<uint32_t>(r), off_lo,
                                    off_hi, seed_lo, seed_hi);
    if (bidx < 0) bidx = v;  // lowest index this thread sees: the tie default
    float sc[4];
    sc[0] = fmaf(x[0], x_scale, noise_log2(w.x));
    sc[1] = fmaf(x[1], x_scale, noise_log2(w.y));
    sc[2] = fmaf(x[2], x_scale, noise_log2(w.z));
    sc[3] = fmaf(x[3], x_scale, noise_log2(w.w));
    const float m = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
    if (m > best) {
      best = m;
      bidx = sc[0] == m ? v : (sc[1] == m ? v + 1 : (sc[2] == m ? v + 2 : v + 3));
    }
  }
  const int tid = threadIdx.x;
  unsigned long long key = (bidx >= 0) ? consensus_key(best, static_cast<uint32_t>(bidx)) : 0ull;
  key = warp_max_u64(key);
  __shared__ unsigned long long red[kConsThreads / 32];
  if ((tid & 31) == 0) red[tid >> 5] = key;
  __syncthreads();
  if (tid < 32) {
    key = tid < kConsThreads / 32 ? red[tid] : 0ull;
    key = warp_max_u64(key);
    if (tid == 0) part[static_cast<long long>(r) * n_chunks + c] = key;
  }
}

__global__ void consensus_finalize_kernel(const unsigned long long* __restrict__ part,
                                          int n_chunks, const int* __restrict__ draft,
                                          const int* __restrict__ cu_block, int B, int max_block,
                                          int* __restrict__ accept_len,
                                          int* __restrict__ next_token,
                                          int* __restrict__ row_argmax,
                                          int* __restrict__ prefix_lens, int row_limit) {
  const int warps = blockDim.x >> 5;
  const int b = blockIdx.x * warps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (b >= B) return;
  const int row0 = cu_block ? cu_block[b] : b * max_block;
  const int Kb = cu_block ? cu_block[b + 1] - row0 : max_block;
  // rows outside the keys the caller's workspace holds: treated as an empty block
  if (Kb <= 0 || row0 < 0 || row0 + Kb > row_limit) {
    if (lane == 0) {
      accept_len[b] = 0;
      next_token[b] = -1;
    }
    return;
  }
  pdl_wait();  // the argmax pass's keys are visible from here on
  int m = Kb;  // leading matches
  int next = -1;
  for (int base = 0; base < Kb; base += 32) {
    const int i = base + lane;
    int t = -1;
    bool miss = false;
    if (i < Kb) {
      unsigned long long k = 0ull;
      const unsigned long long* p = part + static_cast<long long>(row0 + i) * n_chunks;
      for (int c = 0; c < n_chunks; ++c) k = p[c] > k ? p[c] : k;
      t = static_cast<int>(key_index(k));
      if (row_argmax) row_argmax[row0 + i] = t;
      miss = draft[row0 + i] != t;
    }
    const unsigned ballot = __ballot_sync(0xffffffffu, miss);
    if (m == Kb && ballot) m = base + __ffs(ballot) - 1;
    // the committed count is min(m + 1, Kb); its last token lives in this chunk
    const int n = (m + 1 < Kb) ? (m + 1) : Kb;
    const int last = n - 1;
    if (last >= base && last < base + 32 && next < 0) next = __shfl_sync(0xffffffffu, t, last - base);
    if (m < Kb && !row_argmax) break;
  }
  if (lane == 0) {
    const int n = (m + 1 < Kb) ? (m + 1) : Kb;
    accept_len[b] = n;
    next_token[b] = next;
    // Commit of write-then-truncate VERIFY: the cache already holds all K_b
    // rows past L_b, so accepting n of them is advancing the length.
    if (prefix_lens) prefix_lens[b] += n;
  }
}

}  // namespace orthrus
