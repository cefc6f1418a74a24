// Fused LM head + greedy token on sm_100a: tcgen05 GEMM with TMEM
// accumulators, TMA-fed shared-memory ring, and the row argmax in the
// epilogue, so the fp32 logits never reach HBM.
//
// What it computes ("Orthrus: Memory-Efficient Parallel Token Generation via
// Dual-View Diffusion", technical summary §2.3 items 2-3 with §2.1: the frozen
// AR model scores every block row over the vocabulary and its greedy token
// decides acceptance): for every block row r,
//   t_r = argmax_v <hidden[r, :], w_head[v, :]>
// with ties going to the lowest v (the consensus rule's order). The per-row
// winners are packed as order-preserving 64-bit keys (value, then lowest
// index; the same keys as the consensus argmax pass) and max-combined across
// vocabulary tiles with 64-bit atomicMax, which is order independent, so the
// result does not depend on the tile schedule. The consensus finalize kernel
// then turns the keys into accept lengths and next tokens.
//
// Tiling: a tile is mt x 128 rows (mt = 1 or 2 M=128 MMAs sharing one B tile)
// by N vocabulary columns (N <= 256, a multiple of 16), over K = d_model in
// 64-element steps (one 128-byte swizzle atom of bf16). Both operands are
// K-major: hidden [R, d] row-major and w_head [V, d] row-major (the output
// projection's [out, in] layout). A persistent CTA per SM walks tiles
// c, c + grid, ...; consecutive tile ids share their vocabulary tile across
// the row tiles, so the CTAs that read a w_head tile run at about the same
// time and the second read hits L2.
//
// Roles (320 threads, one CTA per SM):
//   warp 0      TMA producer, two lanes: per K step lane 0 arms the stage's
//               barrier and issues the A box (mt*128 rows x 64), lane 1 the B
//               box (N rows x 64). A box issue holds its thread for a few
//               hundred cycles whatever the box size, so one issuing thread
//               capped the ring at about one stage per microsecond; two lanes
//               issue side by side.
//   warp 1      MMA issuer: mt x 4 tcgen05.mma (M=128, N, K=16) per stage into
//               TMEM; commits release the stage and, after a tile's last step,
//               publish the accumulator. Owns the TMEM allocation.
//   warps 2-9   epilogue, two groups of four warps (each group covers the four
//               TMEM lane quarters): with mt = 2 group g reduces accumulator g
//               (rows g*128 + lane); with mt = 1 the two groups split the
//               columns of the one accumulator (at a multiple of 32). Each thread scans its row's
//               columns in increasing order (strict >, so ties keep the lower
//               index and NaN never wins) and atomically maxes its key.
// With mt = 1 the accumulator is double buffered (two 256-column slots), so
// the epilogue of one tile overlaps the MMAs of the next; with mt = 2 the two
// accumulators fill TMEM and the epilogue runs between tiles.
#pragma once

#include <cstdint>
#include <cuda.h>

#include "consensus.cuh"
#include "orthrus.h"
#include "ptx.cuh"

namespace orthrus {

constexpr int kLmThreads = 320;
constexpr int kLmProducerWarp = 0;
constexpr int kLmMmaWarp = 1;
constexpr int kLmEpiWarp0 = 2;
constexpr int kLmKStep = 64;          // bf16 elements per 128-byte swizzle atom
constexpr int kLmABlock = 128 * 128;  // bytes of one 128-row x 64 A block
constexpr int kLmMaxStages = 8;
constexpr uint32_t kLmTmemCols = 512;

struct LmArgs {
  int R, V, d;        // rows of hidden, vocabulary, model dim
  int N;              // vocabulary columns per tile
  int mt;             // 128-row MMA blocks per tile (1 or 2)
  int n_m, n_tiles;   // row tiles, total tiles (n_m * vocabulary tiles)
  int k_steps;        // d / 64
  int stages;
  uint32_t stage_bytes;  // mt * 16 KiB (A) + N * 128 (B)
  uint32_t a_bytes;      // mt * 16 KiB
  uint32_t tx_bytes;     // bytes one stage's two boxes deliver
  uint32_t idesc;        // tcgen05 instruction descriptor, M = 128, N
  unsigned long long* keys;  // [R] packed (value, index) keys, zeroed before the launch
  int* error_flag;
  unsigned long long timeout_ns;
  int fault_inject;   // test hook: 1 drops each CTA's first w_head copy (a wait must time out)
};

struct LmLayout {
  // offsets from the 1024-byte aligned base; barriers after the stages
  __device__ __forceinline__ static uint32_t bar_off(const LmArgs& a) {
    return a.stages * a.stage_bytes;
  }
  // barrier indices
  __device__ __forceinline__ static int full(int s) { return s; }
  __device__ __forceinline__ static int empty(int s) { return kLmMaxStages + s; }
  __device__ __forceinline__ static int acc_full(int j) { return 2 * kLmMaxStages + j; }
  __device__ __forceinline__ static int acc_empty(int j) { return 2 * kLmMaxStages + 2 + j; }
  static constexpr int kDrain = 2 * kLmMaxStages + 4;
  static constexpr int kNumBars = kDrain + 1;
  static constexpr int kMiscBytes = kNumBars * 8 + 16;  // barriers, abort flag, TMEM base
};

__host__ __device__ constexpr size_t lm_smem_bytes(int stages, uint32_t stage_bytes) {
  return 1024 + static_cast<size_t>(stages) * stage_bytes + LmLayout::kMiscBytes;
}

__global__ void __launch_bounds__(kLmThreads, 1)
    lm_head_argmax_kernel(const __grid_constant__ CUtensorMap tm_a,
                          const __grid_constant__ CUtensorMap tm_b, const LmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t base = smem_u32(smem);
  const uint32_t bars = base + LmLayout::bar_off(a);
  volatile int* abort_flag =
      reinterpret_cast<volatile int*>(smem + LmLayout::bar_off(a) + LmLayout::kNumBars * 8);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + LmLayout::bar_off(a) +
                                                    LmLayout::kNumBars * 8 + 4);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  auto bar = [&](int i) { return bars + 8u * static_cast<uint32_t>(i); };
  auto wait = [&](uint32_t b, uint32_t parity) {
    return mbar_wait(b, parity, abort_flag, a.timeout_ns);
  };

  // the finalize pass (a programmatic dependent) may be scheduled now; it
  // reads the keys only after this grid has completed
  pdl_launch_dependents();

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(bar(LmLayout::full(s)), 1);
      mbar_init(bar(LmLayout::empty(s)), 1);
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(bar(LmLayout::acc_full(j)), 1);
      mbar_init(bar(LmLayout::acc_empty(j)), 256);  // every epilogue thread
    }
    mbar_init(bar(LmLayout::kDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kLmProducerWarp && lane == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
  }
  if (warp == kLmMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kLmTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_slots = a.mt == 1 ? 2 : 1;

  if (warp == kLmProducerWarp) {
    if (lane < 2) {
      // Both lanes walk every stage in order (each waits on every phase of
      // every empty barrier, so a parity wait is never two phases ahead).
      // Lane 1's bytes may land before lane 0 arms the barrier: the
      // transaction count goes negative for a moment, and the phase cannot
      // complete before lane 0's arrival.
      int s = 0;
      uint32_t ph = 0;
      long long issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < a.n_tiles; tile += gridDim.x) {
        const int n = tile / a.n_m, m = tile % a.n_m;
        for (int ks = 0; ks < a.k_steps; ++ks) {
          if (!wait(bar(LmLayout::empty(s)), ph ^ 1u)) { ok = false; break; }
          const uint32_t st = base + s * a.stage_bytes;
          if (lane == 0) {
            mbar_arrive_expect_tx(bar(LmLayout::full(s)), a.tx_bytes);
            tma_load_2d(st, &tm_a, bar(LmLayout::full(s)), ks * kLmKStep, m * 128 * a.mt);
          } else if (!(a.fault_inject == 1 && issued == 0)) {
            tma_load_2d(st + a.a_bytes, &tm_b, bar(LmLayout::full(s)), ks * kLmKStep, n * a.N);
          }
          ++issued;
          if (++s == a.stages) { s = 0; ph ^= 1u; }
        }
      }
      if (!ok) {
        // wind down: every copy issued must land before the CTA may exit
        const long long first = issued > a.stages ? issued - a.stages : 0;
        for (long long i = first; i < issued; ++i) {
          const int si = static_cast<int>(i % a.stages);
          const uint32_t pi = static_cast<uint32_t>((i / a.stages) & 1);
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(bar(LmLayout::full(si)), pi) &&
                 global_timer_ns() - t0 < a.timeout_ns) {
          }
        }
      }
    }
  } else if (warp == kLmMmaWarp) {
    int s = 0;
    uint32_t ph = 0;
    int local = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < a.n_tiles; tile += gridDim.x, ++local) {
      const int slot = n_slots == 2 ? (local & 1) : 0;
      const int use = n_slots == 2 ? (local >> 1) : local;
      if (!wait(bar(LmLayout::acc_empty(slot)), static_cast<uint32_t>(use & 1) ^ 1u)) {
        ok = false;
        break;
      }
      tc_fence_after();
      for (int ks = 0; ks < a.k_steps; ++ks) {
        if (!wait(bar(LmLayout::full(s)), ph)) { ok = false; break; }
        tc_fence_after();
        const uint32_t st = base + s * a.stage_bytes;
        // Both loops have compile-time bounds: with a run-time bound around
        // elect.sync + tcgen05.mma each issue cost ~200 cycles (the tensor core
        // starved at ~1600 cycles per K step whatever N); unrolled, the issue
        // runs ahead of the tensor core.
        if (a.mt == 2) {
#pragma unroll
          for (int kk = 0; kk < kLmKStep / 16; ++kk) {
            const uint64_t bd = smem_desc_sw128(st + a.a_bytes + kk * 32, 16, 1024);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const uint64_t ad = smem_desc_sw128(st + j * kLmABlock + kk * 32, 16, 1024);
              if (elect_one())
                mma_bf16_ss(tmem + 256u * j, ad, bd, a.idesc, (ks | kk) ? 1u : 0u);
            }
          }
        } else {
          const uint32_t acc = tmem + 256u * static_cast<uint32_t>(slot);
#pragma unroll
          for (int kk = 0; kk < kLmKStep / 16; ++kk) {
            const uint64_t bd = smem_desc_sw128(st + a.a_bytes + kk * 32, 16, 1024);
            const uint64_t ad = smem_desc_sw128(st + kk * 32, 16, 1024);
            if (elect_one()) mma_bf16_ss(acc, ad, bd, a.idesc, (ks | kk) ? 1u : 0u);
          }
        }
        if (elect_one()) mma_commit(bar(LmLayout::empty(s)));
        __syncwarp();
        if (++s == a.stages) { s = 0; ph ^= 1u; }
      }
      if (!ok) break;
      if (elect_one()) mma_commit(bar(LmLayout::acc_full(slot)));
      __syncwarp();
    }
    if (!ok) {
      // wind down: every MMA issued must finish before TMEM is released
      if (elect_one()) mma_commit(bar(LmLayout::kDrain));
      __syncwarp();
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(bar(LmLayout::kDrain), 0) && global_timer_ns() - t0 < a.timeout_ns) {
      }
    }
  } else {
    const int q = warp & 3;                     // TMEM lane quarter of this warp
    const int g = (warp - kLmEpiWarp0) >> 2;    // epilogue group 0 or 1
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    int local = 0;
    for (int tile = blockIdx.x; tile < a.n_tiles; tile += gridDim.x, ++local) {
      const int slot = n_slots == 2 ? (local & 1) : 0;
      const int use = n_slots == 2 ? (local >> 1) : local;
      if (!wait(bar(LmLayout::acc_full(slot)), static_cast<uint32_t>(use & 1))) break;
      tc_fence_after();
      const int n = tile / a.n_m, m = tile % a.n_m;
      int c0, c1, row;
      uint32_t col;
      if (a.mt == 2) {
        c0 = 0;
        c1 = a.N;
        row = m * 256 + g * 128 + q * 32 + lane;
        col = 256u * static_cast<uint32_t>(g);
      } else {
        // the two groups split the columns at a multiple of 32 (TMEM loads
        // start on 32-column boundaries)
        const int split = ((a.N >> 1) + 31) & ~31;
        c0 = g == 0 ? 0 : split;
        c1 = g == 0 ? split : a.N;
        row = m * 128 + q * 32 + lane;
        col = 256u * static_cast<uint32_t>(slot);
      }
      const int v0 = n * a.N;
      // columns past the vocabulary (zero-filled B rows) never compete
      const int c_end = min(c1, a.V - v0);
      float best = -__int_as_float(0x7f800000);
      int bidx = -1;
      int c = c0;
      if (c_end >= c1) {
        // whole slice inside the vocabulary: 64 columns per TMEM wait, no bounds test
        for (; c + 64 <= c1; c += 64) {
          float x0[32], x1[32];
          tmem_ld32(tmem + lane_addr + col + c, x0);
          tmem_ld32(tmem + lane_addr + col + c + 32, x1);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (x0[e] > best) { best = x0[e]; bidx = v0 + c + e; }
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (x1[e] > best) { best = x1[e]; bidx = v0 + c + 32 + e; }
        }
      }
      for (; c < c1; c += 32) {  // c, c1: multiples of 16, warp-uniform
        float x0[16], x1[16];
        const bool two = c + 16 < c1;
        tmem_ld16(tmem + lane_addr + col + c, x0);
        if (two) tmem_ld16(tmem + lane_addr + col + c + 16, x1);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e)
          if (c + e < c_end && x0[e] > best) { best = x0[e]; bidx = v0 + c + e; }
        if (two) {
#pragma unroll
          for (int e = 0; e < 16; ++e)
            if (c + 16 + e < c_end && x1[e] > best) { best = x1[e]; bidx = v0 + c + 16 + e; }
        }
      }
      tc_fence_before();
      mbar_arrive(bar(LmLayout::acc_empty(slot)));
      // a slice whose values are all NaN (= -inf) still offers its lowest column
      if (bidx < 0 && c0 < c_end) bidx = v0 + c0;
      if (row < a.R && bidx >= 0)
        atomicMax(a.keys + row, consensus_key(best, static_cast<uint32_t>(bidx)));
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kLmMmaWarp) tmem_dealloc(tmem, kLmTmemCols);
  if (threadIdx.x == 0 && *abort_flag && a.error_flag) atomicOr(a.error_flag, ORTHRUS_FLAG_TIMEOUT);
}

}  // namespace orthrus
