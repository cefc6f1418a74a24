// Orthrus block attention on sm_100a: tcgen05 MMAs with TMEM accumulators,
// TMA-fed shared-memory pipeline, warp-specialised roles, split-KV partials.
//
// What it computes ("Orthrus: Memory-Efficient Parallel Token Generation via
// Dual-View Diffusion", technical summary §2.2 mask M_diff for the DIFFUSION
// view and §2.3 item 2 for the VERIFY view): for every sequence b, KV head h,
// block row i and query head h*G+g, softmax attention over the L_b prefix keys
// read through the page table followed by the block's own K_b keys, the block
// keys being all visible (DIFFUSION) or visible up to row i (VERIFY).
//
// Work unit = (sequence b, KV head h). Its G*K_b query rows (token-major:
// row r = i*G + g) form one M = 128 MMA tile that stays in shared memory; the
// unit's keys are cut into 64-key tiles: ceil(L_b/64) prefix tiles, then one
// block tile. The host picks one of four schedules (see plan_attn): one CTA
// per whole unit; proportional chunks (few long units, each cut into
// near-equal chunks in proportion to its tiles); balanced ranges (a CTA per SM
// walks a contiguous range of the global (unit, tile) sequence, so every CTA
// gets the same number of tiles whatever the prefix lengths); or fixed chunks
// of a given number of tokens, walked by at most one CTA per SM. A unit that
// is cut is finished by the combine kernel from the partials (max, sum,
// normalised accumulator) of its pieces.
//
// Roles (384 threads):
//   warp 0      TMA producer, two lanes: lane 0 issues the Q tile per unit
//               and the K tiles into a K ring, lane 1 the V tiles into a
//               separate, deeper V ring (K is released by its QK three tiles
//               before V is released by its PV); both step one tile at a time.
//   warps 1-2   MMA issuers, one per softmax group: S = Q K^T for the group's
//               tiles into its two TMEM S buffers (one own tile ahead), and
//               O += P V into its TMEM accumulator. Two issuing warps overlap
//               the per-tile issue overhead; each keeps its own P/S aliasing
//               in one in-order MMA stream. Warp 1 owns TMEM.
//   warps 3-6   softmax group 0 (even tiles), warps 7-10 softmax group 1 (odd
//               tiles). Each thread owns one query row (= one TMEM lane): it
//               reads its S row from TMEM, applies the view's mask, keeps a
//               running max/sum, writes P (bf16 pairs) back into TMEM over
//               its S row for the PV MMA (A operand from TMEM) and, at the
//               end of a unit, merges the two groups'
//               accumulators and stores the output (or a partial).
//   warp 11     block writer (write-then-truncate VERIFY only): copies the
//               block's K/V rows into the cache slots after the prefix while
//               the pipeline streams that prefix; otherwise idle.
// The two softmax groups keep separate O accumulators (TMEM columns), so they
// never wait on each other inside a unit.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "orthrus.h"
#include "ptx.cuh"

namespace orthrus {

constexpr int kTileN = 64;          // keys per tile
constexpr int kTileM = 128;         // query rows per MMA tile
constexpr int kAttnThreads = 384;   // 12 warps
constexpr int kProducerWarp = 0;
constexpr int kMmaWarp0 = 1;        // warps 1 and 2 issue the MMAs of softmax groups 0 and 1
constexpr int kSoftmaxWarp0 = 3;    // warps 3-6: softmax group 0, warps 7-10: group 1
constexpr int kWriterWarp = 11;     // block K/V -> cache (write-then-truncate VERIFY)
constexpr uint32_t kTmemCols = 512;
constexpr int kSPerGroup = 2;       // S buffers per group: QK runs one own tile ahead
constexpr uint32_t kTmemS = 0;      // S buffer k of group w at column 64*(2w + k)
constexpr uint32_t kTmemO = 256;    // O of group w at column 256 + D*w
constexpr float kRescaleLog2 = 8.0f;  // rescale O only when the max grows by > 2^8

struct AttnArgs {
  int view, B, Hq, Hkv, G, page_size, max_pages, num_pages, max_block, total_rows;
  const int* prefix_lens;
  const int* cu_block;
  const int* page_table;
  __nv_bfloat16* out;
  float* ws_o;     // partial accumulators [parts][4 row blocks][D][32 rows] (see part_o)
  float* ws_lse;   // partial log2-sum-exp  [parts][128]
  int* error_flag;
  float scale_log2;  // softmax scale * log2(e)
  int q_box_rows;    // tokens per Q box: min(max_block, total_rows)
  int blk_box_rows;  // rows per block-K/V box: min(64, total_rows)
  int chunked;       // 0: balanced ranges over num_ctas CTAs; 1: fixed chunks;
                     // 2: proportional chunks (see prop_ctas)
  int chunk_tiles;   // chunked == 1: prefix tiles per chunk
  int max_chunks;    // chunked == 1: chunks per unit (grid = B * Hkv * max_chunks)
  int num_ctas;      // grid size
  unsigned long long timeout_ns;
  int fault_inject;  // test hook: 1 drops each CTA's first V copy (a wait must time out)
  int out_v8;        // out is 32-byte aligned: rows are written with 256-bit stores
  // Write-then-truncate VERIFY: also store block rows [0, K_b) of k/v_block
  // into the cache slots L_b .. L_b + K_b - 1 (the caller commits L_b += n_b).
  int write_block;
  const uint4* kb_rows;  // k_block / v_block as 16-byte chunks
  const uint4* vb_rows;
  uint4* kc_rows;        // k_cache / v_cache as 16-byte chunks
  uint4* vc_rows;
};

// ---------------------------------------------------------------------------
// Schedule: identical arithmetic in every role and in the combine kernel.

// K_b; 0 for a sequence whose row range is malformed (it is skipped and flagged).
__device__ __forceinline__ int seq_block_len(const AttnArgs& a, int b) {
  if (!a.cu_block) return a.max_block;
  const int r0 = a.cu_block[b], r1 = a.cu_block[b + 1];
  if (r0 < 0 || r1 < r0 || r1 > a.total_rows || r1 - r0 > a.max_block) return 0;
  return r1 - r0;
}
__device__ __forceinline__ bool seq_rows_bad(const AttnArgs& a, int b) {
  if (!a.cu_block) return false;
  const int r0 = a.cu_block[b], r1 = a.cu_block[b + 1];
  return r0 < 0 || r1 < r0 || r1 > a.total_rows || r1 - r0 > a.max_block;
}
__device__ __forceinline__ int seq_row0(const AttnArgs& a, int b) {
  return a.cu_block ? a.cu_block[b] : b * a.max_block;
}
// Prefix length clamped to what the page table can address.
__device__ __forceinline__ int seq_prefix_len(const AttnArgs& a, int b) {
  const int L = a.prefix_lens[b];
  const long long cap = (long long)a.max_pages * a.page_size;
  return L < 0 ? 0 : (L > cap ? (int)cap : L);
}
__device__ __forceinline__ bool seq_len_bad(const AttnArgs& a, int b) {
  const int L = a.prefix_lens[b];
  return L < 0 || (long long)L > (long long)a.max_pages * a.page_size;
}
__device__ __forceinline__ int seq_tiles(const AttnArgs& a, int b) {
  if (seq_block_len(a, b) <= 0) return 0;
  return (seq_prefix_len(a, b) + kTileN - 1) / kTileN + 1;
}
// Chunked mode: number of chunks of a unit with nt tiles (block tile joins the last).
__device__ __forceinline__ int unit_chunks(const AttnArgs& a, int nt) {
  const int np = nt - 1;
  const int c = (np + a.chunk_tiles - 1) / a.chunk_tiles;
  return c < 1 ? 1 : c;
}

__device__ __forceinline__ long long range_begin(long long T, int c, int C) {
  return T * c / C;
}

// Proportional chunks (few long units): of the C CTAs, a unit with nt tiles
// gets 1 + floor((C - U) * nt / T), at most nt, where U counts the units with
// tiles and T sums their tiles (so the counts add up to at most C); chunk k of
// c covers the unit's tiles [k*nt/c, (k+1)*nt/c). Units stay whole inside a
// CTA, and equal lengths get equal chunks. Sequence b's units take the CTAs
// after those of sequences 0..b-1, head by head.
constexpr int kMinChunkTiles = 4;  // a split pays a partial and the combine
__device__ __forceinline__ int prop_ctas(long long T, int U, int C, int nt) {
  if (nt <= 0) return 0;
  const long long c = 1 + (long long)(C - U) * nt / T;
  const int cap = nt / kMinChunkTiles > 1 ? nt / kMinChunkTiles : 1;
  return c < cap ? (int)c : cap;
}

// What the schedule needs of sequence b: tiles, clamped prefix length, K_b and
// first block row. The attention kernel computes these once per CTA into a
// shared-memory table (sequences 0 .. kSeqTableCap-1); later sequences are
// read from global memory.
struct SeqInfo {
  int nt, L, Kb, row0;
};
constexpr int kSeqTableCap = 512;

__device__ __forceinline__ SeqInfo seq_info_global(const AttnArgs& a, int b) {
  SeqInfo s;
  s.Kb = seq_block_len(a, b);
  s.L = seq_prefix_len(a, b);
  s.row0 = seq_row0(a, b);
  s.nt = s.Kb <= 0 ? 0 : (s.L + kTileN - 1) / kTileN + 1;
  return s;
}

struct SeqTable {
  const int4* rows;  // shared memory, kSeqTableCap entries {nt, L, Kb, row0}
  __device__ __forceinline__ SeqInfo get(const AttnArgs& a, int b) const {
    if (b < kSeqTableCap) {
      const int4 r = rows[b];
      return SeqInfo{r.x, r.y, r.z, r.w};
    }
    return seq_info_global(a, b);
  }
  __device__ __forceinline__ int nt(const AttnArgs& a, int b) const {
    return b < kSeqTableCap ? rows[b].x : seq_info_global(a, b).nt;
  }
};

struct Segment {
  int b, h, t0, t1, nt;
  int part;  // -1: the CTA covers the whole unit and writes the output
};

struct SegCursor {
  int b, h, t;
  long long remaining;
  int first;
  int cta;  // partial slot: the CTA (balanced, proportional) or the chunk slot (fixed chunks)
};

// Fixed chunks: slot j is chunk j % max_chunks of unit j / max_chunks. The
// grid is at most one CTA per SM, and CTA c takes the slots c, c + grid,
// c + 2 grid, ... that hold tiles, one segment each. Points the cursor at the
// first such slot at or after j; false (remaining = 0) when there is none.
__device__ __forceinline__ bool chunk_seek(const AttnArgs& a, const SeqTable& tab, int j,
                                           SegCursor& c);

// kWalk: the kernel variant whose CTAs walk several fixed-chunk slots. The
// other variant runs every schedule in which a fixed-chunk CTA holds one slot
// (the one-CTA-per-unit plan among them) without the walk's code.
template <bool kWalk>
__device__ __forceinline__ bool cursor_next(const AttnArgs& a, const SeqTable& tab, SegCursor& c,
                                            Segment& s) {
  if (c.remaining <= 0 || c.b >= a.B) return false;
  const int nt = tab.nt(a, c.b);
  long long end = c.t + c.remaining;
  const int t1 = end < nt ? (int)end : nt;
  s.b = c.b;
  s.h = c.h;
  s.t0 = c.t;
  s.t1 = t1;
  s.nt = nt;
  const bool full = (s.t0 == 0 && s.t1 == nt);
  s.part = full ? -1 : (a.chunked ? c.cta : c.cta * 2 + (c.first ? 0 : 1));
  c.first = 0;
  if (kWalk && a.chunked == 1) {
    chunk_seek(a, tab, c.cta + a.num_ctas, c);
    return true;
  }
  c.remaining -= (t1 - c.t);
  c.t = 0;
  if (++c.h == a.Hkv) {
    c.h = 0;
    do {
      ++c.b;
    } while (c.b < a.B && tab.nt(a, c.b) == 0);
  }
  return true;
}

// The host keeps the slot count below 2^31 - 2^16, so 32-bit arithmetic holds.
__device__ __forceinline__ bool chunk_seek(const AttnArgs& a, const SeqTable& tab, int j,
                                           SegCursor& c) {
  const int slots = a.B * a.Hkv * a.max_chunks;
  for (; j < slots; j += a.num_ctas) {
    const int u = j / a.max_chunks;
    const int k = j - u * a.max_chunks;
    const int b = u / a.Hkv;
    const int nt = tab.nt(a, b);
    if (nt <= 0) continue;
    const int nc = unit_chunks(a, nt);
    if (k >= nc) continue;
    c.b = b;
    c.h = u - b * a.Hkv;
    c.t = k * a.chunk_tiles;
    c.remaining = (k == nc - 1) ? nt - c.t : a.chunk_tiles;
    c.cta = j;
    return true;
  }
  c.b = a.B;
  c.remaining = 0;
  return false;
}

// ---------------------------------------------------------------------------
// Shared-memory layout (offsets from a 1024-byte aligned base).

template <int D>
struct AttnLayout {
  static constexpr int DH = D / 64;                 // 64-column panels per row
  static constexpr int kNK = (D == 128) ? 4 : 10;   // K ring depth
  static constexpr int kNV = (D == 128) ? 6 : 12;   // V ring depth
  static constexpr int kQPanel = kTileM * 128;      // bytes of one Q panel
  static constexpr int kQBytes = DH * kQPanel;
  static constexpr int kKVPanel = kTileN * 128;        // bytes of one K (or V) panel
  static constexpr int kKVBytes = DH * kKVPanel;       // one K (or V) tile
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kQBytes;
  static constexpr int kVOff = kKOff + kNK * kKVBytes;
  static constexpr int kXOff = kVOff + kNV * kKVBytes;  // (max, sum) exchange [2][2][128]
  static constexpr int kBarOff = kXOff + 2 * 2 * kTileM * 8;
  // barrier indices
  static constexpr int kBarKFull = 0;
  static constexpr int kBarKEmpty = kBarKFull + kNK;
  static constexpr int kBarVFull = kBarKEmpty + kNK;
  static constexpr int kBarVEmpty = kBarVFull + kNV;
  static constexpr int kBarQFull = kBarVEmpty + kNV;
  static constexpr int kBarQEmpty = kBarQFull + 1;
  static constexpr int kBarSFull = kBarQEmpty + 1;             // [2 groups][kSPerGroup]
  static constexpr int kBarPReady = kBarSFull + 2 * kSPerGroup;  // [2 groups][2]
  static constexpr int kBarOReady = kBarPReady + 4;      // [2]
  static constexpr int kBarOFree = kBarOReady + 2;
  static constexpr int kBarXchg = kBarOFree + 1;
  static constexpr int kBarDrain = kBarXchg + 1;  // [2]
  static constexpr int kNumBars = kBarDrain + 2;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;  // abort flag, TMEM base
  // schedule: start cursor {b, h, t, -, remaining}, scan scratch, sequence table
  static constexpr int kSchedOff = (kMiscOff + 16 + 15) / 16 * 16;
  static constexpr int kScanOff = kSchedOff + 32;
  static constexpr int kSeqOff = kScanOff + 16 * 8;
  static constexpr int kBytes = kSeqOff + kSeqTableCap * 16;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base
  static_assert(kAlloc <= 232448, "shared memory budget exceeded");
  // Each MMA warp runs QK up to two own tiles (four tiles) ahead of PV.
  static_assert(kNK >= 4, "K ring shallower than the QK lead");
  // Tile it goes to ring slot it % depth and belongs to MMA warp / softmax
  // group it & 1. With even depths every fill of a slot belongs to the same
  // consumer, which therefore waits on each phase of that slot's barriers in
  // turn. With an odd depth a consumer would skip the other consumer's fill
  // and wait two phases ahead; copies complete out of order, so that fill
  // could still be in flight and the parity wait would pass early (stale K,
  // and a release committed before the copy landed).
  static_assert(kNK % 2 == 0 && kNV % 2 == 0, "ring depths must be even");
};

// Descriptors of the four MMA operands (all SWIZZLE_128B).
// A = Q (K-major): panel p at +p*kQPanel, 8-row groups 1024 B apart.
// B = K tile (K-major): panel p at +p*kKVPanel.
// A = P: in TMEM (packed bf16 pairs aliasing the first 32 columns of its S buffer).
// B = V tile (MN-major): D-panels kKVPanel apart (LBO), 8-key groups 1024 B apart (SBO).
template <int D>
__device__ __forceinline__ uint64_t desc_q(uint32_t q, int kk) {
  return smem_desc_sw128(q + (kk >> 2) * AttnLayout<D>::kQPanel + (kk & 3) * 32, 16, 1024);
}
template <int D>
__device__ __forceinline__ uint64_t desc_k(uint32_t k, int kk) {
  return smem_desc_sw128(k + (kk >> 2) * AttnLayout<D>::kKVPanel + (kk & 3) * 32, 16, 1024);
}
template <int D>
__device__ __forceinline__ uint64_t desc_v(uint32_t v, int kk) {
  return smem_desc_sw128(v + kk * 16 * 128, AttnLayout<D>::kKVPanel, 1024);
}

// Keys of tile t that exist: 64 for a full prefix tile, fewer for the last
// partial prefix tile, K_b for the block tile.
__device__ __forceinline__ int tile_valid_keys(int t, int L, int np, int Kb) {
  if (t == np) return Kb;
  const int rem = L - t * kTileN;
  return rem < kTileN ? rem : kTileN;
}

// Partial accumulator of query row r (0..127), column c, in part p. Each warp
// of a softmax group holds 32 consecutive rows (one TMEM lane quarter), so
// the layout keeps those 32 rows contiguous per column: one warp-wide store
// of a column writes 128 contiguous bytes, and the combine reads the same way.
template <int D>
__device__ __forceinline__ long long part_o(int p, int r, int c) {
  return ((long long)p * kTileM + (r >> 5) * 32) * D + (long long)c * 32 + (r & 31);
}

__device__ __forceinline__ void raise_flag(const AttnArgs& a, int bits) {
  if (a.error_flag) atomicOr(a.error_flag, bits);
}

// ---------------------------------------------------------------------------
// Schedule prologue, run by the whole CTA before the roles split: the
// per-sequence facts are loaded in parallel into the shared table, a block
// reduction gives the total tile count T, and a block scan over the sequences'
// tile counts finds the unit and tile where this CTA's range starts. Returns
// false (uniformly) when the range is empty.
__device__ __forceinline__ long long block_sum_ll(long long x, long long* scan) {
  constexpr int kWarps = kAttnThreads / 32;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  if ((threadIdx.x & 31) == 0) scan[threadIdx.x >> 5] = x;
  __syncthreads();
  long long t = 0;
#pragma unroll
  for (int k = 0; k < kWarps; ++k) t += scan[k];
  __syncthreads();
  return t;
}

template <int D, bool kWalk>
__device__ __forceinline__ bool schedule_prologue(const AttnArgs& a, uint8_t* smem,
                                                  SeqTable& tab, SegCursor& start) {
  using Lay = AttnLayout<D>;
  constexpr int kWarps = kAttnThreads / 32;
  int* sc = reinterpret_cast<int*>(smem + Lay::kSchedOff);  // b, h, t, chunk slot
  long long* srem = reinterpret_cast<long long*>(smem + Lay::kSchedOff + 16);
  long long* scan = reinterpret_cast<long long*>(smem + Lay::kScanOff);
  int4* rows = reinterpret_cast<int4*>(smem + Lay::kSeqOff);
  tab.rows = rows;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  long long part = 0;
  for (int b = tid; b < a.B; b += kAttnThreads) {
    if (blockIdx.x == 0 && (seq_rows_bad(a, b) || seq_len_bad(a, b)))
      raise_flag(a, ORTHRUS_FLAG_BAD_LENGTH);
    const SeqInfo si = seq_info_global(a, b);
    if (b < kSeqTableCap) rows[b] = make_int4(si.nt, si.L, si.Kb, si.row0);
    part += (long long)a.Hkv * si.nt;
  }
  const long long T = block_sum_ll(part, scan);  // also publishes the table

  if (a.chunked == 2) {
    if (tid == 0) {
      int U = 0;
      for (int bb = 0; bb < a.B; ++bb) U += tab.nt(a, bb) > 0 ? a.Hkv : 0;
      int b = a.B, h = 0, t = 0;
      long long rem = 0, base = 0;
      for (int bb = 0; bb < a.B && U > 0; ++bb) {
        const int nt = tab.nt(a, bb);
        const int c = prop_ctas(T, U, a.num_ctas, nt);
        const long long span = (long long)a.Hkv * c;
        if (blockIdx.x < base + span) {
          const int off = (int)(blockIdx.x - base);
          const int k = off % c;
          b = bb;
          h = off / c;
          t = (int)((long long)k * nt / c);
          rem = (long long)(k + 1) * nt / c - t;
          break;
        }
        base += span;
      }
      sc[0] = b, sc[1] = h, sc[2] = t;
      *srem = rem;
    }
  } else if (a.chunked) {
    if (tid == 0) {
      if (kWalk) {
        SegCursor c;
        chunk_seek(a, tab, (int)blockIdx.x, c);
        sc[0] = c.b, sc[1] = c.h, sc[2] = c.t, sc[3] = c.cta;
        *srem = c.remaining;
      } else {  // one slot per CTA: slot = CTA
        int b = a.B, h = 0, t = 0;
        long long rem = 0;
        const int chunk = blockIdx.x % a.max_chunks;
        const int u = blockIdx.x / a.max_chunks;
        const int bu = u / a.Hkv;
        if (bu < a.B) {
          const int nt = tab.nt(a, bu);
          if (nt > 0 && chunk < unit_chunks(a, nt)) {
            b = bu;
            h = u % a.Hkv;
            t = chunk * a.chunk_tiles;
            rem = (chunk == unit_chunks(a, nt) - 1) ? (nt - t) : a.chunk_tiles;
          }
        }
        sc[0] = b, sc[1] = h, sc[2] = t, sc[3] = (int)blockIdx.x;
        *srem = rem;
      }
    }
  } else {
    const long long g0 = range_begin(T, blockIdx.x, a.num_ctas);
    const long long rem = range_begin(T, blockIdx.x + 1, a.num_ctas) - g0;
    if (tid == 0) {
      sc[0] = a.B, sc[1] = 0, sc[2] = 0;
      *srem = rem;
    }
    if (rem > 0) {
      long long off = 0;  // tiles of the sequences before this chunk of them
      for (int base = 0; base < a.B; base += kAttnThreads) {
        const int b = base + tid;
        const int nt = b < a.B ? tab.nt(a, b) : 0;
        const long long n = (long long)a.Hkv * nt;
        long long x = n;  // inclusive scan within the warp
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const long long y = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += y;
        }
        if (lane == 31) scan[warp] = x;
        __syncthreads();
        long long before = 0, total = 0;
#pragma unroll
        for (int k = 0; k < kWarps; ++k) {
          const long long v = scan[k];
          before += (k < warp) ? v : 0;
          total += v;
        }
        const long long excl = off + before + x - n;
        if (n > 0 && excl <= g0 && g0 < excl + n) {
          sc[0] = b;
          sc[1] = (int)((g0 - excl) / nt);
          sc[2] = (int)((g0 - excl) % nt);
        }
        off += total;
        __syncthreads();
        if (off > g0) break;
      }
    }
  }
  __syncthreads();
  start.cta = (kWalk && a.chunked == 1) ? sc[3] : (int)blockIdx.x;
  start.first = 1;
  start.b = sc[0];
  start.h = sc[1];
  start.t = sc[2];
  start.remaining = *srem;
  if (start.b >= a.B) start.remaining = 0;
  return start.remaining > 0;
}

// ---------------------------------------------------------------------------
// Roles

// Two lanes of the producer warp issue every copy: lane 0 the Q tile of each
// unit and the K tiles into the K ring, lane 1 the V tiles into the V ring.
// Each key tile is one 3-D box per tensor (64 tokens x both 64-column halves
// of D, landing as the two swizzled panels the MMA descriptors expect). A box
// issue holds its thread for a few hundred cycles, so one thread issuing both
// copies plus the page lookup paced the whole pipeline; the two lanes wait
// for their ring slots and issue their boxes side by side, one tile per step.
// Page ids are read four tiles ahead into registers, and the slot and the row
// inside the page are tracked incrementally (no division per tile).
template <int D, bool kWalk>
__device__ __forceinline__ void producer_role(const AttnArgs& a, uint8_t* smem,
                                              const CUtensorMap* tm_q, const CUtensorMap* tm_kc,
                                              const CUtensorMap* tm_vc, const CUtensorMap* tm_kb,
                                              const CUtensorMap* tm_vb, volatile int* abort_flag,
                                              const SeqTable& tab, const SegCursor& start) {
  using Lay = AttnLayout<D>;
  constexpr unsigned kPair = 0x3u;  // lanes 0 (K) and 1 (V)
  const bool is_v = (threadIdx.x & 31) == 1;
  const int depth = is_v ? Lay::kNV : Lay::kNK;
  const uint32_t base = smem_u32(smem);
  const uint32_t bars = base + Lay::kBarOff;
  const uint32_t ring = base + (is_v ? Lay::kVOff : Lay::kKOff);
  const uint32_t full0 = bars + 8u * (is_v ? Lay::kBarVFull : Lay::kBarKFull);
  const uint32_t empty0 = bars + 8u * (is_v ? Lay::kBarVEmpty : Lay::kBarKEmpty);
  const CUtensorMap* tm_cache = is_v ? tm_vc : tm_kc;
  const CUtensorMap* tm_blk = is_v ? tm_vb : tm_kb;
  const uint32_t blk_bytes = Lay::DH * a.blk_box_rows * 128;
  const int tiles_per_page = a.page_size / kTileN;
  const int slab_rows = a.Hkv * a.page_size;  // cache rows per page
  int n = 0, q_issued = 0;  // copies issued into this lane's ring; Q tiles issued
  int s = 0, r = 0;         // ring slot of copy n and how often it was filled before
  bool ok = true;

  SegCursor cur = start;
  Segment sg;
  int si = 0;
  while (ok && cursor_next<kWalk>(a, tab, cur, sg)) {
    const int b = sg.b, h = sg.h;
    const SeqInfo sq = tab.get(a, b);
    const int row0 = sq.row0;
    const int np = (sq.L + kTileN - 1) / kTileN;
    const int* ptab = a.page_table + (long long)b * a.max_pages;
    // Q tile of this unit (rows (i, g) for i < max_block, g < G), by lane 0.
    bool qok = true;
    if (!is_v && si > 0)
      qok = mbar_wait(bars + 8u * Lay::kBarQEmpty, (si - 1) & 1, abort_flag, a.timeout_ns);
    if (!__all_sync(kPair, qok)) {
      ok = false;
      break;
    }
    if (!is_v) {
      mbar_arrive_expect_tx(bars + 8u * Lay::kBarQFull, Lay::DH * a.G * a.q_box_rows * 128);
#pragma unroll
      for (int p = 0; p < Lay::DH; ++p)
        tma_load_3d(base + Lay::kQOff + p * Lay::kQPanel, tm_q, bars + 8u * Lay::kBarQFull,
                    p * 64, h * a.G, row0);
    }
    ++q_issued;
    // Page ids of the next four prefix tiles and the position of tile t0 in
    // its page; ahead_* is the page position of tile t + 4.
    const int t1p = sg.t1 < np ? sg.t1 : np;
    int sub = sg.t0 % tiles_per_page;
    int ahead_pidx = sg.t0 / tiles_per_page, ahead_sub = sub;
    int pq[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      pq[k] = (sg.t0 + k < t1p) ? ptab[ahead_pidx] : 0;
      if (++ahead_sub == tiles_per_page) ahead_sub = 0, ++ahead_pidx;
    }
    for (int t = sg.t0; t < sg.t1; ++t) {
      const bool block = t >= np;
      int row = row0;
      if (!block) {
        int page = pq[0];
        if (page < 0 || page >= a.num_pages) {
          raise_flag(a, ORTHRUS_FLAG_BAD_PAGE);
          page = 0;  // keep the pipeline flowing on an in-bounds page
        }
        row = page * slab_rows + h * a.page_size + sub * kTileN;
      }
      pq[0] = pq[1];
      pq[1] = pq[2];
      pq[2] = pq[3];
      pq[3] = (t + 4 < t1p) ? ptab[ahead_pidx] : 0;
      if (++ahead_sub == tiles_per_page) ahead_sub = 0, ++ahead_pidx;
      if (++sub == tiles_per_page) sub = 0;
      // The slot's previous fill must have been consumed.
      bool wok = true;
      if (r > 0) {
        wok = mbar_wait(empty0 + 8u * s, (r - 1) & 1, abort_flag, a.timeout_ns);
      }
      if (!__all_sync(kPair, wok)) {
        ok = false;
        break;
      }
      // test hook: the first V copy is never issued, so its full barrier never
      // completes and the consumers' bounded waits must give up
      if (!(is_v && a.fault_inject == 1 && n == 0)) {
        const uint32_t fb = full0 + 8u * s;
        const uint32_t dst = ring + s * Lay::kKVBytes;
        mbar_arrive_expect_tx(fb, block ? blk_bytes : (uint32_t)Lay::kKVBytes);
        if (block) {
#pragma unroll
          for (int p = 0; p < Lay::DH; ++p)
            tma_load_3d(dst + p * Lay::kKVPanel, tm_blk, fb, p * 64, h, row);
        } else {
          tma_load_3d(dst, tm_cache, fb, 0, row, 0);
        }
      }
      ++n;
      if (++s == depth) s = 0, ++r;
    }
    ++si;
  }
  if (ok && !*abort_flag) {
    // Producer tail. The MMA warps release ring and Q slots with
    // tcgen05.commit, whose mbarrier arrivals land asynchronously; the last
    // release of each slot is never waited for above. Wait for it, so that no
    // arrival is still in flight when the CTA exits: it would land on the
    // barriers of the next CTA that this SM runs, in the same shared memory.
    for (int ss = 0; ss < depth && ok; ++ss) {
      const int nf = n / depth + (ss < n % depth ? 1 : 0);  // fills of slot ss
      if (nf > 0) ok = mbar_wait(empty0 + 8u * ss, (nf - 1) & 1, abort_flag, a.timeout_ns);
    }
    if (!is_v && ok && q_issued > 0)
      ok = mbar_wait(bars + 8u * Lay::kBarQEmpty, (q_issued - 1) & 1, abort_flag, a.timeout_ns);
  }
  if (!ok || *abort_flag) {
    // Wind down: let every copy this lane started land before the CTA exits.
    volatile int no_abort = 0;
    for (int ss = 0; ss < depth; ++ss) {
      const int nf = n / depth + (ss < n % depth ? 1 : 0);
      if (nf > 0) mbar_wait(full0 + 8u * ss, (nf - 1) & 1, &no_abort, 20000000ull);
    }
    if (!is_v && q_issued > 0)
      mbar_wait(bars + 8u * Lay::kBarQFull, (q_issued - 1) & 1, &no_abort, 20000000ull);
  }
}

// One tile as the MMA issuer sees it: its unit segment, its index inside the
// unit (t) and in the CTA's tile order (it), and the unit's lengths.
struct TileStep {
  SegCursor cur;
  Segment sg;
  int si, t, it, L, np, Kb;
  bool valid;
};

// One MMA warp per softmax group w: it issues QK and PV for the group's tiles
// (global tile index parity w). The issuing thread's scalar work sits between
// consecutive MMAs, so every operand descriptor is a precomputed base plus a
// compile-time step: the 14-bit start-address field holds (smem address >> 4)
// and never carries.
//
// Q bookkeeping covers every segment, own tiles or not: at a segment start the
// warp waits for that unit's Q tile, and after its last QK of the segment it
// commits one arrival on q_empty (two arrivals, one per warp, release Q).
template <int D, bool kWalk>
__device__ __forceinline__ void mma_role(const AttnArgs& a, uint8_t* smem, uint32_t tmem,
                                         volatile int* abort_flag, int w, const SeqTable& tab,
                                         const SegCursor& start) {
  using Lay = AttnLayout<D>;
  const uint32_t base = smem_u32(smem);
  const uint32_t bars = base + Lay::kBarOff;
  constexpr uint32_t kIdescQK = idesc_bf16_f32(kTileM, kTileN, 0);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(kTileM, D, 1);
  const uint64_t dq = smem_desc_sw128(base + Lay::kQOff, 16, 1024);
  const uint64_t dk = smem_desc_sw128(base + Lay::kKOff, 16, 1024);
  const uint64_t dv = smem_desc_sw128(base + Lay::kVOff, Lay::kKVPanel, 1024);
  const uint32_t s_base = tmem + kTmemS + 64u * kSPerGroup * w;
  const uint32_t o_acc = tmem + kTmemO + (uint32_t)(D * w);

  // Every lane polls the barrier (no divergence around the wait); a vote makes
  // the verdict warp-uniform.
  auto wait = [&](uint32_t b, uint32_t parity) -> bool {
    const bool ok = mbar_wait(b, parity, abort_flag, a.timeout_ns);
    return __all_sync(0xffffffffu, ok);
  };

  // QK of own tile m (global tile j) into S buffer m % 2; that buffer last held
  // P of own tile m - 2, whose PV this warp issued before: the tensor pipe runs
  // one thread's MMAs in order, so P is read before it is overwritten.
  auto issue_qk = [&](const TileStep& j, int m) -> bool {
    const int slot = j.it % Lay::kNK;
    if (!wait(bars + 8u * (Lay::kBarKFull + slot), (j.it / Lay::kNK) & 1)) return false;
    tc_fence_after();
    const int sb = m & (kSPerGroup - 1);
    const uint32_t d = s_base + 64u * sb;
    const uint64_t kd = dk + (uint64_t)((slot * Lay::kKVBytes) >> 4);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint64_t aq = dq + (uint64_t)(((kk >> 2) * Lay::kQPanel + (kk & 3) * 32) >> 4);
      const uint64_t bk = kd + (uint64_t)(((kk >> 2) * Lay::kKVPanel + (kk & 3) * 32) >> 4);
      if (elect_one()) mma_bf16_ss(d, aq, bk, kIdescQK, kk > 0 ? 1u : 0u);
    }
    if (elect_one()) {
      mma_commit(bars + 8u * (Lay::kBarSFull + kSPerGroup * w + sb));
      mma_commit(bars + 8u * (Lay::kBarKEmpty + slot));
    }
    __syncwarp();
    return true;
  };

  auto issue_pv = [&](const TileStep& j, int m) -> bool {
    const int slot = j.it % Lay::kNV;
    // p_ready also means the tile's V copy has landed: the softmax group waits
    // for it before publishing P, which keeps that wait off this warp's path.
    if (!wait(bars + 8u * (Lay::kBarPReady + 2 * w + (m & 1)), (m >> 1) & 1)) return false;
    const int nvalid = tile_valid_keys(j.t, j.L, j.np, j.Kb);
    if (nvalid < kTileN) {
      // Rows past the last valid key may hold stale or non-finite data;
      // P is zero there, but 0 * NaN is NaN, so clear those V rows.
      const int lane = threadIdx.x & 31;
      const uint32_t v = base + Lay::kVOff + slot * Lay::kKVBytes;
      const int rows = kTileN - nvalid;
      const int chunks = rows * Lay::DH * 8;  // 16-byte chunks
      for (int c = lane; c < chunks; c += 32) {
        const int p = c / (rows * 8);
        const int rem = c % (rows * 8);
        const int r = nvalid + rem / 8;
        st_shared_v4(v + p * Lay::kKVPanel + r * 128 + (rem % 8) * 16, 0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
      __syncwarp();
    }
    tc_fence_after();
    const uint32_t pa = s_base + 64u * (m & (kSPerGroup - 1));
    const uint64_t vd = dv + (uint64_t)((slot * Lay::kKVBytes) >> 4);
    const uint32_t acc0 = (j.t - j.sg.t0 >= 2) ? 1u : 0u;
#pragma unroll
    for (int kk = 0; kk < kTileN / 16; ++kk) {
      const uint64_t bv = vd + (uint64_t)((kk * 16 * 128) >> 4);
      if (elect_one()) mma_bf16_ts(o_acc, pa + 8u * kk, bv, kIdescPV, (kk > 0) ? 1u : acc0);
    }
    if (elect_one()) {
      mma_commit(bars + 8u * (Lay::kBarOReady + w));
      mma_commit(bars + 8u * (Lay::kBarVEmpty + slot));
    }
    __syncwarp();
    return true;
  };

  // The CTA's range is walked one unit segment at a time, and within a
  // segment this warp's own tiles (CTA tile index it = w, w + 2, ...) in a
  // straight loop: QK(0), QK(1), then PV(m), QK(m + 2) for m = 0, 1, ... (the
  // QKs run two own tiles ahead of the PVs, the depth of the S double buffer).
  // A segment's QKs start only after every PV of the previous segment was
  // issued, so the unit's last PVs (and the epilogue waiting on them) never
  // queue behind the next unit's QKs, which wait for that unit's Q tile.
  // The per-tile bookkeeping is a few integer operations: this warp's issue
  // loop paces the whole pipeline (a general tile walker here, with its
  // branches between the MMA batches, cost about 12% of a Qwen3-8B layer).
  auto commit_q_empty = [&]() {
    if (elect_one()) mma_commit(bars + 8u * Lay::kBarQEmpty);
    __syncwarp();
  };
  SegCursor cur = start;
  Segment sg;
  int si = 0;   // segment index (Q tile and O phases)
  int it0 = 0;  // CTA tile index of the segment's first tile
  int mb = 0;   // own tiles of this warp in earlier segments
  bool ok = true;
  while (ok && cursor_next<kWalk>(a, tab, cur, sg)) {
    const SeqInfo sq = tab.get(a, sg.b);
    TileStep j;
    j.cur = cur;
    j.sg = sg;
    j.si = si;
    j.L = sq.L;
    j.np = (sq.L + kTileN - 1) / kTileN;
    j.Kb = sq.Kb;
    j.valid = true;
    const int n = sg.t1 - sg.t0;
    const int first = (w - it0) & 1;  // segment-local index of the first own tile
    const int n_own = n > first ? (n - first + 1) / 2 : 0;
    auto tile = [&](int m) {  // own tile m of the segment
      TileStep x = j;
      const int loc = first + 2 * m;
      x.t = sg.t0 + loc;
      x.it = it0 + loc;
      return x;
    };
    // Every warp waits for the unit's Q tile, own tiles or not, before it
    // commits its release: one warp never completes a q_empty phase alone.
    if (!wait(bars + 8u * Lay::kBarQFull, si & 1)) { ok = false; break; }
    for (int m = 0; m < 2 && m < n_own && ok; ++m) ok = issue_qk(tile(m), mb + m);
    if (!ok) break;
    if (n_own <= 2) commit_q_empty();
    for (int m = 0; m < n_own && ok; ++m) {
      // the group's first PV of a unit overwrites O: the previous unit's
      // epilogue must have read it
      if (m == 0 && si > 0 && !wait(bars + 8u * Lay::kBarOFree, (si - 1) & 1)) { ok = false; break; }
      ok = issue_pv(tile(m), mb + m);
      if (ok && m + 2 < n_own) {
        ok = issue_qk(tile(m + 2), mb + m + 2);
        if (ok && m + 3 == n_own) commit_q_empty();
      }
    }
    mb += n_own;
    it0 += n;
    ++si;
  }
  // Drain: every MMA issued above completes before TMEM is released.
  if (elect_one()) {
    mma_commit(bars + 8u * (Lay::kBarDrain + w));
    volatile int no_abort = 0;
    mbar_wait(bars + 8u * (Lay::kBarDrain + w), 0, &no_abort, 20000000ull);
  }
  __syncwarp();
}

template <int D, bool kWalk>
__device__ __forceinline__ void softmax_role(const AttnArgs& a, uint8_t* smem, uint32_t tmem,
                                             volatile int* abort_flag, const SeqTable& tab,
                                             const SegCursor& start) {
  using Lay = AttnLayout<D>;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int w = (warp - kSoftmaxWarp0) >> 2;   // softmax group 0 or 1
  const int row = 32 * (warp & 3) + lane;      // query row == TMEM lane
  const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
  const uint32_t base = smem_u32(smem);
  const uint32_t bars = base + Lay::kBarOff;
  auto bar = [&](int i) { return bars + 8u * i; };
  const uint32_t t_o_self = tmem + lane_off + kTmemO + (uint32_t)(D * w);
  const uint32_t t_o0 = tmem + lane_off + kTmemO;
  const uint32_t t_o1 = tmem + lane_off + kTmemO + D;
  const float c = a.scale_log2;
  const float NEG_INF = -__int_as_float(0x7f800000);

  auto wait = [&](uint32_t b, uint32_t parity) -> bool {
    const bool ok = mbar_wait(b, parity, abort_flag, a.timeout_ns);
    return __all_sync(0xffffffffu, ok);
  };

  int cnt = 0;        // tiles this group processed (CTA-wide)
  int pv_waited = 0;  // PV completions of this group already observed

  SegCursor cur = start;
  Segment sg;
  int it = 0, si = 0;
  bool ok = true;
  while (ok && cursor_next<kWalk>(a, tab, cur, sg)) {
    const int b = sg.b, h = sg.h;
    const SeqInfo sq = tab.get(a, b);
    const int Kb = sq.Kb, row0 = sq.row0;
    const int L = sq.L;
    const int np = (L + kTileN - 1) / kTileN;
    const int rows_valid = a.G * Kb;
    const bool my_valid = row < rows_valid;
    const int irow = row / a.G;   // block row (token) of this query row
    const int ntile = sg.t1 - sg.t0;
    const bool has0 = ntile >= 2 || ((it & 1) == 0);
    const bool has1 = ntile >= 2 || ((it & 1) == 1);
    float m_ref = NEG_INF, l_sum = 0.f;
    bool has = false;

    for (int t = sg.t0; t < sg.t1; ++t, ++it) {
      if ((it & 1) != w) continue;
      const int sb = cnt & (kSPerGroup - 1);  // this group's own tile cnt -> S buffer
      if (!wait(bar(Lay::kBarSFull + kSPerGroup * w + sb), (cnt / kSPerGroup) & 1)) { ok = false; break; }
      tc_fence_after();
      float s[64];
      const uint32_t t_s = tmem + lane_off + kTmemS + 64u * (kSPerGroup * w + sb);
      tmem_ld32(t_s, *reinterpret_cast<float(*)[32]>(&s[0]));
      tmem_ld32(t_s + 32, *reinterpret_cast<float(*)[32]>(&s[32]));
      tmem_wait_ld();
      // mask: keys that do not exist or that this row may not see
      int lim = kTileN;
      if (!my_valid) lim = 0;
      else if (t == np) lim = (a.view == ORTHRUS_VIEW_DIFFUSION) ? Kb : (irow + 1);
      else if (t == np - 1) lim = L - t * kTileN;
      if (lim < kTileN) {
#pragma unroll
        for (int k = 0; k < 64; ++k) s[k] = (k < lim) ? s[k] : NEG_INF;
      }
      float mx[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx[k] = s[k];
#pragma unroll
      for (int k = 8; k < 64; k += 2) mx[(k >> 1) & 7] = fmax3(mx[(k >> 1) & 7], s[k], s[k + 1]);
      const float mt = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]),
                             fmaxf(mx[6], mx[7]));
      const float m_new = fmaxf(m_ref, mt * c);
      const bool need = has && (m_new > m_ref + kRescaleLog2);
      if (!has) m_ref = m_new;
      // S of own tile cnt is complete, so are the PVs of own tiles 0 .. cnt-2:
      // the MMA warp issued them before this QK, and one thread's tcgen05
      // operations complete in order. Only the PV of own tile cnt-1 may still
      // run. It is waited for only when O must be rescaled (so this tile's
      // exponentials overlap it) and at the group's last tile of the unit
      // (so at most one PV is pending at the unit's end). Each o_ready wait
      // is for the oldest unobserved phase with at most one phase in flight,
      // so the parity is exact. P_ready alternates between two barriers per
      // group, so P of tile cnt may be published before the MMA warp has
      // taken P of tile cnt-1.
      if (pv_waited < cnt - 1) pv_waited = cnt - 1;
      const bool unit_last = t + 2 >= sg.t1;
      if (unit_last && pv_waited < cnt) {
        if (!wait(bar(Lay::kBarOReady + w), pv_waited & 1)) { ok = false; break; }
        ++pv_waited;
      }
      if (__any_sync(0xffffffffu, need)) {
        if (pv_waited < cnt) {
          if (!wait(bar(Lay::kBarOReady + w), pv_waited & 1)) { ok = false; break; }
          ++pv_waited;
        }
        const float alpha = need ? ex2_approx(m_ref - m_new) : 1.f;
        if (need) {
          l_sum *= alpha;
          m_ref = m_new;
        }
        tc_fence_after();
#pragma unroll 1
        for (int ch = 0; ch < D / 32; ++ch) {
          float o[32];
          tmem_ld32(t_o_self + 32 * ch, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] *= alpha;
          tmem_st32(t_o_self + 32 * ch, o);
        }
        tmem_wait_st();
      }
      const float mref = (m_ref == NEG_INF) ? 0.f : m_ref;
      // Scale-and-subtract and the row sums run as packed fp32 pairs and the
      // maximum as three-input max, which cuts the softmax warps' instruction
      // count per tile by about a third; the arithmetic (fp32 round-to-nearest
      // FMA, the same eight partial sums in the same order) is unchanged.
      float2 ps2[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) ps2[k] = make_float2(0.f, 0.f);
      uint32_t pk[32];
      const float2 c2 = make_float2(c, c), nm2 = make_float2(-mref, -mref);
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const float2 x = ffma2(make_float2(s[2 * k], s[2 * k + 1]), c2, nm2);
        const float2 p = make_float2(ex2_approx(x.x), ex2_approx(x.y));
        ps2[k & 3] = fadd2(ps2[k & 3], p);
        pk[k] = pack_bf16x2(p.x, p.y);
      }
      float psum[8];
#pragma unroll
      for (int k = 0; k < 4; ++k) psum[2 * k] = ps2[k].x, psum[2 * k + 1] = ps2[k].y;
      // P (bf16 pairs) over the first 32 columns of this tile's S buffer
      tmem_st32u(t_s, pk);
      if (!wait(bars + 8u * (Lay::kBarVFull + it % Lay::kNV), (it / Lay::kNV) & 1)) {
        ok = false;
        break;
      }
      l_sum += ((psum[0] + psum[1]) + (psum[2] + psum[3])) + ((psum[4] + psum[5]) + (psum[6] + psum[7]));
      has = true;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(Lay::kBarPReady + 2 * w + (cnt & 1)));
      ++cnt;
    }
    if (!ok) break;

    // ---- end of the unit: merge the two groups, store output or partial ----
    if (pv_waited < cnt) {
      if (!wait(bar(Lay::kBarOReady + w), pv_waited & 1)) { ok = false; break; }
      ++pv_waited;
    }
    float2* xch = reinterpret_cast<float2*>(smem + Lay::kXOff);  // [si & 1][group][row]
    xch[((si & 1) * 2 + w) * kTileM + row] = make_float2(m_ref, l_sum);
    mbar_arrive(bar(Lay::kBarXchg));
    if (!wait(bar(Lay::kBarXchg), si & 1)) { ok = false; break; }
    tc_fence_after();
    const float2 other = xch[((si & 1) * 2 + (1 - w)) * kTileM + row];
    const float m_o = other.x, l_o = other.y;
    const float m0 = w == 0 ? m_ref : m_o, l0 = w == 0 ? l_sum : l_o;
    const float m1 = w == 0 ? m_o : m_ref, l1 = w == 0 ? l_o : l_sum;
    float M = NEG_INF;
    if (has0) M = fmaxf(M, m0);
    if (has1) M = fmaxf(M, m1);
    const float Mr = (M == NEG_INF) ? 0.f : M;
    const float a0 = has0 ? ex2_approx(m0 - Mr) : 0.f;
    const float a1 = has1 ? ex2_approx(m1 - Mr) : 0.f;
    const float Lt = a0 * l0 + a1 * l1;
    const float inv = (Lt > 0.f) ? 1.f / Lt : 0.f;
    const float s0 = a0 * inv, s1 = a1 * inv;
    const int g = row - irow * a.G;
#pragma unroll 1
    for (int ch = 0; ch < D / 64; ++ch) {
      const int col = w * (D / 2) + 32 * ch;
      float o[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) o[k] = 0.f;
      if (has0) {
        float x[32];
        tmem_ld32(t_o0 + col, x);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) o[k] = x[k] * s0;
      }
      if (has1) {
        float x[32];
        tmem_ld32(t_o1 + col, x);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) o[k] = fmaf(x[k], s1, o[k]);
      }
      if (my_valid) {
        if (sg.part < 0) {
          __nv_bfloat16* dst = a.out + ((long long)(row0 + irow) * a.Hq + h * a.G + g) * D + col;
          if (a.out_v8) {
#pragma unroll
            for (int k = 0; k < 2; ++k)
              st_global_v8(dst + 16 * k, pack_bf16x2(o[16 * k + 0], o[16 * k + 1]),
                           pack_bf16x2(o[16 * k + 2], o[16 * k + 3]),
                           pack_bf16x2(o[16 * k + 4], o[16 * k + 5]),
                           pack_bf16x2(o[16 * k + 6], o[16 * k + 7]),
                           pack_bf16x2(o[16 * k + 8], o[16 * k + 9]),
                           pack_bf16x2(o[16 * k + 10], o[16 * k + 11]),
                           pack_bf16x2(o[16 * k + 12], o[16 * k + 13]),
                           pack_bf16x2(o[16 * k + 14], o[16 * k + 15]));
          } else {
            uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              d4[k] = make_uint4(pack_bf16x2(o[8 * k + 0], o[8 * k + 1]),
                                 pack_bf16x2(o[8 * k + 2], o[8 * k + 3]),
                                 pack_bf16x2(o[8 * k + 4], o[8 * k + 5]),
                                 pack_bf16x2(o[8 * k + 6], o[8 * k + 7]));
          }
        } else {
          float* dst = a.ws_o + part_o<D>(sg.part, row, col);
#pragma unroll
          for (int k = 0; k < 32; ++k) dst[32 * k] = o[k];
        }
      }
    }
    if (sg.part >= 0 && w == 0 && my_valid)
      a.ws_lse[(long long)sg.part * kTileM + row] = M + log2f(Lt);
    tc_fence_before();
    mbar_arrive(bar(Lay::kBarOFree));
    ++si;
  }
}

// Block writer (write-then-truncate VERIFY: the AR view writes every block
// row's K/V into the cache as it verifies the block, and the commit only moves
// the prefix length; technical summary §2.3 item 3). For each unit of this
// CTA's range whose block tile the CTA owns, block row i of head h goes to the
// cache slot of position L_b + i. These slots lie past every key the call
// reads from the cache (the prefix ends at L_b; a partial last prefix tile
// masks keys at or past L_b and zeroes their V rows), so the copy runs next to
// the pipeline with no ordering against it. A row whose page index or page id
// is out of range is skipped and flagged. No waits.
template <int D, bool kWalk>
__device__ __forceinline__ void block_writer_role(const AttnArgs& a, const SeqTable& tab,
                                                  SegCursor c) {
  constexpr int kChunks = D / 8;  // 16-byte chunks per head row
  constexpr int U = 8;            // chunk pairs in flight per lane
  const int lane = threadIdx.x & 31;
  Segment sg;
  while (cursor_next<kWalk>(a, tab, c, sg)) {
    if (sg.t1 != sg.nt) continue;  // another CTA owns this unit's block tile
    const SeqInfo si = tab.get(a, sg.b);
    const int items = si.Kb * kChunks;
    const int* table = a.page_table + (long long)sg.b * a.max_pages;
    for (int base = lane; base < items; base += 32 * U) {
      uint4 kv[U], vv[U];
      long long dst[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int e = base + 32 * u;
        dst[u] = -1;
        if (e < items) {
          const int i = e / kChunks, ch = e % kChunks;
          const long long pos = (long long)si.L + i;
          const long long pidx = pos / a.page_size;
          int page = -1;
          if (pidx >= a.max_pages) {
            raise_flag(a, ORTHRUS_FLAG_BAD_LENGTH);
          } else {
            page = table[pidx];
            if (page < 0 || page >= a.num_pages) {
              raise_flag(a, ORTHRUS_FLAG_BAD_PAGE);
              page = -1;
            }
          }
          if (page >= 0) {
            const long long src = ((long long)(si.row0 + i) * a.Hkv + sg.h) * kChunks + ch;
            dst[u] = (((long long)page * a.Hkv + sg.h) * a.page_size + pos % a.page_size) *
                         kChunks + ch;
            kv[u] = a.kb_rows[src];
            vv[u] = a.vb_rows[src];
          }
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (dst[u] >= 0) {
          a.kc_rows[dst[u]] = kv[u];
          a.vc_rows[dst[u]] = vv[u];
        }
      }
    }
  }
}

template <int D, bool kWalk>
__global__ void __launch_bounds__(kAttnThreads, 1)
    block_attn_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_kc,
                      const __grid_constant__ CUtensorMap tm_vc,
                      const __grid_constant__ CUtensorMap tm_kb,
                      const __grid_constant__ CUtensorMap tm_vb, const AttnArgs a) {
  using Lay = AttnLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMiscOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kMiscOff + 4);
  const int warp = threadIdx.x >> 5;

  // The combine kernel may be scheduled as soon as every CTA got here; it
  // waits for this grid's writes before it reads them.
  pdl_launch_dependents();

  // A CTA whose range is empty has nothing to set up.
  SeqTable tab;
  SegCursor start;
  if (!schedule_prologue<D, kWalk>(a, smem, tab, start)) return;

  if (threadIdx.x == 0) {
    const uint32_t bars = smem_u32(smem) + Lay::kBarOff;
    for (int s = 0; s < Lay::kNK; ++s) {
      mbar_init(bars + 8u * (Lay::kBarKFull + s), 1);
      mbar_init(bars + 8u * (Lay::kBarKEmpty + s), 1);
    }
    for (int s = 0; s < Lay::kNV; ++s) {
      mbar_init(bars + 8u * (Lay::kBarVFull + s), 1);
      mbar_init(bars + 8u * (Lay::kBarVEmpty + s), 1);
    }
    mbar_init(bars + 8u * Lay::kBarQFull, 1);
    mbar_init(bars + 8u * Lay::kBarQEmpty, 2);  // one arrival per MMA warp
    for (int k = 0; k < 2 * kSPerGroup; ++k) mbar_init(bars + 8u * (Lay::kBarSFull + k), 1);
    for (int w = 0; w < 2; ++w) {
      mbar_init(bars + 8u * (Lay::kBarPReady + 2 * w), 128);
      mbar_init(bars + 8u * (Lay::kBarPReady + 2 * w + 1), 128);
      mbar_init(bars + 8u * (Lay::kBarOReady + w), 1);
    }
    mbar_init(bars + 8u * Lay::kBarOFree, 256);
    mbar_init(bars + 8u * Lay::kBarXchg, 256);
    mbar_init(bars + 8u * Lay::kBarDrain, 1);
    mbar_init(bars + 8u * (Lay::kBarDrain + 1), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kProducerWarp && (threadIdx.x & 31) == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_kc);
    prefetch_tmap(&tm_vc);
    prefetch_tmap(&tm_kb);
    prefetch_tmap(&tm_vb);
    // Start the cold DRAM reads the first copies depend on while the barriers
    // and tensor memory are set up: the page-table line of the first tiles
    // and the first unit's Q tile (into L2; the copies proper follow).
    const SeqInfo sq = tab.get(a, start.b);
    const int tiles_per_page = a.page_size / kTileN;
    if (start.t < (sq.L + kTileN - 1) / kTileN)  // a prefix tile: its page id is in the table
      prefetch_l2(a.page_table + (long long)start.b * a.max_pages + start.t / tiles_per_page);
#pragma unroll
    for (int p = 0; p < Lay::DH; ++p) tma_prefetch_3d(&tm_q, p * 64, start.h * a.G, sq.row0);
  }
  if (warp == kMmaWarp0) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kProducerWarp) {
    if ((threadIdx.x & 31) < 2)
      producer_role<D, kWalk>(a, smem, &tm_q, &tm_kc, &tm_vc, &tm_kb, &tm_vb, abort_flag, tab, start);
  } else if (warp < kSoftmaxWarp0) {
    mma_role<D, kWalk>(a, smem, tmem, abort_flag, warp - kMmaWarp0, tab, start);
  } else if (warp == kWriterWarp) {
    if (a.write_block) {
      // Start the copies once this CTA's first K tile has landed, off the
      // pipeline's cold start (VERIFY minus DIFFUSION time per call: 1.5 us
      // with the copies at kernel start, 0.7 us from here). The wait is
      // bounded like every other; it gives up only if the pipeline stalled.
      mbar_wait(smem_u32(smem) + Lay::kBarOff + 8u * Lay::kBarKFull, 0, abort_flag,
                a.timeout_ns);
      block_writer_role<D, kWalk>(a, tab, start);
    }
  } else {
    softmax_role<D, kWalk>(a, smem, tmem, abort_flag, tab, start);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp0) tmem_dealloc(tmem, kTmemCols);
  if (threadIdx.x == 0 && *abort_flag) raise_flag(a, ORTHRUS_FLAG_TIMEOUT);
}

// ---------------------------------------------------------------------------
// Combine: merge the partials of every unit that was cut across CTAs.
// grid.x: under a chunked schedule one CTA row per (sequence, KV head) unit;
// under balanced ranges one per boundary between attention CTAs x and x + 1
// (only a boundary inside a unit cuts it, and the first boundary inside a
// unit merges it), so no CTA is launched for the many uncut units.
// grid.y: blocks of 32 query rows; grid.z: column groups. 8 warps per CTA,
// lane = query row. A CTA covers D / gridDim.z columns in slices of 16, and
// its warps split over (slice, partial class): warp w takes slice w / wpc and
// the partials k = w % wpc, w % wpc + wpc, ... (wpc warps per slice). Warp 0
// finds the unit and its partials once per CTA, before griddepcontrol.wait,
// so this overlaps the attention grid's tail.
//
// The reads are latency-bound (a few KB per warp), so a warp issues the loads
// of kBatch partials (log-sum-exp and 16 columns each) together, one round
// trip per batch, and keeps its own running (max, sum, accumulator); the warps
// of a slice are then merged in shared memory with the same log-sum-exp
// identity: O = sum_k 2^(lse_k - M) O_k / sum_k 2^(lse_k - M). Chunked
// schedules use batches of 4 (many partials per unit); balanced ranges leave
// two or three partials per cut unit and use batches of 2, which keeps the
// kernel at 64 registers: four CTAs per SM wait at griddepcontrol.wait
// instead of two.

constexpr int kCombineWarps = 8;
constexpr int kCombineThreads = 32 * kCombineWarps;
constexpr int kCombineSlice = 16;  // columns per warp

__device__ __forceinline__ int cta_of_tile(long long T, int C, long long t) {
  long long c = ((t + 1) * C - 1) / T;
  if (c > C - 1) c = C - 1;
  while (c > 0 && range_begin(T, (int)c, C) > t) --c;
  while (c + 1 < C && range_begin(T, (int)c + 1, C) <= t) ++c;
  return (int)c;
}

template <int D, int kBatch>
__global__ void __launch_bounds__(kCombineThreads, kBatch == 2 ? 4 : 1)
    attn_combine_kernel(const AttnArgs a) {
  __shared__ long long sh_T, sh_su;
  __shared__ int sh_b, sh_h, sh_clo, sh_count, sh_skip;
  __shared__ float sh_m[kCombineWarps][32];
  __shared__ float sh_l[kCombineWarps][32];
  __shared__ float sh_acc[kCombineWarps][32][kCombineSlice + 1];
  const int rb = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (a.chunked) {
    // the unit is the CTA row; a unit without rows in this row block has nothing to merge
    const int b = blockIdx.x / a.Hkv;
    const int Kb = (b < a.B) ? seq_block_len(a, b) : 0;
    if (Kb <= 0 || rb * 32 >= a.G * Kb) return;
  }
  if (warp == 0) {
    int skip = 1, count = 0, c_lo = 0, b = 0, h = 0;
    long long T = 0, s_u = 0;
    if (a.chunked == 2) {
      // the attention kernel's allocation: T, U, then the CTAs of sequences < b
      b = blockIdx.x / a.Hkv;
      h = blockIdx.x % a.Hkv;
      const int nt = seq_tiles(a, b);
      long long t_part = 0;
      int u_part = 0;
      for (int bb = lane; bb < a.B; bb += 32) {
        const int n = seq_tiles(a, bb);
        t_part += (long long)a.Hkv * n;
        u_part += n > 0 ? a.Hkv : 0;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        t_part += __shfl_xor_sync(0xffffffffu, t_part, o);
        u_part += __shfl_xor_sync(0xffffffffu, u_part, o);
      }
      long long before = 0;
      for (int bb = lane; bb < b; bb += 32)
        before += (long long)a.Hkv * prop_ctas(t_part, u_part, a.num_ctas, seq_tiles(a, bb));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) before += __shfl_xor_sync(0xffffffffu, before, o);
      count = prop_ctas(t_part, u_part, a.num_ctas, nt);
      c_lo = (int)(before + (long long)h * count);  // first part (= CTA) of this unit
      skip = count <= 1;
    } else if (a.chunked) {
      b = blockIdx.x / a.Hkv;
      h = blockIdx.x % a.Hkv;
      count = unit_chunks(a, seq_tiles(a, b));
      skip = count <= 1;
    } else {
      // total tiles, then the unit holding the boundary tile g (the first
      // tile of attention CTA x + 1), found by a scan over the sequences
      const int C = a.num_ctas, x = blockIdx.x;
      long long t_part = 0;
      for (int bb = lane; bb < a.B; bb += 32) t_part += (long long)a.Hkv * seq_tiles(a, bb);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) t_part += __shfl_xor_sync(0xffffffffu, t_part, o);
      T = t_part;
      const long long g = T > 0 ? range_begin(T, x + 1, C) : 0;
      long long base = 0, s_b = -1;
      int nt = 0;
      for (int b0 = 0; g < T && b0 < a.B; b0 += 32) {
        const int bb = b0 + lane;
        const int n_t = bb < a.B ? seq_tiles(a, bb) : 0;
        const long long n = (long long)a.Hkv * n_t;
        long long incl = n;  // inclusive scan within the warp
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const long long y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const long long excl = base + incl - n;
        const unsigned hit = __ballot_sync(0xffffffffu, n > 0 && excl <= g && g < excl + n);
        if (hit) {
          const int src = __ffs(hit) - 1;
          s_b = __shfl_sync(0xffffffffu, excl, src);
          nt = __shfl_sync(0xffffffffu, n_t, src);
          b = b0 + src;
          break;
        }
        base += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (s_b >= 0) {
        h = (int)((g - s_b) / nt);
        const long long t = g - s_b - (long long)h * nt;
        s_u = s_b + (long long)h * nt;
        c_lo = cta_of_tile(T, C, s_u);
        // a cut (not a unit start), merged by the first boundary inside the unit
        if (t != 0 && c_lo == x) {
          const int c_hi = cta_of_tile(T, C, s_u + nt - 1);
          count = c_hi - c_lo + 1;
          skip = 0;
        }
      }
    }
    if (lane == 0) {
      sh_T = T;
      sh_su = s_u;
      sh_b = b;
      sh_h = h;
      sh_clo = c_lo;
      sh_count = count;
      sh_skip = skip;
    }
  }
  __syncthreads();
  if (sh_skip) return;
  const int b = sh_b, h = sh_h;
  const int Kb = seq_block_len(a, b);
  const int rows_valid = a.G * Kb;
  if (Kb <= 0 || rb * 32 >= rows_valid) return;
  const int row0 = seq_row0(a, b);
  const long long T = sh_T, s_u = sh_su;
  const int c_lo = sh_clo, count = sh_count;
  const int u = b * a.Hkv + h;

  auto part_of = [&](int k, bool& use) -> int {
    if (a.chunked == 2) {
      use = true;
      return c_lo + k;
    }
    if (a.chunked) {
      use = true;
      return u * a.max_chunks + k;
    }
    const int cc = c_lo + k;
    const long long beg = range_begin(T, cc, a.num_ctas);
    use = beg < range_begin(T, cc + 1, a.num_ctas);
    const int slot = (cc == c_lo && s_u > beg) ? 1 : 0;
    return cc * 2 + slot;
  };

  const int cols = D / gridDim.z;           // columns of this CTA
  const int ncs = cols / kCombineSlice;     // slices
  const int wpc = kCombineWarps / ncs;      // warps per slice
  const int sl = warp / wpc, kw = warp % wpc;
  const int c0 = blockIdx.z * cols + sl * kCombineSlice;
  const int r = rb * 32 + lane;  // query row of this lane (rows past rows_valid are ignored)
  const float NEG_INF = -__int_as_float(0x7f800000);

  pdl_wait();  // partials written by the attention grid are visible from here on
  float m_run = NEG_INF, l_run = 0.f;
  float acc[kCombineSlice];
#pragma unroll
  for (int e = 0; e < kCombineSlice; ++e) acc[e] = 0.f;
  for (int k0 = kw; k0 < count; k0 += wpc * kBatch) {
    float lse[kBatch];
    float x[kBatch][kCombineSlice];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int k = k0 + j * wpc;
      bool use = false;
      const int p = k < count ? part_of(k, use) : 0;
      lse[j] = use ? a.ws_lse[(long long)p * kTileM + r] : NEG_INF;
      const float* src = a.ws_o + part_o<D>(use ? p : 0, r, c0);
#pragma unroll
      for (int e = 0; e < kCombineSlice; ++e) x[j][e] = use ? src[32 * e] : 0.f;
    }
    float mb = m_run;
#pragma unroll
    for (int j = 0; j < kBatch; ++j) mb = fmaxf(mb, lse[j]);
    if (mb != NEG_INF) {
      const float sr = exp2f(m_run - mb);  // 0 while nothing is accumulated
      l_run *= sr;
#pragma unroll
      for (int e = 0; e < kCombineSlice; ++e) acc[e] *= sr;
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const float wj = exp2f(lse[j] - mb);
        l_run += wj;
#pragma unroll
        for (int e = 0; e < kCombineSlice; ++e) acc[e] = fmaf(wj, x[j][e], acc[e]);
      }
      m_run = mb;
    }
  }
  sh_m[warp][lane] = m_run;
  sh_l[warp][lane] = l_run;
#pragma unroll
  for (int e = 0; e < kCombineSlice; ++e) sh_acc[warp][lane][e] = acc[e];
  __syncthreads();
  // merge the wpc warps of each slice: thread -> (slice, row, column pair)
  constexpr int kPairs = kCombineSlice / 2;
  for (int idx = tid; idx < ncs * 32 * kPairs; idx += kCombineThreads) {
    const int e = (idx % kPairs) * 2, rr = (idx / kPairs) % 32, s = idx / (32 * kPairs);
    const int q = rb * 32 + rr;
    if (q >= rows_valid) continue;
    float M = NEG_INF;
    for (int k = s * wpc; k < (s + 1) * wpc; ++k) M = fmaxf(M, sh_m[k][rr]);
    float l = 0.f, x0 = 0.f, x1 = 0.f;
    if (M != NEG_INF) {
      for (int k = s * wpc; k < (s + 1) * wpc; ++k) {
        const float w = exp2f(sh_m[k][rr] - M);
        l = fmaf(w, sh_l[k][rr], l);
        x0 = fmaf(w, sh_acc[k][rr][e], x0);
        x1 = fmaf(w, sh_acc[k][rr][e + 1], x1);
      }
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const int i = q / a.G, g = q - i * a.G;
    const int c = blockIdx.z * cols + s * kCombineSlice + e;
    __nv_bfloat16* dst = a.out + ((long long)(row0 + i) * a.Hq + h * a.G + g) * D + c;
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(x0 * inv, x1 * inv);
  }
}

}  // namespace orthrus
