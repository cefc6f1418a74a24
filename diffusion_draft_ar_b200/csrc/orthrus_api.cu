// Host side of the C ABI declared in include/orthrus.h: argument checks (all
// before any CUDA call), TMA descriptor encoding, launch configuration.
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "block_attn.cuh"
#include "consensus.cuh"
#include "kv_append.cuh"
#include "lm_head.cuh"
#include "orthrus.h"

namespace {

using namespace orthrus;

thread_local std::string g_last_error;

orthrus_status_t fail(orthrus_status_t s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

orthrus_status_t ok() {
  g_last_error.clear();
  return ORTHRUS_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// NVTX range named after the C-ABI call, in the "orthrus" domain, around the
// host side of each call (argument checks and launches). NVTX v3 forwards to
// a profiler only when one is attached; otherwise a push/pop is a predicted
// branch on an unset function pointer.
nvtxDomainHandle_t nvtx_domain() {
  static nvtxDomainHandle_t d = nvtxDomainCreateA("orthrus");
  return d;
}

struct NvtxRange {
  explicit NvtxRange(const char* name) {
    nvtxEventAttributes_t ev = {};
    ev.version = NVTX_VERSION;
    ev.size = NVTX_EVENT_ATTRIB_STRUCT_SIZE;
    ev.messageType = NVTX_MESSAGE_TYPE_ASCII;
    ev.message.ascii = name;
    nvtxDomainRangePushEx(nvtx_domain(), &ev);
  }
  ~NvtxRange() { nvtxDomainRangePop(nvtx_domain()); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

constexpr int kMaxDevices = 64;

int device_sm_count(int* sms) {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v <= 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      return -1;
    cache[dev].store(v, std::memory_order_relaxed);
  }
  *sms = v;
  return dev;
}

// Failure-detection test hook. ORTHRUS_FAULT_INJECT=n, read once per process,
// makes the first n attention or LM-head launches of the process withhold one
// copy per CTA, so that a bounded pipeline wait runs out; every later launch
// is normal. Only a test's child process sets it. A process without it pays
// one load of a cached counter per launch and no getenv.
std::atomic<int>& fault_inject_budget() {
  static std::atomic<int> v([] {
    const char* e = std::getenv("ORTHRUS_FAULT_INJECT");
    const int n = e ? std::atoi(e) : 0;
    return n > 0 ? n : 0;
  }());
  return v;
}

int fault_inject_mode() {
  std::atomic<int>& b = fault_inject_budget();
  int n = b.load(std::memory_order_relaxed);
  while (n > 0) {
    if (b.compare_exchange_weak(n, n - 1, std::memory_order_relaxed)) return 1;
  }
  return 0;
}

unsigned long long wait_timeout_ns() {
  static const unsigned long long v = [] {
    const char* e = std::getenv("ORTHRUS_WAIT_TIMEOUT_MS");
    long long ms = e ? std::atoll(e) : 1000;
    if (ms < 1) ms = 1;
    return static_cast<unsigned long long>(ms) * 1000000ull;
  }();
  return v;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point, so the
// library links no driver library and loads on machines without a GPU.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 tensor map with 128-byte swizzle; dims/strides innermost first, strides
// in bytes for dims 1..rank-1.
bool make_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
              const cuuint64_t* strides, const cuuint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides,
            box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct AttnPlan {
  int G, R_max, grid, chunked, chunk_tiles, max_chunks, parts;
  bool combine;  // units may be cut across CTAs: launch the combine kernel
  size_t ws_o_bytes, ws_lse_bytes, ws_bytes;
};

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Host checks shared by the workspace query and the launch. No CUDA call
// except the SM-count query (skipped when `sms` is given).
orthrus_status_t plan_attn(const orthrus_attn_params* p, int sms, AttnPlan* pl) {
  if (!p) return fail(ORTHRUS_ERR_INVALID_ARG, "params is NULL");
  if (p->view != ORTHRUS_VIEW_DIFFUSION && p->view != ORTHRUS_VIEW_VERIFY)
    return fail(ORTHRUS_ERR_INVALID_ARG, "unknown view %d", p->view);
  if (p->B < 0) return fail(ORTHRUS_ERR_INVALID_ARG, "B = %d < 0", p->B);
  if (p->Hq < 1 || p->Hkv < 1 || p->Hq % p->Hkv)
    return fail(ORTHRUS_ERR_INVALID_ARG, "heads Hq = %d, Hkv = %d", p->Hq, p->Hkv);
  if (p->max_block < 1) return fail(ORTHRUS_ERR_INVALID_ARG, "max_block = %d", p->max_block);
  if (p->page_size < 1 || p->max_pages_per_seq < 0 || p->num_pages < 0)
    return fail(ORTHRUS_ERR_INVALID_ARG, "page geometry");
  if (p->kv_split_tokens < 0 || p->max_ctas < 0)
    return fail(ORTHRUS_ERR_INVALID_ARG, "kv_split_tokens / max_ctas negative");
  if (p->D != 64 && p->D != 128) return fail(ORTHRUS_ERR_UNSUPPORTED, "D = %d (64 or 128)", p->D);
  if (p->page_size % kTileN)
    return fail(ORTHRUS_ERR_UNSUPPORTED, "page_size = %d (a multiple of 64)", p->page_size);
  const int G = p->Hq / p->Hkv;
  if (p->max_block > kTileN || G * p->max_block > kTileM)
    return fail(ORTHRUS_ERR_UNSUPPORTED, "max_block = %d, G = %d (need K <= 64, G*K <= 128)",
                p->max_block, G);
  if (p->kv_split_tokens % kTileN)
    return fail(ORTHRUS_ERR_UNSUPPORTED, "kv_split_tokens = %d (a multiple of 64)",
                p->kv_split_tokens);
  if (static_cast<long long>(p->num_pages) * p->Hkv * p->page_size >= (1ll << 31))
    return fail(ORTHRUS_ERR_UNSUPPORTED, "cache rows exceed 2^31");
  if (static_cast<long long>(p->B) * p->max_block >= (1ll << 31) / p->Hq)
    return fail(ORTHRUS_ERR_UNSUPPORTED, "too many block rows");
  if (p->total_rows < 0) return fail(ORTHRUS_ERR_INVALID_ARG, "total_rows = %d", p->total_rows);
  pl->G = G;
  pl->R_max = p->total_rows > 0 ? p->total_rows : p->B * p->max_block;
  if (!p->cu_block && pl->R_max < p->B * p->max_block)
    return fail(ORTHRUS_ERR_INVALID_ARG, "total_rows %d < B * max_block without cu_block",
                pl->R_max);
  const long long max_tokens = static_cast<long long>(p->max_pages_per_seq) * p->page_size;
  if (p->kv_split_tokens > 0) {
    // Fixed chunks: one partial slot per (unit, chunk). The grid is at most
    // one CTA per SM (or max_ctas), each walking the slots c, c + grid, ...,
    // so the chunks beyond the first wave run in CTAs already set up instead
    // of in a tail of short-lived CTAs.
    pl->chunked = 1;
    pl->chunk_tiles = p->kv_split_tokens / kTileN;
    const long long ptiles = (max_tokens + kTileN - 1) / kTileN;
    long long mc = (ptiles + pl->chunk_tiles - 1) / pl->chunk_tiles;
    if (mc < 1) mc = 1;
    const long long slots = mc * p->Hkv * static_cast<long long>(p->B);
    if (slots >= (1ll << 31) - (1ll << 16)) return fail(ORTHRUS_ERR_UNSUPPORTED, "too many chunks");
    pl->max_chunks = static_cast<int>(mc);
    // With max_ctas = 0 the slots are spread evenly over as few CTAs as give
    // the same number of slots per CTA as one per SM would (520 slots on 148
    // SMs: 4 each over 130 CTAs rather than 3 or 4 over 148).
    long long cap = p->max_ctas > 0 ? p->max_ctas : std::max(sms, 1);
    if (p->max_ctas == 0 && slots > cap) {
      const long long per = (slots + cap - 1) / cap;
      cap = (slots + per - 1) / per;
    }
    cap = std::min(cap, 65535LL);  // the walkers' stride: j + grid stays below 2^31
    pl->grid = static_cast<int>(std::min(slots, cap));
    pl->parts = static_cast<int>(slots);
    pl->combine = true;
  } else if (p->max_ctas == 0 && static_cast<long long>(p->B) * p->Hkv >= (3LL * sms) / 4 &&
             static_cast<long long>(p->B) * p->Hkv <= sms) {
    // When the (sequence, KV head) units number between 3/4 of the SMs and
    // the SM count, one CTA per whole unit leaves a few SMs idle but cuts no
    // unit: no partials, no combine launch, and no unit switch inside a CTA
    // (each switch drains the pipeline while the next unit's Q tile loads).
    // This is the fixed-chunk schedule with one chunk per unit. A batch whose
    // prefix lengths differ widely is better served by max_ctas = SM count.
    const long long ptiles = (max_tokens + kTileN - 1) / kTileN;
    pl->chunked = 1;
    pl->chunk_tiles = static_cast<int>(ptiles > 0 ? ptiles : 1);
    pl->max_chunks = 1;
    pl->grid = p->B * p->Hkv;
    pl->parts = pl->grid;
    pl->combine = false;
  } else if (p->max_ctas == 0 && static_cast<long long>(p->B) * p->Hkv < (3LL * sms) / 4) {
    // Few units (long contexts): every unit gets a share of the SMs in
    // proportion to its tiles, cut into near-equal chunks on the device from
    // the actual lengths. No CTA switches units, which the balanced ranges
    // below do whenever a range boundary falls inside a unit.
    // A chunk is at least kMinChunkTiles tiles (a split pays a partial and
    // the combine); when no unit can be that long, each stays whole in one CTA
    // and the combine kernel is not launched.
    const long long max_nt = (max_tokens + kTileN - 1) / kTileN + 1;
    const bool whole = max_nt / kMinChunkTiles <= 1;
    pl->chunked = 2;
    pl->chunk_tiles = 0;
    pl->max_chunks = 0;
    pl->grid = whole ? p->B * p->Hkv : std::max(sms, 1);
    pl->parts = pl->grid;
    pl->combine = !whole;
  } else {
    pl->chunked = 0;
    pl->chunk_tiles = 0;
    pl->max_chunks = 0;
    // Balanced ranges over one CTA per SM (or max_ctas).
    int c = p->max_ctas > 0 ? p->max_ctas : sms;
    if (c < 1) c = 1;
    if (c > 65535) c = 65535;
    pl->grid = c;
    pl->parts = 2 * c;
    pl->combine = true;
  }
  pl->ws_o_bytes = round_up(static_cast<size_t>(pl->parts) * kTileM * p->D * sizeof(float), 256);
  pl->ws_lse_bytes = round_up(static_cast<size_t>(pl->parts) * kTileM * sizeof(float), 256);
  pl->ws_bytes = pl->ws_o_bytes + pl->ws_lse_bytes;
  return ORTHRUS_OK;
}

template <int D>
orthrus_status_t launch_attn(const orthrus_attn_params* p, const AttnPlan& pl, int dev,
                             cudaStream_t stream, bool write_block) {
  using Lay = AttnLayout<D>;
  static std::atomic<int> smem_set[kMaxDevices];
  if (!smem_set[dev].load()) {
    cudaError_t e = cudaFuncSetAttribute(block_attn_kernel<D, false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kAlloc);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(block_attn_kernel<D, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kAlloc);
    if (e != cudaSuccess)
      return fail(ORTHRUS_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    smem_set[dev].store(1);
  }
  const int R = pl.R_max;  // rows the caller's block buffers hold
  CUtensorMap tq, tkc, tvc, tkb, tvb;
  {
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)p->Hq, (cuuint64_t)R};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)p->Hq * D * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)pl.G, (cuuint32_t)std::min(p->max_block, R)};
    if (!make_map(&tq, p->q_block, 3, dims, strides, box))
      return fail(ORTHRUS_ERR_CUDA, "tensor map for q_block");
  }
  {
    // cache rows (one token of one head) viewed as (64 columns, row, D/64 halves):
    // one box of {64, 64, D/64} lands as D/64 panels of 64 rows x 128 bytes
    const cuuint64_t rows = (cuuint64_t)p->num_pages * p->Hkv * p->page_size;
    const cuuint64_t dims[3] = {64, rows > 0 ? rows : 1, (cuuint64_t)D / 64};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, 128};
    const cuuint32_t box[3] = {64, (cuuint32_t)kTileN, (cuuint32_t)D / 64};
    if (!make_map(&tkc, p->k_cache, 3, dims, strides, box) ||
        !make_map(&tvc, p->v_cache, 3, dims, strides, box))
      return fail(ORTHRUS_ERR_CUDA, "tensor map for the KV cache");
  }
  {
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)p->Hkv, (cuuint64_t)R};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)p->Hkv * D * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)std::min(kTileN, R)};
    if (!make_map(&tkb, p->k_block, 3, dims, strides, box) ||
        !make_map(&tvb, p->v_block, 3, dims, strides, box))
      return fail(ORTHRUS_ERR_CUDA, "tensor map for the block K/V");
  }
  AttnArgs a;
  a.view = p->view;
  a.B = p->B;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.G = pl.G;
  a.page_size = p->page_size;
  a.max_pages = p->max_pages_per_seq;
  a.num_pages = p->num_pages;
  a.max_block = p->max_block;
  a.total_rows = pl.R_max;
  a.prefix_lens = p->prefix_lens;
  a.cu_block = p->cu_block;
  a.page_table = p->page_table;
  a.out = static_cast<__nv_bfloat16*>(p->out);
  a.ws_o = static_cast<float*>(p->workspace);
  a.ws_lse = reinterpret_cast<float*>(static_cast<char*>(p->workspace) + pl.ws_o_bytes);
  a.error_flag = p->error_flag;
  const float scale = p->softmax_scale > 0.f ? p->softmax_scale : 1.f / std::sqrt((float)D);
  a.scale_log2 = scale * 1.4426950408889634f;
  a.q_box_rows = std::min(p->max_block, R);
  a.blk_box_rows = std::min(kTileN, R);
  a.chunked = pl.chunked;
  a.chunk_tiles = pl.chunk_tiles;
  a.max_chunks = pl.max_chunks;
  a.num_ctas = pl.grid;
  a.timeout_ns = wait_timeout_ns();
  a.fault_inject = fault_inject_mode();
  a.out_v8 = aligned(p->out, 32) ? 1 : 0;
  a.write_block = write_block ? 1 : 0;
  a.kb_rows = static_cast<const uint4*>(p->k_block);
  a.vb_rows = static_cast<const uint4*>(p->v_block);
  // The write-then-truncate entry point documents that the cache is written.
  a.kc_rows = static_cast<uint4*>(const_cast<void*>(p->k_cache));
  a.vc_rows = static_cast<uint4*>(const_cast<void*>(p->v_cache));

  // Fixed-chunk CTAs that walk several slots run the walking variant; every
  // other schedule (one slot per CTA included) runs the variant without it.
  const bool walk = pl.chunked == 1 && pl.grid < pl.parts;
  if (walk)
    block_attn_kernel<D, true><<<pl.grid, kAttnThreads, Lay::kAlloc, stream>>>(tq, tkc, tvc, tkb,
                                                                              tvb, a);
  else
    block_attn_kernel<D, false><<<pl.grid, kAttnThreads, Lay::kAlloc, stream>>>(tq, tkc, tvc, tkb,
                                                                               tvb, a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(ORTHRUS_ERR_CUDA, "block_attn launch: %s", cudaGetErrorString(e));
  if (!pl.combine) return ok();
  // The combine kernel is launched as a programmatic dependent of the
  // attention grid: its launch and schedule prologue overlap the attention
  // tail, and it reads the partials only after griddepcontrol.wait.
  const int row_blocks = (pl.G * p->max_block + 31) / 32;
  cudaLaunchConfig_t cfg = {};
  // Chunked schedules: one CTA row per unit and one CTA per 16 columns of a
  // row block (many partials per unit). Balanced ranges: one CTA row per
  // boundary between attention CTAs (two or three partials per cut unit),
  // one CTA per row block, its warps on different columns.
  const bool chunked = pl.chunked != 0;
  cfg.gridDim = chunked ? dim3(p->B * p->Hkv, row_blocks, D / kCombineSlice)
                        : dim3(std::max(pl.grid - 1, 1), row_blocks, 1);
  cfg.blockDim = dim3(kCombineThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = chunked ? cudaLaunchKernelEx(&cfg, attn_combine_kernel<D, 4>, a)
              : cudaLaunchKernelEx(&cfg, attn_combine_kernel<D, 2>, a);
  if (e != cudaSuccess) return fail(ORTHRUS_ERR_CUDA, "combine launch: %s", cudaGetErrorString(e));
  return ok();
}

}  // namespace

extern "C" {

size_t orthrus_block_attn_workspace_size(const orthrus_attn_params* p) {
  int sms = 0;
  if (!p) return 0;
  if (p->kv_split_tokens == 0 && p->max_ctas == 0 && device_sm_count(&sms) < 0) return 0;
  AttnPlan pl;
  if (plan_attn(p, sms, &pl) != ORTHRUS_OK) return 0;
  return pl.ws_bytes;
}

int32_t orthrus_block_attn_kernel_count(const orthrus_attn_params* p) {
  int sms = 0;
  if (!p) return 0;
  if (p->kv_split_tokens == 0 && p->max_ctas == 0 && device_sm_count(&sms) < 0) return 0;
  AttnPlan pl;
  if (plan_attn(p, sms, &pl) != ORTHRUS_OK) return 0;
  return pl.combine ? 2 : 1;
}

orthrus_status_t orthrus_block_attn_plan(const orthrus_attn_params* p, int32_t sm_count,
                                         orthrus_attn_plan* plan) {
  if (!plan) return fail(ORTHRUS_ERR_INVALID_ARG, "plan is NULL");
  int sms = sm_count;
  if (sms <= 0 && device_sm_count(&sms) < 0) return fail(ORTHRUS_ERR_CUDA, "no current CUDA device");
  AttnPlan pl;
  const orthrus_status_t s = plan_attn(p, sms, &pl);
  if (s != ORTHRUS_OK) return s;
  plan->schedule = pl.chunked == 2   ? ORTHRUS_SCHEDULE_PROPORTIONAL
                   : pl.chunked == 1 ? ORTHRUS_SCHEDULE_FIXED_CHUNKS
                                     : ORTHRUS_SCHEDULE_BALANCED;
  plan->grid = pl.grid;
  plan->partial_slots = pl.parts;
  plan->kernels = pl.combine ? 2 : 1;
  plan->walks_chunks = (pl.chunked == 1 && pl.grid < pl.parts) ? 1 : 0;  // as launch_attn
  plan->chunk_tiles = pl.chunked == 1 ? pl.chunk_tiles : 0;
  plan->workspace_bytes = pl.ws_bytes;
  return ok();
}

static orthrus_status_t block_attn_entry(const orthrus_attn_params* p, void* stream, bool write_block) {
  AttnPlan pl;
  orthrus_status_t s = plan_attn(p, 1, &pl);  // geometry checks first, no CUDA call
  if (s != ORTHRUS_OK) return s;
  if (p->B == 0) return ok();
  const void* ptrs[] = {p->q_block, p->k_cache, p->v_cache, p->k_block,
                        p->v_block, p->out,     p->workspace};
  const char* names[] = {"q_block", "k_cache", "v_cache", "k_block", "v_block", "out", "workspace"};
  for (int i = 0; i < 7; ++i) {
    if (!ptrs[i]) return fail(ORTHRUS_ERR_INVALID_ARG, "%s is NULL", names[i]);
    if (!aligned(ptrs[i], 16)) return fail(ORTHRUS_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
  }
  if (!p->prefix_lens || !p->page_table)
    return fail(ORTHRUS_ERR_INVALID_ARG, "prefix_lens / page_table is NULL");
  if (p->max_pages_per_seq < 1 || p->num_pages < 1)
    return fail(ORTHRUS_ERR_INVALID_ARG, "empty page table or cache");
  int sms = 0;
  int dev = 0;
  if (p->max_ctas == 0) {
    dev = device_sm_count(&sms);
    if (dev < 0) return fail(ORTHRUS_ERR_CUDA, "no current CUDA device");
  } else {
    if (cudaGetDevice(&dev) != cudaSuccess || dev >= kMaxDevices)
      return fail(ORTHRUS_ERR_CUDA, "no current CUDA device");
    sms = 1;
  }
  s = plan_attn(p, sms, &pl);
  if (s != ORTHRUS_OK) return s;
  if (p->workspace_bytes < pl.ws_bytes)
    return fail(ORTHRUS_ERR_INVALID_ARG, "workspace %zu bytes < %zu needed", p->workspace_bytes,
                pl.ws_bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return p->D == 128 ? launch_attn<128>(p, pl, dev, st, write_block)
                     : launch_attn<64>(p, pl, dev, st, write_block);
}

orthrus_status_t orthrus_block_attn(const orthrus_attn_params* p, void* stream) {
  NvtxRange r("orthrus_block_attn");
  return block_attn_entry(p, stream, false);
}

orthrus_status_t orthrus_block_attn_verify_write(const orthrus_attn_params* p, void* stream) {
  NvtxRange r("orthrus_block_attn_verify_write");
  if (p && p->view != ORTHRUS_VIEW_VERIFY)
    return fail(ORTHRUS_ERR_INVALID_ARG, "write-then-truncate needs the VERIFY view");
  return block_attn_entry(p, stream, true);
}

size_t orthrus_consensus_workspace_size(int32_t B, int32_t max_block, int32_t V) {
  if (B < 0 || max_block < 1 || V < 1) return 0;
  const long long chunks = (V + kConsChunk - 1) / kConsChunk;
  return static_cast<size_t>(B) * max_block * chunks * sizeof(unsigned long long);
}

static orthrus_status_t consensus_entry(const float* verify_logits, int64_t ld, int32_t V,
                                        const int32_t* draft_tokens, const int32_t* cu_block,
                                        int32_t B, int32_t max_block, int32_t* accept_len,
                                        int32_t* next_token, int32_t* row_argmax,
                                        int32_t* prefix_lens, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  if (B < 0) return fail(ORTHRUS_ERR_INVALID_ARG, "B = %d < 0", B);
  if (V < 1 || ld < V) return fail(ORTHRUS_ERR_INVALID_ARG, "V = %d, ld = %lld", V, (long long)ld);
  if (max_block < 1) return fail(ORTHRUS_ERR_INVALID_ARG, "max_block = %d", max_block);
  if (B == 0) return ok();
  if (!verify_logits || !draft_tokens || !accept_len || !next_token || !workspace)
    return fail(ORTHRUS_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned(verify_logits, 4) || !aligned(workspace, 16))
    return fail(ORTHRUS_ERR_INVALID_ARG, "misaligned logits or workspace");
  const long long R_max = static_cast<long long>(B) * max_block;
  if (R_max >= (1ll << 31)) return fail(ORTHRUS_ERR_UNSUPPORTED, "too many rows");
  const size_t need = orthrus_consensus_workspace_size(B, max_block, V);
  if (workspace_bytes < need)
    return fail(ORTHRUS_ERR_INVALID_ARG, "workspace %zu bytes < %zu needed", workspace_bytes, need);
  const int n_chunks = (V + kConsChunk - 1) / kConsChunk;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto* part = static_cast<unsigned long long*>(workspace);
  dim3 grid(n_chunks, static_cast<unsigned>(R_max));
  if (R_max > 65535) return fail(ORTHRUS_ERR_UNSUPPORTED, "more than 65535 rows");
  consensus_argmax_kernel<<<grid, kConsThreads, 0, st>>>(verify_logits, ld, V, cu_block, B,
                                                          max_block, n_chunks, part);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(ORTHRUS_ERR_CUDA, "consensus launch: %s", cudaGetErrorString(e));
  // finalize is a programmatic dependent of the argmax pass: its launch
  // overlaps the argmax tail and it reads the keys after griddepcontrol.wait
  const int warps = 8;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((B + warps - 1) / warps);
  cfg.blockDim = dim3(warps * 32);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, consensus_finalize_kernel, static_cast<const unsigned long long*>(part),
                         n_chunks, draft_tokens, cu_block, static_cast<int>(B),
                         static_cast<int>(max_block), accept_len, next_token, row_argmax,
                         prefix_lens, static_cast<int>(R_max));
  if (e != cudaSuccess) return fail(ORTHRUS_ERR_CUDA, "consensus launch: %s", cudaGetErrorString(e));
  return ok();
}

orthrus_status_t orthrus_consensus(const float* verify_logits, int64_t ld, int32_t V,
                                   const int32_t* draft_tokens, const int32_t* cu_block,
                                   int32_t B, int32_t max_block, int32_t* accept_len,
                                   int32_t* next_token, int32_t* row_argmax, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  NvtxRange r("orthrus_consensus");
  return consensus_entry(verify_logits, ld, V, draft_tokens, cu_block, B, max_block, accept_len,
                         next_token, row_argmax, nullptr, workspace, workspace_bytes, stream);
}

orthrus_status_t orthrus_consensus_commit(const float* verify_logits, int64_t ld, int32_t V,
                                          const int32_t* draft_tokens, const int32_t* cu_block,
                                          int32_t B, int32_t max_block, int32_t* accept_len,
                                          int32_t* next_token, int32_t* row_argmax,
                                          int32_t* prefix_lens, void* workspace,
                                          size_t workspace_bytes, void* stream) {
  NvtxRange r("orthrus_consensus_commit");
  if (B > 0 && !prefix_lens) return fail(ORTHRUS_ERR_INVALID_ARG, "prefix_lens is NULL");
  return consensus_entry(verify_logits, ld, V, draft_tokens, cu_block, B, max_block, accept_len,
                         next_token, row_argmax, prefix_lens, workspace, workspace_bytes, stream);
}

orthrus_status_t orthrus_consensus_sampled(const float* verify_logits, int64_t ld, int32_t V,
                                           const int32_t* draft_tokens, const int32_t* cu_block,
                                           int32_t B, int32_t max_block, float temperature,
                                           uint64_t seed, uint64_t offset, int32_t* accept_len,
                                           int32_t* next_token, int32_t* row_token,
                                           int32_t* prefix_lens, void* workspace,
                                           size_t workspace_bytes, void* stream) {
  NvtxRange r("orthrus_consensus_sampled");
  if (!(temperature > 0.f) || !std::isfinite(temperature))
    return fail(ORTHRUS_ERR_INVALID_ARG, "temperature = %g (must be finite and > 0)",
                static_cast<double>(temperature));
  // base-2 scores: logits scaled by log2(e) / T (see noise_log2)
  const float x_scale = static_cast<float>(1.4426950408889634 / static_cast<double>(temperature));
  if (!std::isfinite(x_scale))
    return fail(ORTHRUS_ERR_UNSUPPORTED, "temperature = %g is too small for fp32 scores",
                static_cast<double>(temperature));
  if (B < 0) return fail(ORTHRUS_ERR_INVALID_ARG, "B = %d < 0", B);
  if (V < 1 || ld < V) return fail(ORTHRUS_ERR_INVALID_ARG, "V = %d, ld = %lld", V, (long long)ld);
  if (max_block < 1) return fail(ORTHRUS_ERR_INVALID_ARG, "max_block = %d", max_block);
  if (B == 0) return ok();
  if (!verify_logits || !draft_tokens || !accept_len || !next_token || !workspace)
    return fail(ORTHRUS_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned(verify_logits, 4) || !aligned(workspace, 16))
    return fail(ORTHRUS_ERR_INVALID_ARG, "misaligned logits or workspace");
  const long long R_max = static_cast<long long>(B) * max_block;
  if (R_max > 65535) return fail(ORTHRUS_ERR_UNSUPPORTED, "more than 65535 rows");
  const size_t need = orthrus_consensus_workspace_size(B, max_block, V);
  if (workspace_bytes < need)
    return fail(ORTHRUS_ERR_INVALID_ARG, "workspace %zu bytes < %zu needed", workspace_bytes, need);
  const int n_chunks = (V + kConsChunk - 1) / kConsChunk;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto* part = static_cast<unsigned long long*>(workspace);
  dim3 grid(n_chunks, static_cast<unsigned>(R_max));
  consensus_sample_kernel<<<grid, kConsThreads, 0, st>>>(
      verify_logits, ld, V, cu_block, B, max_block, n_chunks, part, x_scale,
      static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32),
      static_cast<uint32_t>(offset), static_cast<uint32_t>(offset >> 32));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(ORTHRUS_ERR_CUDA, "consensus launch: %s", cudaGetErrorString(e));
  const int warps = 8;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((B + warps - 1) / warps);
  cfg.blockDim = dim3(warps * 32);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, consensus_finalize_kernel, static_cast<const unsigned long long*>(part),
                         n_chunks, draft_tokens, cu_block, static_cast<int>(B),
                         static_cast<int>(max_block), accept_len, next_token, row_token,
                         prefix_lens, static_cast<int>(R_max));
  if (e != cudaSuccess) return fail(ORTHRUS_ERR_CUDA, "consensus launch: %s", cudaGetErrorString(e));
  return ok();
}

orthrus_status_t orthrus_kv_append(const void* k_block, const void* v_block,
                                   const int32_t* cu_block, int32_t max_block,
                                   const int32_t* accept_len, int32_t* prefix_lens,
                                   int32_t update_lens, const int32_t* page_table,
                                   int32_t max_pages_per_seq, int32_t num_pages, void* k_cache,
                                   void* v_cache, int32_t B, int32_t Hkv, int32_t D,
                                   int32_t page_size, int32_t* error_flag, void* stream) {
  NvtxRange r("orthrus_kv_append");
  if (B < 0 || Hkv < 1 || D < 8 || D % 8 || page_size < 1 || max_pages_per_seq < 0 ||
      num_pages < 0 || (!cu_block && max_block < 1))
    return fail(ORTHRUS_ERR_INVALID_ARG, "bad sizes (B %d, Hkv %d, D %d, P %d)", B, Hkv, D,
                page_size);
  if (B == 0) return ok();
  if (!k_block || !v_block || !accept_len || !prefix_lens || !page_table || !k_cache || !v_cache)
    return fail(ORTHRUS_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned(k_block, 16) || !aligned(v_block, 16) || !aligned(k_cache, 16) ||
      !aligned(v_cache, 16))
    return fail(ORTHRUS_ERR_INVALID_ARG, "K/V pointers must be 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  kv_append_kernel<<<B, kAppendThreads, 0, st>>>(
      static_cast<const uint4*>(k_block), static_cast<const uint4*>(v_block), cu_block, max_block,
      accept_len, prefix_lens, update_lens, page_table, max_pages_per_seq, num_pages,
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), Hkv, D, page_size, error_flag);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(ORTHRUS_ERR_CUDA, "kv_append launch: %s", cudaGetErrorString(e));
  return ok();
}

// ---------------------------------------------------------------------------
// Consensus for callers that cannot allocate device memory at call time (an
// engine that pre-reserves all of HBM and hands plug-ins no scratch, or a
// decode path that must not pay cudaMalloc's implicit synchronisation). The
// partial keys live in this fixed array instead of a caller workspace.

constexpr long long kNoAllocScratchKeys = 65536;  // 512 KiB of 64-bit keys

static __device__ __align__(256) unsigned long long g_consensus_scratch[kNoAllocScratchKeys];

}  // extern "C"

namespace {

// Device address of g_consensus_scratch in the current device's context. In
// host code the array's name is only a host-side stand-in, so the address is
// looked up with that device current. It is looked up on every call (a symbol
// lookup in the loaded module, no allocation): a cached address would go
// stale if the context were reset and the module loaded again elsewhere.
unsigned long long* noalloc_scratch() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_consensus_scratch) != cudaSuccess || !p) return nullptr;
  return static_cast<unsigned long long*>(p);
}

}  // namespace

extern "C" {

orthrus_status_t orthrus_consensus_noalloc(const float* verify_logits, int64_t ld, int32_t V,
                                           const int32_t* draft_tokens, const int32_t* cu_block,
                                           int32_t B, int32_t max_block, int32_t* accept_len,
                                           int32_t* next_token, int32_t* row_argmax,
                                           void* stream) {
  NvtxRange r("orthrus_consensus_noalloc");
  if (B < 0) return fail(ORTHRUS_ERR_INVALID_ARG, "B = %d < 0", B);
  if (V < 1 || ld < V) return fail(ORTHRUS_ERR_INVALID_ARG, "V = %d, ld = %lld", V, (long long)ld);
  if (max_block < 1) return fail(ORTHRUS_ERR_INVALID_ARG, "max_block = %d", max_block);
  if (B == 0) return ok();
  if (!verify_logits || !draft_tokens || !accept_len || !next_token)
    return fail(ORTHRUS_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned(verify_logits, 4)) return fail(ORTHRUS_ERR_INVALID_ARG, "misaligned logits");
  const long long n_chunks = (V + kConsChunk - 1) / kConsChunk;
  const long long R_max = static_cast<long long>(B) * max_block;
  if (R_max > 65535) return fail(ORTHRUS_ERR_UNSUPPORTED, "more than 65535 rows");
  const long long keys = R_max * n_chunks;
  if (keys > kNoAllocScratchKeys)
    return fail(ORTHRUS_ERR_UNSUPPORTED,
                "request needs %lld scratch keys (B*max_block*ceil(V/16384)); the built-in "
                "array holds %lld",
                keys, kNoAllocScratchKeys);
  unsigned long long* part = noalloc_scratch();
  if (!part) return fail(ORTHRUS_ERR_CUDA, "cannot resolve the scratch array's device address");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  dim3 grid(static_cast<unsigned>(n_chunks), static_cast<unsigned>(R_max));
  consensus_argmax_kernel<<<grid, kConsThreads, 0, st>>>(verify_logits, ld, V, cu_block, B,
                                                          max_block, static_cast<int>(n_chunks),
                                                          part);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(ORTHRUS_ERR_CUDA, "consensus launch: %s", cudaGetErrorString(e));
  const int warps = 8;
  consensus_finalize_kernel<<<(B + warps - 1) / warps, warps * 32, 0, st>>>(
      part, static_cast<int>(n_chunks), draft_tokens, cu_block, B, max_block, accept_len,
      next_token, row_argmax, nullptr, B * max_block);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail(ORTHRUS_ERR_CUDA, "consensus launch: %s", cudaGetErrorString(e));
  return ok();
}

const char* orthrus_status_string(orthrus_status_t s) {
  switch (s) {
    case ORTHRUS_OK: return "ok";
    case ORTHRUS_ERR_INVALID_ARG: return "invalid argument";
    case ORTHRUS_ERR_UNSUPPORTED: return "unsupported configuration";
    case ORTHRUS_ERR_CUDA: return "CUDA error";
    case ORTHRUS_ERR_TIMEOUT: return "device wait timed out";
    case ORTHRUS_ERR_DEVICE_CHECK: return "device-side check failed";
  }
  return "unknown status";
}

const char* orthrus_last_error(void) { return g_last_error.c_str(); }

orthrus_status_t orthrus_status_from_flags(int32_t flags) {
  if (flags == 0) return ORTHRUS_OK;
  if (flags & ORTHRUS_FLAG_TIMEOUT) return ORTHRUS_ERR_TIMEOUT;
  return ORTHRUS_ERR_DEVICE_CHECK;
}

int32_t orthrus_abi_version(void) { return ORTHRUS_ABI_VERSION; }

}  // extern "C"

// ---------------------------------------------------------------------------
// LM head + greedy token

namespace {

struct LmPlan {
  int R, mt, N, n_m, n_n, n_tiles, stages, grid, box_a, box_b;
  uint32_t stage_bytes, a_bytes;
  size_t smem;
};

// Tile shape: with more than 128 rows two M=128 blocks share each w_head tile
// (half the w_head reads per FLOP) and N = 192, the widest tile whose stage
// (32 KB of hidden rows + N x 128 B of w_head) still fits four ring stages.
// Measured on the Qwen3-8B head (512 x 4096 x 151936): 449 us at N = 192
// (4 stages), 460 at 176, 463 at 256 and 466 at 208 (3 stages), 480 at 192
// held to 3 stages. With at most 128 rows the head is memory-bound (one block
// per tile, the accumulator double buffered): a tile's time follows its w_head
// bytes, so N (a multiple of 32 in [128, 256], the two epilogue groups taking
// half each) minimises waves x N; at V = 151936 that is 224 (679 tiles, 4.6
// waves) rather than 256 (594 tiles: 4 full waves and 2 tiles).
orthrus_status_t plan_lm(int R, int d, int V, int sms, LmPlan* pl) {
  if (R < 1 || d < 1 || V < 1) return fail(ORTHRUS_ERR_INVALID_ARG, "R %d, d %d, V %d", R, d, V);
  if (d % kLmKStep)
    return fail(ORTHRUS_ERR_UNSUPPORTED, "d_model = %d (a multiple of 64)", d);
  pl->R = R;
  pl->mt = R > 128 ? 2 : 1;
  if (pl->mt == 1) {
    pl->N = std::min(256, (V + 63) / 64 * 64);
    if (V > 256) {
      long long best = -1;
      for (int N = 256; N >= 128; N -= 32) {
        const long long waves = ((V + N - 1) / N + sms - 1) / sms;
        if (best < 0 || waves * N < best) {
          best = waves * N;
          pl->N = N;
        }
      }
    }
  } else {
    pl->N = std::min(192, (V + 15) / 16 * 16);
  }
  pl->n_m = (R + 128 * pl->mt - 1) / (128 * pl->mt);
  pl->n_n = (V + pl->N - 1) / pl->N;
  const long long tiles = static_cast<long long>(pl->n_m) * pl->n_n;
  if (tiles >= (1ll << 31)) return fail(ORTHRUS_ERR_UNSUPPORTED, "too many tiles");
  pl->n_tiles = static_cast<int>(tiles);
  pl->a_bytes = static_cast<uint32_t>(pl->mt) * kLmABlock;
  pl->stage_bytes = pl->a_bytes + static_cast<uint32_t>(pl->N) * 128u;
  const size_t budget = 232448;  // dynamic shared memory per CTA
  const int st = static_cast<int>((budget - 1024 - LmLayout::kMiscBytes) / pl->stage_bytes);
  pl->stages = std::min(st, kLmMaxStages);
  if (pl->stages < 2) return fail(ORTHRUS_ERR_UNSUPPORTED, "tile does not fit shared memory");
  pl->smem = lm_smem_bytes(pl->stages, pl->stage_bytes);
  pl->grid = std::min(pl->n_tiles, std::max(sms, 1));
  pl->box_a = std::min(128 * pl->mt, R);
  pl->box_b = std::min(pl->N, V);
  return ORTHRUS_OK;
}

}  // namespace

extern "C" {

size_t orthrus_lm_head_workspace_size(int32_t total_rows) {
  if (total_rows < 1) return 0;
  return round_up(static_cast<size_t>(total_rows) * sizeof(unsigned long long), 256);
}

orthrus_status_t orthrus_lm_head_consensus(const void* hidden, const void* w_head,
                                           int32_t d_model, int32_t V, int32_t total_rows,
                                           const int32_t* draft_tokens, const int32_t* cu_block,
                                           int32_t B, int32_t max_block, int32_t* accept_len,
                                           int32_t* next_token, int32_t* row_argmax,
                                           int32_t* prefix_lens, void* workspace,
                                           size_t workspace_bytes, int32_t* error_flag,
                                           void* stream) {
  NvtxRange r("orthrus_lm_head_consensus");
  if (B < 0 || max_block < 1 || total_rows < 0)
    return fail(ORTHRUS_ERR_INVALID_ARG, "B %d, max_block %d, total_rows %d", B, max_block,
                total_rows);
  const long long R64 = total_rows > 0 ? total_rows : static_cast<long long>(B) * max_block;
  if (R64 >= (1ll << 31)) return fail(ORTHRUS_ERR_UNSUPPORTED, "too many rows");
  if (!cu_block && R64 < static_cast<long long>(B) * max_block)
    return fail(ORTHRUS_ERR_INVALID_ARG, "total_rows < B * max_block without cu_block");
  // Shape checks first, with a nominal SM count: no CUDA call before the
  // arguments are known to be valid. The real count only sizes the grid.
  constexpr int kNominalSms = 148;
  LmPlan pl;
  orthrus_status_t s =
      plan_lm(R64 > 0 ? static_cast<int>(R64) : 1, d_model, V, kNominalSms, &pl);
  if (s != ORTHRUS_OK) return s;
  if (B == 0) return ok();
  if (!hidden || !w_head || !draft_tokens || !accept_len || !next_token || !workspace)
    return fail(ORTHRUS_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned(hidden, 16) || !aligned(w_head, 16) || !aligned(workspace, 16))
    return fail(ORTHRUS_ERR_INVALID_ARG, "hidden, w_head and workspace must be 16-byte aligned");
  const int R = static_cast<int>(R64);
  if (workspace_bytes < orthrus_lm_head_workspace_size(R))
    return fail(ORTHRUS_ERR_INVALID_ARG, "workspace %zu bytes < %zu needed", workspace_bytes,
                orthrus_lm_head_workspace_size(R));
  int sms = 0;
  const int dev = device_sm_count(&sms);
  if (dev < 0) return fail(ORTHRUS_ERR_CUDA, "no current CUDA device");
  s = plan_lm(R, d_model, V, sms, &pl);
  if (s != ORTHRUS_OK) return s;
  static std::atomic<size_t> smem_set[kMaxDevices];
  if (smem_set[dev].load() < pl.smem) {
    cudaError_t e = cudaFuncSetAttribute(lm_head_argmax_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(pl.smem));
    if (e != cudaSuccess)
      return fail(ORTHRUS_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    smem_set[dev].store(pl.smem);
  }
  CUtensorMap ta, tb;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(d_model), static_cast<cuuint64_t>(R)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(d_model) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kLmKStep),
                               static_cast<cuuint32_t>(pl.box_a)};
    if (!make_map(&ta, hidden, 2, dims, strides, box))
      return fail(ORTHRUS_ERR_CUDA, "tensor map for hidden");
  }
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(d_model), static_cast<cuuint64_t>(V)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(d_model) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kLmKStep),
                               static_cast<cuuint32_t>(pl.box_b)};
    if (!make_map(&tb, w_head, 2, dims, strides, box))
      return fail(ORTHRUS_ERR_CUDA, "tensor map for w_head");
  }
  LmArgs a;
  a.R = R;
  a.V = V;
  a.d = d_model;
  a.N = pl.N;
  a.mt = pl.mt;
  a.n_m = pl.n_m;
  a.n_tiles = pl.n_tiles;
  a.k_steps = d_model / kLmKStep;
  a.stages = pl.stages;
  a.stage_bytes = pl.stage_bytes;
  a.a_bytes = pl.a_bytes;
  a.tx_bytes = static_cast<uint32_t>(pl.box_a + pl.box_b) * 128u;
  a.idesc = idesc_bf16_f32(128, static_cast<uint32_t>(pl.N), 0);
  a.keys = static_cast<unsigned long long*>(workspace);
  a.error_flag = error_flag;
  a.timeout_ns = wait_timeout_ns();
  a.fault_inject = fault_inject_mode();
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(workspace, 0, static_cast<size_t>(R) * 8, st);
  if (e != cudaSuccess) return fail(ORTHRUS_ERR_CUDA, "key reset: %s", cudaGetErrorString(e));
  lm_head_argmax_kernel<<<pl.grid, kLmThreads, pl.smem, st>>>(ta, tb, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail(ORTHRUS_ERR_CUDA, "lm_head launch: %s", cudaGetErrorString(e));
  const int warps = 8;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((B + warps - 1) / warps);
  cfg.blockDim = dim3(warps * 32);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, consensus_finalize_kernel,
                         static_cast<const unsigned long long*>(workspace), 1, draft_tokens,
                         cu_block, static_cast<int>(B), static_cast<int>(max_block), accept_len,
                         next_token, row_argmax, prefix_lens, R);
  if (e != cudaSuccess) return fail(ORTHRUS_ERR_CUDA, "finalize launch: %s", cudaGetErrorString(e));
  return ok();
}

}  // extern "C"
