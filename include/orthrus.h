/*
 * orthrus.h -- C ABI of the Orthrus block-decoding hot path on NVIDIA B200 (sm_100a).
 *
 * Orthrus ("Orthrus: Memory-Efficient Parallel Token Generation via Dual-View
 * Diffusion") lets a lightweight diffusion view draft a block of K tokens (the
 * anchor plus K-1 mask slots) over the KV cache that a frozen autoregressive
 * (AR) view built, then has the AR view verify the whole block in one pass and
 * keeps the drafts that equal the AR greedy tokens. This library implements the
 * data-parallel steps of one round:
 *
 *   orthrus_block_attn  attention of the block rows over the shared paged prefix
 *                       cache plus the block's own K/V, in the DIFFUSION view
 *                       (bidirectional inside the block) or the VERIFY view
 *                       (causal inside the block);
 *   orthrus_consensus   greedy argmax of the verify logits and the left-to-right
 *                       exact match against the drafts;
 *   orthrus_kv_append   commit: write the accepted rows' K/V into the cache;
 * and fused forms of them:
 *   orthrus_block_attn_verify_write + orthrus_consensus_commit
 *                       write-then-truncate: the VERIFY attention stores the
 *                       whole block's K/V, consensus advances the lengths;
 *   orthrus_lm_head_consensus
 *                       the AR model's LM head (hidden states x output
 *                       projection) with the greedy argmax in its epilogue,
 *                       then the consensus rule; the logits are never written;
 *   orthrus_consensus_sampled
 *                       consensus at temperature > 0 (a sampled AR token).
 *
 * Conventions shared by every call:
 *   - Every pointer marked "device" is a device pointer owned by the caller; the
 *     library never allocates, frees or retains memory and keeps no per-call
 *     state (it caches TMA descriptors' driver entry point and device
 *     attributes only).
 *   - `stream` is a cudaStream_t passed as an opaque pointer (NULL = the legacy
 *     default stream). Every call is asynchronous on it.
 *   - Arguments are checked on the host before anything is launched; a failed
 *     check returns ORTHRUS_ERR_INVALID_ARG or ORTHRUS_ERR_UNSUPPORTED and
 *     launches nothing. A failed launch returns ORTHRUS_ERR_CUDA.
 *   - Data that can only be checked on the device (a page index out of range, a
 *     length beyond the page table, a pipeline wait that ran out of time) is
 *     reported by OR-ing ORTHRUS_FLAG_* bits into the optional device word
 *     `error_flag`; the offending work item skips its writes. No kernel traps.
 *   - bf16 is IEEE binary32's upper 16 bits; all layouts are row-major and
 *     densely packed.
 *   - Outputs must not alias inputs.
 *   - Each compute call pushes an NVTX range named after itself in the
 *     "orthrus" domain around its host-side work (checks and launches); the
 *     range costs nothing measurable unless a profiler is attached.
 */
#ifndef ORTHRUS_H_
#define ORTHRUS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ORTHRUS_ABI_VERSION 1

#if defined(ORTHRUS_BUILD) && defined(__GNUC__)
#define ORTHRUS_API __attribute__((visibility("default")))
#else
#define ORTHRUS_API
#endif

typedef enum {
  ORTHRUS_OK = 0,
  ORTHRUS_ERR_INVALID_ARG = 1,  /* a pointer, size or layout argument is wrong */
  ORTHRUS_ERR_UNSUPPORTED = 2,  /* valid, but outside what the kernels implement */
  ORTHRUS_ERR_CUDA = 3,         /* the CUDA runtime refused a launch or query */
  ORTHRUS_ERR_TIMEOUT = 4,      /* a pipeline wait gave up (orthrus_status_from_flags) */
  ORTHRUS_ERR_DEVICE_CHECK = 5  /* a device-side data check failed (orthrus_status_from_flags) */
} orthrus_status_t;
/* The launch calls return only OK, INVALID_ARG, UNSUPPORTED or CUDA: they are
 * asynchronous, so what the kernels find (ORTHRUS_FLAG_* bits in the caller's
 * error_flag word) is known only once the stream has reached that point.
 * orthrus_status_from_flags turns such a word, read by the caller after a
 * stream synchronisation, into TIMEOUT or DEVICE_CHECK. */

/* Bits OR-ed into *error_flag by the kernels. */
#define ORTHRUS_FLAG_BAD_PAGE 0x1   /* a page_table entry was outside [0, num_pages) */
#define ORTHRUS_FLAG_BAD_LENGTH 0x2 /* prefix_len + rows ran past max_pages_per_seq pages,
                                       or accept_len outside [0, K_b] */
#define ORTHRUS_FLAG_TIMEOUT 0x4    /* a pipeline wait gave up; that CTA wrote nothing */

typedef enum {
  ORTHRUS_VIEW_DIFFUSION = 0, /* block rows see the whole prefix and every block row */
  ORTHRUS_VIEW_VERIFY = 1     /* block row i sees the whole prefix and block rows 0..i */
} orthrus_view_t;

/*
 * Parameters of orthrus_block_attn.
 *
 * Operation (technical summary §2.2 "attention mechanism", mask M_diff, for the
 * DIFFUSION view; §2.3 item 2, the AR view's single-pass check of the populated
 * block, for the VERIFY view). For every sequence b, KV head h, block row i in
 * [0, K_b) and query head hq = h*G + g (G = Hq / Hkv, g in [0, G)):
 *
 *   out[row0_b + i, hq, :] = sum_j softmax_j(scale * <q, k_j>) * v_j
 *
 * with q = q_block[row0_b + i, hq, :] and j running over the visible keys: the
 * prefix positions t in [0, L_b) (k_j = k_cache[page_table[b][t / P], h, t % P, :])
 * followed by the block rows j' in [0, K_b) (k_j = k_block[row0_b + j', h, :]),
 * block row j' being visible to row i always (DIFFUSION) or iff j' <= i (VERIFY).
 * L_b = prefix_lens[b]; row0_b = cu_block[b]; K_b = cu_block[b+1] - cu_block[b].
 * The same indexing gives v_j. Accumulation is fp32, the output is rounded to bf16.
 *
 * Work is split over the prefix (split-KV): each CTA covers a contiguous range
 * of 64-token tiles and writes either the final rows or a partial (row max, sum,
 * normalised accumulator) that a combine kernel merges.
 */
typedef struct {
  int32_t view;              /* orthrus_view_t */
  int32_t B;                 /* sequences, >= 0 (0: nothing to do) */
  int32_t Hq, Hkv;           /* query / KV heads; Hq % Hkv == 0 */
  int32_t D;                 /* head dim: 64 or 128 */
  int32_t page_size;         /* tokens per page P: a multiple of 64 */
  int32_t max_pages_per_seq; /* columns of page_table */
  int32_t num_pages;         /* pages in k_cache / v_cache */
  int32_t max_block;         /* max K_b: 1..64 and G * max_block <= 128 */
  int32_t total_rows;        /* R, rows of q_block, k_block, v_block and out; cu_block[B]
                                must not exceed it (0: R = B * max_block) */
  const void* q_block;       /* device bf16 [R, Hq, D] */
  const void* k_cache;       /* device bf16 [num_pages, Hkv, P, D] */
  const void* v_cache;       /* device bf16 [num_pages, Hkv, P, D] */
  const void* k_block;       /* device bf16 [R, Hkv, D] */
  const void* v_block;       /* device bf16 [R, Hkv, D] */
  const int32_t* prefix_lens; /* device [B] */
  const int32_t* cu_block;   /* device [B+1] row offsets; NULL: every K_b = max_block */
  const int32_t* page_table; /* device [B, max_pages_per_seq] */
  float softmax_scale;       /* <= 0: 1/sqrt(D) */
  int32_t kv_split_tokens;   /* 0: the library's schedule (see max_ctas); > 0: fixed chunks
                                of this many prefix tokens (a multiple of 64), each merged
                                as one partial; at most one CTA per SM (or max_ctas > 0
                                CTAs) walks the chunks, chunk j in CTA j mod grid */
  int32_t max_ctas;          /* 0: library picks: one CTA per (sequence, KV head) unit
                                when the units number between 3/4 of the SM count and
                                the SM count; fewer units: every unit gets SMs in
                                proportion to its tiles, in near-equal chunks (long
                                contexts); more units than SMs: a balanced split over
                                one CTA per SM; > 0: balanced split over this many CTAs
                                (with kv_split_tokens > 0: the chunk walkers' grid) */
  void* out;                 /* device bf16 [R, Hq, D] */
  void* workspace;           /* device scratch, >= orthrus_block_attn_workspace_size() bytes,
                                256-byte aligned; contents need no initialisation */
  size_t workspace_bytes;
  int32_t* error_flag;       /* optional device int32; ORTHRUS_FLAG_* bits are OR-ed in */
} orthrus_attn_params;

/* Scratch bytes orthrus_block_attn needs for these parameters (queries the
 * current device's SM count). 0 when the parameters are invalid. */
ORTHRUS_API size_t orthrus_block_attn_workspace_size(const orthrus_attn_params* p);

/* Number of kernels one orthrus_block_attn call with these parameters launches
 * on the current device: 1 when no (sequence, KV head) unit is cut across CTAs
 * (one CTA per whole unit, chosen when the units number between 3/4 of the SM
 * count and the SM count), 2 otherwise (attention, then the combine kernel
 * that merges the partials). 0 when the parameters are invalid. */
ORTHRUS_API int32_t orthrus_block_attn_kernel_count(const orthrus_attn_params* p);

/* The schedule orthrus_block_attn picks for *p, decided on the host from the
 * parameters alone: the kernels then cut proportional chunks and balanced
 * ranges from the actual prefix lengths on the device.
 *   sm_count  SMs to plan for; <= 0: the current device's (a CUDA query).
 * Returns OK and fills *plan, or INVALID_ARG / UNSUPPORTED as orthrus_block_attn
 * would for these parameters (plan NULL: INVALID_ARG), or CUDA when sm_count
 * <= 0 and there is no current device. No allocation, no launch. */
typedef enum {
  ORTHRUS_SCHEDULE_BALANCED = 0,     /* one contiguous range of the (unit, tile) list per CTA */
  ORTHRUS_SCHEDULE_FIXED_CHUNKS = 1, /* kv_split_tokens chunks, or one chunk per whole unit */
  ORTHRUS_SCHEDULE_PROPORTIONAL = 2  /* few units, each cut in proportion to its tiles */
} orthrus_schedule_t;

typedef struct {
  int32_t schedule;        /* orthrus_schedule_t */
  int32_t grid;            /* attention CTAs */
  int32_t partial_slots;   /* (max, sum, accumulator) partial slots the workspace holds */
  int32_t kernels;         /* launches per call: 1 (no unit cut) or 2 (attention, combine) */
  int32_t walks_chunks;    /* 1: fixed-chunk CTAs take several chunk slots each */
  int32_t chunk_tiles;     /* fixed chunks: 64-key prefix tiles per chunk; else 0 */
  size_t workspace_bytes;  /* as orthrus_block_attn_workspace_size for this SM count */
} orthrus_attn_plan;

ORTHRUS_API orthrus_status_t orthrus_block_attn_plan(const orthrus_attn_params* p,
                                                     int32_t sm_count, orthrus_attn_plan* plan);

/* Launch the block attention described by *p on `stream`.
 * q_block, k_block, v_block and out hold total_rows rows; a sequence whose
 * cu_block range is decreasing, longer than max_block or past total_rows is
 * skipped and flagged (ORTHRUS_FLAG_BAD_LENGTH). All device pointers 16-byte
 * aligned. Errors: INVALID_ARG (null pointer, bad sizes, misalignment, short
 * workspace), UNSUPPORTED (D, page_size, max_block or G*max_block outside the
 * implemented set), CUDA (launch failure). */
ORTHRUS_API orthrus_status_t orthrus_block_attn(const orthrus_attn_params* p, void* stream);

/*
 * Write-then-truncate VERIFY (technical summary §2.3 item 3: the AR view
 * writes the whole block's KV while it verifies it, and the commit truncates
 * the cache to the accepted prefix). Same attention as orthrus_block_attn with
 * p->view == ORTHRUS_VIEW_VERIFY and, in the same launch, for every sequence
 * b, block row i in [0, K_b) and KV head h, with L_b = prefix_lens[b]:
 *
 *   k_cache[page_table[b][(L_b+i)/P], h, (L_b+i) % P, :] = k_block[row0_b + i, h, :]
 *
 * and the same for V. prefix_lens is not changed: orthrus_consensus_commit
 * then advances it by the accepted count, which leaves the cache bytes of
 * every position below the new length identical to orthrus_block_attn
 * followed by orthrus_kv_append, and removes the append launch. Slots
 * L_b + n_b .. L_b + K_b - 1 keep the rejected rows until the next round
 * overwrites them (they lie past the committed length).
 *   - k_cache and v_cache are WRITTEN through the params' const pointers.
 *   - The page table must reach position L_b + K_b - 1; a row past it is
 *     skipped and flags ORTHRUS_FLAG_BAD_LENGTH, a row whose page id is out of
 *     range is skipped and flags ORTHRUS_FLAG_BAD_PAGE. A raised flag means
 *     the round's cache is incomplete: do not commit it.
 *   - The slots written must not be read by any sequence of the same call
 *     (pages holding positions >= L_b are not shared with another sequence's
 *     prefix).
 * Errors: as orthrus_block_attn; INVALID_ARG when p->view is not VERIFY.
 */
ORTHRUS_API orthrus_status_t orthrus_block_attn_verify_write(const orthrus_attn_params* p,
                                                             void* stream);

/*
 * Greedy consensus (technical summary §2.3 item 3: a drafted token is accepted
 * iff it equals the frozen AR view's greedy token, checked left to right; at the
 * first divergence j the prefix up to j-1 is committed and the exact AR
 * correction token appended; agents-report.net commentary, "core design").
 *
 * For every block row r: t_r = argmax_v verify_logits[r, v] (the lowest index
 * among equal maxima; NaN counts as -inf; -0 == +0). For every sequence b with
 * K_b > 0: m_b = number of leading rows r = row0_b + i with draft_tokens[r] ==
 * t_r; accept_len[b] = min(m_b + 1, K_b); next_token[b] = t_{row0_b +
 * accept_len[b] - 1}. A sequence with K_b = 0 gets accept_len 0, next_token -1.
 *
 *   verify_logits  device fp32 [R, ld] (row r at verify_logits + r*ld), V <= ld
 *   draft_tokens   device int32 [R]
 *   cu_block       device int32 [B+1] or NULL (every K_b = max_block)
 *   accept_len, next_token  device int32 [B] (written)
 *   row_argmax     device int32 [R] or NULL (written when given)
 *   workspace      device scratch of orthrus_consensus_workspace_size(B, max_block, V)
 *                  bytes, 16-byte aligned; contents need no initialisation
 * R = cu_block[B] <= B * max_block. Errors: INVALID_ARG, CUDA.
 */
ORTHRUS_API size_t orthrus_consensus_workspace_size(int32_t B, int32_t max_block, int32_t V);
ORTHRUS_API orthrus_status_t orthrus_consensus(const float* verify_logits, int64_t ld, int32_t V,
                                   const int32_t* draft_tokens, const int32_t* cu_block,
                                   int32_t B, int32_t max_block, int32_t* accept_len,
                                   int32_t* next_token, int32_t* row_argmax, void* workspace,
                                   size_t workspace_bytes, void* stream);

/*
 * Consensus plus the commit of write-then-truncate VERIFY (technical summary
 * §2.3 item 3). Same operation, arguments and results as orthrus_consensus,
 * and in the same launches prefix_lens[b] += accept_len[b] for every sequence
 * (a sequence with K_b = 0 is left unchanged). Meant to follow
 * orthrus_block_attn_verify_write, which already stored all K_b block rows
 * past L_b: advancing the length is then the whole commit.
 *   prefix_lens  device int32 [B], updated in place (required)
 * Errors: as orthrus_consensus; INVALID_ARG when prefix_lens is NULL.
 */
ORTHRUS_API orthrus_status_t orthrus_consensus_commit(const float* verify_logits, int64_t ld,
                                                      int32_t V, const int32_t* draft_tokens,
                                                      const int32_t* cu_block, int32_t B,
                                                      int32_t max_block, int32_t* accept_len,
                                                      int32_t* next_token, int32_t* row_argmax,
                                                      int32_t* prefix_lens, void* workspace,
                                                      size_t workspace_bytes, void* stream);

/*
 * Consensus at temperature T > 0. The pages name temperature settings
 * (technical summary §4) but give no sampling rule; this library's rule keeps
 * the greedy rule's exact-match acceptance (§2.3 item 3) and replaces the AR
 * view's greedy token by a sample from softmax(logits / T), drawn with the
 * Gumbel-max rule. For every block row r:
 *
 *   t_r = argmax_v  verify_logits[r, v] / T - ln(-ln u_{r,v})
 *
 * (ties to the lowest v, NaN never chosen), where u_{r,v} in (0, 1) is word
 * v % 4 of Philox4x32-10 (Salmon et al., "Parallel random numbers: as easy as
 * 1, 2, 3", SC 2011) at counter (v / 4, r, offset & 0xffffffff, offset >> 32)
 * and key (seed & 0xffffffff, seed >> 32), as (word >> 8) + 1/2 over 2^24.
 * Then accept_len, next_token (and, when prefix_lens is given, the commit
 * prefix_lens[b] += accept_len[b]) follow orthrus_consensus's rule on t.
 * Every committed token is the AR view's own sample, so the emitted stream is
 * an AR sample at temperature T; give each round a new offset (or seed) so
 * that no position reuses its noise. Scores are fp32 (logits * (1/T) + noise).
 *
 *   temperature  finite, > 0, with 1/T finite in fp32
 *   row_token    device int32 [R] or NULL: the sampled t_r (written when given)
 *   prefix_lens  device int32 [B] or NULL (advanced by accept_len when given)
 *   workspace    as orthrus_consensus (orthrus_consensus_workspace_size)
 * Other arguments as orthrus_consensus. Errors: as orthrus_consensus, and
 * INVALID_ARG / UNSUPPORTED for a temperature outside the range above.
 */
ORTHRUS_API orthrus_status_t orthrus_consensus_sampled(
    const float* verify_logits, int64_t ld, int32_t V, const int32_t* draft_tokens,
    const int32_t* cu_block, int32_t B, int32_t max_block, float temperature, uint64_t seed,
    uint64_t offset, int32_t* accept_len, int32_t* next_token, int32_t* row_token,
    int32_t* prefix_lens, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Fused LM head + greedy consensus (technical summary §2.3 items 2-3 with §2.1:
 * the frozen AR model scores every block row over the vocabulary, and its
 * greedy token decides acceptance). For every block row r in [0, R):
 *
 *   t_r = argmax_v  sum_k hidden[r, k] * w_head[v, k]
 *
 * (bf16 products accumulated in fp32 by the tensor cores, in an unspecified
 * order; ties go to the lowest v, NaN counts as -inf). The logits are never
 * written: each vocabulary tile's row maxima are combined in the workspace.
 * From the t_r, accept_len / next_token / row_argmax (and, when prefix_lens is
 * given, the commit prefix_lens[b] += accept_len[b]) follow the rule of
 * orthrus_consensus exactly.
 *
 *   hidden        device bf16 [R, d_model], row-major (the block rows' final
 *                 hidden states), R = total_rows, or B * max_block when 0
 *   w_head        device bf16 [V, d_model], row-major (one row per vocabulary
 *                 entry: the output projection's [out, in] layout)
 *   d_model       a multiple of 64
 *   draft_tokens  device int32 [R]
 *   cu_block      device int32 [B+1] or NULL (every K_b = max_block); a
 *                 sequence whose rows fall outside [0, R) gets accept_len 0
 *                 and next_token -1
 *   accept_len, next_token  device int32 [B] (written)
 *   row_argmax    device int32 [R] or NULL (written when given)
 *   prefix_lens   device int32 [B] or NULL (advanced by accept_len when given)
 *   workspace     device scratch of orthrus_lm_head_workspace_size(R) bytes,
 *                 16-byte aligned; contents need no initialisation
 *   error_flag    optional device int32: ORTHRUS_FLAG_TIMEOUT if a pipeline
 *                 wait of the GEMM gave up (its rows' results are then invalid)
 * Launches a 8*R-byte memset, the GEMM/argmax kernel (one CTA per SM) and the
 * consensus finalize kernel. Errors: INVALID_ARG (null pointer, misalignment,
 * short workspace, bad sizes), UNSUPPORTED (d_model not a multiple of 64, too
 * many rows), CUDA.
 */
ORTHRUS_API size_t orthrus_lm_head_workspace_size(int32_t total_rows);
ORTHRUS_API orthrus_status_t orthrus_lm_head_consensus(
    const void* hidden, const void* w_head, int32_t d_model, int32_t V, int32_t total_rows,
    const int32_t* draft_tokens, const int32_t* cu_block, int32_t B, int32_t max_block,
    int32_t* accept_len, int32_t* next_token, int32_t* row_argmax, int32_t* prefix_lens,
    void* workspace, size_t workspace_bytes, int32_t* error_flag, void* stream);

/*
 * Commit (technical summary §2.3 item 3, commit the synchronised prefix and
 * truncate the cache; agents-report.net commentary, "core design", the accepted
 * tokens' KV appended to the shared cache). For every sequence b, accepted row
 * i in [0, accept_len[b]) and KV head h, with L_b = prefix_lens[b] on entry:
 *
 *   k_cache[page_table[b][(L_b+i)/P], h, (L_b+i) % P, :] = k_block[cu_block[b]+i, h, :]
 *
 * and the same for V; no other cache byte is written. With update_lens != 0,
 * prefix_lens[b] becomes L_b + accept_len[b] (only when every row of b found its
 * page; otherwise ORTHRUS_FLAG_* is raised and b's length is left unchanged).
 *
 *   k_block, v_block  device bf16 [R, Hkv, D] (the VERIFY view's block K/V)
 *   cu_block          device int32 [B+1], or NULL: every block has max_block rows
 *                     (row0_b = b * max_block)
 *   accept_len        device int32 [B]
 *   prefix_lens       device int32 [B] (read; updated in place iff update_lens)
 *   page_table        device int32 [B, max_pages_per_seq]
 *   k_cache, v_cache  device bf16 [num_pages, Hkv, page_size, D] (updated in place)
 *   error_flag        optional device int32
 * D must be a multiple of 8 and the pointers 16-byte aligned. Errors:
 * INVALID_ARG, CUDA.
 */
ORTHRUS_API orthrus_status_t orthrus_kv_append(const void* k_block, const void* v_block,
                                   const int32_t* cu_block, int32_t max_block,
                                   const int32_t* accept_len, int32_t* prefix_lens,
                                   int32_t update_lens, const int32_t* page_table,
                                   int32_t max_pages_per_seq, int32_t num_pages, void* k_cache,
                                   void* v_cache, int32_t B, int32_t Hkv, int32_t D,
                                   int32_t page_size, int32_t* error_flag, void* stream);

/*
 * Greedy consensus without any device allocation (no counterpart in the
 * paper; it is a deployment convenience of this library).
 *
 * Same operation, arguments and results as orthrus_consensus, minus the
 * workspace. It is meant for callers that cannot allocate device memory when
 * they call in: a serving engine that reserves every byte of HBM at start-up
 * and gives its plug-ins no scratch, or a caller that must not trigger the
 * implicit device synchronisation and latency of cudaMalloc on its decode
 * path. The scratch lives instead in a fixed 512 KiB array inside the library
 * (a file-scope __device__ array, so every GPU that loads the library holds it
 * until the process exits):
 *   - the request must fit: B * max_block * ceil(V / 16384) <= 65536 (for
 *     V = 151936 that is B * max_block <= 6553 rows); larger requests return
 *     ORTHRUS_ERR_UNSUPPORTED and launch nothing;
 *   - every call looks up the array's address in the current device's
 *     context (a runtime symbol lookup, no allocation);
 *   - the array is reserved when the library's device code is loaded on a
 *     device, which under CUDA's lazy module loading can be the first call of
 *     this library there: a caller that reserves nearly all of HBM should make
 *     one library call on each device at start-up, before that reservation,
 *     and also before any stream capture;
 *   - every call on a device uses the same array, so calls whose kernels can
 *     overlap on the GPU (different streams without ordering) race: order them
 *     on one stream or with events. Nothing in the array needs to start at
 *     zero: each call writes every slot it later reads.
 * The call itself allocates nothing (no cudaMalloc, cudaFree or allocating
 * library routine). Errors: as orthrus_consensus, plus UNSUPPORTED above.
 */
ORTHRUS_API orthrus_status_t orthrus_consensus_noalloc(const float* verify_logits, int64_t ld,
                                                       int32_t V, const int32_t* draft_tokens,
                                                       const int32_t* cu_block, int32_t B,
                                                       int32_t max_block, int32_t* accept_len,
                                                       int32_t* next_token, int32_t* row_argmax,
                                                       void* stream);

/* Static description of a status code. */
ORTHRUS_API const char* orthrus_status_string(orthrus_status_t status);

/* Status for a word of ORTHRUS_FLAG_* bits that the kernels OR-ed into a
 * caller's error_flag (read by the caller after synchronising the stream):
 * ORTHRUS_OK for 0, ORTHRUS_ERR_TIMEOUT when ORTHRUS_FLAG_TIMEOUT is set (that
 * CTA's results are missing), ORTHRUS_ERR_DEVICE_CHECK for any other bit (bad
 * page ids or lengths: the flagged work was skipped). Host only; no CUDA call. */
ORTHRUS_API orthrus_status_t orthrus_status_from_flags(int32_t flags);

/* Detail of the last failed call on this host thread ("" when none). */
ORTHRUS_API const char* orthrus_last_error(void);

/* ORTHRUS_ABI_VERSION of the loaded library. */
ORTHRUS_API int32_t orthrus_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ORTHRUS_H_ */
