/*
 * Orthrus hot-path oracle: a plain, slow, obviously correct CPU implementation
 * of what the block-decoding path computes, in fp64.
 *
 * TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and the CPU-baseline
 * leg of bench.py may load this library. It shares no code, header, table or
 * helper with the CUDA path; the two meet only through the seeded input
 * generators, which hold none of the method's arithmetic.
 *
 * Source of each definition ("Orthrus: Memory-Efficient Parallel Token
 * Generation via Dual-View Diffusion", technical summary pages, Spanish and
 * German editions; agents-report.net commentary "core design"):
 *   - oracle_block_attn, DIFFUSION view: technical summary §2.2, "attention
 *     mechanism" bullet, mask M_diff: block positions attend to the whole clean
 *     context before the anchor and bidirectionally to each other.
 *   - oracle_block_attn, VERIFY view: technical summary §2.3 item 2 (the frozen
 *     AR view reads the populated block in one pass under its usual causal
 *     attention).
 *   - oracle_block_attn_split: the split-KV partial/merge identity of the
 *     library's own split schedule (not on the pages; a restatement of the
 *     softmax over a union of key sets).
 *   - oracle_consensus: technical summary §2.3 item 3 (strict left-to-right
 *     check, accept iff equal to the AR greedy token, at the first divergence j
 *     commit up to j-1 and append the AR correction token).
 *   - oracle_kv_append: technical summary §2.3 item 3 ("truncates the cache")
 *     and the commentary's "appends their KV state to the shared cache".
 *   - oracle_lm_head, oracle_greedy_tokens: technical summary §2.3 items 2-3
 *     (the frozen AR view scores the populated block; its greedy token per row
 *     is the largest of those scores). The scores are the AR model's output
 *     projection of each row's final hidden state (technical summary §2.1: the
 *     AR view is the unchanged base model).
 *   - oracle_accept: the left-to-right rule of oracle_consensus on given
 *     greedy tokens (technical summary §2.3 item 3).
 *
 * Layouts (all row-major, caller-owned host memory):
 *   q_block  [R, Hq, D]                   bf16 bits (uint16)
 *   k_cache, v_cache [num_pages, Hkv, P, D] bf16 bits
 *   k_block, v_block [R, Hkv, D]          bf16 bits
 *   prefix_lens [B], cu_block [B+1], page_table [B, max_pages_per_seq] int32
 *   logits [R, ld] fp32, draft [R] int32
 * Query head hq reads KV head hq / G with G = Hq / Hkv. Block row i of
 * sequence b is global row cu_block[b] + i.
 *
 * Every bf16 value is widened exactly to double; all arithmetic is double.
 */
#include <math.h>
#include <pthread.h>
#include <stdatomic.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_VIEW_DIFFUSION 0
#define ORACLE_VIEW_VERIFY 1

/* ------------------------------------------------------------------------- */
/* bf16 bits -> double: the bf16 value is the top half of an IEEE binary32.   */
static double bf16_to_double(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* ------------------------------------------------------------------------- */
/* A minimal dynamic parallel-for over [0, n) on plain pthreads.             */
typedef void (*task_fn)(void* ctx, int64_t index);

typedef struct {
  task_fn fn;
  void* ctx;
  int64_t n;
  atomic_llong next;
} pool_job;

static void* pool_worker(void* arg) {
  pool_job* job = (pool_job*)arg;
  for (;;) {
    int64_t i = atomic_fetch_add(&job->next, 1);
    if (i >= job->n) break;
    job->fn(job->ctx, i);
  }
  return NULL;
}

static void parallel_for(int64_t n, task_fn fn, void* ctx, int threads) {
  if (threads < 1) threads = 1;
  if (threads > 256) threads = 256;
  if ((int64_t)threads > n) threads = (int)(n > 0 ? n : 1);
  pool_job job;
  job.fn = fn;
  job.ctx = ctx;
  job.n = n;
  atomic_init(&job.next, 0);
  if (threads == 1) {
    pool_worker(&job);
    return;
  }
  pthread_t tid[256];
  int started = 0;
  for (int t = 1; t < threads; ++t) {
    if (pthread_create(&tid[started], NULL, pool_worker, &job) == 0) ++started;
  }
  pool_worker(&job);
  for (int t = 0; t < started; ++t) pthread_join(tid[t], NULL);
}

/* ------------------------------------------------------------------------- */
/* Attention                                                                 */

typedef struct {
  int view, B, Hq, Hkv, D, page_size, max_pages_per_seq, num_pages;
  const uint16_t *q_block, *k_cache, *v_cache, *k_block, *v_block;
  const int32_t *prefix_lens, *cu_block, *page_table;
  double scale;
  int64_t chunk_tokens; /* <= 0: one softmax over all keys (no split) */
  int64_t n_items;
  const int64_t* sel_rows; /* NULL: every (row, head) pair in order */
  const int32_t* sel_heads;
  double* out;
  atomic_int bad; /* set when an index read from the inputs is out of range */
} attn_job;

/* Sequence that owns global block row r (cu_block is nondecreasing). */
static int seq_of_row(const int32_t* cu_block, int B, int64_t r) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) / 2;
    if ((int64_t)cu_block[mid] <= r) lo = mid; else hi = mid - 1;
  }
  return lo;
}

/* Pointer to the key (or value) vector of key j for (sequence b, kv head h).
 * Keys 0..L-1 are prefix positions read through the page table, keys
 * L..L+K_b-1 are the block's own rows. Returns NULL on a bad page index. */
static const uint16_t* key_row(const attn_job* a, const uint16_t* cache, const uint16_t* blk,
                               int b, int h, int64_t L, int64_t j) {
  if (j < L) {
    int64_t pidx = j / a->page_size;
    if (pidx >= a->max_pages_per_seq) return NULL;
    int32_t page = a->page_table[(int64_t)b * a->max_pages_per_seq + pidx];
    if (page < 0 || page >= a->num_pages) return NULL;
    int64_t slot = j % a->page_size;
    return cache + (((int64_t)page * a->Hkv + h) * a->page_size + slot) * a->D;
  }
  int64_t row = (int64_t)a->cu_block[b] + (j - L);
  return blk + (row * a->Hkv + h) * a->D;
}

static double dot_q_k(const uint16_t* q, const uint16_t* k, int D) {
  double s = 0.0;
  for (int d = 0; d < D; ++d) s += bf16_to_double(q[d]) * bf16_to_double(k[d]);
  return s;
}

static void attn_item(void* ctx, int64_t item) {
  attn_job* a = (attn_job*)ctx;
  int64_t r;
  int hq;
  if (a->sel_rows) {
    r = a->sel_rows[item];
    hq = a->sel_heads[item];
  } else {
    r = item / a->Hq;
    hq = (int)(item % a->Hq);
  }
  const int D = a->D;
  double* o = a->out + item * D;
  for (int d = 0; d < D; ++d) o[d] = 0.0;

  const int G = a->Hq / a->Hkv;
  const int h = hq / G;
  const int b = seq_of_row(a->cu_block, a->B, r);
  const int64_t i = r - a->cu_block[b];
  const int64_t L = a->prefix_lens[b];
  const int64_t Kb = (int64_t)a->cu_block[b + 1] - a->cu_block[b];
  /* visible keys: the whole prefix, then block rows 0..Kb-1 (DIFFUSION) or
   * 0..i (VERIFY, causal inside the block) */
  const int64_t n_block_vis = (a->view == ORACLE_VIEW_DIFFUSION) ? Kb : (i + 1);
  const int64_t n_keys = L + n_block_vis;
  const uint16_t* q = a->q_block + (r * a->Hq + hq) * D;

  double* z = (double*)malloc(sizeof(double) * (size_t)(n_keys > 0 ? n_keys : 1));
  double* acc = (double*)malloc(sizeof(double) * (size_t)D);
  if (!z || !acc) {
    atomic_store(&a->bad, 2);
    free(z);
    free(acc);
    return;
  }
  /* scores z_j = scale * <q, k_j> */
  for (int64_t j = 0; j < n_keys; ++j) {
    const uint16_t* k = key_row(a, a->k_cache, a->k_block, b, h, L, j);
    if (!k) {
      atomic_store(&a->bad, 1);
      free(z);
      free(acc);
      return;
    }
    z[j] = a->scale * dot_q_k(q, k, D);
  }

  /* key chunks: a single chunk holding every key when no split is asked for;
   * otherwise prefix chunks [c*S, (c+1)*S) and the block keys in the last one */
  int64_t S = a->chunk_tokens;
  int64_t n_chunks = 1;
  if (S > 0) {
    n_chunks = (L + S - 1) / S;
    if (n_chunks < 1) n_chunks = 1;
  }
  double m_all = -INFINITY, l_all = 0.0; /* merge state across chunks */
  for (int64_t c = 0; c < n_chunks; ++c) {
    int64_t j0, j1;
    if (S <= 0) {
      j0 = 0;
      j1 = n_keys;
    } else {
      j0 = c * S;
      j1 = (c == n_chunks - 1) ? n_keys : (c + 1) * S;
    }
    /* partial softmax of this chunk: m_c, l_c, acc_c */
    double m_c = -INFINITY;
    for (int64_t j = j0; j < j1; ++j) if (z[j] > m_c) m_c = z[j];
    double l_c = 0.0;
    for (int d = 0; d < D; ++d) acc[d] = 0.0;
    for (int64_t j = j0; j < j1; ++j) {
      double w = exp(z[j] - m_c);
      l_c += w;
      const uint16_t* v = key_row(a, a->v_cache, a->v_block, b, h, L, j);
      for (int d = 0; d < D; ++d) acc[d] += w * bf16_to_double(v[d]);
    }
    /* merge: m = max(m, m_c); rescale both sides to the new reference */
    double m_new = (m_c > m_all) ? m_c : m_all;
    double f_old = (l_all > 0.0) ? exp(m_all - m_new) : 0.0;
    double f_new = exp(m_c - m_new);
    l_all = l_all * f_old + l_c * f_new;
    for (int d = 0; d < D; ++d) o[d] = o[d] * f_old + acc[d] * f_new;
    m_all = m_new;
  }
  for (int d = 0; d < D; ++d) o[d] /= l_all;
  free(z);
  free(acc);
}

static int run_attn(attn_job* a, int threads) {
  if (a->B < 1 || a->Hq < 1 || a->Hkv < 1 || a->Hq % a->Hkv || a->D < 1 || a->page_size < 1)
    return -1;
  atomic_init(&a->bad, 0);
  parallel_for(a->n_items, attn_item, a, threads);
  return atomic_load(&a->bad);
}

/* Attention of every (row, query head) pair, or of the n_sel pairs listed in
 * (sel_rows, sel_heads). out is [R, Hq, D] (all) or [n_sel, D] (selection).
 * scale <= 0 means 1/sqrt(D). Returns 0, or nonzero when a page index read
 * from page_table is out of range. */
int oracle_block_attn(int view, int B, int Hq, int Hkv, int D, int page_size,
                      int max_pages_per_seq, int num_pages,
                      const uint16_t* q_block, const uint16_t* k_cache, const uint16_t* v_cache,
                      const uint16_t* k_block, const uint16_t* v_block,
                      const int32_t* prefix_lens, const int32_t* cu_block,
                      const int32_t* page_table, double scale,
                      int64_t n_sel, const int64_t* sel_rows, const int32_t* sel_heads,
                      double* out, int threads) {
  attn_job a;
  memset(&a, 0, sizeof a);
  a.view = view; a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.D = D; a.page_size = page_size;
  a.max_pages_per_seq = max_pages_per_seq; a.num_pages = num_pages;
  a.q_block = q_block; a.k_cache = k_cache; a.v_cache = v_cache;
  a.k_block = k_block; a.v_block = v_block;
  a.prefix_lens = prefix_lens; a.cu_block = cu_block; a.page_table = page_table;
  a.scale = (scale > 0.0) ? scale : 1.0 / sqrt((double)D);
  a.chunk_tokens = 0;
  a.sel_rows = (n_sel >= 0) ? sel_rows : NULL;
  a.sel_heads = (n_sel >= 0) ? sel_heads : NULL;
  a.n_items = (n_sel >= 0) ? n_sel : (int64_t)cu_block[B] * Hq;
  a.out = out;
  return run_attn(&a, threads);
}

/* Same result computed as per-chunk partial softmaxes (m_c, l_c, acc_c) over
 * prefix chunks of chunk_tokens keys (block keys join the last chunk), merged
 * with m = max m_c, l = sum l_c e^(m_c - m), o = sum acc_c e^(m_c - m) / l. */
int oracle_block_attn_split(int view, int B, int Hq, int Hkv, int D, int page_size,
                            int max_pages_per_seq, int num_pages,
                            const uint16_t* q_block, const uint16_t* k_cache,
                            const uint16_t* v_cache, const uint16_t* k_block,
                            const uint16_t* v_block, const int32_t* prefix_lens,
                            const int32_t* cu_block, const int32_t* page_table, double scale,
                            int64_t chunk_tokens, int64_t n_sel, const int64_t* sel_rows,
                            const int32_t* sel_heads, double* out, int threads) {
  if (chunk_tokens < 1) return -1;
  attn_job a;
  memset(&a, 0, sizeof a);
  a.view = view; a.B = B; a.Hq = Hq; a.Hkv = Hkv; a.D = D; a.page_size = page_size;
  a.max_pages_per_seq = max_pages_per_seq; a.num_pages = num_pages;
  a.q_block = q_block; a.k_cache = k_cache; a.v_cache = v_cache;
  a.k_block = k_block; a.v_block = v_block;
  a.prefix_lens = prefix_lens; a.cu_block = cu_block; a.page_table = page_table;
  a.scale = (scale > 0.0) ? scale : 1.0 / sqrt((double)D);
  a.chunk_tokens = chunk_tokens;
  a.sel_rows = (n_sel >= 0) ? sel_rows : NULL;
  a.sel_heads = (n_sel >= 0) ? sel_heads : NULL;
  a.n_items = (n_sel >= 0) ? n_sel : (int64_t)cu_block[B] * Hq;
  a.out = out;
  return run_attn(&a, threads);
}

/* ------------------------------------------------------------------------- */
/* Consensus                                                                 */

typedef struct {
  const float* logits;
  int64_t ld;
  int V;
  int32_t* row_argmax;
} argmax_job;

/* Greedy token of one row: the first index holding the largest value. NaN
 * counts as -inf; -0 and +0 compare equal (plain IEEE comparison). */
static void argmax_row(void* ctx, int64_t r) {
  argmax_job* a = (argmax_job*)ctx;
  const float* x = a->logits + r * a->ld;
  double best = -INFINITY;
  int32_t idx = 0;
  for (int v = 0; v < a->V; ++v) {
    double xv = (double)x[v];
    if (isnan(xv)) xv = -INFINITY;
    if (xv > best) {
      best = xv;
      idx = v;
    }
  }
  a->row_argmax[r] = idx;
}

/* For each sequence b with block rows row0 .. row0+K_b-1 and greedy tokens t:
 *   m_b  = number of leading rows whose draft equals t_r
 *   n_b  = min(m_b + 1, K_b)     (accepted drafts plus the AR correction)
 *   next = t_{row0 + n_b - 1}    (the token that becomes the next anchor)
 * A sequence with K_b = 0 gets n_b = 0 and next = -1. */
void oracle_accept(const int32_t* t, const int32_t* draft, const int32_t* cu_block, int B,
                   int32_t* accept_len, int32_t* next_token) {
  for (int b = 0; b < B; ++b) {
    int64_t row0 = cu_block[b];
    int64_t Kb = (int64_t)cu_block[b + 1] - row0;
    if (Kb <= 0) {
      accept_len[b] = 0;
      next_token[b] = -1;
      continue;
    }
    int64_t m = 0;
    while (m < Kb && draft[row0 + m] == t[row0 + m]) ++m;
    int64_t n = (m + 1 < Kb) ? (m + 1) : Kb;
    accept_len[b] = (int32_t)n;
    next_token[b] = t[row0 + n - 1];
  }
}

int oracle_consensus(const float* logits, int64_t ld, int V, const int32_t* draft,
                     const int32_t* cu_block, int B, int32_t* accept_len, int32_t* next_token,
                     int32_t* row_argmax, int threads) {
  if (V < 1 || ld < V || B < 0) return -1;
  int64_t R = (B > 0) ? cu_block[B] : 0;
  int32_t* t = row_argmax;
  int32_t* own = NULL;
  if (!t) {
    own = (int32_t*)malloc(sizeof(int32_t) * (size_t)(R > 0 ? R : 1));
    if (!own) return -2;
    t = own;
  }
  argmax_job a = {logits, ld, V, t};
  parallel_for(R, argmax_row, &a, threads);
  oracle_accept(t, draft, cu_block, B, accept_len, next_token);
  free(own);
  return 0;
}

/* ------------------------------------------------------------------------- */
/* KV append                                                                 */

/* For each sequence b and i < accept_len[b], every kv head h:
 *   cache[page_table[b][(L_b+i)/P], h, (L_b+i) % P, :] = block[cu_block[b]+i, h, :]
 * for K and V, with L_b = prefix_lens[b] before the call. Slots outside the
 * appended range are left untouched. With update_lens, prefix_lens[b] += n_b.
 * Returns 0, or nonzero when an index is out of range: that write is skipped
 * and that sequence's length is left as it was. */
int oracle_kv_append(const uint16_t* k_block, const uint16_t* v_block, const int32_t* cu_block,
                     const int32_t* accept_len, int32_t* prefix_lens, int update_lens,
                     const int32_t* page_table, int max_pages_per_seq, int num_pages,
                     uint16_t* k_cache, uint16_t* v_cache, int B, int Hkv, int D,
                     int page_size) {
  int bad = 0;
  for (int b = 0; b < B; ++b) {
    int64_t L = prefix_lens[b];
    int64_t row0 = cu_block[b];
    int64_t Kb = (int64_t)cu_block[b + 1] - row0;
    int64_t n = accept_len[b];
    int seq_bad = 0;
    if (n < 0 || n > Kb) {
      bad = 1;
      continue;
    }
    for (int64_t i = 0; i < n; ++i) {
      int64_t pos = L + i;
      int64_t pidx = pos / page_size;
      if (pidx >= max_pages_per_seq) {
        seq_bad = 1;
        continue;
      }
      int32_t page = page_table[(int64_t)b * max_pages_per_seq + pidx];
      if (page < 0 || page >= num_pages) {
        seq_bad = 1;
        continue;
      }
      int64_t slot = pos % page_size;
      for (int h = 0; h < Hkv; ++h) {
        int64_t dst = (((int64_t)page * Hkv + h) * page_size + slot) * D;
        int64_t src = ((row0 + i) * Hkv + h) * D;
        for (int d = 0; d < D; ++d) {
          k_cache[dst + d] = k_block[src + d];
          v_cache[dst + d] = v_block[src + d];
        }
      }
    }
    /* the length grows only when every row of the sequence found its slot */
    if (update_lens && !seq_bad) prefix_lens[b] = (int32_t)(L + n);
    bad |= seq_bad;
  }
  return bad;
}

/* ------------------------------------------------------------------------- */
/* LM head: the AR view's scores of the block rows                            */

typedef struct {
  const uint16_t* hidden;  /* [R, d] bf16 bits */
  const uint16_t* w;       /* [V, d] bf16 bits, one row per vocabulary entry */
  int d, V;
  const int64_t* rows;     /* the rows of hidden to score */
  double* logits;          /* [nrows, V] */
  double* absdot;          /* [nrows, V] or NULL */
  int64_t vchunk, n_vchunks;
} lmhead_job;

/* logits[i, v] = sum_k hidden[rows[i], k] * w[v, k], and absdot[i, v] =
 * sum_k |hidden[rows[i], k] * w[v, k]| (the scale of the rounding error of any
 * shorter-precision evaluation of the same sum). Every bf16 product is exact
 * in double; the sum runs over k in increasing order. */
static void lmhead_task(void* ctx, int64_t task) {
  lmhead_job* a = (lmhead_job*)ctx;
  int64_t i = task / a->n_vchunks;
  int64_t c = task % a->n_vchunks;
  const uint16_t* h = a->hidden + a->rows[i] * (int64_t)a->d;
  int64_t v0 = c * a->vchunk;
  int64_t v1 = v0 + a->vchunk < a->V ? v0 + a->vchunk : a->V;
  double* hv = (double*)malloc(sizeof(double) * (size_t)a->d);
  if (!hv) return;
  for (int k = 0; k < a->d; ++k) hv[k] = bf16_to_double(h[k]);
  for (int64_t v = v0; v < v1; ++v) {
    const uint16_t* wr = a->w + v * (int64_t)a->d;
    double s = 0.0, sa = 0.0;
    for (int k = 0; k < a->d; ++k) {
      double x = hv[k] * bf16_to_double(wr[k]);
      s += x;
      sa += fabs(x);
    }
    a->logits[i * (int64_t)a->V + v] = s;
    if (a->absdot) a->absdot[i * (int64_t)a->V + v] = sa;
  }
  free(hv);
}

int oracle_lm_head(const uint16_t* hidden, const uint16_t* w_head, int d_model, int V,
                   const int64_t* rows, int64_t nrows, double* logits, double* absdot,
                   int threads) {
  if (d_model < 1 || V < 1 || nrows < 0) return -1;
  lmhead_job a = {hidden, w_head, d_model, V, rows, logits, absdot, 4096, 0};
  a.n_vchunks = (V + a.vchunk - 1) / a.vchunk;
  parallel_for(nrows * a.n_vchunks, lmhead_task, &a, threads);
  return 0;
}

/* Greedy token of each row of fp64 scores [nrows, V]: the first index holding
 * the largest value (NaN counts as -inf, -0 == +0). */
void oracle_greedy_tokens(const double* logits, int64_t nrows, int V, int32_t* t) {
  for (int64_t i = 0; i < nrows; ++i) {
    const double* x = logits + i * (int64_t)V;
    double best = -INFINITY;
    int32_t idx = 0;
    for (int v = 0; v < V; ++v) {
      double xv = isnan(x[v]) ? -INFINITY : x[v];
      if (xv > best) {
        best = xv;
        idx = v;
      }
    }
    t[i] = idx;
  }
}

/* ------------------------------------------------------------------------- */
/* Temperature > 0 consensus (the pages fix no sampling rule; this is the
 * reading taken): the frozen AR view's token of row r is a sample from
 * softmax(logits[r] / T), drawn by the Gumbel-max rule
 *     t_r = argmax_v ( logits[r, v] / T + g_{r,v} ),   g = -ln(-ln u),
 * with u_{r,v} in (0, 1) from the counter-based generator Philox4x32-10
 * (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3",
 * SC 2011), and a draft is accepted iff it equals that sample, left to right,
 * exactly as in the greedy rule (technical summary §2.3 item 3). Every
 * committed token is the AR view's own sample, so the emitted stream is an
 * AR sample at temperature T. Scores here are in fp64. */

/* One Philox4x32 round and the key schedule, as published. */
static void philox_round(uint32_t c[4], const uint32_t k[2]) {
  const uint64_t p0 = (uint64_t)0xD2511F53u * c[0];
  const uint64_t p1 = (uint64_t)0xCD9E8D57u * c[2];
  const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
  const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
  const uint32_t n0 = hi1 ^ c[1] ^ k[0];
  const uint32_t n2 = hi0 ^ c[3] ^ k[1];
  c[0] = n0;
  c[1] = lo1;
  c[2] = n2;
  c[3] = lo0;
}

/* Philox4x32-10: ten rounds, the key bumped by the Weyl constants between
 * rounds. out may alias ctr. */
void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  uint32_t c[4] = {ctr[0], ctr[1], ctr[2], ctr[3]};
  uint32_t k[2] = {key[0], key[1]};
  for (int i = 0; i < 10; ++i) {
    if (i > 0) {
      k[0] += 0x9E3779B9u;
      k[1] += 0xBB67AE85u;
    }
    philox_round(c, k);
  }
  for (int i = 0; i < 4; ++i) out[i] = c[i];
}

/* u_{r,v}: word (v mod 4) of Philox4x32-10 at counter (v / 4, r, offset low,
 * offset high) and key (seed low, seed high); its top 24 bits plus one half,
 * over 2^24: a value in (0, 1), never 0 or 1. */
static double sample_uniform(int64_t r, int v, uint64_t seed, uint64_t offset) {
  const uint32_t ctr[4] = {(uint32_t)(v >> 2), (uint32_t)r, (uint32_t)offset,
                           (uint32_t)(offset >> 32)};
  const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  uint32_t w[4];
  oracle_philox4x32_10(ctr, key, w);
  return ((double)(w[v & 3] >> 8) + 0.5) / 16777216.0;
}

typedef struct {
  const float* logits;
  int64_t ld;
  int V;
  double T;
  uint64_t seed, offset;
  int32_t* tokens;
  double* margin;  /* best score minus the runner-up's (may be NULL) */
} sample_job;

static void sample_row(void* ctx, int64_t r) {
  sample_job* a = (sample_job*)ctx;
  const float* x = a->logits + r * a->ld;
  double best = -INFINITY, second = -INFINITY;
  int32_t idx = 0;
  for (int v = 0; v < a->V; ++v) {
    double xv = (double)x[v];
    if (isnan(xv)) xv = -INFINITY;
    const double u = sample_uniform(r, v, a->seed, a->offset);
    const double s = xv / a->T - log(-log(u));
    if (s > best) {
      second = best;
      best = s;
      idx = v;
    } else if (s > second) {
      second = s;
    }
  }
  a->tokens[r] = idx;
  if (a->margin) a->margin[r] = best - second;
}

/* Sampled AR tokens of rows 0 .. R-1 (and each row's winning margin). */
int oracle_sampled_tokens(const float* logits, int64_t ld, int V, int64_t R, double T,
                          uint64_t seed, uint64_t offset, int32_t* tokens, double* margin,
                          int threads) {
  if (V < 1 || ld < V || R < 0 || !(T > 0.0)) return -1;
  sample_job a = {logits, ld, V, T, seed, offset, tokens, margin};
  parallel_for(R, sample_row, &a, threads);
  return 0;
}

/* Consensus at temperature T: the sampled tokens, then the greedy rule's
 * left-to-right acceptance on them. */
int oracle_consensus_sampled(const float* logits, int64_t ld, int V, const int32_t* draft,
                             const int32_t* cu_block, int B, double T, uint64_t seed,
                             uint64_t offset, int32_t* accept_len, int32_t* next_token,
                             int32_t* tokens, int threads) {
  if (B < 0) return -1;
  const int64_t R = (B > 0) ? cu_block[B] : 0;
  const int rc = oracle_sampled_tokens(logits, ld, V, R, T, seed, offset, tokens, NULL, threads);
  if (rc) return rc;
  oracle_accept(tokens, draft, cu_block, B, accept_len, next_token);
  return 0;
}
