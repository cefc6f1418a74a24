"""Orthrus hot-path oracle (fp64, CPU).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. It shares no code with
the CUDA path (``diffusion_draft_ar_b200``); the two meet only through the seeded
input generators in ``diffusion_draft_ar_b200.workloads``.

The arithmetic lives in ``orthrus_oracle.c`` (plain C, fp64, one scalar loop per
definition); this module compiles it with gcc on first use and marshals numpy
arrays to it. bf16 tensors travel as their raw 16-bit patterns (``numpy.uint16``).

Definitions followed (Orthrus: Memory-Efficient Parallel Token Generation via
Dual-View Diffusion, technical summary):

* ``block_attn(view=DIFFUSION)`` -- §2.2, mask M_diff: every block row sees the
  whole clean prefix and every other block row.
* ``block_attn(view=VERIFY)`` -- §2.3 item 2: the frozen AR view runs causal
  attention over the populated block (row i sees block rows 0..i).
* ``block_attn_split`` -- partial softmax per prefix chunk, merged by the
  max/sum identity; equal to ``block_attn`` up to rounding.
* ``consensus`` -- §2.3 item 3: strict left-to-right greedy match, commit up to
  j-1 plus the AR correction token.
* ``kv_append`` -- §2.3 item 3 (commit and truncate the cache) and the
  agents-report.net commentary, "core design" (accepted tokens' KV appended to
  the shared cache).
* ``lm_head_logits`` / ``greedy_tokens`` -- §2.3 items 2-3 with §2.1: the
  frozen AR model's output projection scores each block row over the
  vocabulary, and its greedy token is the first index of the largest score.
* ``accept_from_tokens`` -- the §2.3 item 3 rule of ``consensus`` applied to
  given greedy tokens.
* ``consensus_sampled`` / ``sampled_tokens`` -- temperature > 0 (the pages
  name temperature settings, §4, but give no sampling rule; the reading
  taken): the AR token of each row is a Gumbel-max sample from
  softmax(logits / T), with uniforms from Philox4x32-10 (``philox4x32_10``,
  Salmon et al., SC 2011), and the §2.3 item 3 acceptance runs on it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

VIEW_DIFFUSION = 0
VIEW_VERIFY = 1

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "orthrus_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liborthrus_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``orthrus_oracle.c`` into ``liborthrus_oracle.so`` (gcc, -O2, no fast-math)."""
    stale = (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
               "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def default_threads() -> int:
    env = os.environ.get("ORTHRUS_ORACLE_THREADS")
    if env:
        return max(1, int(env))
    return max(1, os.cpu_count() or 1)


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        p = ctypes.c_void_p
        i32, i64, dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.oracle_block_attn.restype = i32
        lib.oracle_block_attn.argtypes = [i32] * 8 + [p] * 5 + [p] * 3 + [dbl, i64, p, p, p, i32]
        lib.oracle_block_attn_split.restype = i32
        lib.oracle_block_attn_split.argtypes = [i32] * 8 + [p] * 5 + [p] * 3 + [dbl, i64, i64, p, p, p, i32]
        lib.oracle_consensus.restype = i32
        lib.oracle_consensus.argtypes = [p, i64, i32, p, p, i32, p, p, p, i32]
        lib.oracle_kv_append.restype = i32
        lib.oracle_kv_append.argtypes = [p, p, p, p, p, i32, p, i32, i32, p, p, i32, i32, i32, i32]
        lib.oracle_accept.restype = None
        lib.oracle_accept.argtypes = [p, p, p, i32, p, p]
        lib.oracle_lm_head.restype = i32
        lib.oracle_lm_head.argtypes = [p, p, i32, i32, p, i64, p, p, i32]
        lib.oracle_greedy_tokens.restype = None
        lib.oracle_greedy_tokens.argtypes = [p, i64, i32, p]
        u64 = ctypes.c_uint64
        lib.oracle_philox4x32_10.restype = None
        lib.oracle_philox4x32_10.argtypes = [p, p, p]
        lib.oracle_sampled_tokens.restype = i32
        lib.oracle_sampled_tokens.argtypes = [p, i64, i32, i64, dbl, u64, u64, p, p, i32]
        lib.oracle_consensus_sampled.restype = i32
        lib.oracle_consensus_sampled.argtypes = [p, i64, i32, p, p, i32, dbl, u64, u64, p, p, p,
                                                 i32]
        _lib = lib
        return lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _attn_common(view, q_block, k_cache, v_cache, k_block, v_block, prefix_lens, cu_block,
                 page_table, sel):
    q = _c(q_block, np.uint16)
    kc = _c(k_cache, np.uint16)
    vc = _c(v_cache, np.uint16)
    kb = _c(k_block, np.uint16)
    vb = _c(v_block, np.uint16)
    pl = _c(prefix_lens, np.int32)
    cu = _c(cu_block, np.int32)
    pt = _c(page_table, np.int32)
    if pt.ndim != 2:
        raise ValueError("page_table must be [B, max_pages_per_seq]")
    R, Hq, D = q.shape
    num_pages, Hkv, P, D2 = kc.shape
    if D2 != D or vc.shape != kc.shape or kb.shape != (R, Hkv, D) or vb.shape != kb.shape:
        raise ValueError("inconsistent attention shapes")
    B = pl.shape[0]
    if cu.shape[0] != B + 1 or int(cu[-1]) != R or pt.shape[0] != B:
        raise ValueError("inconsistent batch metadata")
    if sel is None:
        n_sel, rows, heads = -1, None, None
        out = np.zeros((R, Hq, D), np.float64)
    else:
        rows = _c(sel[0], np.int64)
        heads = _c(sel[1], np.int32)
        n_sel = rows.shape[0]
        out = np.zeros((n_sel, D), np.float64)
    arrays = (q, kc, vc, kb, vb, pl, cu, pt, rows, heads, out)
    dims = (int(view), B, Hq, Hkv, D, P, pt.shape[1], num_pages)
    return dims, arrays, n_sel


def block_attn(view, q_block, k_cache, v_cache, k_block, v_block, prefix_lens, cu_block,
               page_table, scale: float = 0.0, sel=None, threads: int | None = None) -> np.ndarray:
    """fp64 attention of the block rows over prefix + block keys.

    ``sel`` = (rows int64[n], heads int32[n]) restricts the computation to those
    (global block row, query head) pairs and returns [n, D]; otherwise [R, Hq, D].
    """
    lib = _load()
    dims, arrs, n_sel = _attn_common(view, q_block, k_cache, v_cache, k_block, v_block,
                                     prefix_lens, cu_block, page_table, sel)
    q, kc, vc, kb, vb, pl, cu, pt, rows, heads, out = arrs
    rc = lib.oracle_block_attn(*dims, _ptr(q), _ptr(kc), _ptr(vc), _ptr(kb), _ptr(vb),
                               _ptr(pl), _ptr(cu), _ptr(pt), float(scale), n_sel,
                               _ptr(rows), _ptr(heads), _ptr(out),
                               threads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle_block_attn: bad input (code {rc})")
    return out


def block_attn_split(view, q_block, k_cache, v_cache, k_block, v_block, prefix_lens, cu_block,
                     page_table, chunk_tokens: int, scale: float = 0.0, sel=None,
                     threads: int | None = None) -> np.ndarray:
    """Same as :func:`block_attn`, computed as merged per-chunk partial softmaxes."""
    lib = _load()
    dims, arrs, n_sel = _attn_common(view, q_block, k_cache, v_cache, k_block, v_block,
                                     prefix_lens, cu_block, page_table, sel)
    q, kc, vc, kb, vb, pl, cu, pt, rows, heads, out = arrs
    rc = lib.oracle_block_attn_split(*dims, _ptr(q), _ptr(kc), _ptr(vc), _ptr(kb), _ptr(vb),
                                     _ptr(pl), _ptr(cu), _ptr(pt), float(scale),
                                     int(chunk_tokens), n_sel, _ptr(rows), _ptr(heads),
                                     _ptr(out), threads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle_block_attn_split: bad input (code {rc})")
    return out


def consensus(logits, draft_tokens, cu_block, threads: int | None = None):
    """Greedy consensus. Returns (accept_len[B], next_token[B], row_argmax[R]) as int32."""
    lib = _load()
    x = np.asarray(logits, dtype=np.float32)
    if x.ndim != 2:
        raise ValueError("logits must be [R, ld]")
    if not x.flags.c_contiguous:
        x = np.ascontiguousarray(x)
    R, V = x.shape
    dr = _c(draft_tokens, np.int32)
    cu = _c(cu_block, np.int32)
    B = cu.shape[0] - 1
    if dr.shape[0] != R or int(cu[-1]) != R:
        raise ValueError("inconsistent consensus shapes")
    acc = np.zeros(B, np.int32)
    nxt = np.zeros(B, np.int32)
    am = np.zeros(R, np.int32)
    rc = lib.oracle_consensus(_ptr(x), V, V, _ptr(dr), _ptr(cu), B, _ptr(acc), _ptr(nxt),
                              _ptr(am), threads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle_consensus: bad input (code {rc})")
    return acc, nxt, am


def kv_append(k_block, v_block, cu_block, accept_len, prefix_lens, page_table, k_cache, v_cache,
              update_lens: bool = True) -> int:
    """In-place append of the accepted rows into numpy caches (uint16 bf16 bits).

    ``prefix_lens`` (int32 numpy) is updated in place when ``update_lens``.
    Returns the C status (0 = every index in range).
    """
    lib = _load()
    for name, arr, dt in (("k_cache", k_cache, np.uint16), ("v_cache", v_cache, np.uint16),
                          ("prefix_lens", prefix_lens, np.int32)):
        if arr.dtype != dt or not arr.flags.c_contiguous:
            raise ValueError(f"{name} must be a contiguous {np.dtype(dt).name} array (updated in place)")
    kb = _c(k_block, np.uint16)
    vb = _c(v_block, np.uint16)
    cu = _c(cu_block, np.int32)
    al = _c(accept_len, np.int32)
    pt = _c(page_table, np.int32)
    num_pages, Hkv, P, D = k_cache.shape
    B = cu.shape[0] - 1
    return lib.oracle_kv_append(_ptr(kb), _ptr(vb), _ptr(cu), _ptr(al), _ptr(prefix_lens),
                                int(bool(update_lens)), _ptr(pt), pt.shape[1], num_pages,
                                _ptr(k_cache), _ptr(v_cache), B, Hkv, D, P)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def accept_from_tokens(tokens, draft_tokens, cu_block):
    """The consensus rule on given greedy tokens: (accept_len[B], next_token[B])."""
    lib = _load()
    t = _c(tokens, np.int32)
    dr = _c(draft_tokens, np.int32)
    cu = _c(cu_block, np.int32)
    B = cu.shape[0] - 1
    if t.shape[0] < int(cu[-1]) or dr.shape[0] < int(cu[-1]):
        raise ValueError("inconsistent accept shapes")
    acc = np.zeros(B, np.int32)
    nxt = np.zeros(B, np.int32)
    lib.oracle_accept(_ptr(t), _ptr(dr), _ptr(cu), B, _ptr(acc), _ptr(nxt))
    return acc, nxt


def lm_head_logits(hidden, w_head, rows=None, with_absdot: bool = False,
                   threads: int | None = None):
    """fp64 scores of the AR view's LM head: logits[i, v] = <hidden[rows[i]], w_head[v]>.

    ``hidden`` [R, d] and ``w_head`` [V, d] are bf16 bit patterns (uint16).
    Returns logits [n, V] (and, with ``with_absdot``, the sums of |products|).
    """
    lib = _load()
    h = _c(hidden, np.uint16)
    w = _c(w_head, np.uint16)
    if h.ndim != 2 or w.ndim != 2 or h.shape[1] != w.shape[1]:
        raise ValueError("hidden [R, d] and w_head [V, d] expected")
    R, d = h.shape
    V = w.shape[0]
    r = np.arange(R, dtype=np.int64) if rows is None else _c(rows, np.int64)
    if r.size and (r.min() < 0 or r.max() >= R):
        raise ValueError("row index out of range")
    out = np.empty((r.shape[0], V), np.float64)
    ab = np.empty((r.shape[0], V), np.float64) if with_absdot else None
    rc = lib.oracle_lm_head(_ptr(h), _ptr(w), d, V, _ptr(r), r.shape[0], _ptr(out), _ptr(ab),
                            threads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle_lm_head: bad input (code {rc})")
    return (out, ab) if with_absdot else out


def greedy_tokens(logits64):
    """First index of the largest fp64 score per row (NaN as -inf)."""
    lib = _load()
    x = _c(logits64, np.float64)
    n, V = x.shape
    t = np.zeros(n, np.int32)
    lib.oracle_greedy_tokens(_ptr(x), n, V, _ptr(t))
    return t


def philox4x32_10(counter, key):
    """Philox4x32-10 of one 4-word counter under a 2-word key (uint32 words)."""
    lib = _load()
    c = _c(counter, np.uint32)
    k = _c(key, np.uint32)
    if c.shape != (4,) or k.shape != (2,):
        raise ValueError("counter has 4 words, key 2")
    out = np.zeros(4, np.uint32)
    lib.oracle_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def sampled_tokens(logits, temperature: float, seed: int, offset: int,
                   threads: int | None = None):
    """Gumbel-max samples of softmax(logits / T) per row (fp64 scores) and each
    row's margin between the winning score and the runner-up's."""
    lib = _load()
    x = np.ascontiguousarray(np.asarray(logits, dtype=np.float32))
    if x.ndim != 2:
        raise ValueError("logits must be [R, V]")
    R, V = x.shape
    t = np.zeros(R, np.int32)
    margin = np.zeros(R, np.float64)
    rc = lib.oracle_sampled_tokens(_ptr(x), V, V, R, float(temperature), int(seed) & (2**64 - 1),
                                   int(offset) & (2**64 - 1), _ptr(t), _ptr(margin),
                                   threads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle_sampled_tokens: bad input (code {rc})")
    return t, margin


def consensus_sampled(logits, draft_tokens, cu_block, temperature: float, seed: int, offset: int,
                      threads: int | None = None):
    """Consensus at temperature T > 0: (accept_len[B], next_token[B], tokens[R])."""
    lib = _load()
    x = np.ascontiguousarray(np.asarray(logits, dtype=np.float32))
    if x.ndim != 2:
        raise ValueError("logits must be [R, V]")
    R, V = x.shape
    dr = _c(draft_tokens, np.int32)
    cu = _c(cu_block, np.int32)
    B = cu.shape[0] - 1
    if dr.shape[0] != R or int(cu[-1]) != R:
        raise ValueError("inconsistent consensus shapes")
    acc = np.zeros(B, np.int32)
    nxt = np.zeros(B, np.int32)
    t = np.zeros(R, np.int32)
    rc = lib.oracle_consensus_sampled(_ptr(x), V, V, _ptr(dr), _ptr(cu), B, float(temperature),
                                      int(seed) & (2**64 - 1), int(offset) & (2**64 - 1),
                                      _ptr(acc), _ptr(nxt), _ptr(t), threads or default_threads())
    if rc != 0:
        raise ValueError(f"oracle_consensus_sampled: bad input (code {rc})")
    return acc, nxt, t
