"""CPU oracle of the page indexer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package.  The product path
(``page_scoring_top_b200``) never imports it, and this package imports nothing
from the product: the two meet only at the seeded inputs.

The arithmetic lives in ``oracle.c`` (plain C, single-threaded, double
precision, explicit loops, a library sort); this module only compiles it with
gcc, marshals numpy arrays into it, and states the two acceptance measures the
pages name:

* the score bound ``|s_gpu - S| <= 1e-5 * A`` per valid entry, with S the exact
  (double) score and A = sum_h sum_d |q_hd * c_pd| its scale;
* recall@m ("Iterate Topk", benchmark protocol: recall is reported at
  floor(3K/4) and at K) = |GPU top-m  intersect  oracle top-m| / min(m, #selectable).

Every function states the passage of the pages it follows in ``oracle.c``.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

SCORE_REL_BOUND = 1e-5  # |s_gpu - S| <= SCORE_REL_BOUND * A, per entry


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` (gcc, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
             "-fPIC", "-shared", "-fvisibility=hidden", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        L = ctypes.c_int64
        lib.oracle_scores.argtypes = [P, P, P, I, I, I, I, I, L, P, P]
        lib.oracle_scores_tokens.argtypes = [P, P, P, I, I, I, I, I, L, P, P]
        lib.oracle_pool.argtypes = [P, P, I, I, I, I, L, P]
        lib.oracle_kmeans_assign.argtypes = [P, P, I, I, I, P, P, P, P]
        lib.oracle_argmax_rows_f32.argtypes = [P, I, I, P]
        lib.oracle_topk_f64.argtypes = [P, I, I, P, P]
        lib.oracle_topk_f32.argtypes = [P, I, I, P, P]
        lib.oracle_topk_rows_f32.argtypes = [P, P, I, I, L, I, P, P]
        lib.oracle_topk_rows_f64.argtypes = [P, P, I, I, L, I, P, P]
        for f in ("oracle_scores", "oracle_scores_tokens", "oracle_pool", "oracle_topk_f64",
                  "oracle_topk_f32", "oracle_topk_rows_f32", "oracle_topk_rows_f64",
                  "oracle_kmeans_assign", "oracle_argmax_rows_f32"):
            getattr(lib, f).restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def scores(q_bits, c_bits, lengths=None):
    """Exact scores S and bound scales A, both double [B][T][N].

    ``q_bits``: uint16 bf16 patterns [B][T][Q][D]; ``c_bits``: uint16 [B][N][D];
    ``lengths``: int32 [B] in [0, N], int32 [B][T] (a valid page count per
    token: multi-token causal decode), or None (all valid).
    """
    q = _c(q_bits, np.uint16)
    c = _c(c_bits, np.uint16)
    B, T, Q, D = q.shape
    Bc, N, Dc = c.shape
    assert Bc == B and Dc == D
    S = np.empty((B, T, N), np.float64)
    A = np.empty((B, T, N), np.float64)
    if lengths is not None and np.ndim(lengths) == 2:
        # per (request, token) valid page counts: multi-token causal decode
        ln = _c(lengths, np.int32)
        assert ln.shape == (B, T)
        rc = _load().oracle_scores_tokens(_ptr(q), _ptr(c), _ptr(ln), B, T, Q, D, N, N * D,
                                          _ptr(S), _ptr(A))
    else:
        ln = None if lengths is None else _c(lengths, np.int32)
        rc = _load().oracle_scores(_ptr(q), _ptr(c), _ptr(ln), B, T, Q, D, N, N * D,
                                   _ptr(S), _ptr(A))
    if rc != 0:
        raise ValueError("oracle_scores: arguments outside the contract")
    return S, A


def pool(key_bits, key_counts, P, N):
    """Exact page centroids (double [B][N][D]): the mean of each page's valid
    keys; ``key_bits`` uint16 bf16 [B][L][D], ``key_counts`` int32 [B] (<= L,
    <= N*P), pages of P keys."""
    k = _c(key_bits, np.uint16)
    B, L, D = k.shape
    kc = _c(key_counts, np.int32)
    means = np.empty((B, N, D), np.float64)
    rc = _load().oracle_pool(_ptr(k), _ptr(kc), B, D, P, N, L * D, _ptr(means))
    if rc != 0:
        raise ValueError("oracle_pool: arguments outside the contract")
    return means


def scores_paged(q_bits, pool_bits, page_table, lengths=None):
    """Scores when page p of request b is row page_table[b, p] of a shared
    block pool (the block-pool table of "Iterate Centroids Score"): the
    gather is a library fancy index, the arithmetic is ``scores``'s."""
    pool = _c(pool_bits, np.uint16)
    pt = np.asarray(page_table)
    B, N = pt.shape
    live = np.ones((B, N), bool)
    if lengths is not None:
        live = np.arange(N)[None, :] < np.asarray(lengths)[:, None]
    # The page only defines a table of valid block ids: an id outside the pool
    # on a live page has no meaning, so it is an error here, not a value.
    if np.any(live & ((pt < 0) | (pt >= pool.shape[0]))):
        raise ValueError("scores_paged: page-table entry outside the block pool")
    gathered = pool[np.where(live, pt, 0)]  # [B][N][D]; dead pages read block 0, then masked
    gathered = np.where(live[:, :, None], gathered, np.uint16(0))
    return scores(q_bits, gathered, lengths)


def kmeans_assign(x_bits, c_bits, full=False):
    """Nearest centroid of every point (the KMeans assignment of "Export Cake
    KMeans plan-runtime suite"): argmax_c (x.c - |c|^2/2) in double, ties to
    the lower centroid.  ``x_bits`` uint16 bf16 [M][D], ``c_bits`` [C][D].
    Returns (assign int32 [M], best double [M]) and, with ``full``, also the
    score matrix S and its error-bound scale A, double [M][C]."""
    x = _c(x_bits, np.uint16)
    c = _c(c_bits, np.uint16)
    M, D = x.shape
    C, Dc = c.shape
    assert Dc == D
    assign = np.empty(M, np.int32)
    best = np.empty(M, np.float64)
    S = np.empty((M, C), np.float64) if full else None
    A = np.empty((M, C), np.float64) if full else None
    rc = _load().oracle_kmeans_assign(_ptr(x), _ptr(c), M, C, D, _ptr(assign), _ptr(best),
                                      _ptr(S), _ptr(A))
    if rc != 0:
        raise ValueError("oracle_kmeans_assign: arguments outside the contract")
    return (assign, best, S, A) if full else (assign, best)


def argmax_rows(scores_f32):
    """Column of the largest entry of every row of an fp32 matrix (ties to the
    lower column, NaN never wins)."""
    s = _c(scores_f32, np.float32)
    M, C = s.shape
    arg = np.empty(M, np.int32)
    rc = _load().oracle_argmax_rows_f32(_ptr(s), M, C, _ptr(arg))
    if rc != 0:
        raise ValueError("oracle_argmax_rows_f32: arguments outside the contract")
    return arg


def topk(row, K, length=None):
    """Top-K of one row (float32 or float64).  Returns (idx int32[K], val[K], K')."""
    row = np.asarray(row)
    n = row.shape[0] if length is None else int(length)
    idx = np.empty(K, np.int32)
    if row.dtype == np.float32:
        r = _c(row, np.float32)
        val = np.empty(K, np.float32)
        kk = _load().oracle_topk_f32(_ptr(r), n, K, _ptr(idx), _ptr(val))
    else:
        r = _c(row, np.float64)
        val = np.empty(K, np.float64)
        kk = _load().oracle_topk_f64(_ptr(r), n, K, _ptr(idx), _ptr(val))
    if kk < 0:
        raise ValueError("oracle_topk: arguments outside the contract")
    return idx, val, kk


def topk_rows(scores_2d, K, lengths=None):
    """Top-K of every row of a [rows][N] array; lengths per row or None."""
    s = np.asarray(scores_2d)
    rows, N = s.shape
    ln = None if lengths is None else _c(lengths, np.int32)
    idx = np.empty((rows, K), np.int32)
    if s.dtype == np.float32:
        s = _c(s, np.float32)
        val = np.empty((rows, K), np.float32)
        rc = _load().oracle_topk_rows_f32(_ptr(s), _ptr(ln), rows, N, N, K, _ptr(idx), _ptr(val))
    else:
        s = _c(s, np.float64)
        val = np.empty((rows, K), np.float64)
        rc = _load().oracle_topk_rows_f64(_ptr(s), _ptr(ln), rows, N, N, K, _ptr(idx), _ptr(val))
    if rc != 0:
        raise ValueError("oracle_topk_rows: arguments outside the contract")
    return idx, val


def score_bound_violations(s_gpu, S, A, rel=SCORE_REL_BOUND):
    """Number of entries breaking the score bound.

    Valid entries (S finite) need |s_gpu - S| <= rel * A; padded entries
    (S == -inf) need s_gpu == -inf exactly.
    """
    s_gpu = np.asarray(s_gpu, np.float64)
    S = np.asarray(S, np.float64)
    A = np.asarray(A, np.float64)
    pad = np.isneginf(S)
    bad_pad = np.count_nonzero(pad & ~np.isneginf(s_gpu))
    with np.errstate(invalid="ignore"):
        err = np.abs(s_gpu - S)
    bad_val = np.count_nonzero(~pad & ~(err <= rel * A))
    return int(bad_pad + bad_val)


def recall(gpu_idx, oracle_idx, m):
    """recall@m of one row: |GPU top-m & oracle top-m| / min(m, #selectable).

    Both inputs are index lists in rank order, padded with -1 past K'.
    Returns 1.0 when nothing is selectable.
    """
    g = np.asarray(gpu_idx)[:m]
    o = np.asarray(oracle_idx)[:m]
    o = o[o >= 0]
    g = g[g >= 0]
    if o.size == 0:
        return 1.0
    return np.intersect1d(g, o).size / float(o.size)
