"""Thin Python binding of libidx.so (the C ABI in include/idx.h).

Argument marshalling only: every step of the indexer runs in the CUDA
library.  The functions keep the C names; tensors are torch CUDA tensors (bf16
inputs may be given as bfloat16, int16 or uint16 tensors), and the stream
defaults to torch's current stream on the tensor's device.

If libidx.so is missing the first call raises ``RuntimeError``: there is no
fallback of any kind.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libidx.so")

IDX_OK, IDX_EINVAL, IDX_EUNSUPPORTED, IDX_ENOWORKSPACE, IDX_ECUDA, IDX_EDEVICE = 0, -1, -2, -3, -4, -5
IDX_MAX_K = 2048

# Every symbol include/idx.h declares, with its ctypes signature.
_P = ctypes.c_void_p
_I = ctypes.c_int
_L = ctypes.c_int64
SIGNATURES = {
    "idx_init": (_I, [ctypes.POINTER(_P), _I, _I, _I, _I]),
    "idx_destroy": (_I, [_P]),
    "centroid_score": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _L, _P, _P]),
    "topk_select": (_I, [_P, _P, _P, _I, _I, _L, _I, _P, _P, _P]),
    "score_topk_fused": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _L, _I, _P, _P, _P]),
    "centroid_score_tokens": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _L, _P, _P]),
    "score_topk_fused_tokens": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _L, _I, _P, _P, _P]),
    "centroid_pool": (_I, [_P, _P, _P, _I, _I, _I, _I, _L, _P, _L, _P]),
    "centroid_score_paged": (_I, [_P, _P, _P, _I, _P, _L, _P, _I, _I, _I, _I, _I, _P, _P]),
    "score_topk_fused_paged": (_I, [_P, _P, _P, _I, _P, _L, _P, _I, _I, _I, _I, _I, _I, _P, _P,
                                    _P]),
    "idx_get_status": (_I, [_P, _P, ctypes.POINTER(_I)]),
    "idx_strerror": (ctypes.c_char_p, [_I]),
    "idx_num_sms": (_I, [_P]),
    "topk_select_noalloc": (_I, [_P, _P, _I, _I, _L, _I, _P, _P, _P]),
    "kmeans_assign": (_I, [_P, _P, _P, _I, _I, _I, _P, _P, _P]),
    "kmeans_scores": (_I, [_P, _P, _P, _I, _I, _I, _P, _P]),
}

_lib = None


class IdxError(RuntimeError):
    def __init__(self, code, what):
        self.code = code
        super().__init__("%s failed: %s (%d)" % (what, strerror(code), code))


def lib():
    """The loaded CDLL with argtypes set (raises if libidx.so was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libidx.so not found at %s: build it with "
                               "`python -m page_scoring_top_b200.build`" % LIB_PATH)
        dll = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(dll, name)
            fn.restype = res
            fn.argtypes = args
        _lib = dll
    return _lib


def strerror(code):
    return lib().idx_strerror(int(code)).decode()


def _check(rc, what):
    if rc != IDX_OK:
        raise IdxError(rc, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    if isinstance(stream, torch.cuda.Stream):
        stream = stream.cuda_stream
    return ctypes.c_void_p(int(stream))


class Context:
    """An idx_ctx: device, limits and the workspace allocated once by idx_init."""

    def __init__(self, device=0, max_rows=1, max_n=1, max_k=1):
        if isinstance(device, torch.device):
            device = device.index if device.index is not None else torch.cuda.current_device()
        self.device = int(device)
        self.max_rows, self.max_n, self.max_k = int(max_rows), int(max_n), int(max_k)
        handle = ctypes.c_void_p()
        _check(lib().idx_init(ctypes.byref(handle), self.device, self.max_rows, self.max_n,
                              self.max_k), "idx_init")
        self.handle = handle

    def close(self):
        if getattr(self, "handle", None) is not None and self.handle.value:
            _check(lib().idx_destroy(self.handle), "idx_destroy")
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    @property
    def num_sms(self):
        return lib().idx_num_sms(self.handle)


def idx_init(device, max_rows, max_n, max_k):
    return Context(device, max_rows, max_n, max_k)


def idx_destroy(ctx):
    ctx.close()


def _score_shapes(q, c):
    if q.dim() != 4 or c.dim() != 3:
        raise ValueError("q must be [B][T][Q][D] and c [B][N][D]")
    B, T, Q, D = q.shape
    Bc, N, Dc = c.shape
    if Bc != B or Dc != D:
        raise ValueError("q and c disagree on B or D")
    if not q.is_contiguous() or c.stride(2) != 1 or c.stride(1) != D:
        raise ValueError("q must be contiguous and c's pages contiguous rows of D")
    return B, T, Q, D, N, c.stride(0)


def centroid_score(ctx, q, c, lengths, scores, stream=None):
    """scores[b][t][p] (fp32 [B][T][N]) = sum_h q[b,t,h,:] . c[b,p,:]; -inf past lengths."""
    B, T, Q, D, N, ldc = _score_shapes(q, c)
    if tuple(scores.shape) != (B, T, N) or scores.dtype != torch.float32 or not scores.is_contiguous():
        raise ValueError("scores must be contiguous fp32 [B][T][N]")
    _check(lib().centroid_score(ctx.handle, _ptr(q), _ptr(c), _ptr(lengths), B, T, Q, D, N, ldc,
                                _ptr(scores), _stream(stream, q.device)), "centroid_score")
    return scores


def topk_select(ctx, scores, lengths, K, idx_out, val_out=None, stream=None):
    """Top-K of each row of a 2-D fp32 tensor (row stride = scores.stride(0))."""
    if scores.dim() != 2 or scores.stride(1) != 1:
        raise ValueError("scores must be 2-D with unit column stride")
    rows, N = scores.shape
    _check(lib().topk_select(ctx.handle, _ptr(scores), _ptr(lengths), rows, N, scores.stride(0), K,
                             _ptr(idx_out), _ptr(val_out), _stream(stream, scores.device)),
           "topk_select")
    return idx_out, val_out


def topk_select_noalloc(scores, lengths, K, idx_out, val_out=None, stream=None):
    """topk_select without a context: scratch in a static device array (see idx.h)."""
    if scores.dim() != 2 or scores.stride(1) != 1:
        raise ValueError("scores must be 2-D with unit column stride")
    rows, N = scores.shape
    # the C call works on the current device: make it the one holding the data
    with torch.cuda.device(scores.device):
        _check(lib().topk_select_noalloc(_ptr(scores), _ptr(lengths), rows, N, scores.stride(0),
                                         K, _ptr(idx_out), _ptr(val_out),
                                         _stream(stream, scores.device)),
               "topk_select_noalloc")
    return idx_out, val_out


def score_topk_fused(ctx, q, c, lengths, K, idx_out, val_out=None, stream=None):
    """idx_out[b*T+t] = top-K pages of request b for token t (int32 [B*T][K])."""
    B, T, Q, D, N, ldc = _score_shapes(q, c)
    _check(lib().score_topk_fused(ctx.handle, _ptr(q), _ptr(c), _ptr(lengths), B, T, Q, D, N, ldc,
                                  K, _ptr(idx_out), _ptr(val_out), _stream(stream, q.device)),
           "score_topk_fused")
    return idx_out, val_out


def _token_lengths(token_lengths, B, T):
    if (tuple(token_lengths.shape) not in ((B, T), (B * T,)) or token_lengths.dtype != torch.int32
            or not token_lengths.is_contiguous()):
        raise ValueError("token_lengths must be contiguous int32 [B][T]")
    return token_lengths


def centroid_score_tokens(ctx, q, c, token_lengths, scores, stream=None):
    """centroid_score with a valid page count per (request, token) row."""
    B, T, Q, D, N, ldc = _score_shapes(q, c)
    _token_lengths(token_lengths, B, T)
    if tuple(scores.shape) != (B, T, N) or scores.dtype != torch.float32 or not scores.is_contiguous():
        raise ValueError("scores must be contiguous fp32 [B][T][N]")
    _check(lib().centroid_score_tokens(ctx.handle, _ptr(q), _ptr(c), _ptr(token_lengths), B, T, Q,
                                       D, N, ldc, _ptr(scores), _stream(stream, q.device)),
           "centroid_score_tokens")
    return scores


def score_topk_fused_tokens(ctx, q, c, token_lengths, K, idx_out, val_out=None, stream=None):
    """score_topk_fused with a valid page count per (request, token) row."""
    B, T, Q, D, N, ldc = _score_shapes(q, c)
    _token_lengths(token_lengths, B, T)
    _check(lib().score_topk_fused_tokens(ctx.handle, _ptr(q), _ptr(c), _ptr(token_lengths), B, T,
                                         Q, D, N, ldc, K, _ptr(idx_out), _ptr(val_out),
                                         _stream(stream, q.device)),
           "score_topk_fused_tokens")
    return idx_out, val_out


def idx_get_status(ctx, stream=None):
    """(status code, raised bits) of the context; synchronises the stream."""
    bits = ctypes.c_int(0)
    rc = lib().idx_get_status(ctx.handle, _stream(stream, torch.device("cuda", ctx.device)),
                              ctypes.byref(bits))
    return rc, bits.value


def centroid_pool(ctx, keys, key_counts, P, c, stream=None):
    """c[b,p,:] = bf16 mean of the valid keys of page p (P keys per page).
    keys: bf16 bits (int16) [B][L][D]; key_counts: int32 [B]; c: int16 [B][N][D]."""
    if keys.dim() != 3 or keys.dtype != torch.int16 or not keys.is_contiguous():
        raise ValueError("keys must be contiguous bf16 bits (int16) [B][L][D]")
    B, Lk, D = keys.shape
    if c.dim() != 3 or c.dtype != torch.int16 or not c.is_contiguous() or c.shape[0] != B \
            or c.shape[2] != D:
        raise ValueError("c must be contiguous bf16 bits (int16) [B][N][D]")
    N = c.shape[1]
    if tuple(key_counts.shape) != (B,) or key_counts.dtype != torch.int32:
        raise ValueError("key_counts must be int32 [B]")
    _check(lib().centroid_pool(ctx.handle, _ptr(keys), _ptr(key_counts), B, D, P, N, Lk * D,
                               _ptr(c), N * D, _stream(stream, keys.device)), "centroid_pool")
    return c


def _kmeans_shapes(x, centroids):
    for name, t in (("x", x), ("centroids", centroids)):
        if t.dim() != 2 or t.dtype not in (torch.int16, torch.bfloat16) or not t.is_contiguous():
            raise ValueError("%s must be contiguous bf16 (or its int16 bits) [rows][D]" % name)
    M, D = x.shape
    C, Dc = centroids.shape
    if Dc != D:
        raise ValueError("x and centroids differ in D")
    return M, C, D


def kmeans_assign(ctx, x, centroids, assign_out, score_out=None, stream=None):
    """assign_out[i] = nearest centroid of point i (int32 [M]); score_out, if
    given, gets the winning x.c - |c|^2/2 (fp32 [M])."""
    M, C, D = _kmeans_shapes(x, centroids)
    _check(lib().kmeans_assign(ctx.handle, _ptr(x), _ptr(centroids), M, C, D, _ptr(assign_out),
                               _ptr(score_out), _stream(stream, x.device)), "kmeans_assign")
    return assign_out, score_out


def kmeans_scores(ctx, x, centroids, scores, stream=None):
    """scores[i, c] = x_i.c - |c|^2/2 (fp32 [M][C])."""
    M, C, D = _kmeans_shapes(x, centroids)
    if tuple(scores.shape) != (M, C) or scores.dtype != torch.float32 or not scores.is_contiguous():
        raise ValueError("scores must be contiguous fp32 [M][C]")
    _check(lib().kmeans_scores(ctx.handle, _ptr(x), _ptr(centroids), M, C, D, _ptr(scores),
                               _stream(stream, x.device)), "kmeans_scores")
    return scores


def _paged_shapes(q, pool, page_table):
    if q.dim() != 4 or q.dtype != torch.int16 or not q.is_contiguous():
        raise ValueError("q must be contiguous bf16 bits (int16) [B][T][Q][D]")
    if pool.dim() != 2 or pool.dtype != torch.int16 or not pool.is_contiguous():
        raise ValueError("pool must be contiguous bf16 bits (int16) [n_blocks][D]")
    if page_table.dim() != 2 or page_table.dtype != torch.int32 or not page_table.is_contiguous():
        raise ValueError("page_table must be contiguous int32 [B][N]")
    B, T, Q, D = q.shape
    if pool.shape[1] != D or page_table.shape[0] != B:
        raise ValueError("shape mismatch")
    return B, T, Q, D, page_table.shape[1], pool.shape[0]


def centroid_score_paged(ctx, q, pool, page_table, lengths, scores, stream=None):
    """centroid_score with page p of request b read from pool[page_table[b, p]]."""
    B, T, Q, D, N, nb = _paged_shapes(q, pool, page_table)
    if tuple(scores.shape) != (B, T, N) or scores.dtype != torch.float32 or not scores.is_contiguous():
        raise ValueError("scores must be contiguous fp32 [B][T][N]")
    _check(lib().centroid_score_paged(ctx.handle, _ptr(q), _ptr(pool), nb, _ptr(page_table), N,
                                      _ptr(lengths), B, T, Q, D, N, _ptr(scores),
                                      _stream(stream, q.device)), "centroid_score_paged")
    return scores


def score_topk_fused_paged(ctx, q, pool, page_table, lengths, K, idx_out, val_out=None,
                           stream=None):
    """score_topk_fused with page p of request b read from pool[page_table[b, p]]."""
    B, T, Q, D, N, nb = _paged_shapes(q, pool, page_table)
    _check(lib().score_topk_fused_paged(ctx.handle, _ptr(q), _ptr(pool), nb, _ptr(page_table), N,
                                        _ptr(lengths), B, T, Q, D, N, K, _ptr(idx_out),
                                        _ptr(val_out), _stream(stream, q.device)),
           "score_topk_fused_paged")
    return idx_out, val_out
