"""Seeded synthetic inputs for the page indexer.

This module is shared by the tests, the benchmark and the oracle checks, and
holds none of the indexer's arithmetic: it only draws numbers.  It imports
neither the CUDA library nor the oracle.

Generator (all of it counter-based, so any slice can be drawn on its own):

* splitmix64: the i-th draw (i = 0, 1, ...) of stream ``s`` under seed ``S`` is
  ``mix64(key + (i + 1) * 0x9E3779B97F4A7C15)`` with
  ``key = mix64(S * 0x9E3779B97F4A7C15 + s)`` and ``mix64`` the splitmix64
  finaliser (shifts 30/27/31, multipliers 0xBF58476D1CE4E5B9 /
  0x94D049BB133111EB), all modulo 2^64.
* uniform in [0, 1): ``(x >> 11) * 2^-53`` (53-bit) or ``(x >> 40) * 2^-24``
  (24-bit, exact in fp32).
* normal: Box-Muller in double on consecutive draws (u1, u2):
  ``r = sqrt(-2 ln(1 - u1))``, ``z0 = r cos(2 pi u2)``, ``z1 = r sin(2 pi u2)``
  (host libm), rounded to fp32 (round-to-nearest-even), then to bf16 (RNE).

The workloads below are the five indexer configurations: a tiny decode batch,
a batch with per-page bias (heavy-tailed scores), the ragged decode batch, the
standalone top-K sweep over eleven score distributions, and the prefill chunk.
"""

from __future__ import annotations

import numpy as np

GOLDEN = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_MASK = (1 << 64) - 1
_CHUNK = 1 << 22  # draws per numpy block (bounds host memory)

BF16_NAN_POISON = 0xFFFF  # written into padded centroid rows


def _mix_int(z: int) -> int:
    z &= _MASK
    z = ((z ^ (z >> 30)) * _M1) & _MASK
    z = ((z ^ (z >> 27)) * _M2) & _MASK
    return z ^ (z >> 31)


def _mix_np(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * np.uint64(_M1)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(_M2)
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, stream: int) -> int:
    return _mix_int((seed * GOLDEN + stream) & _MASK)


def u64(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    """Draws start .. start+count-1 of stream ``stream`` under ``seed``."""
    key = np.uint64(stream_key(seed, stream))
    out = np.empty(count, np.uint64)
    with np.errstate(over="ignore"):
        for off in range(0, count, _CHUNK):
            n = min(_CHUNK, count - off)
            i = np.arange(start + off + 1, start + off + n + 1, dtype=np.uint64)
            out[off:off + n] = _mix_np(key + i * np.uint64(GOLDEN))
    return out


def uniform53(x: np.ndarray) -> np.ndarray:
    return (x >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def uniform24(x: np.ndarray) -> np.ndarray:
    return (x >> np.uint64(40)).astype(np.float64) * (2.0 ** -24)


def normal(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    """``count`` standard normals (double): numbers start .. start+count-1 of
    the stream's normal sequence (pair k = draws 2k, 2k+1)."""
    if start % 2:
        return normal(seed, stream, start - 1, count + 1)[1:]
    npairs = (count + 1) // 2
    out = np.empty(2 * npairs, np.float64)
    for off in range(0, npairs, _CHUNK // 2):
        n = min(_CHUNK // 2, npairs - off)
        x = u64(seed, stream, start + 2 * off, 2 * n)
        u1 = uniform53(x[0::2])
        u2 = uniform53(x[1::2])
        r = np.sqrt(-2.0 * np.log1p(-u1))
        th = 2.0 * np.pi * u2
        out[2 * off:2 * (off + n):2] = r * np.cos(th)
        out[2 * off + 1:2 * (off + n):2] = r * np.sin(th)
    return out[:count]


def f32_to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16, nearest-even; returns the uint16 bit patterns."""
    u = np.ascontiguousarray(x32, np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    return f32_to_bf16_bits(normal(seed, stream, start, count).astype(np.float32))


# --------------------------------------------------------------------------
# Indexer inputs: q [B][T][Q][D] bf16 bits, c [B][N][D] bf16 bits, lengths [B]
# --------------------------------------------------------------------------

def decode_inputs(seed, B, T, Q, D, N, lengths=None, len_range=None, page_bias=False,
                  poison_padding=True):
    """Indexer inputs for one workload.

    Streams: 0 = ragged lengths (drawn first), 1 = q, 2 = c, 3 = per-page bias.
    * ``lengths``: explicit int array, or None;
    * ``len_range=(lo, hi)``: len[b] uniform on the integers lo..hi inclusive
      (``lo + floor(u53 * (hi - lo + 1))``);
    * neither: every page valid (len = N).
    * ``page_bias``: c[b,p,d] = bf16(fp32(bf16(z)) + beta[b,p]) with
      beta[b,p] = bf16(0.5 * z') one scalar per page (one rounding of the fp32 sum).
    Padded pages (p >= len[b]) are filled with a bf16 NaN pattern when
    ``poison_padding`` so that any read of them would show in a score.
    """
    if lengths is None:
        if len_range is not None:
            lo, hi = len_range
            u = uniform53(u64(seed, 0, 0, B))
            lengths = lo + np.floor(u * (hi - lo + 1)).astype(np.int64)
        else:
            lengths = np.full(B, N, np.int64)
    lengths = np.asarray(lengths, np.int32)
    q = normal_bf16(seed, 1, 0, B * T * Q * D).reshape(B, T, Q, D)
    c = np.empty((B, N, D), np.uint16)
    for b in range(B):
        n_valid = int(min(max(lengths[b], 0), N))
        # each request owns the slice [b*N*D, (b+1)*N*D) of stream 2
        if page_bias:
            z = normal(seed, 2, b * N * D, n_valid * D).astype(np.float32)
            zb = bf16_bits_to_f32(f32_to_bf16_bits(z)).reshape(n_valid, D)
            beta = bf16_bits_to_f32(f32_to_bf16_bits(
                (0.5 * normal(seed, 3, b * N, max(n_valid, 1))[:n_valid]).astype(np.float32)))
            s = (zb + beta[:, None]).astype(np.float32)
            c[b, :n_valid] = f32_to_bf16_bits(s).reshape(n_valid, D)
        else:
            c[b, :n_valid] = normal_bf16(seed, 2, b * N * D, n_valid * D).reshape(n_valid, D)
        c[b, n_valid:] = BF16_NAN_POISON if poison_padding else 0
    return {"q": q, "c": c, "lengths": lengths}


def causal_token_lengths(pos0, T, page_tokens, N):
    """Valid page counts per (request, token) of a multi-token decode step.

    Request b has ``pos0[b]`` tokens of context before this step and decodes
    T new tokens; token t sits at position pos0[b] + t and sees the keys at
    positions 0 .. pos0[b] + t, i.e. the first ceil((pos0[b] + t + 1) /
    page_tokens) pages (capped at N).  This is the per-token "dead" tail of a
    multi-token chunk, with pages of ``page_tokens`` keys each.  Returns int32
    [B][T]; the last token's count is the request's page count."""
    pos0 = np.asarray(pos0, np.int64)
    t = np.arange(T, dtype=np.int64)
    n = (pos0[:, None] + t[None, :] + page_tokens) // page_tokens
    return np.minimum(n, N).astype(np.int32)


# --------------------------------------------------------------------------
# Standalone top-K sweep: fp32 score rows from eleven distributions
# --------------------------------------------------------------------------

DISTRIBUTIONS = (
    "normal", "uniform", "lognormal", "cauchy", "exponential", "bimodal",
    "levels16", "all_equal", "sorted_asc", "sorted_desc", "neg_inf_90",
)

SWEEP_ROWS = (1, 8, 32, 128)
SWEEP_N = (4096, 16384, 65536, 262144)


def score_rows(seed, rows, N, dist):
    """fp32 [rows][N] score rows of one distribution.

    Streams: 1 = the values (row r owns draws [r*N, (r+1)*N)); 2 = auxiliary
    draws (bimodal component, shuffle keys).
    * normal N(0,1); uniform U[0,1) (24-bit); lognormal exp(N(0,1));
      cauchy tan(pi (u - 1/2)); exponential -ln(1 - u);
      bimodal N(0,1) - 2 or + 2 with probability 1/2 each;
      levels16 floor(16 u) / 16; all_equal 1.0; sorted_asc / sorted_desc a
      sorted N(0,1) row; neg_inf_90: exactly floor(0.9 N) positions, the first
      of a seeded random permutation, set to -inf, the rest N(0,1).
    """
    out = np.empty((rows, N), np.float32)
    for r in range(rows):
        if dist in ("normal", "sorted_asc", "sorted_desc", "neg_inf_90", "bimodal",
                    "lognormal"):
            z = normal(seed, 1, r * N, N)
        if dist == "normal":
            v = z
        elif dist == "uniform":
            v = uniform24(u64(seed, 1, r * N, N))
        elif dist == "lognormal":
            v = np.exp(z)
        elif dist == "cauchy":
            v = np.tan(np.pi * (uniform53(u64(seed, 1, r * N, N)) - 0.5))
        elif dist == "exponential":
            v = -np.log1p(-uniform53(u64(seed, 1, r * N, N)))
        elif dist == "bimodal":
            side = uniform53(u64(seed, 2, r * N, N)) < 0.5
            v = z + np.where(side, -2.0, 2.0)
        elif dist == "levels16":
            v = np.floor(16.0 * uniform53(u64(seed, 1, r * N, N))) / 16.0
        elif dist == "all_equal":
            v = np.ones(N)
        elif dist == "sorted_asc":
            v = np.sort(z.astype(np.float32))
        elif dist == "sorted_desc":
            v = np.sort(z.astype(np.float32))[::-1]
        elif dist == "neg_inf_90":
            v = z.copy()
            perm = np.argsort(u64(seed, 2, r * N, N), kind="stable")
            v[perm[: (9 * N) // 10]] = -np.inf
        else:
            raise ValueError(dist)
        out[r] = np.asarray(v).astype(np.float32)
    return out


def sweep_cases():
    """(case number, rows, N, distribution) for the whole top-K sweep."""
    case = 0
    for rows in SWEEP_ROWS:
        for n in SWEEP_N:
            for dist in DISTRIBUTIONS:
                yield case, rows, n, dist
                case += 1


# --------------------------------------------------------------------------
# The five indexer workloads
# --------------------------------------------------------------------------

WORKLOADS = {
    "tiny_decode": dict(seed=101, B=1, T=1, Q=4, D=128, N=4096, K=256),
    "batch_decode_bias": dict(seed=102, B=8, T=1, Q=4, D=128, N=16384, K=256, page_bias=True),
    "ragged_decode": dict(seed=103, B=32, T=1, Q=4, D=128, N=65536, K=256,
                          len_range=(1024, 65536)),
    "prefill_chunk": dict(seed=105, B=4, T=16, Q=8, D=128, N=131072, K=512),
    # multi-token causal decode: 4 new tokens after a ragged context of
    # U{64*1024 .. 64*65536 - 4} keys, pages of 64 keys (token lengths drawn
    # from stream 4 of the seed)
    "causal_decode": dict(seed=106, B=32, T=4, Q=4, D=128, N=65536, K=256,
                          pos0_range=(64 * 1024, 64 * 65536 - 4), page_tokens=64),
}
SWEEP_SEED = 104


def workload(name, **override):
    """Inputs of a named indexer workload (``override`` changes any field)."""
    spec = dict(WORKLOADS[name])
    spec.update(override)
    K = spec.pop("K")
    if "pos0_range" in spec:
        lo, hi = spec.pop("pos0_range")
        page_tokens = spec.pop("page_tokens")
        u = uniform53(u64(spec["seed"], 4, 0, spec["B"]))
        pos0 = lo + np.floor(u * (hi - lo + 1)).astype(np.int64)
        tl = causal_token_lengths(pos0, spec["T"], page_tokens, spec["N"])
        inputs = decode_inputs(spec.pop("seed"), spec.pop("B"), spec.pop("T"), spec.pop("Q"),
                               spec.pop("D"), spec.pop("N"), lengths=tl[:, -1], **spec)
        inputs["token_lengths"] = tl
        inputs["K"] = K
        return inputs
    inputs = decode_inputs(spec.pop("seed"), spec.pop("B"), spec.pop("T"), spec.pop("Q"),
                           spec.pop("D"), spec.pop("N"), **spec)
    inputs["K"] = K
    return inputs


# --------------------------------------------------------------------------
# KMeans assignment inputs (the second workload)
# --------------------------------------------------------------------------

KMEANS = dict(seed=109, M=262144, C=1024, D=128)


def kmeans_inputs(seed, M, C, D, spread=0.5):
    """Clustered points for an assignment: centroids ~ N(0,1) (stream 1), each
    point a centroid chosen uniformly (stream 2) plus ``spread`` * N(0,1)
    noise (stream 3), rounded once to bf16.  Returns bf16 bits x [M][D],
    centroids [C][D] and the generating centroid of every point."""
    cf = normal(seed, 1, 0, C * D).astype(np.float32).reshape(C, D)
    cent = f32_to_bf16_bits(cf)
    cf = bf16_bits_to_f32(cent)
    pick = (u64(seed, 2, 0, M) % np.uint64(C)).astype(np.int64)
    noise = normal(seed, 3, 0, M * D).astype(np.float32).reshape(M, D)
    x = f32_to_bf16_bits((cf[pick] + np.float32(spread) * noise).astype(np.float32))
    return {"x": x, "centroids": cent, "pick": pick.astype(np.int32)}
