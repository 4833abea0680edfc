"""GPU parity: the CUDA path (called through the C ABI) against the CPU oracle.

Bars:
* scores: |s_gpu - S| <= 1e-5 * sum_h sum_d |q*c| per valid entry, -inf exactly
  on padding;
* indices: bit-exact against the oracle's select run on the GPU's own fp32
  scores; values bit-equal to those scores;
* recall@floor(3K/4) and recall@K against the oracle's double-precision top-K
  >= 0.999.
Small cases span several tiles and a ragged tail; output slots are poisoned
with 0xa5 before each call so an unwritten slot shows.
"""

import numpy as np
import pytest

import oracle
from page_scoring_top_b200 import synth
from helpers import (check_recall, check_select_bit_exact, poisoned_outputs, to_dev,
                     to_dev_bf16)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def ctx():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from page_scoring_top_b200 import binding
    c = binding.Context(0, max_rows=256, max_n=262144, max_k=2048)
    yield c
    c.close()


def _status_clean(ctx):
    from page_scoring_top_b200 import binding
    rc, bits = binding.idx_get_status(ctx)
    assert rc == 0 and bits == 0, "device status raised: %d" % bits


def run_scores(ctx, d):
    from page_scoring_top_b200 import binding
    B, T, Q, D = d["q"].shape
    N = d["c"].shape[1]
    q, c = to_dev_bf16(d["q"]), to_dev_bf16(d["c"])
    ln = to_dev(d["lengths"])
    s = torch.full((B, T, N), 12345.0, device="cuda")
    binding.centroid_score(ctx, q, c, ln, s)
    return s.cpu().numpy()


def run_fused(ctx, d, K):
    from page_scoring_top_b200 import binding
    B, T, Q, D = d["q"].shape
    q, c = to_dev_bf16(d["q"]), to_dev_bf16(d["c"])
    ln = to_dev(d["lengths"])
    idx, val = poisoned_outputs(B * T, K)
    binding.score_topk_fused(ctx, q, c, ln, K, idx, val)
    return idx.cpu().numpy(), val.cpu().numpy()


def check_indexer(ctx, d, K, recall_floor=0.999):
    B, T, Q, D = d["q"].shape
    N = d["c"].shape[1]
    s_gpu = run_scores(ctx, d)
    S, A = oracle.scores(d["q"], d["c"], d["lengths"])
    assert oracle.score_bound_violations(s_gpu, S, A) == 0
    idx, val = run_fused(ctx, d, K)
    rows_len = np.repeat(d["lengths"], T)
    check_select_bit_exact(s_gpu.reshape(B * T, N), rows_len, K, idx, val)
    check_recall(idx, S.reshape(B * T, N), rows_len, K, recall_floor)
    _status_clean(ctx)


# ------------------------------------------------------------------ scoring + fused, small shapes

@pytest.mark.parametrize("D", [128, 64, 256, 8, 96])
@pytest.mark.parametrize("Q", [4, 1, 8])
def test_decode_shapes(ctx, D, Q):
    d = synth.decode_inputs(200 + D + Q, B=3, T=1, Q=Q, D=D, N=3000, lengths=[3000, 1777, 33])
    check_indexer(ctx, d, K=64)


@pytest.mark.parametrize("T", [1, 2, 3, 4, 5])
def test_multi_token_decode(ctx, T):
    d = synth.decode_inputs(300 + T, B=2, T=T, Q=4, D=128, N=2500, lengths=[2500, 901])
    check_indexer(ctx, d, K=100)


@pytest.mark.parametrize("K", [1, 7, 256, 1000, 2048])
def test_k_values(ctx, K):
    d = synth.decode_inputs(400 + K, B=4, T=1, Q=4, D=128, N=9000,
                            lengths=[9000, 4097, 2048, 5])
    check_indexer(ctx, d, K=K)


def test_ragged_many_requests(ctx):
    # many short rows (chunks span many requests), empty rows, single-page rows
    rng = np.random.default_rng(5)
    lengths = rng.integers(0, 700, 200).astype(np.int32)
    lengths[[0, 17, 199]] = 0
    lengths[[3, 4]] = 1
    lengths[5] = 700
    d = synth.decode_inputs(500, B=200, T=1, Q=4, D=128, N=700, lengths=lengths)
    check_indexer(ctx, d, K=32)


def test_all_rows_empty(ctx):
    d = synth.decode_inputs(501, B=3, T=2, Q=4, D=128, N=64, lengths=[0, 0, 0])
    s = run_scores(ctx, d)
    assert np.all(np.isneginf(s))
    idx, val = run_fused(ctx, d, 16)
    assert np.all(idx == -1) and np.all(np.isneginf(val))


def test_long_rows_many_chunks(ctx):
    # rows longer than a CTA's on-chip score capacity: multi-chunk rows and merges
    d = synth.decode_inputs(502, B=2, T=1, Q=4, D=128, N=200000, lengths=[200000, 150001])
    check_indexer(ctx, d, K=256)


def test_heavy_ties_in_scores(ctx):
    # all-zero q: every score is +-0, so the select is decided by ties alone
    d = synth.decode_inputs(503, B=2, T=1, Q=4, D=128, N=5000, lengths=[5000, 3000])
    d["q"][:] = 0
    s = run_scores(ctx, d)
    assert np.all(s[0, 0] == 0) and np.all(s[1, 0, :3000] == 0)
    idx, _ = run_fused(ctx, d, 300)
    assert list(idx[0]) == list(range(300)) and list(idx[1]) == list(range(300))


def test_fused_without_values(ctx):
    from page_scoring_top_b200 import binding
    d = synth.decode_inputs(504, B=2, T=1, Q=4, D=128, N=4000, lengths=[4000, 2500])
    idx_v, _ = run_fused(ctx, d, 50)
    idx = torch.full((2, 50), -7, dtype=torch.int32, device="cuda")
    binding.score_topk_fused(ctx, to_dev_bf16(d["q"]), to_dev_bf16(d["c"]), to_dev(d["lengths"]),
                             50, idx, None)
    assert np.array_equal(idx.cpu().numpy(), idx_v)


def test_repeat_calls_are_identical(ctx):
    # counters reset by the kernels themselves: back-to-back calls agree
    d = synth.decode_inputs(505, B=4, T=1, Q=4, D=128, N=30000, len_range=(1000, 30000))
    a = run_fused(ctx, d, 256)
    for _ in range(3):
        b = run_fused(ctx, d, 256)
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1].view(np.uint32),
                                                             b[1].view(np.uint32))


# ------------------------------------------------------------------ standalone top-K

@pytest.mark.parametrize("dist", synth.DISTRIBUTIONS)
@pytest.mark.parametrize("N", [1, 255, 2049, 20000])
def test_topk_distributions(ctx, dist, N):
    from page_scoring_top_b200 import binding
    rows = 5
    s = synth.score_rows(600 + N, rows, N, dist)
    lengths = np.array([N, max(N - 1, 0), N // 2, 1, 0], np.int32)
    for K in (1, 64, 256):
        idx, val = poisoned_outputs(rows, K)
        binding.topk_select(ctx, to_dev(s), to_dev(lengths), K, idx, val)
        check_select_bit_exact(s, lengths, K, idx.cpu().numpy(), val.cpu().numpy())
    _status_clean(ctx)


def test_topk_row_stride_and_null_lengths(ctx):
    from page_scoring_top_b200 import binding
    s = synth.score_rows(700, 6, 5003, "normal")
    big = np.full((6, 5120), 7.0, np.float32)
    big[:, :5003] = s
    dev = to_dev(big)[:, :5003]
    idx, val = poisoned_outputs(6, 128)
    binding.topk_select(ctx, dev, None, 128, idx, val)
    check_select_bit_exact(s, None, 128, idx.cpu().numpy(), val.cpu().numpy())


def test_topk_signed_zero_and_nan(ctx):
    from page_scoring_top_b200 import binding
    row = np.array([0.0, -0.0, np.nan, -0.0, 1.0, -np.inf, 0.0, np.nan], np.float32)
    s = np.tile(row, (2, 1))
    idx, val = poisoned_outputs(2, 6)
    binding.topk_select(ctx, to_dev(s), None, 6, idx, val)
    got = idx.cpu().numpy()
    assert list(got[0]) == [4, 0, 1, 3, 6, -1]
    v = val.cpu().numpy()
    assert v[0, 2].tobytes() == np.float32(-0.0).tobytes()   # the row's own -0 bits


# ------------------------------------------------------------------ the ABI's error paths

def test_abi_errors(ctx):
    from page_scoring_top_b200 import binding
    L = binding.lib()
    d = synth.decode_inputs(800, B=2, T=1, Q=4, D=128, N=64)
    q, c = to_dev_bf16(d["q"]), to_dev_bf16(d["c"])
    s = torch.empty((2, 1, 64), device="cuda")
    h = ctx.handle
    st = None
    P = lambda t: None if t is None else t.data_ptr()
    assert L.centroid_score(h, None, P(c), None, 2, 1, 4, 128, 64, 64 * 128, P(s), st) == -1
    assert L.centroid_score(h, P(q), P(c), None, 2, 1, 4, 12, 64, 64 * 16, P(s), st) == -2
    assert L.centroid_score(h, P(q), P(c), None, 2, 1, 4, 264, 16, 16 * 264, P(s), st) == -2
    assert L.centroid_score(h, P(q), P(c), None, 2, 1, 4, 128, 64, 64 * 128 - 8, P(s), st) == -1
    assert L.centroid_score(h, P(q) + 2, P(c), None, 2, 1, 4, 128, 64, 64 * 128, P(s), st) == -1
    assert L.centroid_score(h, P(q), P(c), None, 2, 1, 4, 128, 300000, 300000 * 128, P(s), st) == -3
    idx = torch.empty((2, 16), dtype=torch.int32, device="cuda")
    flat = s.view(2, 64)
    assert L.topk_select(h, P(flat), None, 2, 64, 64, 0, P(idx), None, st) == -1
    assert L.topk_select(h, P(flat), None, 2, 64, 64, 4096, P(idx), None, st) == -2
    assert L.topk_select(h, P(flat), None, 2, 64, 32, 16, P(idx), None, st) == -1
    assert L.topk_select(h, P(flat), None, 1000, 64, 64, 16, P(idx), None, st) == -3
    assert L.score_topk_fused(h, P(q), P(c), None, 2, 1, 4, 128, 64, 64 * 128, 16, None, None, st) == -1
    assert L.score_topk_fused(None, P(q), P(c), None, 2, 1, 4, 128, 64, 64 * 128, 16, P(idx), None, st) == -1
    torch.cuda.synchronize()
    _status_clean(ctx)


def test_length_out_of_range_is_clamped_and_reported(ctx):
    from page_scoring_top_b200 import binding
    d = synth.decode_inputs(801, B=2, T=1, Q=4, D=128, N=300, lengths=[300, 300])
    ref_idx, ref_val = run_fused(ctx, d, 10)
    ln = to_dev(np.array([400, -5], np.int32))
    idx, val = poisoned_outputs(2, 10)
    binding.score_topk_fused(ctx, to_dev_bf16(d["q"]), to_dev_bf16(d["c"]), ln, 10, idx, val)
    rc, bits = binding.idx_get_status(ctx)
    assert rc == binding.IDX_EDEVICE and bits & 1
    got = idx.cpu().numpy()
    assert np.array_equal(got[0], ref_idx[0])        # 400 clamped to N = 300
    assert np.all(got[1] == -1)                      # -5 clamped to 0 pages
    _status_clean(ctx)


# ------------------------------------------------------------------ fused select, adversarial orders

def _ordered_inputs(order, B, N, lengths, seed):
    """Inputs whose scores are set by two centroid coordinates: q puts 1 on
    dim 0 and 2^-8 on dim 1 of head 0 (zeros elsewhere), so every score is
    c[p,0] + c[p,1] / 256 exactly in fp32.  Orders:
    ascending / descending: strictly monotone scores along the row (each page
        beats every earlier one, or none), the worst and best visiting orders
        of an online filter;
    one_bin: all scores in [1, 1 + 1/256): one 12-bit digit bin, ~128 distinct
        values, so the boundary bin is crowded and ties are everywhere;
    few_values: scores in {-1, 0, 1, 2}."""
    d = synth.decode_inputs(seed, B=B, T=1, Q=4, D=128, N=N, lengths=lengths)
    q = np.zeros_like(d["q"])
    q[:, :, 0, 0] = 0x3F80          # 1.0
    q[:, :, 0, 1] = 0x3B80          # 2^-8
    d["q"] = q
    rng = np.random.default_rng(seed)
    c = d["c"]
    for b in range(B):
        n = int(lengths[b])
        c[b, :n, :] = 0
        p = np.arange(n)
        if order == "ascending":
            c[b, :n, 0] = 0x3F80 + (p % 16000)      # bf16 patterns, increasing
            c[b, :n, 1] = 0
        elif order == "descending":
            c[b, :n, 0] = 0x3F80 + ((n - 1 - p) % 16000)
        elif order == "one_bin":
            c[b, :n, 0] = 0x3F80
            c[b, :n, 1] = 0x3F00 + rng.integers(0, 128, n)  # bf16 in [0.5, 1)
        else:
            c[b, :n, 0] = np.array([0xBF80, 0x0000, 0x3F80, 0x4000], np.uint16)[
                rng.integers(0, 4, n)]
    return d


@pytest.mark.parametrize("order", ["ascending", "descending", "one_bin", "few_values"])
@pytest.mark.parametrize("K", [256, 1000])
def test_fused_adversarial_orders_long_rows(ctx, order, K):
    lengths = np.array([16000, 15001], np.int32)
    d = _ordered_inputs(order, 2, 16000, lengths, 610)
    check_indexer(ctx, d, K=K)


@pytest.mark.parametrize("order", ["ascending", "one_bin", "few_values"])
def test_fused_adversarial_orders_short_rows(ctx, order):
    rng = np.random.default_rng(611)
    lengths = rng.integers(1, 3000, 64).astype(np.int32)
    d = _ordered_inputs(order, 64, 3000, lengths, 612)
    check_indexer(ctx, d, K=300)
