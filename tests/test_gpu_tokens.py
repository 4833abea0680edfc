"""GPU parity of the per-token calls (multi-token causal decode): scores and
fused selection against the CPU oracle, with a valid page count per
(request, token) row.

Bars as in test_gpu_parity: scores within 1e-5 * sum |q*c| (exactly -inf past
each token's count), indices bit-exact against the oracle's select of the
GPU's own fp32 scores, values bit-equal to those scores, recall >= 0.999
against the oracle's double scores."""

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
    c = binding.Context(0, max_rows=512, max_n=70000, max_k=1024)
    yield c
    c.close()


def _inputs(seed, B, T, Q, D, N, pos0, page_tokens):
    tl = synth.causal_token_lengths(pos0, T, page_tokens, N)
    d = synth.decode_inputs(seed, B=B, T=T, Q=Q, D=D, N=N, lengths=tl[:, -1])
    return d, tl


def _run(ctx, d, tl, K):
    from page_scoring_top_b200 import binding
    B, T, Q, D = d["q"].shape
    N = d["c"].shape[1]
    q, c = to_dev_bf16(d["q"]), to_dev_bf16(d["c"])
    tld = to_dev(tl)
    s = torch.full((B, T, N), 12345.0, device="cuda")
    binding.centroid_score_tokens(ctx, q, c, tld, s)
    idx, val = poisoned_outputs(B * T, K)
    binding.score_topk_fused_tokens(ctx, q, c, tld, K, idx, val)
    rc, bits = binding.idx_get_status(ctx)
    assert rc == 0 and bits == 0
    return s.cpu().numpy(), idx.cpu().numpy(), val.cpu().numpy()


def _check(ctx, d, tl, K):
    B, T, Q, D = d["q"].shape
    N = d["c"].shape[1]
    s_gpu, idx, val = _run(ctx, d, tl, K)
    S, A = oracle.scores(d["q"], d["c"], tl)
    assert oracle.score_bound_violations(s_gpu, S, A) == 0
    rows_len = tl.reshape(-1)
    check_select_bit_exact(s_gpu.reshape(B * T, N), rows_len, K, idx, val)
    check_recall(idx, S.reshape(B * T, N), rows_len, K, 0.999)


@pytest.mark.parametrize("T", [1, 2, 3, 4])
@pytest.mark.parametrize("D", [128, 96])
def test_causal_decode_tokens(ctx, T, D):
    # ragged contexts: short, page-boundary and long; pages of 64 keys
    rng = np.random.default_rng(700 + T)
    pos0 = rng.integers(0, 64 * 3000, 6)
    pos0[:3] = [0, 63, 64 * 1500 - T]
    B, N = 6, 3000
    d, tl = _inputs(701 + T + D, B, T, 4, D, N, pos0, 64)
    _check(ctx, d, tl, K=256)


def test_tokens_fall_back_to_score_then_select(ctx):
    # T = 6 is past the fused path's token limit, and T*Q = 32 with D = 128
    # is a prefill shape: per-token rows still go through the decode kernels
    # and a per-row select
    rng = np.random.default_rng(710)
    pos0 = rng.integers(0, 32 * 2000, 5)
    d, tl = _inputs(711, 5, 6, 4, 128, 2000, pos0, 32)
    _check(ctx, d, tl, K=128)
    d, tl = _inputs(712, 3, 8, 4, 128, 1500, [0, 31 * 100, 32 * 1400], 32)
    _check(ctx, d, tl, K=64)


def test_tokens_long_rows_many_chunks(ctx):
    # rows spread over many CTAs: per-token masks inside the multi-chunk merges
    d, tl = _inputs(720, 2, 4, 4, 128, 65536, [64 * 65000, 64 * 40000 + 5], 64)
    _check(ctx, d, tl, K=256)


def test_tokens_match_request_lengths_when_all_equal(ctx):
    # every token row with the request's count: the per-token calls equal the
    # whole-request ones bit for bit
    from page_scoring_top_b200 import binding
    B, T, N, K = 4, 3, 5000, 200
    lengths = np.array([5000, 4097, 33, 0], np.int32)
    d = synth.decode_inputs(730, B=B, T=T, Q=4, D=128, N=N, lengths=lengths)
    tl = np.repeat(lengths[:, None], T, axis=1).astype(np.int32)
    s_tok, idx_tok, val_tok = _run(ctx, d, tl, K)
    q, c = to_dev_bf16(d["q"]), to_dev_bf16(d["c"])
    s = torch.full((B, T, N), 1.0, device="cuda")
    binding.centroid_score(ctx, q, c, to_dev(lengths), s)
    idx, val = poisoned_outputs(B * T, K)
    binding.score_topk_fused(ctx, q, c, to_dev(lengths), K, idx, val)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_tok.view(np.uint32))
    assert np.array_equal(idx.cpu().numpy(), idx_tok)
    assert np.array_equal(val.cpu().numpy().view(np.uint32), val_tok.view(np.uint32))


def test_tokens_argument_errors(ctx):
    from page_scoring_top_b200 import binding
    L = binding.lib()
    q = torch.zeros((2, 2, 4, 128), dtype=torch.int16, device="cuda")
    c = torch.zeros((2, 64, 128), dtype=torch.int16, device="cuda")
    s = torch.zeros((2, 2, 64), device="cuda")
    idx = torch.zeros((4, 8), dtype=torch.int32, device="cuda")
    rc = L.centroid_score_tokens(ctx.handle, q.data_ptr(), c.data_ptr(), None, 2, 2, 4, 128, 64,
                                 64 * 128, s.data_ptr(), None)
    assert rc == binding.IDX_EINVAL
    rc = L.score_topk_fused_tokens(ctx.handle, q.data_ptr(), c.data_ptr(), None, 2, 2, 4, 128, 64,
                                   64 * 128, 8, idx.data_ptr(), None, None)
    assert rc == binding.IDX_EINVAL
