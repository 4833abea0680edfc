"""GPU parity of centroid_pool (page centroids by key mean-pooling) against
the CPU oracle's exact means.

The kernel sums in fp32 and rounds the mean to bf16 once; the fp32 error is
far below half a bf16 ulp, so the result equals bf16_rne(exact mean) except
where the exact mean lies within that error of a rounding boundary: every
element must be within one bf16 ulp and all but a handful exactly equal.
Pages without a valid key must stay untouched (poisoned)."""

import numpy as np
import pytest

import oracle
from page_scoring_top_b200 import synth
from helpers import to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

POISON = np.uint16(0xA5A5)


@pytest.fixture(scope="module")
def ctx():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from page_scoring_top_b200 import binding
    c = binding.Context(0, max_rows=8, max_n=1024, max_k=64)
    yield c
    c.close()


def _bf16_ulp_diff(a_bits, b_bits):
    # distance in representable bf16 steps (same sign assumed for nonzero)
    def ordered(x):
        x = x.astype(np.int32)
        return np.where(x & 0x8000, 0x8000 - (x & 0x7FFF), 0x8000 + (x & 0x7FFF))
    return np.abs(ordered(a_bits) - ordered(b_bits))


def _run(ctx, keys, counts, P, N):
    from page_scoring_top_b200 import binding
    B, L, D = keys.shape
    kd = torch.from_numpy(keys.view(np.int16)).cuda()
    cd = torch.from_numpy(np.full((B, N, D), POISON, np.uint16).view(np.int16)).cuda()
    binding.centroid_pool(ctx, kd, to_dev(counts), P, cd)
    rc, bits = binding.idx_get_status(ctx)
    assert rc == 0 and bits == 0
    return cd.cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("D,P", [(128, 64), (64, 16), (96, 7), (256, 1), (8, 33)])
def test_pool_matches_exact_means(ctx, D, P):
    B, N = 3, 40
    L = N * P
    keys = synth.normal_bf16(800 + D + P, 1, 0, B * L * D).reshape(B, L, D)
    counts = np.array([L, P * 17 + P // 2 + 1, 0], np.int32)
    got = _run(ctx, keys, counts, P, N)
    want = synth.f32_to_bf16_bits(oracle.pool(keys, counts, P, N).astype(np.float32))
    for b in range(B):
        pages = (counts[b] + P - 1) // P
        assert np.all(got[b, pages:] == POISON), "page past the keys was written"
        diff = _bf16_ulp_diff(got[b, :pages], want[b, :pages])
        assert diff.max(initial=0) <= 1
        assert np.count_nonzero(diff) <= max(2, diff.size // 1000)


def test_pooled_centroids_feed_the_scorer(ctx):
    # pool, then score and select on the pooled table: equal to the oracle on
    # the same (GPU-pooled) centroids
    from page_scoring_top_b200 import binding
    from helpers import check_select_bit_exact, poisoned_outputs, to_dev_bf16
    B, P, N, D, Q, K = 2, 16, 600, 128, 4, 32
    keys = synth.normal_bf16(850, 1, 0, B * N * P * D).reshape(B, N * P, D)
    counts = np.array([N * P, 333 * P + 5], np.int32)
    c = _run(ctx, keys, counts, P, N)
    lengths = ((counts + P - 1) // P).astype(np.int32)
    c[1, lengths[1]:] = 0
    q = synth.normal_bf16(851, 1, 0, B * Q * D).reshape(B, 1, Q, D)
    s = torch.empty((B, 1, N), device="cuda")
    binding.centroid_score(ctx, to_dev_bf16(q), to_dev_bf16(c), to_dev(lengths), s)
    S, A = oracle.scores(q, c, lengths)
    assert oracle.score_bound_violations(s.cpu().numpy(), S, A) == 0
    idx, val = poisoned_outputs(B, K)
    binding.score_topk_fused(ctx, to_dev_bf16(q), to_dev_bf16(c), to_dev(lengths), K, idx, val)
    check_select_bit_exact(s.cpu().numpy().reshape(B, N), lengths, K, idx.cpu().numpy(),
                           val.cpu().numpy())
