"""GPU parity of the tensor-core (tcgen05) prefill-chunk path against the oracle.

A request's T*Q query rows form the MMA's M dimension (T*Q >= 32, Q a power
of two, D = 128); the head-sum happens on the fp32 accumulators.  Bars as for
decode: scores within 1e-5 * sum|q*c|, indices bit-exact against the oracle's
select on the GPU's own scores, recall >= 0.999 against the oracle's top-K.
"""

import numpy as np
import pytest

import oracle
from page_scoring_top_b200 import synth
from helpers import check_recall, check_select_bit_exact, poisoned_outputs, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def ctx():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from page_scoring_top_b200 import binding
    c = binding.Context(0, max_rows=64, max_n=131072, max_k=512)
    yield c
    c.close()


def _run(ctx, d, K):
    from page_scoring_top_b200 import binding
    B, T, Q, D = d["q"].shape
    N = d["c"].shape[1]
    q, c, ln = to_dev_bf16(d["q"]), to_dev_bf16(d["c"]), to_dev(d["lengths"])
    s = torch.full((B, T, N), 777.0, device="cuda")
    binding.centroid_score(ctx, q, c, ln, s)
    idx, val = poisoned_outputs(B * T, K)
    binding.score_topk_fused(ctx, q, c, ln, K, idx, val)
    rc, bits = binding.idx_get_status(ctx)
    assert rc == 0, bits
    return s.cpu().numpy(), idx.cpu().numpy(), val.cpu().numpy()


@pytest.mark.parametrize("B,T,Q,N,lengths", [
    (2, 16, 8, 3000, [3000, 1111]),        # the prefill-chunk shape, ragged, partial tiles
    (3, 8, 4, 777, [777, 5, 300]),          # 32 rows, N not a multiple of 4 or 256
    (1, 1, 32, 513, [513]),                 # one token of 32 heads
    (2, 4, 16, 1024, [1024, 0]),            # 64 rows, an empty request
    (2, 32, 4, 2049, [2049, 2048]),         # 128 rows of 4 heads
])
def test_prefill_shapes(ctx, B, T, Q, N, lengths):
    from page_scoring_top_b200 import binding
    # the tensor-core path is the one taken for these shapes
    assert T * Q >= 32
    d = synth.decode_inputs(900 + T * Q + N, B=B, T=T, Q=Q, D=128, N=N, lengths=lengths)
    K = 64
    s, idx, val = _run(ctx, d, K)
    S, A = oracle.scores(d["q"], d["c"], d["lengths"])
    assert oracle.score_bound_violations(s, S, A) == 0
    rows_len = np.repeat(d["lengths"], T)
    check_select_bit_exact(s.reshape(B * T, N), rows_len, K, idx, val)
    check_recall(idx, S.reshape(B * T, N), rows_len, K)


def test_prefill_full_size_sampled(ctx):
    """The prefill-chunk workload at full size (B=4, T=16, Q=8, N=131072, K=512),
    in the launch configuration the benchmark uses; the oracle checks whole
    score rows and selections of sampled (request, token) pairs."""
    d = synth.workload("prefill_chunk")
    K = d["K"]
    B, T, Q, D = d["q"].shape
    N = d["c"].shape[1]
    s, idx, val = _run(ctx, d, K)
    rng = np.random.default_rng(0)
    for b, t in [(0, 0), (3, 15)] + [tuple(x) for x in rng.integers(0, [B, T], size=(2, 2))]:
        S, A = oracle.scores(d["q"][b:b + 1, t:t + 1], d["c"][b:b + 1], d["lengths"][b:b + 1])
        assert oracle.score_bound_violations(s[b, t], S[0, 0], A[0, 0]) == 0
        r = b * T + t
        check_select_bit_exact(s[b, t][None], d["lengths"][b:b + 1], K, idx[r:r + 1], val[r:r + 1])
        check_recall(idx[r:r + 1], S[0], d["lengths"][b:b + 1], K)
