"""GPU parity of the KMeans assignment (tcgen05 product + h, argmax in the
epilogue) against the CPU oracle ("Export Cake KMeans plan-runtime suite":
every point to its nearest centroid).

* scores: every s[i,c] of kmeans_scores within 1e-5 * (sum_d |x*c| + h) of
  the oracle's exact double score;
* assignment: bit-exact against the oracle's row argmax of the GPU's own
  scores (ties to the lower centroid), and the returned score bit-equal to
  the GPU score of the chosen centroid;
* against the exact assignment: a chosen centroid's exact score is within
  twice the bound of the best, and the two agree on nearly every point;
* the full-size workload (262144 points, 1024 centroids, D=128) on sampled
  points; duplicate centroids go to the lower index; tiny scores; argument
  errors."""

import numpy as np
import pytest

import oracle
from page_scoring_top_b200 import synth
from helpers import to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def ctx():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from page_scoring_top_b200 import binding
    c = binding.Context(0, max_rows=8, max_n=1024, max_k=64)  # workspace >= 8192 centroids
    yield c
    c.close()


def _run(ctx, x, cent):
    from page_scoring_top_b200 import binding
    M, C = x.shape[0], cent.shape[0]
    xd, cd = to_dev_bf16(x), to_dev_bf16(cent)
    s = torch.full((M, C), float("nan"), device="cuda")
    binding.kmeans_scores(ctx, xd, cd, s)
    assign = torch.full((M,), -7, dtype=torch.int32, device="cuda")
    score = torch.full((M,), float("nan"), device="cuda")
    binding.kmeans_assign(ctx, xd, cd, assign, score)
    torch.cuda.synchronize()
    rc, bits = binding.idx_get_status(ctx)
    assert rc == 0, bits
    return s.cpu().numpy(), assign.cpu().numpy(), score.cpu().numpy()


def _check(ctx, x, cent):
    s, assign, score = _run(ctx, x, cent)
    a_ex, best, S, A = oracle.kmeans_assign(x, cent, full=True)
    # every score within the bound
    assert oracle.score_bound_violations(s, S, A) == 0
    # bit-exact argmax of the GPU's own scores; the score is that entry
    want = oracle.argmax_rows(s)
    assert np.array_equal(assign, want)
    rows = np.arange(x.shape[0])
    assert np.array_equal(score.view(np.int32), s[rows, assign].view(np.int32))
    # against the exact assignment: near-optimal everywhere, equal almost everywhere
    bound = 1e-5 * A.max(axis=1)
    assert np.all(S[rows, assign] >= best - 2 * bound)
    assert np.mean(assign == a_ex) >= 0.999
    return assign


@pytest.mark.parametrize("M,C,D", [
    (1000, 300, 128),   # ragged point and centroid tiles
    (4096, 256, 128),   # one centroid tile
    (257, 513, 64),     # one K block
    (300, 1000, 112),   # D not a multiple of 64: zero-filled columns
    (129, 1, 8),        # a single centroid, tiny D
    (2048, 777, 96),
])
def test_kmeans_shapes(ctx, M, C, D):
    d = synth.kmeans_inputs(1000 + M + C + D, M, C, D)
    _check(ctx, d["x"], d["centroids"])


def test_kmeans_unclustered_scores(ctx):
    # points and centroids drawn independently: many near-ties between centroids
    x = synth.normal_bf16(31, 1, 0, 700 * 128).reshape(700, 128)
    c = synth.normal_bf16(31, 2, 0, 600 * 128).reshape(600, 128)
    _check(ctx, x, c)


def test_kmeans_duplicate_centroids_go_low(ctx):
    d = synth.kmeans_inputs(77, 600, 40, 128)
    cent = d["centroids"].copy()
    cent[[30, 31, 39]] = cent[5]  # copies of centroid 5 after it
    assign = _check(ctx, d["x"], cent)
    assert not np.any(np.isin(assign, [30, 31, 39]))
    assert np.any(assign == 5)


def test_kmeans_tiny_scores(ctx):
    # inputs scaled by 2^-60: scores near 2^-114, far below the usual range,
    # with exact ties inside the first 32-column chunk
    d = synth.kmeans_inputs(91, 500, 300, 128)
    scale = np.float32(2.0 ** -60)

    def shrink(a):
        f = (a.astype(np.uint32) << 16).view(np.float32) * scale
        return (f.view(np.uint32) >> 16).astype(np.uint16)  # exact: a power-of-two scaling
    x, cent = shrink(d["x"]), shrink(d["centroids"])
    cent[[7, 8]] = cent[3]  # ties inside the first chunk
    assign = _check(ctx, x, cent)
    assert not np.any(np.isin(assign, [7, 8]))


def test_kmeans_full_workload_sampled(ctx):
    from page_scoring_top_b200 import binding
    spec = synth.KMEANS
    d = synth.kmeans_inputs(spec["seed"], spec["M"], spec["C"], spec["D"])
    M, C = spec["M"], spec["C"]
    big = binding.Context(0, max_rows=1, max_n=C, max_k=1)
    assign = torch.full((M,), -7, dtype=torch.int32, device="cuda")
    score = torch.full((M,), float("nan"), device="cuda")
    binding.kmeans_assign(big, to_dev_bf16(d["x"]), to_dev_bf16(d["centroids"]), assign, score)
    torch.cuda.synchronize()
    rc, bits = binding.idx_get_status(big)
    assert rc == 0, bits
    assign, score = assign.cpu().numpy(), score.cpu().numpy()
    assert assign.min() >= 0 and assign.max() < C
    rng = np.random.default_rng(5)
    pts = np.sort(rng.choice(M, 512, replace=False))
    a_ex, best, S, A = oracle.kmeans_assign(d["x"][pts], d["centroids"], full=True)
    rows = np.arange(len(pts))
    got = assign[pts]
    bound = 1e-5 * A.max(axis=1)
    assert np.all(S[rows, got] >= best - 2 * bound)
    assert np.mean(got == a_ex) >= 0.99
    # the returned score is the chosen centroid's score, within the bound
    assert np.all(np.abs(score[pts] - S[rows, got]) <= 1e-5 * A[rows, got])
    big.close()


def test_kmeans_argument_errors(ctx):
    from page_scoring_top_b200 import binding
    L = binding.lib()
    x = torch.zeros((4, 128), dtype=torch.int16, device="cuda")
    c = torch.zeros((4, 128), dtype=torch.int16, device="cuda")
    out = torch.zeros(4, dtype=torch.int32, device="cuda")
    assert L.kmeans_assign(ctx.handle, x.data_ptr(), c.data_ptr(), 4, 4, 136, out.data_ptr(), None,
                           None) == binding.IDX_EUNSUPPORTED  # D beyond 128
    assert L.kmeans_assign(ctx.handle, x.data_ptr(), c.data_ptr(), 4, 4, 100, out.data_ptr(), None,
                           None) == binding.IDX_EINVAL       # D not a multiple of 8
    assert L.kmeans_assign(ctx.handle, x.data_ptr(), c.data_ptr(), 0, 4, 128, out.data_ptr(), None,
                           None) == binding.IDX_EINVAL
    assert L.kmeans_assign(ctx.handle, x.data_ptr(), c.data_ptr(), 4, 10 ** 6, 128, out.data_ptr(),
                           None, None) == binding.IDX_ENOWORKSPACE
