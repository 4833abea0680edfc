"""Pins of the CPU oracle against things other than itself.

* worked examples computed by hand (tests/golden/worked_examples.json);
* exact rational arithmetic (fractions) on tiny random bf16 inputs;
* a library dot product (numpy einsum in float64, another summation order);
* the top-K definition checked pairwise (O(N^2), no sorting) for N <= 64 and
  every K in 1..N+2, on random, tied, signed-zero and -inf rows;
* invariants: min selected >= max unselected, K >= #valid returns exactly the
  valid set, page permutation, padding never selected, q scaled by 2, score
  linearity;
* the checkers themselves reject planted mistakes (a mistake planted in a copy
  of the oracle's output, on the CPU).
"""

import itertools
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from page_scoring_top_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def _num(x):
    if isinstance(x, str):
        return {"-inf": -np.inf, "+inf": np.inf, "nan": np.nan, "-0.0": -0.0}[x]
    return float(x)


def _bf16(values):
    arr = np.asarray(values, np.float32)
    bits = synth.f32_to_bf16_bits(arr)
    assert np.array_equal(synth.bf16_bits_to_f32(bits), arr), "example value not exact in bf16"
    return bits


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


# ---------------------------------------------------------------- worked examples

@pytest.mark.parametrize("ex", _golden()["score_examples"], ids=lambda e: e["name"])
def test_worked_score_examples(ex):
    T, Q, D = ex["T"], ex["Q"], ex["D"]
    q = _bf16(ex["q"]).reshape(1, T, Q, D)
    c = _bf16(ex["c"]).reshape(1, -1, D)
    S, A = oracle.scores(q, c, np.array([ex["len"]], np.int32))
    want_s = np.array([[_num(v) for v in row] for row in ex["s"]])
    want_a = np.array([[_num(v) for v in row] for row in ex["A"]])
    assert np.array_equal(S[0], want_s)
    assert np.array_equal(A[0], want_a)
    for case in ex["topk"]:
        K = case["K"]
        want = np.array(case["idx"]).reshape(T, K)
        for t in range(T):
            idx, val, kk = oracle.topk(S[0, t], K)
            assert list(idx) == list(want[t])
            assert kk == int(np.count_nonzero(want[t] >= 0))
            # the value slots follow the indices
            for k in range(K):
                if idx[k] >= 0:
                    assert val[k] == S[0, t, idx[k]]
                else:
                    assert val[k] == -np.inf


@pytest.mark.parametrize("ex", _golden()["select_examples"], ids=lambda e: e["name"])
@pytest.mark.parametrize("dtype", [np.float32, np.float64])
def test_worked_select_examples(ex, dtype):
    row = np.array([_num(v) for v in ex["row"]], dtype)
    idx, val, _ = oracle.topk(row, ex["K"])
    assert list(idx) == ex["idx"]
    for k, i in enumerate(idx):
        if i >= 0:
            # bit-exact value, signed zero kept
            assert np.asarray(val[k], dtype).tobytes() == np.asarray(row[i], dtype).tobytes()


# ---------------------------------------------------------------- scores: exact arithmetic

def _exact_scores(qb, cb, length):
    """Scores by exact rational arithmetic on the bf16 values."""
    qf = synth.bf16_bits_to_f32(qb).astype(np.float64)
    cf = synth.bf16_bits_to_f32(cb).astype(np.float64)
    B, T, Q, D = qf.shape
    N = cf.shape[1]
    out = np.empty((T, N), object)
    for t in range(T):
        for p in range(N):
            if p >= length:
                out[t, p] = None
                continue
            acc = Fraction(0)
            for h in range(Q):
                for d in range(D):
                    acc += Fraction(qf[0, t, h, d]) * Fraction(cf[0, p, d])
            out[t, p] = acc
    return out


@pytest.mark.parametrize("seed", range(6))
def test_scores_match_exact_rationals(seed):
    rng = np.random.default_rng(seed)
    T, Q, D, N = int(rng.integers(1, 3)), int(rng.integers(1, 5)), int(rng.integers(1, 17)), 7
    length = int(rng.integers(0, N + 1))
    q = synth.f32_to_bf16_bits(rng.standard_normal((1, T, Q, D)).astype(np.float32) * 3)
    c = synth.f32_to_bf16_bits(rng.standard_normal((1, N, D)).astype(np.float32) * 3)
    S, A = oracle.scores(q, c, np.array([length], np.int32))
    exact = _exact_scores(q, c, length)
    for t in range(T):
        for p in range(N):
            if p >= length:
                assert S[0, t, p] == -np.inf and A[0, t, p] == 0.0
            else:
                # a double sum of exact products: error <= terms * 2^-53 * A
                err = abs(Fraction(S[0, t, p]) - exact[t, p])
                assert err <= Fraction(Q * D) * Fraction(2.0 ** -53) * Fraction(A[0, t, p])


def test_scores_match_library_dot_product():
    d = synth.decode_inputs(7, B=3, T=2, Q=4, D=64, N=50, lengths=[50, 17, 0])
    S, A = oracle.scores(d["q"], d["c"], d["lengths"])
    qf = synth.bf16_bits_to_f32(d["q"]).astype(np.float64)
    cf = synth.bf16_bits_to_f32(d["c"]).astype(np.float64)
    ref = np.einsum("bthd,bpd->btp", qf, np.where(np.isnan(cf), 0.0, cf))
    aref = np.einsum("bthd,bpd->btp", np.abs(qf), np.abs(np.where(np.isnan(cf), 0.0, cf)))
    for b, length in enumerate(d["lengths"]):
        assert np.all(np.abs(S[b, :, :length] - ref[b, :, :length]) <= 1e-12 * A[b, :, :length] + 1e-300)
        assert np.allclose(A[b, :, :length], aref[b, :, :length], rtol=1e-12, atol=0)
        assert np.all(np.isneginf(S[b, :, length:]))


def test_one_hot_closed_form():
    # q = e_h (one head nonzero, one dim), c = one-hot row: each score equals one q entry
    Q, D, N = 3, 8, 8
    q = np.zeros((1, 1, Q, D), np.float32)
    q[0, 0, 1, :] = np.arange(1, D + 1, dtype=np.float32) * 0.5
    c = np.eye(N, D, dtype=np.float32)[None]
    S, _ = oracle.scores(_bf16(q), _bf16(c), None)
    assert np.array_equal(S[0, 0], np.arange(1, D + 1) * 0.5)


def test_scores_scale_and_head_order():
    d = synth.decode_inputs(11, B=2, T=1, Q=4, D=32, N=40)
    S, A = oracle.scores(d["q"], d["c"], d["lengths"])
    q2 = synth.f32_to_bf16_bits(2 * synth.bf16_bits_to_f32(d["q"]))
    S2, A2 = oracle.scores(q2, d["c"], d["lengths"])
    assert np.array_equal(S2, 2 * S) and np.array_equal(A2, 2 * A)   # exact: scaling by 2
    Sp, _ = oracle.scores(d["q"][:, :, ::-1].copy(), d["c"], d["lengths"])
    assert np.all(np.abs(Sp - S) <= 1e-12 * A)                      # heads commute


def test_scores_linear_in_q():
    # q = qa + qb where qa, qb use disjoint dims: exact sums, so S(q) = S(qa) + S(qb)
    d = synth.decode_inputs(12, B=1, T=1, Q=2, D=16, N=30)
    qa = d["q"].copy()
    qb = d["q"].copy()
    qa[..., 8:] = 0
    qb[..., :8] = 0
    S, A = oracle.scores(d["q"], d["c"])
    Sa, _ = oracle.scores(qa, d["c"])
    Sb, _ = oracle.scores(qb, d["c"])
    assert np.all(np.abs(S - (Sa + Sb)) <= 1e-12 * A)


# ---------------------------------------------------------------- top-K by definition

def _selectable(row, length):
    return [p for p in range(length) if not np.isnan(row[p]) and row[p] != -np.inf]


def check_topk_definition(row, length, K, idx, val):
    """Raise AssertionError unless (idx, val) is THE top-K of row[:length]
    under (value desc, index asc); checked pairwise, without sorting."""
    sel = _selectable(row, length)
    kk = min(K, len(sel))
    idx = list(idx)
    assert len(idx) == K
    chosen = idx[:kk]
    assert all(i >= 0 for i in chosen) and all(i == -1 for i in idx[kk:])
    assert len(set(chosen)) == kk and set(chosen) <= set(sel)
    for k in range(kk, K):
        assert val[k] == -np.inf
    for k, i in enumerate(chosen):
        assert np.asarray(val[k]).tobytes() == np.asarray(row[i], np.asarray(val).dtype).tobytes()
    rest = set(sel) - set(chosen)
    for i in chosen:
        for j in rest:
            assert row[i] > row[j] or (row[i] == row[j] and i < j)
    for a, b in zip(chosen, chosen[1:]):
        assert row[a] > row[b] or (row[a] == row[b] and a < b)


def _adversarial_rows(rng, n):
    yield rng.standard_normal(n)
    yield rng.integers(-3, 4, n).astype(np.float64)              # small-integer ties
    yield np.where(rng.random(n) < 0.5, 0.0, -0.0)                  # signed zeros only
    r = rng.standard_normal(n)
    r[rng.random(n) < 0.4] = -np.inf
    yield r                                                          # -inf mixed in
    r = rng.integers(0, 2, n).astype(np.float64)
    r[rng.random(n) < 0.2] = np.nan
    yield r                                                          # NaN mixed in
    yield np.full(n, 1.5)                                            # all equal
    yield np.arange(n, dtype=np.float64)                             # ascending


@pytest.mark.parametrize("n", [1, 2, 3, 5, 8, 13, 31, 64])
@pytest.mark.parametrize("dtype", [np.float32, np.float64])
def test_topk_brute_force_every_k(n, dtype):
    rng = np.random.default_rng(1000 + n)
    for row in _adversarial_rows(rng, n):
        row = row.astype(dtype)
        for length in sorted({n, max(0, n - 1), n // 2, 0}):
            for K in range(1, n + 3):
                idx, val, kk = oracle.topk(row, K, length)
                check_topk_definition(row, length, K, idx, val)


def test_topk_exhaustive_tiny_rows():
    # every row over the value set {-inf, -1, -0.0, 0.0, 1} of length <= 4, every K
    values = [-np.inf, -1.0, -0.0, 0.0, 1.0]
    for n in range(1, 5):
        for combo in itertools.product(values, repeat=n):
            row = np.array(combo)
            for K in range(1, n + 2):
                idx, val, _ = oracle.topk(row, K)
                check_topk_definition(row, n, K, idx, val)


# ---------------------------------------------------------------- invariants

def test_invariants_min_selected_and_all_valid():
    rng = np.random.default_rng(5)
    for _ in range(20):
        n = int(rng.integers(1, 300))
        row = rng.standard_normal(n).astype(np.float32)
        row[rng.random(n) < 0.3] = -np.inf
        length = int(rng.integers(0, n + 1))
        K = int(rng.integers(1, n + 5))
        idx, val, kk = oracle.topk(row, K, length)
        sel = set(_selectable(row, length))
        chosen = set(int(i) for i in idx[:kk])
        if chosen and sel - chosen:
            assert min(row[list(chosen)]) >= max(row[list(sel - chosen)])
        assert not any(i >= length for i in chosen)           # padding never selected
        assert not any(row[i] == -np.inf for i in chosen)      # -inf never selected
        idx_all, _, kk_all = oracle.topk(row, len(sel) + 3, length)
        assert set(int(i) for i in idx_all[:kk_all]) == sel    # K >= #valid: all valid


def test_invariant_page_permutation():
    rng = np.random.default_rng(6)
    for _ in range(10):
        n = 200
        row = rng.standard_normal(n)                    # distinct values
        perm = rng.permutation(n)
        K = 37
        a, _, _ = oracle.topk(row, K)
        b, _, _ = oracle.topk(row[perm], K)
        # page perm[j] moved to position j: the selected pages are relabelled
        assert sorted(perm[b].tolist()) == sorted(a.tolist())
        assert list(perm[b]) == list(a)                 # and the order is kept
    # with ties the selected VALUES are invariant, and ties re-resolve by new index
    row = rng.integers(0, 5, 100).astype(np.float64)
    perm = rng.permutation(100)
    a, va, _ = oracle.topk(row, 30)
    b, vb, _ = oracle.topk(row[perm], 30)
    assert np.array_equal(va, vb)


def test_invariant_scaling_q_keeps_indices():
    d = synth.decode_inputs(21, B=2, T=1, Q=4, D=32, N=300, lengths=[300, 123])
    S, _ = oracle.scores(d["q"], d["c"], d["lengths"])
    q2 = synth.f32_to_bf16_bits(2 * synth.bf16_bits_to_f32(d["q"]))
    S2, _ = oracle.scores(q2, d["c"], d["lengths"])
    for b in range(2):
        assert np.array_equal(oracle.topk(S[b, 0], 50)[0], oracle.topk(S2[b, 0], 50)[0])


def test_rows_api_matches_single_rows():
    rng = np.random.default_rng(8)
    s = rng.standard_normal((5, 77)).astype(np.float32)
    lengths = np.array([77, 0, 1, 40, 76], np.int32)
    idx, val = oracle.topk_rows(s, 16, lengths)
    for r in range(5):
        i1, v1, _ = oracle.topk(s[r], 16, lengths[r])
        assert np.array_equal(idx[r], i1) and np.array_equal(val[r], v1)


# ---------------------------------------------------------------- acceptance measures

def test_recall_definition():
    assert oracle.recall([3, 1, 2, 0], [1, 2, 3, 4], 4) == 0.75
    assert oracle.recall([1, 2, 9, 8], [1, 2, 3, 4], 2) == 1.0
    assert oracle.recall([1, -1, -1], [1, -1, -1], 3) == 1.0      # denominator min(m, #selectable)
    assert oracle.recall([-1], [-1], 1) == 1.0


def test_score_bound_measure():
    S = np.array([1.0, -np.inf, 2.0])
    A = np.array([10.0, 0.0, 1.0])
    assert oracle.score_bound_violations(np.array([1.0 + 9e-5, -np.inf, 2.0]), S, A) == 0
    assert oracle.score_bound_violations(np.array([1.0 + 2e-4, -np.inf, 2.0]), S, A) == 1
    assert oracle.score_bound_violations(np.array([1.0, 0.0, 2.0]), S, A) == 1     # padding must be -inf
    assert oracle.score_bound_violations(np.array([1.0, -np.inf, np.nan]), S, A) == 1


# ---------------------------------------------------------------- the checkers catch planted mistakes

def test_checker_rejects_planted_mistakes():
    rng = np.random.default_rng(9)
    row = rng.integers(0, 4, 40).astype(np.float64)
    idx, val, _ = oracle.topk(row, 12)
    check_topk_definition(row, 40, 12, idx, val)
    # ties to the higher index
    ties = [i for i in range(40) if row[i] == row[idx[11]]]
    bad = idx.copy()
    bad[11] = max(t for t in ties if t not in idx[:11]) if len(ties) > 1 else bad[11]
    if bad[11] != idx[11]:
        with pytest.raises(AssertionError):
            check_topk_definition(row, 40, 12, bad, val)
    # order reversed
    with pytest.raises(AssertionError):
        check_topk_definition(row, 40, 12, idx[::-1].copy(), val[::-1].copy())
    # an unselected better page swapped in for the worst
    bad = idx.copy()
    bad[0] = [i for i in range(40) if i not in idx][0]
    with pytest.raises(AssertionError):
        check_topk_definition(row, 40, 12, bad, val)
    # a padded page selected
    with pytest.raises(AssertionError):
        check_topk_definition(row, 30, 12, idx, val) if max(idx) >= 30 else \
            check_topk_definition(row, 40, 12, np.r_[idx[:-1], 45], val)


def test_exact_check_rejects_planted_score_mistakes():
    # a dropped head, a flipped sign and a transposed operand all break the pins
    rng = np.random.default_rng(10)
    q = synth.f32_to_bf16_bits(rng.standard_normal((1, 1, 3, 4)).astype(np.float32))
    c = synth.f32_to_bf16_bits(rng.standard_normal((1, 5, 4)).astype(np.float32))
    S, A = oracle.scores(q, c)
    exact = _exact_scores(q, c, 5)
    qf = synth.bf16_bits_to_f32(q).astype(np.float64)[0, 0]
    cf = synth.bf16_bits_to_f32(c).astype(np.float64)[0]
    mistakes = {
        "dropped_head": (qf[:2].sum(0) @ cf.T),
        "sign": (qf.sum(0) @ (-cf.T)),
        # the page table read as [D][N] instead of [N][D]
        "transposed": (qf.sum(0) @ cf.reshape(-1).reshape(4, 5)),
    }
    for name, wrong in mistakes.items():
        n = len(wrong)
        ok = all(abs(Fraction(float(wrong[p])) - exact[0, p]) <= Fraction(1, 10 ** 6) for p in range(n))
        assert not ok, name
    for p in range(5):
        assert abs(Fraction(S[0, 0, p]) - exact[0, p]) <= Fraction(12) * Fraction(2.0 ** -53) * Fraction(A[0, 0, p])


# ------------------------------------------------------------------ per-token (multi-token decode) rows

def test_causal_token_lengths_worked_example():
    # pages of 4 keys; context 5 tokens, 4 new tokens at positions 5, 6, 7, 8:
    # they see 6, 7, 8, 9 keys -> 2, 2, 2, 3 pages.  Context 0: 1..4 keys -> 1 page.
    # Context 7: 8 keys -> 2 pages, then 9, 10, 11 keys -> 3 pages.  Capped at N.
    got = synth.causal_token_lengths([5, 0, 7, 100], 4, 4, 26)
    want = [[2, 2, 2, 3], [1, 1, 1, 1], [2, 3, 3, 3], [26, 26, 26, 26]]
    assert got.tolist() == want


def test_token_lengths_scores_by_hand():
    # Q=1, D=2, q_t = [t+1, 0]: token t's score of page p is (t+1) * c[p,0];
    # token 0 sees 1 page, token 1 sees 3 pages.
    q = _bf16([[[[1.0, 0.0]], [[2.0, 0.0]]]])          # [1][2][1][2]
    c = _bf16([[[1.0, 5.0], [3.0, -1.0], [-2.0, 4.0]]])  # [1][3][2]
    S, A = oracle.scores(q, c, np.array([[1, 3]], np.int32))
    assert S[0, 0].tolist() == [1.0, -np.inf, -np.inf]
    assert S[0, 1].tolist() == [2.0, 6.0, -4.0]
    assert A[0, 0].tolist() == [1.0, 0.0, 0.0]
    idx, val, kk = oracle.topk(S[0, 1], 2)
    assert idx.tolist() == [1, 0] and kk == 2


@pytest.mark.parametrize("seed", [21, 22])
def test_token_lengths_equal_masked_request_rows(seed):
    # a token row is its request row with the pages past the token's count at -inf
    B, T, N = 3, 4, 40
    d = synth.decode_inputs(seed, B=B, T=T, Q=2, D=16, N=N, lengths=[N, 30, 0])
    tl = synth.causal_token_lengths([150, 113, 0], T, 4, N)
    tl[2] = 0
    S_req, A_req = oracle.scores(d["q"], d["c"], tl[:, -1])
    S_tok, A_tok = oracle.scores(d["q"], d["c"], tl)
    live = np.arange(N)[None, None, :] < tl[:, :, None]
    assert np.array_equal(S_tok, np.where(live, S_req, -np.inf))
    assert np.array_equal(A_tok, np.where(live, A_req, 0.0))
    # and the per-row select sees exactly the live pages
    idx, _ = oracle.topk_rows(S_tok.reshape(B * T, N), 8, tl.reshape(-1))
    for r in range(B * T):
        sel = idx[r][idx[r] >= 0]
        assert np.all(sel < tl.reshape(-1)[r])
        assert len(sel) == min(8, tl.reshape(-1)[r])


# ------------------------------------------------------------------ page centroids (key mean-pooling)

def test_pool_worked_example():
    # pages of 2 keys over 5 keys: (1,2)+(3,4) -> (2,3); (5,6)+(7,8) -> (6,7);
    # the partial last page holds (9,10) alone; page 3 has no key -> 0
    k = _bf16([[[1, 2], [3, 4], [5, 6], [7, 8], [9, 10]]])
    m = oracle.pool(k, np.array([5], np.int32), 2, 4)
    assert m[0].tolist() == [[2, 3], [6, 7], [9, 10], [0, 0]]


def test_pool_closed_forms():
    rng = np.random.default_rng(31)
    k = synth.normal_bf16(32, 1, 0, 2 * 40 * 8).reshape(2, 40, 8)
    counts = np.array([40, 23], np.int32)
    # one key per page: the centroid is the key itself
    m1 = oracle.pool(k, counts, 1, 40)
    kf = synth.bf16_bits_to_f32(k).astype(np.float64)
    assert np.array_equal(m1[0], kf[0]) and np.array_equal(m1[1, :23], kf[1, :23])
    # constant keys: the centroid is the constant, whatever the page size
    c = np.full((1, 12, 8), synth.f32_to_bf16_bits(np.array([0.375], np.float32))[0], np.uint16)
    assert np.all(oracle.pool(c, np.array([12], np.int32), 5, 3) == 0.375)
    # the mean is linear: pooling 2*k (exact in bf16) doubles it
    k2 = synth.f32_to_bf16_bits((2 * synth.bf16_bits_to_f32(k)).astype(np.float32))
    assert np.array_equal(oracle.pool(k2, counts, 4, 10), 2 * oracle.pool(k, counts, 4, 10))
    # a library mean over the same keys
    lib = kf[1, 20:23].mean(axis=0)
    assert np.allclose(oracle.pool(k, counts, 4, 10)[1, 5], lib, rtol=0, atol=1e-15)


# ------------------------------------------------------------------ paged centroid table

def test_paged_scores_gather_the_pool():
    # a pool of 3 blocks; request 0 reads blocks [2, 0, 2], request 1 reads [1]
    q = _bf16([[[[1.0, 2.0]]], [[[0.5, -1.0]]]])          # [2][1][1][2]
    pool = _bf16([[1.0, 0.0], [0.0, 1.0], [3.0, 1.0]])     # [3][2]
    pt = np.array([[2, 0, 2], [1, 0, 0]], np.int32)
    S, _ = oracle.scores_paged(q, pool, pt, np.array([3, 1], np.int32))
    assert S[0, 0].tolist() == [5.0, 1.0, 5.0]
    assert S[1, 0].tolist() == [-1.0, -np.inf, -np.inf]


def test_paged_identity_table_equals_contiguous():
    d = synth.decode_inputs(41, B=2, T=1, Q=2, D=16, N=30, lengths=[30, 17])
    pool = d["c"].reshape(60, 16)
    pt = np.arange(60, dtype=np.int32).reshape(2, 30)
    S1, A1 = oracle.scores(d["q"], d["c"], d["lengths"])
    S2, A2 = oracle.scores_paged(d["q"], pool, pt, d["lengths"])
    assert np.array_equal(S1, S2) and np.array_equal(A1, A2)


def test_paged_scores_reject_ids_outside_the_pool():
    # The block-pool table ("Iterate Centroids Score", the ctx argument)
    # names valid blocks only: a live page pointing outside the pool is an
    # error for the oracle, while entries past a request's length are never read.
    q = _bf16([[[[1.0, 2.0]]]])
    pool = _bf16([[1.0, 0.0], [0.0, 1.0]])
    with pytest.raises(ValueError):
        oracle.scores_paged(q, pool, np.array([[0, 2]], np.int32), np.array([2], np.int32))
    with pytest.raises(ValueError):
        oracle.scores_paged(q, pool, np.array([[-1, 0]], np.int32), np.array([2], np.int32))
    S, _ = oracle.scores_paged(q, pool, np.array([[1, 99]], np.int32), np.array([1], np.int32))
    assert S[0, 0].tolist() == [2.0, -np.inf]


# ------------------------------------------------------------------ KMeans assignment
# "Export Cake KMeans plan-runtime suite" (summary): assignments =
# compute(x, centroids), each point to its nearest centroid.

def test_kmeans_worked_example():
    # centroids (0,0), (2,0), (0,2); by hand:
    #   (1.5, 0.25): squared distances 2.3125, 0.3125, 5.3125 -> centroid 1,
    #                score x.c - |c|^2/2 = 3 - 2 = 1
    #   (0.25, 0.25): 0.125, 3.125, 3.125 -> centroid 0, score 0
    #   (1, 1): 2, 2, 2 -> a three-way tie, the lowest index 0, score 0
    x = _bf16([[1.5, 0.25], [0.25, 0.25], [1.0, 1.0]])
    c = _bf16([[0.0, 0.0], [2.0, 0.0], [0.0, 2.0]])
    assign, best = oracle.kmeans_assign(x, c)
    assert assign.tolist() == [1, 0, 0]
    assert best.tolist() == [1.0, 0.0, 0.0]


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_kmeans_matches_nearest_by_distance(seed):
    # an independent formulation: argmin of the squared Euclidean distance,
    # library arithmetic in double (exact for these bf16 inputs), first minimum
    rng = np.random.default_rng(seed)
    M, C, D = 37, 11, 16
    xf = rng.integers(-8, 9, size=(M, D)).astype(np.float32) / 4
    cf = rng.integers(-8, 9, size=(C, D)).astype(np.float32) / 4
    x, c = synth.f32_to_bf16_bits(xf), synth.f32_to_bf16_bits(cf)
    assign, best, S, A = oracle.kmeans_assign(x, c, full=True)
    d2 = ((xf.astype(np.float64)[:, None, :] - cf.astype(np.float64)[None, :, :]) ** 2).sum(-1)
    assert np.array_equal(assign, np.argmin(d2, axis=1))
    # the score is the library's x c^T - |c|^2 / 2, and the winner's score is best
    lib = xf.astype(np.float64) @ cf.astype(np.float64).T - 0.5 * (cf.astype(np.float64) ** 2).sum(1)
    assert np.array_equal(S, lib)
    assert np.array_equal(best, S[np.arange(M), assign])
    assert np.all(A >= np.abs(S))


def test_kmeans_invariants():
    rng = np.random.default_rng(7)
    M, C, D = 50, 9, 8
    cf = rng.standard_normal((C, D)).astype(np.float32)
    c = synth.f32_to_bf16_bits(cf)
    # a point on a centroid goes to it (distinct centroids)
    x = c[[4, 0, 8]]
    assert oracle.kmeans_assign(x, c)[0].tolist() == [4, 0, 8]
    # permuting the centroids permutes the assignment (no ties at random)
    x = synth.f32_to_bf16_bits(rng.standard_normal((M, D)).astype(np.float32))
    a0, _ = oracle.kmeans_assign(x, c)
    perm = rng.permutation(C)
    a1, _ = oracle.kmeans_assign(x, c[perm])
    assert np.array_equal(perm[a1], a0)
    # doubling x (exact in bf16) and centroids leaves the nearest centroid
    x2 = synth.f32_to_bf16_bits(2 * synth.bf16_bits_to_f32(x))
    c2 = synth.f32_to_bf16_bits(2 * synth.bf16_bits_to_f32(c))
    assert np.array_equal(oracle.kmeans_assign(x2, c2)[0], a0)


def test_argmax_rows_ties_and_nan():
    s = np.array([[1.0, 3.0, 3.0, 2.0], [np.nan, -1.0, np.nan, -1.0],
                  [np.nan, np.nan, np.nan, np.nan], [-0.0, 0.0, 0.0, -5.0]], np.float32)
    assert oracle.argmax_rows(s).tolist() == [1, 1, -1, 0]


def test_kmeans_checker_rejects_planted_mistakes():
    # a plausible wrong rule (no half on |c|^2, or + instead of -) changes
    # the assignment on this example
    x = _bf16([[1.5, 0.25], [0.25, 0.25]])
    c = _bf16([[0.0, 0.0], [2.0, 0.0]])
    xf, cf = synth.bf16_bits_to_f32(x).astype(np.float64), synth.bf16_bits_to_f32(c).astype(np.float64)
    good = oracle.kmeans_assign(x, c)[0]
    no_half = np.argmax(xf @ cf.T - (cf ** 2).sum(1), axis=1)
    plus = np.argmax(xf @ cf.T + 0.5 * (cf ** 2).sum(1), axis=1)
    assert good.tolist() == [1, 0]
    assert no_half.tolist() != good.tolist() and plus.tolist() != good.tolist()
