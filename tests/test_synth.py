"""The seeded input generator: determinism, slicing, rounding and shapes."""

import numpy as np

from page_scoring_top_b200 import synth


def test_splitmix64_reference_values():
    # splitmix64 from state 0: the published first outputs of the generator
    # (Vigna's reference implementation seeded with 0)
    z = 0
    outs = []
    for _ in range(3):
        z = (z + synth.GOLDEN) & ((1 << 64) - 1)
        outs.append(synth._mix_int(z))
    assert outs[0] == 0xE220A8397B1DCDAF
    assert outs[1] == 0x6E789E6AA1B965F4
    assert outs[2] == 0x06C45D188009454F
    # the numpy path agrees with the integer path
    x = synth._mix_np(np.array([synth.GOLDEN, 2 * synth.GOLDEN & ((1 << 64) - 1)], np.uint64))
    assert int(x[0]) == outs[0] and int(x[1]) == outs[1]


def test_counter_based_slices():
    full = synth.u64(3, 5, 0, 1000)
    assert np.array_equal(synth.u64(3, 5, 400, 100), full[400:500])
    nfull = synth.normal(3, 5, 0, 1000)
    assert np.array_equal(synth.normal(3, 5, 200, 300), nfull[200:500])
    assert np.array_equal(synth.normal(3, 5, 201, 299), nfull[201:500])   # odd start
    assert not np.array_equal(synth.u64(3, 6, 0, 10), full[:10])   # streams differ


def test_normal_moments():
    z = synth.normal(1, 1, 0, 400000)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01


def test_bf16_rounding_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5, 0.0, -0.0], np.float32)
    bits = synth.f32_to_bf16_bits(x)
    back = synth.bf16_bits_to_f32(bits)
    # 1+2^-8 is a tie between 1 and 1+2^-7: even mantissa (1.0) wins;
    # 1+3*2^-8 ties between 1+2^-7 and 1+2^-6... rounds to even 1+2^-6
    assert list(back) == [1.0, 1.0, 1.0 + 2 ** -6, 1.0, -2.5, 0.0, -0.0]
    assert bits[6] == 0x8000


def test_decode_inputs_shapes_and_poison():
    d = synth.decode_inputs(103, B=4, T=1, Q=4, D=16, N=64, len_range=(10, 64))
    assert d["q"].shape == (4, 1, 4, 16) and d["c"].shape == (4, 64, 16)
    assert np.all((d["lengths"] >= 10) & (d["lengths"] <= 64))
    for b, n in enumerate(d["lengths"]):
        assert np.all(d["c"][b, n:] == synth.BF16_NAN_POISON)
        assert not np.any(d["c"][b, :n] == synth.BF16_NAN_POISON)
    d2 = synth.decode_inputs(103, B=4, T=1, Q=4, D=16, N=64, len_range=(10, 64))
    assert all(np.array_equal(d[k], d2[k]) for k in ("q", "c", "lengths"))


def test_page_bias_is_one_scalar_per_page():
    d = synth.decode_inputs(102, B=1, T=1, Q=1, D=8, N=200, page_bias=True)
    plain = synth.decode_inputs(102, B=1, T=1, Q=1, D=8, N=200)
    cb = synth.bf16_bits_to_f32(d["c"][0]).astype(np.float64)
    cp = synth.bf16_bits_to_f32(plain["c"][0]).astype(np.float64)
    beta = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(
        (0.5 * synth.normal(102, 3, 0, 200)).astype(np.float32))).astype(np.float64)
    # c = bf16(z + beta_p): one rounding of the sum, half a bf16 ulp at most
    assert np.all(np.abs(cb - (cp + beta[:, None])) <= np.abs(cb) * 2.0 ** -8)
    assert np.std(beta) > 0.3


def test_score_row_distributions():
    n = 4096
    for dist in synth.DISTRIBUTIONS:
        r = synth.score_rows(104, 2, n, dist)
        assert r.shape == (2, n) and r.dtype == np.float32
        if dist == "neg_inf_90":
            assert np.all(np.count_nonzero(np.isneginf(r), axis=1) == (9 * n) // 10)
        else:
            assert np.all(np.isfinite(r))
    assert np.all(synth.score_rows(104, 1, n, "all_equal") == 1.0)
    lv = synth.score_rows(104, 1, n, "levels16")
    assert len(np.unique(lv)) == 16
    asc = synth.score_rows(104, 1, n, "sorted_asc")[0]
    assert np.all(np.diff(asc) >= 0)
    u = synth.score_rows(104, 1, n, "uniform")[0]
    assert u.min() >= 0 and u.max() < 1
    assert len(list(synth.sweep_cases())) == 4 * 4 * 11
