"""Pins for the FP8 (E4M3) quantisation oracle.

* every finite E4M3 code, decoded from its bit fields, is a fixed point of
  the rounding, and the decoded set is exactly the rounding's range;
* a value half-way between two neighbours rounds to the one with the even
  mantissa; values past 448 saturate; the subnormal grid is 2^-9;
* a block's largest magnitude quantises to +-448; data already on the E4M3
  grid at a power-of-two scale quantises exactly;
* the K smoothing shifts every score of a row by one constant, so the
  softmax over the smoothed keys equals the softmax over the raw keys, and
  the quantised K of grid-valued keys does not change when one vector is
  added to every key;
* every dequantised Q, K and V element is within half an E4M3 step of its
  input at its group's scale (2^-4 relative, or s * 2^-10 on the subnormal
  range).
"""

import numpy as np

from oracle import fp8


def _finite_values():
    vals = [fp8.e4m3_decode(c) for c in range(256)]
    return np.array([v for v in vals if not np.isnan(v)])


def test_codes_are_fixed_points_and_the_whole_range():
    vals = _finite_values()
    assert len(vals) == 254                               # 0x7F and 0xFF are NaN
    assert np.array_equal(fp8.e4m3_round(vals), vals)
    assert vals.max() == 448.0 and vals.min() == -448.0
    assert sorted(set(np.abs(vals))) [1] == 2.0 ** -9     # smallest subnormal
    rng = np.random.default_rng(0)
    x = rng.standard_normal(20000) * rng.choice([1e-3, 1.0, 100.0], 20000)
    assert np.isin(fp8.e4m3_round(x), vals).all()


def test_ties_to_even_and_saturation():
    pos = np.unique(np.abs(_finite_values()))             # 0 and the 126 positive values
    codes = {fp8.e4m3_decode(c): c for c in range(0x7F)}
    for lo, hi in zip(pos[:-1], pos[1:]):
        mid = 0.5 * (lo + hi)
        want = lo if (codes[lo] & 1) == 0 else hi
        assert fp8.e4m3_round(mid) == want, (lo, hi)
        assert fp8.e4m3_round(-mid) == -want
        assert fp8.e4m3_round(np.nextafter(mid, 0)) == lo
        assert fp8.e4m3_round(np.nextafter(mid, np.inf)) == hi
    for big in (448.0, 460.0, 464.0, 500.0, 1e9):
        assert fp8.e4m3_round(big) == 448.0 and fp8.e4m3_round(-big) == -448.0
    assert fp8.e4m3_round(2.0 ** -10) == 0.0               # tie between 0 and 2^-9
    assert fp8.e4m3_round(3 * 2.0 ** -10) == 2 * 2.0 ** -9


def test_block_absmax_maps_to_448_and_grid_data_is_exact():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((256, 64)).astype(np.float32)
    codes, scales = fp8.quantize_q(x, bq=128)
    for b in range(2):
        blk = codes[b * 128:(b + 1) * 128]
        assert np.max(np.abs(blk)) == 448.0
    # data on the E4M3 grid scaled by 2^-5, with an element of magnitude 448 * 2^-5
    vals = _finite_values()
    g = rng.choice(vals, size=(128, 64)).astype(np.float32) * np.float32(2.0 ** -5)
    g[0, 0] = np.float32(448.0 * 2.0 ** -5)
    c, s = fp8.quantize_q(g, bq=128)
    assert s[0] == np.float32(2.0 ** -5)
    assert np.array_equal(c * np.float64(s[0]), g.astype(np.float64))
    z = np.zeros((128, 8), dtype=np.float32)
    cz, sz = fp8.quantize_q(z)
    assert sz[0] == 1.0 and not cz.any()


def test_smoothing_leaves_the_softmax_unchanged():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((16, 32)).astype(np.float32)
    k = (rng.standard_normal((40, 32)) + 3.0).astype(np.float32)
    ks = fp8.smooth_k(k)
    def softmax(s):
        e = np.exp(s - s.max(axis=1, keepdims=True))
        return e / e.sum(axis=1, keepdims=True)
    a = softmax(q.astype(np.float64) @ k.astype(np.float64).T)
    b = softmax(q.astype(np.float64) @ ks.astype(np.float64).T)
    assert np.allclose(a, b, atol=1e-9)
    assert np.all(np.abs(ks.astype(np.float64).mean(axis=0)) < 1e-4)


def test_quantised_k_is_invariant_to_a_common_key_shift():
    # keys on a 1/8 grid with a grid-valued shift: the fp32 mean and the
    # subtraction are exact, so smoothing removes the shift exactly
    rng = np.random.default_rng(3)
    k = (rng.integers(-40, 41, size=(64, 32)) / 8.0).astype(np.float32)
    c = (rng.integers(-16, 17, size=32) / 4.0).astype(np.float32)
    c0, s0 = fp8.quantize_k(k)
    c1, s1 = fp8.quantize_k(k + c)
    assert s0 == s1 and np.array_equal(c0, c1)


def test_dequantised_operands_within_half_a_step():
    # |x - x^| <= half an E4M3 step at x / s: 2^-4 |x| on the normal range,
    # s * 2^-10 on the subnormal range; nothing saturates since |x| / s <= 448
    rng = np.random.default_rng(4)
    q = (rng.standard_normal((300, 128)) * rng.choice([0.01, 1.0, 30.0], (300, 1))).astype(np.float32)
    k = (rng.standard_normal((300, 128)) + 2.0).astype(np.float32)
    v = (rng.standard_normal((300, 128)) * rng.choice([0.1, 5.0], (1, 128))).astype(np.float32)
    q_hat, k_hat, v_hat = fp8.dequantized_head(q, k, v)
    _, qs = fp8.quantize_q(q)
    _, ks = fp8.quantize_k(k)
    _, vs = fp8.quantize_v(v)
    s_q = np.repeat(qs.astype(np.float64), 128)[:300, None]
    ksm = fp8.smooth_k(k).astype(np.float64)
    for x, xh, s in ((q.astype(np.float64), q_hat, s_q), (ksm, k_hat, np.float64(ks)),
                     (v.astype(np.float64), v_hat, vs.astype(np.float64)[None, :])):
        bound = np.maximum(2.0 ** -4 * np.abs(x), s * 2.0 ** -10) * (1 + 1e-6)
        assert np.all(np.abs(x - xh) <= bound)
        # the largest magnitude of each scaling group maps to exactly 448
    assert np.max(np.abs(q_hat[:128])) == np.float64(qs[0]) * 448.0


def test_smoothing_mean_is_the_exact_mean_rounded_once():
    # the same exact-fraction fixture as the int4 estimate's: smooth_k must
    # subtract the correctly rounded fp32 mean (an fp32 sum, or a sum rounded
    # to fp32 before the division, gives other values on these keys)
    from test_oracle_sale import exact_mean_fixture
    k, want = exact_mean_fixture(seed=12, L=2999, d=64)
    np.testing.assert_array_equal(fp8.smooth_k(k), (k - want).astype(np.float32))
