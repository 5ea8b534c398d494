"""Pins for the oracle's SALE selection.

* The corrected threshold rewrite agrees with the exp/divide form of the
  Relative Attention Score on 10^6 random draws, near-ties included, and the
  printed form of Eq. (4) gives different decisions.
* Integer inputs in [-7, 7] whose blocks reach absmax 7 (and whose K columns
  have zero mean) quantise exactly, so S~ equals the exact scaled score.
* Quantisation properties: codes in [-7, 7], absmax element at +-7, error at
  most half a step; K smoothing makes the result invariant to adding one
  vector to every key.
* A hand-derived example (tests/golden/sale_handmade.json) fixes em/el over
  the sink-local area, the threshold, the block maximum and tie handling.
* Nesting in tau.
* The smoothing mean (the per-head K mean over the sequence) equals the
  correctly rounded fp32 value of the exact rational mean, computed here with
  exact fractions, on bf16-valued keys with a non-zero mean and a length that
  is not a power of two -- inputs on which an fp32 sum, or rounding the sum
  to fp32 before dividing, lands on a different fp32 value.
"""

import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import selection as osel
from workloads import C0_TINY, bf16_bits_to_f32, generate

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_threshold_rewrite_matches_relative_score():
    rng = np.random.default_rng(0)
    n = 1_000_000
    em = rng.normal(0, 5, n)
    el = np.exp(rng.uniform(0, 8, n))           # el >= 1 (it contains exp(em - em))
    tau = np.exp(rng.uniform(np.log(1e-6), 0, n))
    s = em + rng.normal(0, 6, n)
    # planted near-ties: S~ within 1e-7 of the threshold
    tie = rng.random(n) < 0.1
    t = osel.sale_threshold(em, el, tau)
    s = np.where(tie, t + rng.uniform(-1e-7, 1e-7, n), s)
    by_log = s >= osel.sale_threshold(em, el, tau)
    p = np.exp(s - em) / el                     # Relative Attention Score
    by_exp = p >= tau
    disagree = by_log != by_exp
    # disagreement only where S~ sits within rounding of the threshold
    assert np.all(np.abs(s - t)[disagree] < 1e-12 * (1 + np.abs(t[disagree])) + 1e-12)
    assert disagree.mean() < 1e-4
    printed = s >= osel.sale_threshold_as_printed(em, el, tau)
    assert (printed != by_exp).mean() > 0.05


def test_relative_score_definition():
    s = np.array([[1.0, 2.0, 0.5]])
    em = np.array([2.0])
    el = np.array([1.0 + math.exp(-1.0)])
    p = osel.relative_score(s, em, el)
    np.testing.assert_allclose(p, np.exp(s - 2.0) / el[0], rtol=0, atol=0)


def test_integer_inputs_quantise_exactly():
    rng = np.random.default_rng(1)
    L, d, bq, bk = 256, 128, 128, 32
    q = rng.integers(-7, 8, (L, d)).astype(np.float32)
    for blk in range(L // bq):
        q[blk * bq, 0] = 7.0                    # every Q block reaches absmax 7
    half = rng.integers(-7, 8, (L // 2, d)).astype(np.float32)
    for blk in range((L // 2) // bk):
        half[blk * bk, 1] = 7.0                 # every K block reaches absmax 7
    k = np.concatenate([half, -half])           # zero column means, exactly
    prep = osel.sale_prepare(q, k, bq=bq, bk=bk)
    np.testing.assert_array_equal(prep.kmean, np.zeros(d, dtype=np.float32))
    np.testing.assert_array_equal(prep.qscales, np.ones(L // bq, dtype=np.float32))
    np.testing.assert_array_equal(prep.kscales, np.ones(L // bk, dtype=np.float32))
    np.testing.assert_array_equal(prep.qcodes, q.astype(np.int8))
    np.testing.assert_array_equal(prep.kcodes, k.astype(np.int8))
    s = osel.sale_scores(prep.qcodes[:bq], 1.0, prep.kcodes, np.ones(L), 1 / math.sqrt(d))
    np.testing.assert_allclose(s, (q[:bq].astype(np.float64) @ k.T.astype(np.float64)) / math.sqrt(d),
                               rtol=0, atol=1e-12)


def test_quantisation_properties_on_generated_data():
    inp = generate(C0_TINY, seq_len=1000)
    q32 = bf16_bits_to_f32(inp.q[0, 0])
    k32 = bf16_bits_to_f32(inp.k[0, 0])
    for x32, rows in ((q32, 128), (k32, 32)):
        codes, scales = osel._quantize_rows_fp32(x32, rows)
        assert codes.min() >= -7 and codes.max() <= 7
        for blk in range(len(scales)):
            part = x32[blk * rows:(blk + 1) * rows]
            c = codes[blk * rows:(blk + 1) * rows]
            assert np.abs(c).max() == 7
            err = np.abs(part.astype(np.float64) - c.astype(np.float64) * float(scales[blk]))
            assert err.max() <= 0.5 * float(scales[blk]) * (1 + 1e-6)


def test_smoothing_invariance_to_common_key_shift():
    rng = np.random.default_rng(4)
    L, d = 512, 128
    k = rng.integers(-20, 21, (L, d)).astype(np.float32)
    shift = rng.integers(-5, 6, d).astype(np.float32)
    q = rng.integers(-7, 8, (L, d)).astype(np.float32)
    a = osel.sale_prepare(q, k, bq=128, bk=32)
    b = osel.sale_prepare(q, k + shift, bq=128, bk=32)
    np.testing.assert_array_equal(a.kcodes, b.kcodes)
    np.testing.assert_array_equal(a.kscales, b.kscales)
    for qb in range(1, 4):
        ra = osel.sale_block(a, qb, L=L, bq=128, bk=32, sink=32, local=128, tau=1e-3)
        rb = osel.sale_block(b, qb, L=L, bq=128, bk=32, sink=32, local=128, tau=1e-3)
        np.testing.assert_array_equal(ra.kept_blocks, rb.kept_blocks)


def _handmade():
    with open(os.path.join(GOLDEN, "sale_handmade.json")) as f:
        g = json.load(f)
    L, d = g["seq_len"], g["head_dim"]
    q = np.zeros((L, d), dtype=np.float32)
    q[:, 0] = g["q_e0"]
    k = np.zeros((L, d), dtype=np.float32)
    k[: g["sink"], 0] = g["k_e0_sink"]
    for lo, hi, c in g["k_e0_ranges"]:
        k[lo:hi, 0] = c
    for j, c in g["k_e0_special"].items():
        k[int(j), 0] = c
    return g, q, k


def test_handmade_sale_cases():
    g, q, k = _handmade()
    prep = osel.sale_prepare(q, k, bq=g["block_q"], bk=g["block_k"])
    a = 49.0 / math.sqrt(g["head_dim"])
    for case in g["cases"]:
        r = osel.sale_block(prep, g["qb"], L=g["seq_len"], bq=g["block_q"], bk=g["block_k"],
                            sink=g["sink"], local=g["local"], tau=case["tau"])
        np.testing.assert_array_equal(r.cand_blocks, np.arange(*g["candidate_blocks"]))
        np.testing.assert_array_equal(r.kept_blocks, np.array(case["kept_blocks"], dtype=np.int64),
                                      err_msg=str(case))
        rows = np.arange(384, 512)
        np.testing.assert_allclose(r.em, np.full(128, a), rtol=0, atol=1e-12)
        np.testing.assert_allclose(r.el, 32 + (rows - 383) * math.exp(-a), rtol=1e-13, atol=0)


def test_nesting_in_tau():
    inp = generate(C0_TINY, seq_len=2048)
    q32 = bf16_bits_to_f32(inp.q[0, 0])
    k32 = bf16_bits_to_f32(inp.k[0, 0])
    prep = osel.sale_prepare(q32, k32, bq=128, bk=32)
    for qb in (4, 9, 15):
        prev = None
        for tau in (1e-1, 3e-2, 1e-2, 3e-3, 1e-3, 1e-4):
            kept = set(osel.sale_block(prep, qb, L=2048, bq=128, bk=32, sink=64, local=128,
                                       tau=tau).kept_blocks)
            if prev is not None:
                assert prev <= kept
            prev = kept


def test_tiny_tau_keeps_every_candidate_block():
    inp = generate(C0_TINY, seq_len=1024)
    prep = osel.sale_prepare(bf16_bits_to_f32(inp.q[0, 0]), bf16_bits_to_f32(inp.k[0, 0]),
                             bq=128, bk=32)
    r = osel.sale_block(prep, 6, L=1024, bq=128, bk=32, sink=64, local=128, tau=1e-300)
    np.testing.assert_array_equal(r.kept_blocks, r.cand_blocks)


def _bf16_valued(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest even) and return them as fp32."""
    b = x.astype(np.float32).view(np.uint32).astype(np.uint64)
    b = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16) << 16
    return b.astype(np.uint32).view(np.float32)


def _nearest_fp32(fr: Fraction) -> np.float32:
    """The fp32 value nearest to an exact rational (no ties allowed here)."""
    f = np.float32(float(fr))
    cands = [np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))]
    dist = sorted((abs(Fraction(float(c)) - fr), n) for n, c in enumerate(cands))
    assert dist[0][0] != dist[1][0], "the fixture must avoid an fp32 tie"
    # the mean is rounded twice (fp64 division, then fp32): a result within
    # 2^-50 (relative) of an fp32 midpoint could round either way
    half_gap = abs(Fraction(float(cands[2])) - Fraction(float(cands[1]))) / 2
    assert abs(dist[0][0] - half_gap) > abs(fr) * Fraction(1, 2 ** 50)
    return cands[dist[0][1]]


def exact_mean_fixture(seed: int = 11, L: int = 3000, d: int = 128):
    """bf16-valued keys with a non-zero mean, and their exact per-column means
    rounded once to fp32."""
    rng = np.random.default_rng(seed)
    k = _bf16_valued(rng.normal(0, 1, (L, d)).astype(np.float32) + np.float32(2.5))
    want = np.array([_nearest_fp32(sum(Fraction(float(v)) for v in k[:, c]) / L)
                     for c in range(d)], dtype=np.float32)
    return k, want


def test_smoothing_mean_is_the_exact_mean_rounded_once():
    k, want = exact_mean_fixture()
    L = k.shape[0]
    # the fixture separates the reading from its plausible slips
    assert np.count_nonzero(k.sum(axis=0, dtype=np.float32) / np.float32(L) != want) > 0
    assert np.count_nonzero(k.astype(np.float64).sum(axis=0).astype(np.float32) /
                            np.float32(L) != want) > 0
    np.testing.assert_array_equal(osel.sale_smooth_mean(k), want)
    # and the smoothed keys the codes are taken from are K minus that mean (fp32)
    codes, scales, mean = osel.sale_quantize_k(k, 32)
    np.testing.assert_array_equal(mean, want)
    for blk in range(L // 32):
        ks = k[blk * 32:(blk + 1) * 32] - want
        amax = np.float32(np.abs(ks).max())
        assert scales[blk] == np.float32(amax / np.float32(7.0))
