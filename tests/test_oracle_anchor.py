"""Pins for the oracle's anchor (stripe) selection.

Each check ties ``oracle.selection.anchor_block`` (and the kept-set assembly in
``oracle.attention``) to something other than itself:

* a hand-derived example (tests/golden/anchor_handmade.json) that fixes the
  sink/local geometry, the causal cut inside the local block, the mean over a
  ragged block, the scale and the direction of the comparison;
* theta -> +inf reduces to dense causal softmax attention (closed form);
* theta -> -inf reduces to sink + block-local window attention, checked against
  a mask written directly as an L x L matrix;
* avgpool linearity: the pooled score equals the row-mean of the full scores;
* nesting in theta and sink/local inclusion.
"""

import json
import math
import os

import numpy as np
import pytest

from oracle import attention as oatt
from oracle import selection as osel
from workloads import C0_TINY, generate

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _handmade():
    with open(os.path.join(GOLDEN, "anchor_handmade.json")) as f:
        g = json.load(f)
    L, d = g["seq_len"], g["head_dim"]
    q = np.zeros((L, d))
    q[:, 0] = g["q_e0"]
    k = np.zeros((L, d))
    k[:, 0] = g["k_e0_default"]
    k[: g["sink"], 0] = g["k_e0_sink"]
    for j, c in g["k_e0_special"].items():
        k[int(j), 0] = c
    return g, q, k


def _ranges_to_keys(ranges):
    if not ranges:
        return np.zeros(0, dtype=np.int64)
    return np.concatenate([np.arange(a, b) for a, b in ranges])


def test_handmade_anchor_cases():
    g, q, k = _handmade()
    for case in g["cases"]:
        blk = osel.anchor_block(q, k, case["qb"], bq=g["block_q"], sink=g["sink"],
                                local=g["local"], theta=case["theta"])
        assert blk.xbar_a == pytest.approx(math.sqrt(2) * case["xbar_over_sqrt2"], abs=1e-12), case
        lo, hi = case["candidates"]
        np.testing.assert_array_equal(blk.cand, np.arange(lo, hi))
        np.testing.assert_array_equal(blk.kept, _ranges_to_keys(case["kept_ranges"]), err_msg=str(case))


def _small_case(L=700, seed_cfg=C0_TINY):
    w = seed_cfg.with_(sink=64, local=256)
    inp = generate(w, seq_len=L)
    q, k, v = inp.as_f64()
    return w, q[0, 0], k[0, 0], v[0, 0]


def test_theta_plus_inf_equals_dense_causal():
    w, qh, kh, vh = _small_case()
    L = qh.shape[0]
    bq = w.block_q
    sel = {}
    for qb in range((L + bq - 1) // bq):
        blk = osel.anchor_block(qh, kh, qb, bq=bq, sink=w.sink, local=w.local, theta=math.inf)
        np.testing.assert_array_equal(blk.kept, blk.cand)
        sel[qb] = blk.kept
    rows = range(L)
    o_s, lse_s = oatt.attend_rows(qh, kh, vh, rows, lambda i: i // bq, lambda b: sel[b],
                                  bq=bq, sink=w.sink, local=w.local)
    o_d, lse_d = oatt.dense_causal_rows(qh, kh, vh, rows)
    np.testing.assert_allclose(o_s, o_d, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse_s, lse_d, atol=1e-12, rtol=0)


def test_theta_minus_inf_is_sink_plus_local_window():
    w, qh, kh, vh = _small_case(L=650)
    L, d = qh.shape
    bq, sink, local = w.block_q, w.sink, w.local
    sel = {}
    for qb in range((L + bq - 1) // bq):
        blk = osel.anchor_block(qh, kh, qb, bq=bq, sink=sink, local=local, theta=-math.inf)
        assert blk.kept.size == 0
        sel[qb] = blk.kept
    o_s, lse_s = oatt.attend_rows(qh, kh, vh, range(L), lambda i: i // bq, lambda b: sel[b],
                                  bq=bq, sink=sink, local=local)
    # StreamingLLM-style mask written directly over the whole L x L score matrix.
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    window_start = np.maximum(0, (i // bq + 1) * bq - local)
    allowed = (j <= i) & ((j < sink) | (j >= window_start))
    scores = (qh @ kh.T) / math.sqrt(d)
    scores = np.where(allowed, scores, -np.inf)
    top = scores.max(axis=1, keepdims=True)
    w_ = np.exp(scores - top)
    o_ref = (w_ @ vh) / w_.sum(axis=1, keepdims=True)
    lse_ref = top[:, 0] + np.log(w_.sum(axis=1))
    np.testing.assert_allclose(o_s, o_ref, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse_s, lse_ref, atol=1e-12, rtol=0)


def test_avgpool_linearity():
    w, qh, kh, _ = _small_case(L=900)
    d = qh.shape[1]
    bq = w.block_q
    for qb in range(2, (900 + bq - 1) // bq):
        blk = osel.anchor_block(qh, kh, qb, bq=bq, sink=w.sink, local=w.local, theta=3.0)
        rows = np.arange(qb * bq, min((qb + 1) * bq, 900))
        full = (qh[rows] @ kh[blk.cand].T) / math.sqrt(d)
        np.testing.assert_allclose(blk.sbar, full.mean(axis=0), atol=1e-12, rtol=0)


def test_nesting_in_theta():
    w, qh, kh, _ = _small_case(L=1500)
    bq = w.block_q
    thetas = [-1.0, 0.5, 2.0, 2.5, 3.0, 3.5, 5.0]
    for qb in range(3, 12):
        prev = None
        for th in thetas:
            kept = set(osel.anchor_block(qh, kh, qb, bq=bq, sink=w.sink, local=w.local, theta=th).kept)
            if prev is not None:
                assert prev <= kept
            prev = kept


def test_every_row_keeps_sink_and_local():
    w, qh, kh, _ = _small_case(L=800)
    L = qh.shape[0]
    bq = w.block_q
    for qb in range((L + bq - 1) // bq):
        blk = osel.anchor_block(qh, kh, qb, bq=bq, sink=w.sink, local=w.local, theta=-math.inf)
        ls = max(0, (qb + 1) * bq - w.local)
        for i in range(qb * bq, min((qb + 1) * bq, L)):
            keys = set(oatt.kept_keys_for_row(i, qb, L, bq=bq, sink=w.sink, local=w.local,
                                              selected=blk.kept))
            assert set(range(min(w.sink, i + 1))) <= keys
            assert set(range(ls, i + 1)) <= keys
            assert max(keys) == i


def test_margin_sign_matches_decision():
    w, qh, kh, _ = _small_case(L=1200)
    blk = osel.anchor_block(qh, kh, 7, bq=w.block_q, sink=w.sink, local=w.local, theta=3.0)
    np.testing.assert_array_equal(blk.cand[blk.margin >= 0], blk.kept)


def test_handmade_exact_ties_keep():
    g, q, k = _handmade()
    tc = g["tie_cases"]
    q = q / g["q_e0"] * tc["q_e0"]
    for case in tc["cases"]:
        blk = osel.anchor_block(q, k, case["qb"], bq=g["block_q"], sink=g["sink"],
                                local=g["local"], theta=case["theta"], scale=tc["scale"])
        assert blk.xbar_a == case["xbar"]
        np.testing.assert_array_equal(blk.kept, _ranges_to_keys(case["kept_ranges"]), err_msg=str(case))


def test_anchor_head_equals_per_block():
    w, qh, kh, _ = _small_case(L=1100)
    blocks = [0, 1, 2, 5, 8]
    many = osel.anchor_head(qh, kh, blocks, bq=w.block_q, sink=w.sink, local=w.local, theta=2.7)
    for qb in blocks:
        one = osel.anchor_block(qh, kh, qb, bq=w.block_q, sink=w.sink, local=w.local, theta=2.7)
        np.testing.assert_array_equal(many[qb].kept, one.kept)
        np.testing.assert_allclose(many[qb].margin, one.margin, atol=1e-12, rtol=0)
        assert many[qb].xbar_a == one.xbar_a


def test_step_grouping_pins():
    w, qh, kh, _ = _small_case(L=2000)
    L, bq = 2000, w.block_q
    nqb = (L + bq - 1) // bq
    own = osel.anchor_head(qh, kh, range(nqb), bq=bq, sink=w.sink, local=w.local, theta=2.6)
    sel = lambda b: own[b].kept
    for qb in range(nqb):
        geo = osel.block_geometry(qb, L, bq, w.sink, w.local)
        # step 1 is the identity
        np.testing.assert_array_equal(
            osel.step_union(sel, qb, step=1, nqb=nqb, cand_lo=geo.cand_lo, cand_hi=geo.cand_hi),
            own[qb].kept)
        # nesting: a block keeps at least its own selection, and more with larger groups
        # (groups of 2 sit inside groups of 4, which sit inside groups of 16)
        prev = set(own[qb].kept)
        for step in (2, 4, 16):
            cur = set(osel.step_union(sel, qb, step=step, nqb=nqb, cand_lo=geo.cand_lo,
                                      cand_hi=geo.cand_hi))
            assert prev <= cur
            assert all(geo.cand_lo <= j < geo.cand_hi for j in cur)
            prev = cur
        # a group covering the whole layer: the union of every block's selection,
        # clipped to this block's candidates
        allkeys = np.unique(np.concatenate([own[b].kept for b in range(nqb)]))
        expect = allkeys[(allkeys >= geo.cand_lo) & (allkeys < geo.cand_hi)]
        np.testing.assert_array_equal(
            osel.step_union(sel, qb, step=nqb, nqb=nqb, cand_lo=geo.cand_lo,
                            cand_hi=geo.cand_hi), expect)
