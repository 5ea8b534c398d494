"""Pins for the oracle's masked softmax attention.

``oracle.attention.attend_row`` is checked against a brute-force evaluation in
plain Python (no max subtraction, exp and sums by loop) on tiny inputs with
random kept sets, including single-key rows; the dense causal reference is
checked the same way; permuting the kept keys must not change the result; and
the closed-form kept-pair count is checked against explicit enumeration.
"""

import math
import random

import numpy as np
import pytest

from oracle import attention as oatt


def _brute(q_i, kh, vh, keys, scale):
    e = []
    for j in keys:
        s = 0.0
        for t in range(len(q_i)):
            s += q_i[t] * kh[j][t]
        e.append(math.exp(s * scale))
    z = sum(e)
    out = [sum(e[n] * vh[keys[n]][t] for n in range(len(keys))) / z for t in range(len(vh[0]))]
    return out, math.log(z)


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_attend_row_brute_force(seed):
    rng = np.random.default_rng(seed)
    L, d = 48, 16
    qh = rng.standard_normal((L, d))
    kh = rng.standard_normal((L, d))
    vh = rng.standard_normal((L, d))
    scale = 1.0 / math.sqrt(d)
    pyr = random.Random(seed)
    for i in range(L):
        n = 1 if i % 7 == 0 else pyr.randint(1, i + 1)
        keys = sorted(pyr.sample(range(i + 1), n))
        o, lse = oatt.attend_row(qh[i], kh, vh, np.array(keys), scale)
        o_b, lse_b = _brute(qh[i].tolist(), kh.tolist(), vh.tolist(), keys, scale)
        np.testing.assert_allclose(o, o_b, atol=1e-12, rtol=0)
        assert lse == pytest.approx(lse_b, abs=1e-12)


def test_single_key_row_returns_that_value():
    rng = np.random.default_rng(5)
    kh = rng.standard_normal((8, 4))
    vh = rng.standard_normal((8, 4))
    q = rng.standard_normal(4)
    o, lse = oatt.attend_row(q, kh, vh, np.array([3]), 0.5)
    np.testing.assert_allclose(o, vh[3], atol=0, rtol=0)
    assert lse == pytest.approx(0.5 * float(q @ kh[3]), abs=1e-15)


def test_dense_causal_brute_force():
    rng = np.random.default_rng(11)
    L, d = 40, 8
    qh, kh, vh = (rng.standard_normal((L, d)) for _ in range(3))
    o, lse = oatt.dense_causal_rows(qh, kh, vh, range(L))
    for i in range(L):
        o_b, lse_b = _brute(qh[i].tolist(), kh.tolist(), vh.tolist(), list(range(i + 1)),
                            1.0 / math.sqrt(d))
        np.testing.assert_allclose(o[i], o_b, atol=1e-12, rtol=0)
        assert lse[i] == pytest.approx(lse_b, abs=1e-12)


def test_permuting_kept_keys_leaves_output_unchanged():
    rng = np.random.default_rng(3)
    L, d = 300, 128
    qh, kh, vh = (rng.standard_normal((L, d)) for _ in range(3))
    keys = np.sort(rng.choice(L, size=120, replace=False))
    o1, l1 = oatt.attend_row(qh[-1], kh, vh, keys, 1 / math.sqrt(d))
    o2, l2 = oatt.attend_row(qh[-1], kh, vh, rng.permutation(keys), 1 / math.sqrt(d))
    np.testing.assert_allclose(o1, o2, atol=1e-12, rtol=0)
    assert l1 == pytest.approx(l2, abs=1e-12)


@pytest.mark.parametrize("L,sink,local", [(1000, 64, 128), (777, 128, 256), (300, 0, 128),
                                          (2000, 300, 384)])
def test_kept_pairs_closed_form(L, sink, local):
    bq = 128
    rng = np.random.default_rng(L)
    for qb in range((L + bq - 1) // bq):
        ls = max(0, (qb + 1) * bq - local)
        cand = np.arange(sink, max(sink, ls))
        sel = np.sort(rng.choice(cand, size=min(len(cand), 17), replace=False)) if len(cand) else cand
        explicit = sum(len(oatt.kept_keys_for_row(i, qb, L, bq=bq, sink=sink, local=local,
                                                  selected=sel))
                       for i in range(qb * bq, min((qb + 1) * bq, L)))
        assert oatt.kept_pairs_block(qb, L, bq=bq, sink=sink, local=local,
                                     n_selected=len(sel)) == explicit
