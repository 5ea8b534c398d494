"""Pins for the decode-shaped reuse oracle (SpotAttention Fig. 2 / Sec. 3;
KVpop Sec. 3, transposed attention).

* a decode query at p = L - 1 has exactly the prefill kept set of row L - 1;
* with every candidate selected (theta -> +inf) the decode key set is every
  key up to p, and decode attention equals textbook causal softmax attention
  of the extended sequence at position p;
* with nothing selected it is the sink plus the grown local window, checked
  against a mask written as a whole vector;
* the per-key attention mass from the prefill LSE sums to the number of
  rows, and equals the column sums of the explicit masked-softmax matrix
  (dense and with a random selection).
"""

import numpy as np
import pytest

from oracle import decode as odec
from oracle.attention import attend_rows, dense_causal_rows, kept_keys_for_row
from oracle.selection import block_geometry


def _qkv(L, d=16, seed=0):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((L, d)), rng.standard_normal((L, d)),
            rng.standard_normal((L, d)))


def _random_selection(L, bq, sink, local, seed):
    rng = np.random.default_rng(seed)
    sel = {}
    for qb in range((L + bq - 1) // bq):
        ls = block_geometry(qb, L, bq, sink, local).ls
        cand = np.arange(sink, max(sink, ls))
        sel[qb] = np.sort(rng.choice(cand, size=len(cand) // 3, replace=False)) if len(cand) else cand
    return sel


@pytest.mark.parametrize("L,bq,sink,local", [(37, 8, 4, 8), (64, 16, 3, 32), (9, 8, 2, 8)])
def test_decode_at_last_prefill_row_is_that_row(L, bq, sink, local):
    sel = _random_selection(L, bq, sink, local, seed=L)
    qb = (L - 1) // bq
    got = odec.decode_keys(L - 1, L, sel[qb], bq=bq, sink=sink, local=local)
    want = kept_keys_for_row(L - 1, qb, L, bq=bq, sink=sink, local=local, selected=sel[qb])
    assert np.array_equal(got, want)


@pytest.mark.parametrize("L,extra", [(40, 0), (40, 5), (17, 12)])
def test_all_selected_decode_is_dense_causal_attention(L, extra):
    bq, sink, local = 8, 3, 16
    q, k, v = _qkv(L + extra, seed=L + extra)
    qb = (L - 1) // bq
    ls = block_geometry(qb, L, bq, sink, local).ls
    everything = np.arange(sink, max(sink, ls))
    p = L - 1 + extra
    keys = odec.decode_keys(p, L, everything, bq=bq, sink=sink, local=local)
    assert np.array_equal(keys, np.arange(p + 1))
    o, lse = odec.decode_attend(q[p], k, v, keys)
    o_ref, lse_ref = dense_causal_rows(q, k, v, [p])
    assert np.allclose(o, o_ref[0], atol=1e-12) and abs(lse - lse_ref[0]) < 1e-12


def test_nothing_selected_decode_is_sink_plus_window():
    L, extra, bq, sink, local = 50, 7, 8, 4, 16
    p = L - 1 + extra
    keys = odec.decode_keys(p, L, np.array([], dtype=np.int64), bq=bq, sink=sink, local=local)
    idx = np.arange(p + 1)
    window_start = ((L - 1) // bq + 1) * bq - local
    mask = (idx < sink) | (idx >= window_start)
    assert np.array_equal(keys, idx[mask])


@pytest.mark.parametrize("seed", [0, 1])
def test_key_mass_equals_masked_softmax_column_sums(seed):
    L, bq, sink, local = 48, 8, 3, 16
    q, k, v = _qkv(L, seed=seed)
    sel = _random_selection(L, bq, sink, local, seed=seed + 10)
    rows = range(L)
    _, lse = attend_rows(q, k, v, rows, lambda i: i // bq, lambda b: sel[b], bq=bq, sink=sink,
                         local=local)
    keys_of_row = odec.prefill_keys_of_row(L, lambda b: sel[b], bq=bq, sink=sink, local=local)
    mass = odec.key_mass(q, k, lse, rows, keys_of_row)
    # the whole probability matrix, from logits masked to -inf outside each kept set
    scale = 1.0 / np.sqrt(q.shape[1])
    logits = (q @ k.T) * scale
    masked = np.full((L, L), -np.inf)
    for i in rows:
        kk = keys_of_row(i)
        masked[i, kk] = logits[i, kk]
    probs = np.exp(masked - masked.max(axis=1, keepdims=True))
    probs /= probs.sum(axis=1, keepdims=True)
    assert np.allclose(mass, probs.sum(axis=0), atol=1e-12)
    assert abs(mass.sum() - L) < 1e-9


def test_key_mass_dense_is_causal_softmax_column_sums():
    L, bq, sink, local = 33, 8, 2, 8
    q, k, v = _qkv(L, seed=5)
    everything = lambda b: np.arange(sink, max(sink, block_geometry(b, L, bq, sink, local).ls))
    _, lse = dense_causal_rows(q, k, v, range(L))
    mass = odec.key_mass(q, k, lse, range(L),
                         odec.prefill_keys_of_row(L, everything, bq=bq, sink=sink, local=local))
    scale = 1.0 / np.sqrt(q.shape[1])
    s = (q @ k.T) * scale
    s[np.triu_indices(L, 1)] = -np.inf
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    assert np.allclose(mass, p.sum(axis=0), atol=1e-12)
