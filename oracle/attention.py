"""Attention over a kept key set, in fp64 (oracle; test infrastructure only).

AnchorAttention Sec. 3.4 ("fine-grained sparse computation") and SALE's
Computation Pass both run ordinary softmax attention restricted to the kept
keys; pruned entries are treated as -inf.  For row i of query block b the kept
set is

    K_i = (Sk u Lo_b u I_b) n {j <= i},

with Sk the sink keys, Lo_b the block-aligned local window and I_b the block's
selected candidate keys (AnchorAttention Eq. (3); for SALE the union of the
kept key blocks).  Sink and local keys are always kept.  Because local >= bq,
the local window contains the block's own diagonal, so no row is ever empty.

``attend_rows`` is the masked softmax (the FlashAttention output, computed
directly rather than online); ``dense_causal_rows`` is an independently written
dense causal softmax used as the theta -> +inf pin.
"""

from __future__ import annotations

from typing import Iterable, Tuple

import numpy as np

from .selection import block_geometry, default_scale


def kept_keys_for_row(i: int, qb: int, L: int, *, bq: int, sink: int, local: int,
                      selected: np.ndarray) -> np.ndarray:
    """Ascending K_i for row ``i`` of block ``qb`` given the block's selected keys."""
    geo = block_geometry(qb, L, bq, sink, local)
    assert geo.row_lo <= i < geo.row_hi
    sink_part = np.arange(0, min(sink, i + 1))
    local_part = np.arange(geo.ls, i + 1)
    sel = np.asarray(selected, dtype=np.int64)
    sel = sel[sel <= i]
    return np.union1d(np.union1d(sink_part, local_part), sel)


def attend_row(q_i: np.ndarray, kh: np.ndarray, vh: np.ndarray, keys: np.ndarray,
               scale: float) -> Tuple[np.ndarray, float]:
    """O_i = sum_j softmax_j(s_ij) v_j over ``keys``; returns (O_i, LSE_i) in fp64.

    LSE_i = m + ln(sum_j exp(s_ij - m)) with m the row maximum (natural log).
    """
    s = (kh[keys] @ q_i) * scale
    m = s.max()
    p = np.exp(s - m)
    den = p.sum()
    return (p @ vh[keys]) / den, float(m + np.log(den))


def attend_rows(qh: np.ndarray, kh: np.ndarray, vh: np.ndarray, rows: Iterable[int],
                qb_of_row, selected_of_block, *, bq: int, sink: int, local: int,
                scale: float = 0.0) -> Tuple[np.ndarray, np.ndarray]:
    """Sparse attention for the given rows of one q head.

    ``selected_of_block(qb)`` returns the block's selected candidate keys.
    """
    L, d = qh.shape
    sc = default_scale(d, scale)
    rows = list(rows)
    out = np.zeros((len(rows), vh.shape[1]))
    lse = np.zeros(len(rows))
    for n, i in enumerate(rows):
        qb = qb_of_row(i)
        keys = kept_keys_for_row(i, qb, L, bq=bq, sink=sink, local=local,
                                 selected=selected_of_block(qb))
        out[n], lse[n] = attend_row(qh[i], kh, vh, keys, sc)
    return out, lse


def dense_causal_rows(qh: np.ndarray, kh: np.ndarray, vh: np.ndarray,
                      rows: Iterable[int], scale: float = 0.0
                      ) -> Tuple[np.ndarray, np.ndarray]:
    """Textbook causal softmax attention softmax(q_i K[:i+1]^T * scale) V[:i+1].

    Written with the log-sum-exp first and the weights exp(s - lse) second, so
    that it shares no step with ``attend_row`` beyond the definition itself.
    """
    d = qh.shape[1]
    sc = default_scale(d, scale)
    rows = list(rows)
    out = np.zeros((len(rows), vh.shape[1]))
    lse = np.zeros(len(rows))
    for n, i in enumerate(rows):
        logits = sc * np.einsum("d,jd->j", qh[i], kh[: i + 1])
        top = np.max(logits)
        lse_i = top + np.log(np.sum(np.exp(logits - top)))
        w = np.exp(logits - lse_i)
        out[n] = np.einsum("j,jd->d", w, vh[: i + 1])
        lse[n] = lse_i
    return out, lse


def kept_pairs_block(qb: int, L: int, *, bq: int, sink: int, local: int,
                     n_selected: int) -> int:
    """sum_i |K_i| over the block's valid rows (each selected key is below every row)."""
    geo = block_geometry(qb, L, bq, sink, local)
    total = 0
    for i in range(geo.row_lo, geo.row_hi):
        # sink keys below the local window, the causal part of the window, the selection
        total += geo.sink_end + (i + 1 - geo.ls) + n_selected
    return total
