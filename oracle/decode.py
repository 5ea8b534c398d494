"""Decode-shaped reuse of a prefill plan, in fp64 (oracle; test infrastructure only).

Two uses of a finished prefill's selection and its log-sum-exp output, as
the pages describe them for decoding after a sparse prefill:

* SpotAttention (Fig. 2 and Sec. 3): a decode query attends to a sink prefix,
  a recency window and a set of selected content blocks only.  Reading (no
  learned selector here): the decode query at absolute position p >= L - 1
  reuses the selection of the last prefill query block qb = (L - 1) // bq,
  so its key set is

      D(p) = Sk u I_qb u [ls_qb, p],

  the sink, that block's kept candidates, and every key from that block's
  local start up to p (its local window grown by the decoded tokens).  For
  p = L - 1 this is exactly the prefill kept set of row L - 1.

* KVpop (Sec. 3, "transposed attention"): the attention mass a key receives
  from a set of query rows, sum_i exp(s_ij - LSE_i) over the rows i whose kept
  set holds j, computed from Q, K and the prefill's LSE without recomputing
  the softmax normalisers.  Over all rows these masses sum to the number of
  rows, since each row's probabilities sum to one.
"""

from __future__ import annotations

from typing import Callable, Iterable, Tuple

import numpy as np

from .attention import attend_row, kept_keys_for_row
from .selection import block_geometry, default_scale


def decode_keys(p: int, L: int, last_selected: np.ndarray, *, bq: int, sink: int,
                local: int) -> np.ndarray:
    """Ascending D(p) for a decode query at position p >= L - 1 (keys 0..p exist)."""
    assert L >= 1 and p >= L - 1
    qb = (L - 1) // bq
    geo = block_geometry(qb, L, bq, sink, local)
    sel = np.asarray(last_selected, dtype=np.int64)
    return np.union1d(np.union1d(np.arange(0, min(sink, p + 1)), sel),
                      np.arange(geo.ls, p + 1))


def decode_attend(q: np.ndarray, kh: np.ndarray, vh: np.ndarray, keys: np.ndarray,
                  scale: float = 0.0) -> Tuple[np.ndarray, float]:
    """Softmax attention of one query over ``keys``: (O, LSE) in fp64."""
    return attend_row(q, kh, vh, keys, default_scale(q.shape[0], scale))


def key_mass(qh: np.ndarray, kh: np.ndarray, lse: np.ndarray, rows: Iterable[int],
             keys_of_row: Callable[[int], np.ndarray], scale: float = 0.0) -> np.ndarray:
    """Attention mass each key receives from ``rows``: sum_i exp(s_ij - LSE_i).

    ``lse[n]`` is the log-sum-exp of the n-th row of ``rows`` over its kept
    set ``keys_of_row(i)``; keys outside every kept set receive 0.
    """
    sc = default_scale(qh.shape[1], scale)
    mass = np.zeros(kh.shape[0])
    for n, i in enumerate(rows):
        keys = keys_of_row(i)
        mass[keys] += np.exp((kh[keys] @ qh[i]) * sc - lse[n])
    return mass


def prefill_keys_of_row(L: int, selected_of_block, *, bq: int, sink: int, local: int):
    """keys_of_row for the prefill rows of a plan (K_i of AnchorAttention Eq. (3))."""
    def keys(i: int) -> np.ndarray:
        qb = i // bq
        return kept_keys_for_row(i, qb, L, bq=bq, sink=sink, local=local,
                                 selected=selected_of_block(qb))
    return keys
