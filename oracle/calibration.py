"""SALE per-head threshold calibration, in fp64 (oracle; test infrastructure only).

SALE Sec. 3.3 and Appendix C: each head's tau starts at tau0 = 0.008 and is
halved until the L1 error of SALE's output against full attention,
Err(tau) = ||O - O~||_1 / N, is below theta_L1 on every calibration sample
(the paper uses five samples; theta_L1 = 0.4 for Llama-3.1, 2.0 for
Qwen-2.5).  Readings: ||.||_1 sums absolute differences over all query rows
and the head dimension, N is the number of query rows; the returned tau is
the largest tau0 / 2^k (k <= max_halvings) meeting the bound, or the last one
tried when none does.
"""

from __future__ import annotations

from typing import List, Sequence, Tuple

import numpy as np

from .attention import attend_rows, dense_causal_rows
from .selection import sale_block, sale_blocks_to_keys, sale_prepare


def err_l1(o_sparse: np.ndarray, o_dense: np.ndarray) -> float:
    """Err = ||O - O~||_1 / N over N query rows."""
    return float(np.abs(o_sparse - o_dense).sum() / o_sparse.shape[0])


def sale_head_output(q32, k32, q64, k64, v64, *, bq: int, bk: int, sink: int, local: int,
                     tau: float) -> np.ndarray:
    L = q64.shape[0]
    prep = sale_prepare(q32, k32, bq=bq, bk=bk)
    sel = {}
    for qb in range((L + bq - 1) // bq):
        r = sale_block(prep, qb, L=L, bq=bq, bk=bk, sink=sink, local=local, tau=tau)
        sel[qb] = sale_blocks_to_keys(r.kept_blocks, bk)
    o, _ = attend_rows(q64, k64, v64, range(L), lambda i: i // bq, lambda b: sel[b], bq=bq,
                       sink=sink, local=local)
    return o


def calibrate_head(samples: Sequence[Tuple[np.ndarray, np.ndarray, np.ndarray]], *, bq: int,
                   bk: int, sink: int, local: int, theta_l1: float, tau0: float = 0.008,
                   max_halvings: int = 12) -> Tuple[float, List[float], List[List[float]]]:
    """samples: (q, k, v) of one head as fp32 arrays widened from bf16.

    Returns (tau, per-sample errors at tau, error history per halving step).
    """
    dense = []
    for q, k, v in samples:
        q64, k64, v64 = (x.astype(np.float64) for x in (q, k, v))
        o, _ = dense_causal_rows(q64, k64, v64, range(q.shape[0]))
        dense.append(o)
    history = []
    tau = tau0
    for step in range(max_halvings + 1):
        tau = tau0 / (2.0 ** step)
        errs = []
        for (q, k, v), od in zip(samples, dense):
            o = sale_head_output(q, k, q.astype(np.float64), k.astype(np.float64),
                                 v.astype(np.float64), bq=bq, bk=bk, sink=sink, local=local,
                                 tau=tau)
            errs.append(err_l1(o, od))
        history.append(errs)
        if max(errs) < theta_l1:
            return tau, errs, history
    return tau, history[-1], history
