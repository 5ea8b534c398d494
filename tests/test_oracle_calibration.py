"""Pins for the oracle's SALE per-head tau calibration (SALE Sec. 3.3 / App. C).

* a bound that the first tau already meets returns tau0 after one step;
* an unreachable bound (theta = 0) halves max_halvings times and returns the
  last tau;
* the error at the returned tau is the L1 definition recomputed from the
  outputs, and every earlier step's error is at or above the bound;
* tau -> 0 keeps every candidate block, so the error vanishes (SALE equals
  dense attention), a closed form.
"""

import numpy as np

from oracle import calibration as ocal
from workloads import bf16_bits_to_f32


def _samples(n=2, L=1024, q_bias=8.0, sink_bias=12.0):
    from workloads import calibration_samples
    out = []
    for inp in calibration_samples(n, heads_q=1, heads_kv=1, seq_len=L, sink=64, local=128,
                                   q_bias=q_bias, sink_bias=sink_bias):
        out.append(tuple(bf16_bits_to_f32(x[0, 0]) for x in (inp.q, inp.k, inp.v)))
    return out


def test_loose_bound_stops_at_tau0():
    s = _samples()
    tau, errs, hist = ocal.calibrate_head(s, bq=128, bk=32, sink=64, local=128, theta_l1=1e9)
    assert tau == 0.008 and len(hist) == 1


def test_unreachable_bound_halves_to_the_end():
    s = _samples(n=1)
    tau, errs, hist = ocal.calibrate_head(s, bq=128, bk=32, sink=64, local=128, theta_l1=0.0,
                                          max_halvings=3)
    assert tau == 0.008 / 8 and len(hist) == 4


def test_returned_tau_is_first_meeting_the_bound():
    s = _samples()
    _, _, hist = ocal.calibrate_head(s, bq=128, bk=32, sink=64, local=128, theta_l1=0.0,
                                     max_halvings=8)
    maxes = [max(e) for e in hist]
    assert maxes[0] > 0.0, "the samples must make SALE prune at tau0"
    assert maxes[-1] < maxes[0], "halving tau must reduce the error on these samples"
    k = next(i for i in range(1, len(maxes)) if maxes[i] < min(maxes[:i]))
    theta = 0.5 * (maxes[k] + min(maxes[:k]))
    tau, errs, hist2 = ocal.calibrate_head(s, bq=128, bk=32, sink=64, local=128,
                                           theta_l1=theta, max_halvings=8)
    assert tau == 0.008 / 2 ** k
    assert max(errs) < theta
    assert all(max(e) >= theta for e in hist2[:-1])


def test_tiny_tau_error_vanishes():
    s = _samples(n=1, L=512)
    q, k, v = s[0]
    o_sale = ocal.sale_head_output(q, k, q.astype(np.float64), k.astype(np.float64),
                                   v.astype(np.float64), bq=128, bk=32, sink=64, local=128,
                                   tau=1e-300)
    from oracle.attention import dense_causal_rows
    o_dense, _ = dense_causal_rows(q.astype(np.float64), k.astype(np.float64),
                                   v.astype(np.float64), range(512))
    assert ocal.err_l1(o_sale, o_dense) < 1e-12
