"""GPU: SALE per-head tau calibration through the library vs the oracle's.

The library version runs SALE mode and the same attention kernel in dense
mode and halves each head's tau until the L1 error is below theta_L1 on every
sample; the oracle does the same in fp64.  The library's Err carries the bf16
noise of its two outputs, measured here as its error with every candidate
kept (where the exact error is zero).  The bound theta_L1 is placed where the
oracle's errors of every head and halving step are farthest from it; with
that margin above the noise band the chosen taus must be identical, and the
library's errors must follow the oracle's within the band.
"""

import numpy as np
import pytest
import torch

from block_sparse_long_sm_b200.calibrate import (calibrate_sale_tau, dense_outputs,
                                                 sale_l1_errors)
from oracle import calibration as ocal
from workloads import bf16_bits_to_f32, calibration_samples

from gpu_common import to_dev

pytestmark = pytest.mark.gpu

HALVINGS = 5


def _choose_theta(hists):
    """Midpoint between two error values, farthest from every (head, step) error;
    among the best, prefer one at which the heads stop at different steps."""
    vals = sorted({e for hist in hists for e in hist})
    best = None
    for a, b in zip(vals, vals[1:]):
        theta = 0.5 * (a + b)
        ks = [next((i for i, e in enumerate(hist) if e < theta), len(hist) - 1) for hist in hists]
        if ks[0] == 0:
            continue                       # tau0 already meets it: nothing is calibrated
        key = (len(set(ks)) > 1, 0.5 * (b - a))
        if best is None or key > best[0]:
            best = (key, theta, ks)
    return best[1], best[2], best[0][1]


@pytest.mark.parametrize("hq,hkv,diffuse", [(1, 1, ()), (4, 2, (1,))])
def test_calibration_matches_oracle(hq, hkv, diffuse):
    """With a diffuse kv head, its q heads meet the bound at tau0 while the
    sink heads need halvings: the per-head taus differ."""
    L, sink, local = 1024, 64, 128
    group = hq // hkv
    samples = calibration_samples(2, heads_q=hq, heads_kv=hkv, seq_len=L, sink=sink, local=local,
                                  q_bias=6.0, sink_bias=11.0, diffuse_kv_heads=diffuse)
    hists = []
    for h in range(hq):
        per = [tuple(bf16_bits_to_f32(x[0, i]) for x, i in ((s.q, h), (s.k, h // group),
                                                          (s.v, h // group)))
               for s in samples]
        _, _, hist = ocal.calibrate_head(per, bq=128, bk=32, sink=sink, local=local,
                                         theta_l1=0.0, max_halvings=HALVINGS)
        hists.append([max(e) for e in hist])
    theta, k_oracle, margin = _choose_theta(hists)

    dev = [(to_dev(s.q), to_dev(s.k), to_dev(s.v)) for s in samples]
    dense = dense_outputs(dev, sink=sink, local=local)
    floor, _ = sale_l1_errors(dev, dense, [1e-30] * hq, sink=sink, local=local)
    # |Err_gpu - Err| is bounded by the mean L1 of the two outputs' rounding
    # noise, which the floor measures where the key sets agree; the band takes
    # 1.5x the floor plus 2e-3 of slack for the sets that differ
    band = 1.5 * max(floor) + 2e-3
    assert margin > band, (margin, band, hists)

    taus, errs, hist_gpu = calibrate_sale_tau(dev, sink=sink, local=local, theta_l1=theta,
                                              block_k=32, max_halvings=HALVINGS, dense=dense)
    torch.cuda.synchronize()
    k_gpu = [int(round(np.log2(0.008 / t))) for t in taus]
    assert k_gpu == k_oracle, (k_gpu, k_oracle, theta, hists, hist_gpu)
    for h in range(hq):
        for i in range(k_gpu[h] + 1):
            assert abs(hist_gpu[i][h] - hists[h][i]) < band, (h, i, hist_gpu[i][h], hists[h][i], band)
        assert errs[h] < theta
