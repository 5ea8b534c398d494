"""Offline per-head threshold calibration for SALE mode (host procedure).

SALE Sec. 3.3 / Appendix C: every head's tau starts at 0.008 and is halved
until the L1 error of the sparse output against full attention,
Err(tau) = ||O - O~||_1 / N (N = query rows), is below theta_L1 on every
calibration sample.  Both outputs come from this library (SALE mode and the
same attention kernel in DENSE mode); the error itself is a small torch
reduction on the device, since calibration is an offline host loop and not
part of the prefill path.  The result feeds ``spa_params.tau_per_head``.

Both outputs are bf16, so Err carries a noise floor of its own (the two
kernels round differently where their key sets agree); ``sale_l1_errors``
with a vanishing tau (every candidate kept, exact Err = 0) measures it.
"""

from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

from . import binding as spa


def _shape(samples):
    q0 = samples[0][0]
    B, Hq, L, _ = q0.shape
    return B, Hq, samples[0][1].shape[1], L, q0.device


def dense_outputs(samples: Sequence[Tuple[object, object, object]], *, sink: int, local: int,
                  stream=None) -> List[object]:
    """Full causal attention of every sample (DENSE mode), as fp32 tensors."""
    import torch
    B, Hq, Hkv, L, dev = _shape(samples)
    pd = spa.make_params(B, Hq, Hkv, L, mode="dense", sink=sink, local=local)
    wsd = torch.empty(spa.sparse_prefill_workspace_bytes(pd), dtype=torch.uint8, device=dev)
    out = []
    for q, k, v in samples:
        o = torch.empty_like(q)
        spa.check(spa.sparse_prefill_plan(pd, q, k, wsd, stream=stream), "plan dense")
        spa.check(spa.sparse_prefill_attn(pd, q, k, v, wsd, o, None, stream=stream), "attn dense")
        out.append(o.float())
    return out


def sale_l1_errors(samples: Sequence[Tuple[object, object, object]], dense: Sequence[object],
                   taus: Sequence[float], *, sink: int, local: int, block_k: int = 32,
                   stream=None, workspace=None) -> Tuple[List[float], object]:
    """Per q head, the max over samples of Err at the given per-head taus.

    Returns (errors, workspace); pass the workspace back in to reuse it.
    """
    import torch
    B, Hq, Hkv, L, dev = _shape(samples)
    p = spa.make_params(B, Hq, Hkv, L, mode="sale", sink=sink, local=local, tau=float(taus[0]),
                        block_k=block_k, tau_per_head=list(taus))
    ws = workspace
    if ws is None:
        ws = torch.empty(spa.sparse_prefill_workspace_bytes(p), dtype=torch.uint8, device=dev)
    errs = torch.zeros(Hq, dtype=torch.float64, device=dev)
    for (q, k, v), od in zip(samples, dense):
        o = torch.empty_like(q)
        spa.check(spa.sparse_prefill_plan(p, q, k, ws, stream=stream), "plan sale")
        spa.check(spa.sparse_prefill_attn(p, q, k, v, ws, o, None, stream=stream), "attn sale")
        e = (o.float() - od).abs().double().sum(dim=(2, 3)) / L      # [B, Hq]
        errs = torch.maximum(errs, e.max(dim=0).values)
    return errs.tolist(), ws


def calibrate_sale_tau(samples: Sequence[Tuple[object, object, object]], *, sink: int, local: int,
                       theta_l1: float, block_k: int = 32, tau0: float = 0.008,
                       max_halvings: int = 12, stream=None,
                       dense: Optional[Sequence[object]] = None):
    """samples: list of (q, k, v) bf16 device tensors of one layer shape.

    Returns (tau per q head, error per q head at that tau, history) where the
    history holds, per halving step, the per-head max-over-samples error.
    """
    _, Hq, _, _, _ = _shape(samples)
    if dense is None:
        dense = dense_outputs(samples, sink=sink, local=local, stream=stream)
    taus = [float(tau0)] * Hq
    done = [False] * Hq
    final_err = [float("inf")] * Hq
    history: List[List[float]] = []
    ws = None
    for step in range(max_halvings + 1):
        errs_h, ws = sale_l1_errors(samples, dense, taus, sink=sink, local=local,
                                    block_k=block_k, stream=stream, workspace=ws)
        history.append(errs_h)
        for h in range(Hq):
            if done[h]:
                continue
            final_err[h] = errs_h[h]
            if errs_h[h] < theta_l1:
                done[h] = True
            elif step < max_halvings:
                taus[h] = taus[h] / 2.0
        if all(done):
            break
    return taus, final_err, history
