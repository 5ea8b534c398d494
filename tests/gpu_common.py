"""Shared helpers for the GPU parity tests (CUDA path through the C ABI vs oracle).

Tolerances (from the target definition of the path):
* selection: bit-exact except at entries whose oracle margin to the
  threshold is below 1e-3 (such near-ties may go either way);
* outputs, computed by the oracle on the GPU's own kept sets: max abs error
  <= 1e-2 and mean abs error <= 1e-3 against fp64;
* LSE: <= 2e-3 absolute (fp32 accumulation of up to 1.3e5 exponentials plus
  the bf16-rounded probabilities; natural-log units).
"""

from __future__ import annotations

import math
from typing import Dict, Iterable, List, Sequence, Tuple

import numpy as np
import torch

import block_sparse_long_sm_b200 as spa
from block_sparse_long_sm_b200.binding import WorkspaceView
from oracle import attention as oatt
from oracle import selection as osel
from workloads import Inputs, bf16_bits_to_f32

MASK_MARGIN = 1e-3
O_MAX_ABS = 1e-2
O_MEAN_ABS = 1e-3
LSE_ABS = 2e-3


def to_dev(u16: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).cuda().view(torch.bfloat16)


class Run:
    """One plan + attn through the C ABI on device copies of ``inputs``."""

    def __init__(self, inputs: Inputs, *, mode: str, sink: int, local: int, theta: float = 5.0,
                 tau: float = 1e-3, block_k=None, do_attn: bool = True, lse: bool = True,
                 dev=None, step: int = 1, debug_flags: int = 0):
        B, Hq, L, _ = inputs.q.shape
        Hkv = inputs.k.shape[1]
        self.B, self.Hq, self.Hkv, self.L = B, Hq, Hkv, L
        self.group = Hq // Hkv
        self.params = spa.make_params(B, Hq, Hkv, L, mode=mode, sink=sink, local=local,
                                      theta=theta, tau=tau, block_k=block_k, step=step,
                                      debug_flags=debug_flags)
        self.q, self.k, self.v = dev if dev is not None else (
            to_dev(inputs.q), to_dev(inputs.k), to_dev(inputs.v))
        nbytes = spa.sparse_prefill_workspace_bytes(self.params)
        assert nbytes > 0
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        spa.check(spa.sparse_prefill_plan(self.params, self.q, self.k, self.ws), "plan")
        self.o = None
        self.lse = None
        if do_attn:
            self.o = torch.empty((B, Hq, L, 128), dtype=torch.bfloat16, device="cuda")
            self.lse = torch.empty((B, Hq, L), dtype=torch.float32, device="cuda") if lse else None
            spa.check(spa.sparse_prefill_attn(self.params, self.q, self.k, self.v, self.ws,
                                              self.o, self.lse), "attn")
        st, self.stats = spa.sparse_prefill_stats(self.params, self.ws)
        spa.check(st, "stats")
        torch.cuda.synchronize()
        self.view = WorkspaceView(self.params, self.ws)
        self.counts = self.view.counts.cpu().numpy()
        self._lists = None

    def lists_host(self) -> np.ndarray:
        if self._lists is None:
            self._lists = self.view.lists.cpu().numpy()
        return self._lists

    def block_list(self, b: int, h: int, qb: int) -> np.ndarray:
        n = int(self.counts[self.view.block_index(b, h, qb)])
        off = self.view.list_offset(b, h, qb)
        return self.lists_host()[off:off + n].astype(np.int64)

    def selected_keys(self, b: int, h: int, qb: int) -> np.ndarray:
        lst = self.block_list(b, h, qb)
        if self.params.mode == spa.SPA_MODE_SALE:
            return osel.sale_blocks_to_keys(lst, self.params.block_k)
        return lst


def head_f64(x_u16: np.ndarray, b: int, h: int) -> np.ndarray:
    return bf16_bits_to_f32(x_u16[b, h]).astype(np.float64)


def check_list_shape(lst: np.ndarray, lo: int, hi: int):
    assert np.all(np.diff(lst) > 0), "list not strictly ascending"
    if lst.size:
        assert lst[0] >= lo and lst[-1] < hi, (lst[0], lst[-1], lo, hi)


def compare_anchor_masks(run: Run, inputs: Inputs, heads: Sequence[Tuple[int, int]],
                         blocks_of=None, theta: float = None) -> Dict[str, int]:
    """Selection parity for the given (b, h) heads; returns mismatch counts.

    With step > 1 the oracle's selection of a block is the union over its
    group (oracle.selection.step_union); a key may differ only if its decision
    is a near-tie in some block of the group.
    """
    p = run.params
    theta = p.theta if theta is None else theta
    step = int(p.step)
    nqb = (run.L + 127) // 128
    total = dict(blocks=0, kept=0, mismatches=0, near_tie=0)
    for b, h in heads:
        qh = head_f64(inputs.q, b, h)
        kh = head_f64(inputs.k, b, h // run.group)
        blocks = list(range(nqb)) if blocks_of is None else list(blocks_of(b, h))
        need = sorted({g for qb in blocks
                       for g in range((qb // step) * step, min((qb // step) * step + step, nqb))})
        ora = osel.anchor_head(qh, kh, need, bq=128, sink=p.sink, local=p.local, theta=theta)
        for qb in blocks:
            o = ora[qb]
            kept = osel.step_union(lambda x: ora[x].kept, qb, step=step, nqb=nqb,
                                   cand_lo=o.cand[0] if o.cand.size else p.sink,
                                   cand_hi=(o.cand[-1] + 1) if o.cand.size else p.sink)
            g = run.block_list(b, h, qb)
            check_list_shape(g, o.cand[0] if o.cand.size else p.sink, (o.cand[-1] + 1) if o.cand.size else p.sink)
            diff = np.setxor1d(g, kept)
            if diff.size:
                g0 = (qb // step) * step
                m = np.full(diff.shape, np.inf)
                for b2 in range(g0, min(g0 + step, nqb)):
                    c2 = ora[b2].cand
                    inside = (diff >= p.sink) & (diff < p.sink + c2.size)
                    m[inside] = np.minimum(m[inside], np.abs(ora[b2].margin[diff[inside] - p.sink]))
                bad = np.abs(m) >= MASK_MARGIN
                assert not bad.any(), (
                    f"mask mismatch b={b} h={h} qb={qb}: keys {diff[bad][:8]} margins {m[bad][:8]}")
                total["near_tie"] += int(diff.size)
            total["blocks"] += 1
            total["kept"] += int(g.size)
    return total


def compare_sale_masks(run: Run, inputs: Inputs, heads: Sequence[Tuple[int, int]],
                       blocks_of=None) -> Dict[str, int]:
    p = run.params
    bk = p.block_k
    nqb = (run.L + 127) // 128
    total = dict(blocks=0, kept=0, near_tie=0)
    for b, h in heads:
        q32 = bf16_bits_to_f32(inputs.q[b, h])
        k32 = bf16_bits_to_f32(inputs.k[b, h // run.group])
        prep = osel.sale_prepare(q32, k32, bq=128, bk=bk)
        blocks = list(range(nqb)) if blocks_of is None else list(blocks_of(b, h))
        for qb in blocks:
            o = osel.sale_block(prep, qb, L=run.L, bq=128, bk=bk, sink=p.sink, local=p.local,
                                tau=p.tau)
            g = run.block_list(b, h, qb)
            lo = o.cand_blocks[0] if o.cand_blocks.size else 0
            hi = (o.cand_blocks[-1] + 1) if o.cand_blocks.size else 0
            check_list_shape(g, lo, hi)
            diff = np.setxor1d(g, o.kept_blocks)
            if diff.size:
                m = o.margin[diff - lo]
                bad = np.abs(m) >= MASK_MARGIN
                assert not bad.any(), (
                    f"SALE mismatch b={b} h={h} qb={qb}: blocks {diff[bad][:8]} margins {m[bad][:8]}")
                total["near_tie"] += int(diff.size)
            total["blocks"] += 1
            total["kept"] += int(g.size)
    return total


def compare_outputs(run: Run, inputs: Inputs, rows_of: Dict[Tuple[int, int], Iterable[int]],
                    dense: bool = False, bound: str = "stated") -> Dict[str, float]:
    """Output parity on the GPU's own kept sets (or dense causal), given rows per head.

    ``bound="stated"`` applies the fixed tolerances above.  ``bound="bf16"``
    applies instead, element by element, the error bound of the kernel's
    arithmetic, for inputs whose attention is concentrated on a few keys
    (a strong sink): the probabilities enter the PV product rounded to bf16
    (relative error <= 2^-8 each) and the output is rounded to bf16, so
    |dO_i| <= 2^-8 (sum_j p_ij |v_j| / l_i + 2 |O_i|) + 1e-4, where the
    weighted mean of |v| is the oracle's attention over |V|.
    """
    p = run.params
    o_gpu = run.o.float().cpu().numpy() if run.o is not None else None
    lse_gpu = run.lse.cpu().numpy() if run.lse is not None else None
    errs: List[np.ndarray] = []
    lse_err = 0.0
    for (b, h), rows in rows_of.items():
        rows = sorted(set(int(r) for r in rows))
        qh = head_f64(inputs.q, b, h)
        kh = head_f64(inputs.k, b, h // run.group)
        vh = head_f64(inputs.v, b, h // run.group)
        if dense:
            o_ref, lse_ref = oatt.dense_causal_rows(qh, kh, vh, rows)
        else:
            cache = {}

            def sel(qb):
                if qb not in cache:
                    cache[qb] = run.selected_keys(b, h, qb)
                return cache[qb]
            o_ref, lse_ref = oatt.attend_rows(qh, kh, vh, rows, lambda i: i // 128, sel, bq=128,
                                              sink=p.sink, local=p.local)
        d = np.abs(o_gpu[b, h, rows].astype(np.float64) - o_ref)
        if bound == "bf16":
            if dense:
                w_ref, _ = oatt.dense_causal_rows(qh, kh, np.abs(vh), rows)
            else:
                w_ref, _ = oatt.attend_rows(qh, kh, np.abs(vh), rows, lambda i: i // 128, sel,
                                            bq=128, sink=p.sink, local=p.local)
            lim = 2.0 ** -8 * (w_ref + 2.0 * np.abs(o_ref)) + 1e-4
            worst = float(np.max(d / lim))
            assert worst <= 1.0, (f"b={b} h={h}: error above the bf16 bound", worst)
        errs.append(d.ravel())
        if lse_gpu is not None:
            lse_err = max(lse_err, float(np.max(np.abs(lse_gpu[b, h, rows] - lse_ref))))
    e = np.concatenate(errs)
    res = dict(max_abs=float(e.max()), mean_abs=float(e.mean()), lse_max=lse_err, n=int(e.size))
    if bound == "stated":
        assert res["max_abs"] <= O_MAX_ABS, res
    assert res["mean_abs"] <= O_MEAN_ABS, res
    assert res["lse_max"] <= LSE_ABS, res
    return res


def sample_rows(L: int, n: int, seed: int, must: Sequence[int] = ()) -> List[int]:
    rng = np.random.default_rng(seed)
    rows = set(int(r) for r in must if 0 <= r < L)
    rows.update(int(r) for r in rng.integers(0, L, size=n))
    return sorted(rows)


def edge_blocks(L: int, extra: int, seed: int) -> List[int]:
    nqb = (L + 127) // 128
    rng = np.random.default_rng(seed)
    s = {0, 1, 2, 3, nqb // 2, nqb - 2, nqb - 1}
    s.update(int(x) for x in rng.integers(0, nqb, size=extra))
    return sorted(x for x in s if 0 <= x < nqb)


def sale_scratch(run: Run) -> Dict[str, np.ndarray]:
    """The SALE plan's quantised operands, read back from the workspace.

    Offsets follow the workspace layout of SALE mode: after the header, the
    counts and the lists come the fp64 K-mean partial sums (64 chunks x 128
    per (b, kv head)), the fp32 K mean [B*Hkv][128], the int8 Q codes
    [B*Hq][L][128], the int8 K codes [B*Hkv][L][128], the fp32 Q scales
    [B*Hq*nqb] and the fp32 K scales [B*Hkv][nkb]; every region starts on a
    256-byte boundary.
    """
    p = run.params
    assert p.mode == spa.SPA_MODE_SALE
    B, Hq, Hkv, L, bk = run.B, run.Hq, run.Hkv, run.L, p.block_k
    nqb, nkb = (L + 127) // 128, (L + bk - 1) // bk
    view = run.view
    a = lambda x: (x + 255) // 256 * 256
    off = a(256 + 4 * view.nb)                       # lists
    off = a(off + 4 * B * Hq * view.per_head)        # K-mean partials
    off = a(off + B * Hkv * 64 * 128 * 8)            # K mean
    kmean_at = off
    off = a(off + B * Hkv * 128 * 4)
    q8_at = off
    off = a(off + B * Hq * L * 128)
    k8_at = off
    off = a(off + B * Hkv * L * 128)
    sq_at = off
    off = a(off + view.nb * 4)
    sk_at = off
    ws = run.ws.cpu().numpy()
    take = lambda at, n, dt: ws[at:at + n * np.dtype(dt).itemsize].view(dt)
    return dict(kmean=take(kmean_at, B * Hkv * 128, np.float32).reshape(B, Hkv, 128),
                qcodes=take(q8_at, B * Hq * L * 128, np.int8).reshape(B, Hq, L, 128),
                kcodes=take(k8_at, B * Hkv * L * 128, np.int8).reshape(B, Hkv, L, 128),
                qscales=take(sq_at, view.nb, np.float32).reshape(B, Hq, nqb),
                kscales=take(sk_at, B * Hkv * nkb, np.float32).reshape(B, Hkv, nkb))
