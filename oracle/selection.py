"""Key selection for one query block, in fp64 (oracle; test infrastructure only).

Notation (both selection modes):

* scores s_ij = scale * q_i . k_j, natural-log units; scale defaults to 1/sqrt(d);
* query block b covers rows [b*bq, min((b+1)*bq, L));
* sink set Sk = [0, sink);
* block-aligned local set Lo_b = [ls_b, (b+1)*bq), ls_b = max(0, (b+1)*bq - local);
* sink-local set of row i: SL(i) = (Sk u Lo_b) n {j <= i};
* candidates C_b = [sink, ls_b): every key that is neither sink nor local.

Readings taken where the pages are silent or garbled (each one is listed in
the design notes):

* the local region is block aligned (AnchorAttention Eq. (1) speaks of "the
  local key block"; SALE's "most recent up to 256 tokens, at least 128" is what
  a block-aligned 256-key window gives with bq = 128);
* the anchor is the row maximum M of the scaled logits, causally masked inside
  the local block (AnchorAttention, Algorithm 2 with M in place of Acc);
* avgpool is the arithmetic mean over the block's valid rows;
* ``<= theta`` keeps (ties keep); theta = +inf keeps every candidate and
  theta = -inf keeps none;
* SALE uses the corrected threshold ln(tau * el_i) + em_i (the printed
  ln(tau * el_i + em_i) is rejected), keeps a block when its largest relative
  score reaches tau (ties keep), and takes em/el over SL(i);
* SALE quantisation (the pages name only SageAttention2): K is smoothed by its
  per-head mean over the sequence (the mean is summed in fp64, divided by L in
  fp64 and rounded once to fp32); symmetric per-block int4 with
  scale = absmax / 7 in fp32, codes = round-half-even(x / scale) in fp32,
  clamped to [-7, 7]; an all-zero block gets scale 1.  Q blocks are bq rows,
  K blocks bk rows.  This one step runs in fp32 so the codes are bit-exact;
  everything after it is fp64.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np


@dataclasses.dataclass(frozen=True)
class BlockGeometry:
    """Row and key ranges of one query block."""

    row_lo: int      # first row of the block
    row_hi: int      # one past the last valid row (ragged last block)
    ls: int          # start of the block-aligned local window
    sink_end: int    # min(sink, ls): the sink keys not already local
    cand_lo: int     # candidates are [cand_lo, cand_hi)
    cand_hi: int


def block_geometry(qb: int, L: int, bq: int, sink: int, local: int) -> BlockGeometry:
    row_lo = qb * bq
    row_hi = min((qb + 1) * bq, L)
    ls = max(0, (qb + 1) * bq - local)
    sink_end = min(sink, ls)
    cand_lo = sink
    cand_hi = max(sink, ls)
    return BlockGeometry(row_lo, row_hi, ls, sink_end, cand_lo, cand_hi)


def default_scale(d: int, scale: float = 0.0) -> float:
    return 1.0 / math.sqrt(d) if scale == 0.0 else float(scale)


def sink_local_keys(geo: BlockGeometry, sink: int) -> np.ndarray:
    """Sorted keys of Sk u Lo_b restricted to j < row_hi (no causal cut yet)."""
    sk = np.arange(0, min(sink, geo.row_hi))
    lo = np.arange(geo.ls, geo.row_hi)
    return np.union1d(sk, lo)


# ---------------------------------------------------------------------------
# AnchorAttention: anchor + difference-aware stripe selection
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class AnchorBlock:
    kept: np.ndarray       # ascending kept candidate keys (the index set I, Eq. (3))
    cand: np.ndarray       # all candidate keys [sink, ls_b)
    margin: np.ndarray     # theta - (xbar_a - sbar_j) per candidate (>= 0 <=> kept)
    x_a: np.ndarray        # anchor per valid row (Eq. (1))
    xbar_a: float          # avgpool of the anchor over the block's rows
    qbar: np.ndarray       # avgpool(Q) over the block's rows, fp64 [d]
    sbar: np.ndarray       # pooled score per candidate


def anchor_block(qh: np.ndarray, kh: np.ndarray, qb: int, *, bq: int, sink: int,
                 local: int, theta: float, scale: float = 0.0) -> AnchorBlock:
    """Stripe selection for query block ``qb`` of one q head.

    ``qh`` [L, d] is the q head, ``kh`` [L, d] its kv head, both fp64.

    AnchorAttention Eq. (1): x_a[i] = max_{j in SL(i)} s_ij.
    AnchorAttention Eq. (2): keep j in C_b iff avgpool(x_a) - avgpool(Q) k_j^T * scale <= theta.
    AnchorAttention Eq. (3): the kept set is the list of discrete key coordinates.
    """
    L, d = qh.shape
    sc = default_scale(d, scale)
    geo = block_geometry(qb, L, bq, sink, local)
    rows = np.arange(geo.row_lo, geo.row_hi)
    slk = sink_local_keys(geo, sink)
    s = (qh[rows] @ kh[slk].T) * sc                       # [n_rows, |Sk u Lo|]
    causal = slk[None, :] <= rows[:, None]
    x_a = np.where(causal, s, -np.inf).max(axis=1)        # Eq. (1), row max M
    xbar_a = float(x_a.mean())                            # avgpool(x_a)
    qbar = qh[rows].mean(axis=0)                          # avgpool(Q)
    cand = np.arange(geo.cand_lo, geo.cand_hi)
    sbar = (kh[cand] @ qbar) * sc                         # avgpool(Q) K^T / sqrt(d)
    diff = xbar_a - sbar
    with np.errstate(invalid="ignore"):
        margin = theta - diff
    keep = diff <= theta                                  # Eq. (2), ties keep
    return AnchorBlock(kept=cand[keep], cand=cand, margin=margin, x_a=x_a,
                       xbar_a=xbar_a, qbar=qbar, sbar=sbar)


def anchor_head(qh: np.ndarray, kh: np.ndarray, blocks, *, bq: int, sink: int, local: int,
                theta: float, scale: float = 0.0):
    """``anchor_block`` for several blocks of one head, the pooled scores of all
    of them taken with a single matrix product avgpool(Q)_blocks K^T.

    Returns {qb: AnchorBlock}; equal to calling ``anchor_block`` per block.
    """
    L, d = qh.shape
    sc = default_scale(d, scale)
    blocks = list(blocks)
    out = {}
    qbars = []
    for qb in blocks:
        geo = block_geometry(qb, L, bq, sink, local)
        qbars.append(qh[geo.row_lo:geo.row_hi].mean(axis=0))
    cand_hi_max = max((block_geometry(qb, L, bq, sink, local).cand_hi for qb in blocks), default=sink)
    cand_all = np.arange(sink, max(sink, cand_hi_max))
    sbar_all = (np.stack(qbars) @ kh[cand_all].T) * sc if blocks else None
    for n, qb in enumerate(blocks):
        geo = block_geometry(qb, L, bq, sink, local)
        rows = np.arange(geo.row_lo, geo.row_hi)
        slk = sink_local_keys(geo, sink)
        s = (qh[rows] @ kh[slk].T) * sc
        causal = slk[None, :] <= rows[:, None]
        x_a = np.where(causal, s, -np.inf).max(axis=1)
        xbar_a = float(x_a.mean())
        cand = np.arange(geo.cand_lo, geo.cand_hi)
        sbar = sbar_all[n, : cand.size]
        diff = xbar_a - sbar
        with np.errstate(invalid="ignore"):
            margin = theta - diff
        keep = diff <= theta
        out[qb] = AnchorBlock(kept=cand[keep], cand=cand, margin=margin, x_a=x_a,
                              xbar_a=xbar_a, qbar=qbars[n], sbar=sbar)
    return out


# ---------------------------------------------------------------------------
# SALE: 4-bit estimate + Relative Attention Score block selection
# ---------------------------------------------------------------------------

def _quantize_rows_fp32(x32: np.ndarray, block_rows: int):
    """Symmetric per-block int4 codes of fp32 rows (fp32 arithmetic throughout)."""
    n = x32.shape[0]
    nblk = (n + block_rows - 1) // block_rows
    codes = np.zeros(x32.shape, dtype=np.int8)
    scales = np.ones(nblk, dtype=np.float32)
    seven = np.float32(7.0)
    for blk in range(nblk):
        part = x32[blk * block_rows:(blk + 1) * block_rows]
        amax = np.float32(np.abs(part).max()) if part.size else np.float32(0.0)
        if amax > 0:
            sc = np.float32(amax / seven)                 # fp32 IEEE division
            c = np.rint(part / sc)                        # fp32 division, half-to-even
            codes[blk * block_rows:(blk + 1) * block_rows] = np.clip(c, -7, 7).astype(np.int8)
            scales[blk] = sc
    return codes, scales


def sale_smooth_mean(kh32: np.ndarray) -> np.ndarray:
    """Per-head mean of K over the sequence: fp64 sum / L, rounded once to fp32."""
    L = kh32.shape[0]
    return (kh32.astype(np.float64).sum(axis=0) / float(L)).astype(np.float32)


def sale_quantize_k(kh32: np.ndarray, bk: int):
    """Smooth K by its sequence mean, then int4-quantise per bk-row block."""
    mean = sale_smooth_mean(kh32)
    ks = (kh32.astype(np.float32) - mean).astype(np.float32)   # fp32 subtraction
    codes, scales = _quantize_rows_fp32(ks, bk)
    return codes, scales, mean


def sale_quantize_q(qh32: np.ndarray, bq: int):
    """int4-quantise Q per bq-row block (no smoothing)."""
    return _quantize_rows_fp32(qh32.astype(np.float32), bq)


def sale_scores(qcodes: np.ndarray, qscale: float, kcodes: np.ndarray,
                kscales_per_key: np.ndarray, scale: float) -> np.ndarray:
    """S~ = (q^ . k^) * s_q * s_k * scale in fp64.

    The integer dot products are formed with an fp64 matmul of the codes; every
    partial sum is an integer of magnitude <= 7*7*d < 2^53, so it is exact.
    """
    dots = qcodes.astype(np.float64) @ kcodes.astype(np.float64).T
    return dots * (float(qscale) * kscales_per_key.astype(np.float64)[None, :] * scale)


def sale_threshold(em: np.ndarray, el: np.ndarray, tau: float) -> np.ndarray:
    """Corrected SALE Eq. (4): P~ >= tau  <=>  S~ >= ln(tau * el) + em."""
    return em + np.log(tau * el)


def sale_threshold_as_printed(em: np.ndarray, el: np.ndarray, tau: float) -> np.ndarray:
    """SALE Eq. (4) exactly as printed, ln(tau * el + em); kept only to show it differs."""
    with np.errstate(invalid="ignore"):
        return np.log(tau * el + em)


def relative_score(s: np.ndarray, em: np.ndarray, el: np.ndarray) -> np.ndarray:
    """SALE Relative Attention Score P~[i, j] = exp(S~[i, j] - em_i) / el_i."""
    return np.exp(s - em[:, None]) / el[:, None]


@dataclasses.dataclass
class SaleBlock:
    kept_blocks: np.ndarray   # ascending kept key-block ids (each covers bk keys)
    cand_blocks: np.ndarray   # all candidate key-block ids
    margin: np.ndarray        # max over the block of (S~ - t_i); kept <=> >= 0
    em: np.ndarray            # per valid row
    el: np.ndarray
    t: np.ndarray             # ln(tau * el) + em


@dataclasses.dataclass
class SaleHead:
    """Quantised tensors of one (q head, kv head) pair."""

    qcodes: np.ndarray
    qscales: np.ndarray
    kcodes: np.ndarray
    kscales: np.ndarray
    kmean: np.ndarray


def sale_prepare(qh32: np.ndarray, kh32: np.ndarray, *, bq: int, bk: int) -> SaleHead:
    qc, qs = sale_quantize_q(qh32, bq)
    kc, ks, km = sale_quantize_k(kh32, bk)
    return SaleHead(qc, qs, kc, ks, km)


def sale_block(prep: SaleHead, qb: int, *, L: int, bq: int, bk: int, sink: int,
               local: int, tau: float, scale: float = 0.0,
               d: int = 128) -> SaleBlock:
    """SALE block selection for query block ``qb`` of one q head.

    SALE Sec. 3.3: em_i, el_i are the max and the sum of exp(S~ - em_i) over
    the sink-local area SL(i).  Eq. (4) (corrected): keep (qb, kb) iff some
    valid row i and candidate key j in kb have S~_ij >= ln(tau * el_i) + em_i.
    """
    sc = default_scale(d, scale)
    geo = block_geometry(qb, L, bq, sink, local)
    rows = np.arange(geo.row_lo, geo.row_hi)
    kscale_key = np.repeat(prep.kscales, bk)[:L]
    qcode = prep.qcodes[rows]
    qscale = prep.qscales[qb]
    slk = sink_local_keys(geo, sink)
    s_sl = sale_scores(qcode, qscale, prep.kcodes[slk], kscale_key[slk], sc)
    causal = slk[None, :] <= rows[:, None]
    s_sl = np.where(causal, s_sl, -np.inf)
    em = s_sl.max(axis=1)
    el = np.exp(s_sl - em[:, None]).sum(axis=1)
    t = sale_threshold(em, el, tau)
    kb_lo = geo.cand_lo // bk
    kb_hi = geo.cand_hi // bk
    cand_blocks = np.arange(kb_lo, kb_hi)
    margin = np.full(cand_blocks.shape, -np.inf)
    if cand_blocks.size:
        keys = np.arange(kb_lo * bk, kb_hi * bk)
        s_c = sale_scores(qcode, qscale, prep.kcodes[keys], kscale_key[keys], sc)
        excess = (s_c - t[:, None]).max(axis=0)             # max over rows
        margin = excess.reshape(-1, bk).max(axis=1)         # max over the block
    kept = cand_blocks[margin >= 0.0]
    return SaleBlock(kept_blocks=kept, cand_blocks=cand_blocks, margin=margin,
                     em=em, el=el, t=t)


def sale_blocks_to_keys(kept_blocks: np.ndarray, bk: int) -> np.ndarray:
    if kept_blocks.size == 0:
        return np.zeros(0, dtype=np.int64)
    return (kept_blocks[:, None] * bk + np.arange(bk)[None, :]).reshape(-1)


# ---------------------------------------------------------------------------
# Query-block grouping (AnchorAttention's ``step``)
# ---------------------------------------------------------------------------

def step_union(selected_of_block, qb: int, *, step: int, nqb: int, cand_lo: int,
               cand_hi: int) -> np.ndarray:
    """Selection of block ``qb`` when query blocks are grouped ``step`` at a time.

    AnchorAttention (Sec. 3.4; Appendix C, Algorithm 2 with the ``step``
    parameter): the identification runs for groups of ``step`` consecutive
    query blocks and a key selected by any block of the group is active for
    every block of the group.  Reading taken here: the group of block b is
    [floor(b / step) * step, ... + step) (clipped to the layer), the union is
    taken over the blocks' own selections, and it is restricted to block b's
    own candidate range [cand_lo, cand_hi) so that no key outside b's causal
    candidates (or inside its always-kept sink/local windows) is added.
    ``selected_of_block(b)`` returns block b's own selection (keys, or key-block
    ids with a range given in the same units).
    """
    g0 = (qb // step) * step
    parts = [np.asarray(selected_of_block(b), dtype=np.int64)
             for b in range(g0, min(g0 + step, nqb))]
    keys = np.unique(np.concatenate(parts)) if parts else np.zeros(0, dtype=np.int64)
    return keys[(keys >= cand_lo) & (keys < cand_hi)]
