"""FP8 (E4M3) quantised attention, in fp64 (oracle; test infrastructure only).

SALE runs its Computation Pass on quantised operands "SageAttention-style"
(the review of SALE, Summary).  Reading for a B200 tensor-core version
(tcgen05 kind::f8f6f4, E4M3 operands, fp32 accumulation):

* E4M3 (OCP FP8, "fn" variant): 1 sign, 4 exponent bits with bias 7, 3
  mantissa bits, subnormals, no infinities; largest finite value 448.
  Rounding is to nearest, ties to even, saturating to +-448 ("satfinite").
* Q: one scale per (b, h, 128-row block), s_q = absmax / 448 in fp32.
* K: smoothed by its per-(b, kv head) sequence mean (as the int4 estimate;
  the shift adds a constant to every score of a row, which cancels in the
  softmax), then one scale per (b, kv head): s_k = absmax / 448.
* V: one scale per (b, kv head, channel c): s_v[c] = absmax_j |V[j, c]| / 448.
* code = E4M3(x / s) with the division in IEEE fp32; an all-zero block or
  channel gets s = 1.
* Attention is the kept-set softmax of the dequantised operands in fp64.  A
  kernel also rounds the probabilities to E4M3 before the PV product; that
  rounding (relative error <= 2^-4 per probability) is left to the
  comparison's error bound, not modelled here.
"""

from __future__ import annotations

from typing import Tuple

import numpy as np

E4M3_MAX = 448.0
E4M3_MIN_NORMAL = 2.0 ** -6
E4M3_SUBNORMAL_STEP = 2.0 ** -9


def e4m3_round(x) -> np.ndarray:
    """Round to the nearest E4M3 value (ties to even), saturating at +-448.

    Works on the exact value of ``x`` (fp32 or fp64 input); returns fp64.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    out = np.zeros_like(a)
    sub = a < E4M3_MIN_NORMAL
    out[sub] = np.rint(a[sub] / E4M3_SUBNORMAL_STEP) * E4M3_SUBNORMAL_STEP
    nrm = ~sub
    if nrm.any():
        e = np.floor(np.log2(a[nrm]))
        step = np.exp2(e - 3.0)                      # 3 mantissa bits
        q = np.rint(a[nrm] / step) * step            # may carry into the next binade
        out[nrm] = q
    out = np.minimum(out, E4M3_MAX)
    return np.copysign(out, x)


def e4m3_decode(code: int) -> float:
    """The value of an 8-bit E4M3 code, from its sign / exponent / mantissa fields."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * m * 2.0 ** -9                     # subnormal: m/8 * 2^(1-7)
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def scale_of(absmax: np.float32) -> np.float32:
    """s = absmax / 448 in fp32 (1 for an all-zero block)."""
    absmax = np.float32(absmax)
    return np.float32(1.0) if absmax == 0 else np.float32(absmax / np.float32(E4M3_MAX))


def quantize(x32: np.ndarray, scale: np.float32) -> np.ndarray:
    """E4M3 values of x / scale (fp32 division), as fp64."""
    return e4m3_round(np.asarray(x32, dtype=np.float32) / np.float32(scale))


def quantize_q(qh32: np.ndarray, bq: int = 128) -> Tuple[np.ndarray, np.ndarray]:
    """Q of one head: codes (as values) per 128-row block and the block scales."""
    L = qh32.shape[0]
    codes = np.zeros(qh32.shape)
    scales = np.zeros((L + bq - 1) // bq, dtype=np.float32)
    for b in range(len(scales)):
        blk = qh32[b * bq:(b + 1) * bq]
        scales[b] = scale_of(np.max(np.abs(blk)))
        codes[b * bq:(b + 1) * bq] = quantize(blk, scales[b])
    return codes, scales


def smooth_k(kh32: np.ndarray) -> np.ndarray:
    """K minus its sequence mean (fp64 sum / L rounded once to fp32), in fp32."""
    mean = np.float32(kh32.astype(np.float64).sum(axis=0) / kh32.shape[0])
    return (kh32 - mean).astype(np.float32)


def quantize_k(kh32: np.ndarray) -> Tuple[np.ndarray, np.float32]:
    ks = smooth_k(kh32)
    s = scale_of(np.max(np.abs(ks)))
    return quantize(ks, s), s


def quantize_v(vh32: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    scales = np.array([scale_of(np.max(np.abs(vh32[:, c]))) for c in range(vh32.shape[1])],
                      dtype=np.float32)
    codes = np.stack([quantize(vh32[:, c], scales[c]) for c in range(vh32.shape[1])], axis=1)
    return codes, scales


def dequantized_head(qh32, kh32, vh32, bq: int = 128):
    """(Q^, K^, V^) in fp64: the operands the FP8 attention multiplies."""
    qc, qs = quantize_q(qh32, bq)
    q_hat = qc * np.repeat(qs.astype(np.float64), bq)[: qh32.shape[0], None]
    kc, ks = quantize_k(kh32)
    vc, vs = quantize_v(vh32)
    return q_hat, kc * np.float64(ks), vc * vs.astype(np.float64)[None, :]
