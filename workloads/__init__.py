"""Seeded synthetic inputs for block-sparse long-context prefill.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests.  It holds only data: the workload shapes and a deterministic
generator of bf16 Q/K/V.  It contains none of the selection or attention
arithmetic.

The pages measure on RULER, LongBench, InfiniteBench and Needle-in-a-Haystack
with Llama-3.1-8B / Qwen models (AnchorAttention, Sec. 4; SALE, Sec. 4.1).
Neither the datasets nor the weights are used here; the generator reproduces
only the layer shapes (Llama-3.1-8B: 32 q heads / 8 kv heads, d = 128;
Qwen3-32B: 64 q heads / 8 kv heads) and the structure the methods rely on:
an attention sink on the first tokens and planted "needle" keys standing in for
retrieval targets.

Recipe (per batch element b and kv head g, one independent PCG64 stream seeded
from ``1000 + config id`` and spawned per (b, g)):

* u ~ uniform random unit vector in R^128 (normalised N(0, I) draw);
* for each q head of the group: q_i = z + 2u, z ~ N(0, I);
* k_j = z + 3u for j < 64 (the biased sink region), else k_j = z;
  (the two bias factors are fields of the workload; the five layer
  configurations use 2 and 3, calibration samples a stronger sink);
* v_j = z;
* needles, drawn after the base tensors, per q head h of the group:
  m ~ U[128, L), j ~ U[64, m) with j distinct within the kv head;
  k_j <- 1.5 * q_m (q_m taken from head h, in fp32 before rounding);
* "diffuse" kv heads: q, k ~ N(0, 0.5) (variance 0.5), no bias, no needles;
* every value is drawn in fp32 and rounded to bf16 with round-to-nearest-even.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

HEAD_DIM = 128
SINK_BIAS_ROWS = 64


@dataclasses.dataclass(frozen=True)
class Workload:
    """One prefill attention layer plus its selection settings."""

    name: str
    cid: int                      # config id, seeds the generator (1000 + cid)
    batch: int
    heads_q: int
    heads_kv: int
    seq_len: int
    sink: int
    local: int
    theta: float = 5.0
    tau: float = 1e-3
    block_k: int = 32             # SALE key-block size
    block_q: int = 128
    needles_per_head: int = 16
    diffuse_kv_heads: Tuple[int, ...] = ()
    head_dim: int = HEAD_DIM
    q_bias: float = 2.0           # q_i = z + q_bias * u
    sink_bias: float = 3.0        # k_j = z + sink_bias * u for j < 64

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def nqb(self) -> int:
        return (self.seq_len + self.block_q - 1) // self.block_q


# The five layer configurations (names give the shape; sizes as stated).
C0_TINY = Workload("1h-L4096", 0, 1, 1, 1, 4096, sink=64, local=128, theta=5.0,
                   needles_per_head=16)
C1_LLAMA_32K = Workload("llama3.1-8b-L32768", 1, 1, 32, 8, 32768, sink=128,
                        local=256, theta=5.0, needles_per_head=512)
C2_LLAMA_128K = Workload("llama3.1-8b-L131072", 2, 1, 32, 8, 131072, sink=128,
                         local=256, theta=5.0, tau=1e-3, block_k=32,
                         needles_per_head=512)
C3_QWEN_64K = Workload("qwen3-32b-L65536-half-diffuse", 3, 1, 64, 8, 65536,
                       sink=128, local=256, theta=5.0, needles_per_head=16,
                       diffuse_kv_heads=(4, 5, 6, 7))
C4_SWEEP_128K = C2_LLAMA_128K.with_(name="llama3.1-8b-L131072-sweep", cid=4)
C4_B4_16K = Workload("llama3.1-8b-B4-L16384", 4, 4, 32, 8, 16384, sink=128,
                     local=256, theta=5.0, needles_per_head=512)

CONFIGS: Dict[str, Workload] = {w.name: w for w in
                                (C0_TINY, C1_LLAMA_32K, C2_LLAMA_128K,
                                 C3_QWEN_64K, C4_SWEEP_128K, C4_B4_16K)}
THETA_SWEEP_128K = (3.0, 5.0, 7.0)
THETA_DENSITY_SWEEP = (math.inf, 7.0, 5.0, 4.0, 3.0, 2.5, 2.0)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round-to-nearest-even); returns uint16 bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass
class Inputs:
    """bf16 bit patterns, layout [B, H, L, d] row-major (d innermost)."""

    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    needles: List[Tuple[int, int, int, int]]   # (b, q_head, m, j)

    def as_f64(self) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
        return (bf16_bits_to_f32(self.q).astype(np.float64),
                bf16_bits_to_f32(self.k).astype(np.float64),
                bf16_bits_to_f32(self.v).astype(np.float64))


def _group_streams(w: Workload) -> List[np.random.Generator]:
    root = np.random.SeedSequence(1000 + w.cid)
    return [np.random.Generator(np.random.PCG64(s))
            for s in root.spawn(w.batch * w.heads_kv)]


def generate(w: Workload, seq_len: Optional[int] = None,
             kv_groups: Optional[Sequence[int]] = None) -> Inputs:
    """Draw the workload's Q/K/V.

    ``seq_len`` overrides the length (used for reduced-size parity cases);
    ``kv_groups`` restricts generation to a subset of kv heads (other heads are
    left zero), which keeps CPU-side checks of very long layers cheap.
    """
    L = w.seq_len if seq_len is None else int(seq_len)
    d = w.head_dim
    group = w.heads_q // w.heads_kv
    q = np.zeros((w.batch, w.heads_q, L, d), dtype=np.uint16)
    k = np.zeros((w.batch, w.heads_kv, L, d), dtype=np.uint16)
    v = np.zeros((w.batch, w.heads_kv, L, d), dtype=np.uint16)
    needles: List[Tuple[int, int, int, int]] = []
    streams = _group_streams(w)
    for b in range(w.batch):
        for g in range(w.heads_kv):
            if kv_groups is not None and g not in kv_groups:
                continue
            rng = streams[b * w.heads_kv + g]
            diffuse = g in w.diffuse_kv_heads
            u = rng.standard_normal(d, dtype=np.float32)
            u /= np.float32(np.linalg.norm(u.astype(np.float64)))
            qf = []
            for hh in range(group):
                if diffuse:
                    qh = rng.standard_normal((L, d), dtype=np.float32) * np.float32(math.sqrt(0.5))
                else:
                    qh = rng.standard_normal((L, d), dtype=np.float32) + np.float32(w.q_bias) * u
                qf.append(qh)
            if diffuse:
                kf = rng.standard_normal((L, d), dtype=np.float32) * np.float32(math.sqrt(0.5))
            else:
                kf = rng.standard_normal((L, d), dtype=np.float32)
                nb = min(SINK_BIAS_ROWS, L)
                kf[:nb] += np.float32(w.sink_bias) * u
            vf = rng.standard_normal((L, d), dtype=np.float32)
            if not diffuse and L > 128 + 1:
                used = set()
                for hh in range(group):
                    planted = 0
                    tries = 0
                    while planted < w.needles_per_head and tries < 50 * w.needles_per_head:
                        tries += 1
                        m = int(rng.integers(128, L))
                        j = int(rng.integers(SINK_BIAS_ROWS, m))
                        if j in used:
                            continue
                        used.add(j)
                        kf[j] = np.float32(1.5) * qf[hh][m]
                        needles.append((b, g * group + hh, m, j))
                        planted += 1
            for hh in range(group):
                q[b, g * group + hh] = f32_to_bf16_bits(qf[hh])
            k[b, g] = f32_to_bf16_bits(kf)
            v[b, g] = f32_to_bf16_bits(vf)
    return Inputs(q=q, k=k, v=v, needles=needles)


def random_bf16(shape, seed: int, scale: float = 1.0, mean: float = 0.0) -> np.ndarray:
    """Plain N(mean, scale^2) bf16 tensor (bit patterns) for edge-case tests."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.standard_normal(shape, dtype=np.float32) * np.float32(scale) + np.float32(mean)
    return f32_to_bf16_bits(x)


def calibration_samples(n: int, *, heads_q: int, heads_kv: int, seq_len: int, sink: int,
                        local: int, first_cid: int = 60, q_bias: float = 8.0,
                        sink_bias: float = 12.0, diffuse_kv_heads: Tuple[int, ...] = ()):
    """Stand-ins for SALE's calibration samples (five Retrieve.KV inputs in the
    paper): independent draws with a strong attention sink and planted needles,
    so that SALE at tau = 0.008 really prunes and halving tau matters."""
    out = []
    for s in range(n):
        w = Workload(f"calib-{s}", first_cid + s, 1, heads_q, heads_kv, seq_len, sink=sink,
                     local=local, needles_per_head=8, diffuse_kv_heads=diffuse_kv_heads,
                     q_bias=q_bias, sink_bias=sink_bias)
        out.append(generate(w))
    return out
