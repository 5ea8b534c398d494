"""GPU parity of the FP8 (E4M3) attention path (SALE review, Summary: the
Computation Pass on quantised operands, SageAttention-style).

* Quantisation, bit-exact: the E4M3 codes of Q (per 128-row block), K (mean
  smoothed, per kv head) and V (per channel), their fp32 scales and the fp32 K
  mean equal ``oracle.fp8`` on the same bf16 inputs.
* Attention: against the oracle's fp64 attention of the dequantised operands
  (Q^, K^ + mean, V^) over the GPU's own kept set, element by element within
  the bound of the kernel's arithmetic: the probabilities enter the PV product
  rounded to E4M3 (relative error <= 2^-4 each) and O is rounded to bf16, so
  |dO| <= 2^-4 (sum_j p_j |v^_j|) / l + 2^-8 |O| + 1e-4; LSE within 2e-3.
"""

import numpy as np
import pytest
import torch

import block_sparse_long_sm_b200 as spa
from oracle import attention as oatt
from oracle import fp8 as ofp8
from workloads import C0_TINY, bf16_bits_to_f32, generate

from gpu_common import LSE_ABS, Run

pytestmark = pytest.mark.gpu

E4M3_VALUES = np.array([ofp8.e4m3_decode(c) for c in range(256)])


class Fp8Run:
    def __init__(self, run: Run):
        p = run.params
        B, Hq, Hkv, L = run.B, run.Hq, run.Hkv, run.L
        self.run = run
        self.q8 = torch.empty((B, Hq, L, 128), dtype=torch.uint8, device="cuda")
        self.k8 = torch.empty((B, Hkv, L, 128), dtype=torch.uint8, device="cuda")
        self.v8 = torch.empty((B, Hkv, L, 128), dtype=torch.uint8, device="cuda")
        self.scales = torch.empty(spa.sparse_fp8_scales_floats(p), dtype=torch.float32,
                                  device="cuda")
        scratch = torch.empty(spa.sparse_fp8_scratch_bytes(p), dtype=torch.uint8, device="cuda")
        spa.check(spa.sparse_fp8_quantize(p, run.q, run.k, run.v, self.q8, self.k8, self.v8,
                                          self.scales, scratch), "fp8 quantize")
        self.o = torch.empty((B, Hq, L, 128), dtype=torch.bfloat16, device="cuda")
        self.lse = torch.empty((B, Hq, L), dtype=torch.float32, device="cuda")
        spa.check(spa.sparse_prefill_attn_fp8(p, self.q8, self.k8, self.v8, self.scales, run.ws,
                                              self.o, self.lse), "fp8 attn")
        st, _ = spa.sparse_prefill_stats(p, run.ws)
        spa.check(st, "stats")
        torch.cuda.synchronize()
        nqb = (L + 127) // 128
        sc = self.scales.cpu().numpy()
        n_qs = B * Hq * nqb
        self.qs = sc[:n_qs].reshape(B, Hq, nqb)
        self.ks = sc[n_qs:n_qs + B * Hkv].reshape(B, Hkv)
        self.vs = sc[n_qs + B * Hkv:n_qs + B * Hkv * 129].reshape(B, Hkv, 128)
        self.kmean = sc[n_qs + B * Hkv * 129:].reshape(B, Hkv, 128)


def _check_quantisation(fr: Fp8Run, inp, b, h):
    g = h // fr.run.group
    q32 = bf16_bits_to_f32(inp.q[b, h])
    k32 = bf16_bits_to_f32(inp.k[b, g])
    v32 = bf16_bits_to_f32(inp.v[b, g])
    qc, qs = ofp8.quantize_q(q32)
    assert np.array_equal(fr.qs[b, h], qs)
    assert np.array_equal(E4M3_VALUES[fr.q8[b, h].cpu().numpy()], qc)
    mean = np.float32(k32.astype(np.float64).sum(axis=0) / k32.shape[0])
    assert np.array_equal(fr.kmean[b, g], mean)
    kc, ks = ofp8.quantize_k(k32)
    assert fr.ks[b, g] == ks
    assert np.array_equal(E4M3_VALUES[fr.k8[b, g].cpu().numpy()], kc)
    vc, vs = ofp8.quantize_v(v32)
    assert np.array_equal(fr.vs[b, g], vs)
    assert np.array_equal(E4M3_VALUES[fr.v8[b, g].cpu().numpy()], vc)


def _check_outputs(fr: Fp8Run, inp, b, h, rows):
    run, p = fr.run, fr.run.params
    g = h // run.group
    q32 = bf16_bits_to_f32(inp.q[b, h])
    k32 = bf16_bits_to_f32(inp.k[b, g])
    v32 = bf16_bits_to_f32(inp.v[b, g])
    q_hat, k_hat, v_hat = ofp8.dequantized_head(q32, k32, v32)
    k_full = k_hat + np.float32(k32.astype(np.float64).sum(axis=0) / k32.shape[0])[None, :]
    scale = 128 ** -0.5
    o_gpu = fr.o[b, h].float().cpu().numpy()
    lse_gpu = fr.lse[b, h].cpu().numpy()
    worst, lse_err = 0.0, 0.0
    for i in rows:
        qb = i // 128
        if p.mode == spa.SPA_MODE_DENSE:
            keys = np.arange(i + 1)
        else:
            keys = oatt.kept_keys_for_row(i, qb, run.L, bq=128, sink=p.sink, local=p.local,
                                          selected=run.selected_keys(b, h, qb))
        o_ref, lse_ref = oatt.attend_row(q_hat[i], k_full, v_hat, keys, scale)
        s = (k_full[keys] @ q_hat[i]) * scale
        w = np.exp(s - s.max())
        w /= w.sum()
        lim = 2.0 ** -4 * (w @ np.abs(v_hat[keys])) + 2.0 ** -8 * np.abs(o_ref) + 1e-4
        worst = max(worst, float(np.max(np.abs(o_gpu[i] - o_ref) / lim)))
        lse_err = max(lse_err, abs(float(lse_gpu[i]) - lse_ref))
    assert worst <= 1.0, ("FP8 output outside the E4M3 bound", worst)
    assert lse_err <= LSE_ABS, lse_err


# Hq / Hkv = 2: the paired schedule (two q heads per CTA over the union
# lists); 3: the one-head schedule (also every DENSE call).
@pytest.mark.parametrize("mode,L,theta,bk,hq", [
    ("anchor", 1000, 2.5, None, 4), ("anchor", 129, 3.0, None, 4), ("sale", 1500, 0.0, 32, 4),
    ("dense", 700, 0.0, None, 4), ("anchor", 1000, 2.5, None, 6), ("sale", 900, 0.0, 64, 6)])
def test_fp8_quantisation_and_attention(mode, L, theta, bk, hq):
    w = C0_TINY.with_(heads_q=hq, heads_kv=2, sink=64, local=256)
    inp = generate(w, seq_len=L)
    run = Run(inp, mode=mode, sink=64, local=256, theta=theta, tau=1e-2, block_k=bk,
              do_attn=False)
    fr = Fp8Run(run)
    for h in range(hq):
        _check_quantisation(fr, inp, 0, h)
    rows = sorted(set(range(0, L, max(1, L // 40))) | {L - 1, min(L - 1, 127), min(L - 1, 128)})
    for h in (0, 1, hq - 1):
        _check_outputs(fr, inp, 0, h, rows)


def test_fp8_llama_32k_sampled():
    from workloads import C1_LLAMA_32K
    from gpu_common import sample_rows
    w = C1_LLAMA_32K
    inp = generate(w)
    run = Run(inp, mode="anchor", sink=w.sink, local=w.local, theta=w.theta, do_attn=False)
    fr = Fp8Run(run)
    for h in (0, 13, 31):
        _check_quantisation(fr, inp, 0, h)
        _check_outputs(fr, inp, 0, h, sample_rows(w.seq_len, 16, h, must=(0, 128, w.seq_len - 1)))


def test_fp8_batch_of_two():
    w = C0_TINY.with_(batch=2, heads_q=4, heads_kv=2, sink=64, local=256)
    L = 900
    inp = generate(w, seq_len=L)
    run = Run(inp, mode="anchor", sink=64, local=256, theta=2.5, do_attn=False)
    fr = Fp8Run(run)
    for b in range(2):
        _check_quantisation(fr, inp, b, 3)
        _check_outputs(fr, inp, b, 3, list(range(0, L, 17)) + [L - 1])


def test_fp8_diffuse_heads():
    # attention spread thinly over many keys (no sink bias): the regime where
    # the E4M3 rounding of many small probabilities matters most
    w = C0_TINY.with_(heads_q=4, heads_kv=2, sink=64, local=256, diffuse_kv_heads=(0, 1))
    L = 1200
    inp = generate(w, seq_len=L)
    run = Run(inp, mode="anchor", sink=64, local=256, theta=1.0, do_attn=False)
    fr = Fp8Run(run)
    for h in (0, 2):
        _check_quantisation(fr, inp, 0, h)
        _check_outputs(fr, inp, 0, h, list(range(0, L, 11)) + [L - 1])
