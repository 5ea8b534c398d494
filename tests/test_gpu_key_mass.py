"""GPU parity of the key mass from the prefill LSE (KVpop, Sec. 3: transposed
attention with the sparse LSE normalisers, aggregated over the query heads
of a kv head), through the C ABI.

mass[b, g, j] = sum over q heads h of kv head g and rows i whose kept set
holds j with i - j >= window of exp(s_ij - LSE_i).  The oracle
(``oracle.decode.key_mass``) sums the same terms in fp64 over the GPU's own
kept sets.  With the oracle's LSE as input, every term reaches the column
sums as a bf16 probability (relative error <= 2^-8) and the sums are
accumulated in fp32, so |d mass_j| <= (2^-8 + 2^-12) mass_j + 1e-6; with the
attention kernel's own LSE (within 2e-3) the relative part grows by
exp(2e-3) - 1.
"""

import math

import numpy as np
import pytest
import torch

import block_sparse_long_sm_b200 as spa
from oracle import attention as oatt
from oracle import decode as odec
from workloads import C0_TINY, generate

from gpu_common import Run, head_f64

pytestmark = pytest.mark.gpu

REL = 2.0 ** -8 + 2.0 ** -12


def _oracle(run: Run, inp, window: int):
    p = run.params
    L, G = run.L, run.group
    scale = 1.0 / math.sqrt(128)
    mass = np.zeros((run.B, run.Hkv, L))
    lse = np.zeros((run.B, run.Hq, L))
    for b in range(run.B):
        for h in range(run.Hq):
            g = h // G
            qh, kh, vh = head_f64(inp.q, b, h), head_f64(inp.k, b, g), head_f64(inp.v, b, g)
            if p.mode == spa.SPA_MODE_DENSE:
                keys_of = lambda i: np.arange(i + 1)
            else:
                keys_of = odec.prefill_keys_of_row(L, lambda qb: run.selected_keys(b, h, qb),
                                                   bq=128, sink=p.sink, local=p.local)
            lse[b, h] = [oatt.attend_row(qh[i], kh, vh, keys_of(i), scale)[1] for i in range(L)]
            within = lambda i: keys_of(i)[i - keys_of(i) >= window]
            mass[b, g] += odec.key_mass(qh, kh, lse[b, h], range(L), within)
    return mass, lse


def _gpu_mass(run: Run, lse: torch.Tensor, window: int) -> np.ndarray:
    mass = torch.empty((run.B, run.Hkv, run.L), dtype=torch.float32, device="cuda")
    spa.check(spa.sparse_key_mass(run.params, run.q, run.k, lse, window, run.ws, mass),
              "key mass")
    st, _ = spa.sparse_prefill_stats(run.params, run.ws)
    spa.check(st, "stats")
    return mass.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("mode,L,theta,bk,window", [
    ("anchor", 1000, 2.5, None, 0), ("anchor", 1000, 2.5, None, 128), ("anchor", 129, 3.0, None, 0),
    ("sale", 900, 0.0, 32, 0), ("dense", 500, 0.0, None, 40)])
def test_key_mass_with_oracle_lse(mode, L, theta, bk, window):
    w = C0_TINY.with_(heads_q=4, heads_kv=2, sink=64, local=256)
    inp = generate(w, seq_len=L)
    run = Run(inp, mode=mode, sink=64, local=256, theta=theta, tau=1e-2, block_k=bk)
    ref, lse = _oracle(run, inp, window)
    got = _gpu_mass(run, torch.from_numpy(lse.astype(np.float32)).cuda(), window)
    assert np.all(np.abs(got - ref) <= REL * ref + 1e-6), float(np.max(np.abs(got - ref) - REL * ref))
    # every row's probabilities sum to one, so with window 0 the masses sum to Hq * L
    if window == 0:
        assert abs(got.sum() - run.Hq * L) <= 1e-3 * run.Hq * L


def test_key_mass_with_the_attention_lse():
    L = 1000
    w = C0_TINY.with_(heads_q=4, heads_kv=2, sink=64, local=256)
    inp = generate(w, seq_len=L)
    run = Run(inp, mode="anchor", sink=64, local=256, theta=2.5)
    ref, _ = _oracle(run, inp, 0)
    got = _gpu_mass(run, run.lse, 0)
    rel = REL + math.expm1(2e-3)
    assert np.all(np.abs(got - ref) <= rel * ref + 1e-6)


def test_key_mass_llama_32k_conserves_the_rows():
    # every row's probabilities over its kept set sum to one, so the masses of
    # a kv head sum to (its q heads) x L, up to the bf16 probabilities and the
    # attention's LSE (both within the relative bound used above)
    from workloads import C1_LLAMA_32K
    w = C1_LLAMA_32K
    inp = generate(w)
    run = Run(inp, mode="anchor", sink=w.sink, local=w.local, theta=w.theta)
    got = _gpu_mass(run, run.lse, 0)
    per_kv = got.sum(axis=2)[0]
    want = run.group * w.seq_len
    assert np.all(np.abs(per_kv - want) <= (REL + math.expm1(2e-3)) * want), per_kv
    assert np.all(got >= 0)


def test_key_mass_batch_of_two():
    w = C0_TINY.with_(batch=2, heads_q=4, heads_kv=2, sink=64, local=256)
    inp = generate(w, seq_len=700)
    run = Run(inp, mode="anchor", sink=64, local=256, theta=2.5)
    ref, lse = _oracle(run, inp, 0)
    got = _gpu_mass(run, torch.from_numpy(lse.astype(np.float32)).cuda(), 0)
    assert np.all(np.abs(got - ref) <= REL * ref + 1e-6)
