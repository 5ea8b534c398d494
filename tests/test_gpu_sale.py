"""GPU parity: SALE-mode block selection and attention vs the fp64 oracle."""

import numpy as np
import pytest

from workloads import C0_TINY, C2_LLAMA_128K, generate
from workloads import bf16_bits_to_f32

from gpu_common import (Run, compare_outputs, compare_sale_masks, edge_blocks, sample_rows)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("L,tau,bk,sink", [(2048, 1e-3, 32, 64), (2048, 0.05, 32, 64),
                                           (1900, 0.02, 16, 32), (3000, 0.01, 64, 128),
                                           (2500, 0.03, 128, 128)])
def test_sale_small_all_blocks(L, tau, bk, sink):
    w = C0_TINY.with_(sink=sink, local=256)
    inp = generate(w, seq_len=L)
    run = Run(inp, mode="sale", sink=sink, local=256, tau=tau, block_k=bk)
    compare_sale_masks(run, inp, [(0, 0)])
    compare_outputs(run, inp, {(0, 0): range(L)})


@pytest.mark.parametrize("B,hq,hkv,L,bk", [(1, 1, 1, 2048, 32), (1, 4, 2, 1900, 16),
                                            (2, 2, 1, 1000, 64)])
def test_sale_quantisation_codes_bit_exact(B, hq, hkv, L, bk):
    """The int4 codes, their fp32 scales and the fp32 K mean that the plan
    leaves in the workspace equal the oracle's, bit for bit (the quantisation
    step is fp32 on both sides; the K sum is exact in fp64 for bf16 keys)."""
    from oracle import selection as osel
    from gpu_common import sale_scratch
    w = C0_TINY.with_(batch=B, heads_q=hq, heads_kv=hkv, sink=64, local=256)
    inp = generate(w, seq_len=L)
    run = Run(inp, mode="sale", sink=64, local=256, tau=1e-3, block_k=bk, do_attn=False)
    got = sale_scratch(run)
    for b in range(B):
        for h in range(hq):
            g = h // (hq // hkv)
            prep = osel.sale_prepare(bf16_bits_to_f32(inp.q[b, h]), bf16_bits_to_f32(inp.k[b, g]),
                                     bq=128, bk=bk)
            np.testing.assert_array_equal(got["qcodes"][b, h], prep.qcodes)
            np.testing.assert_array_equal(got["qscales"][b, h], prep.qscales)
            np.testing.assert_array_equal(got["kcodes"][b, g], prep.kcodes)
            np.testing.assert_array_equal(got["kscales"][b, g], prep.kscales)
            np.testing.assert_array_equal(got["kmean"][b, g], prep.kmean)
    # the selection built on them, bit-exact away from near-ties
    compare_sale_masks(run, inp, [(b, h) for b in range(B) for h in range(hq)])


def test_sale_c2_shape_16k_two_heads_all_blocks():
    w = C2_LLAMA_128K
    L = 16384
    inp = generate(w, seq_len=L)
    run = Run(inp, mode="sale", sink=w.sink, local=w.local, tau=w.tau, block_k=w.block_k)
    compare_sale_masks(run, inp, [(0, 0), (0, 21)])
    rows = {(0, h): sample_rows(L, 24, h, must=(L - 1,)) for h in (0, 21)}
    compare_outputs(run, inp, rows)


def test_sale_c2_full_size_sampled():
    w = C2_LLAMA_128K
    inp = generate(w)
    run = Run(inp, mode="sale", sink=w.sink, local=w.local, tau=w.tau, block_k=w.block_k)
    heads = [(0, 0), (0, 31)]
    compare_sale_masks(run, inp, heads, blocks_of=lambda b, h: edge_blocks(w.seq_len, 2, h))
    rows = {hd: sample_rows(w.seq_len, 12, hd[1], must=(w.seq_len - 1,)) for hd in heads}
    compare_outputs(run, inp, rows)


@pytest.mark.parametrize("hq,tau", [(1, 0.008), (2, 0.008), (2, 0.002), (4, 0.008)])
def test_sale_strong_sink_local128(hq, tau):
    """Calibration-style inputs (strong attention sink, planted needles, local
    window of one block): SALE really prunes here and the heads of a group keep
    different blocks, so the paired kernel's per-head membership tags matter."""
    from workloads import calibration_samples
    L, sink, local = 1024, 64, 128
    inp = calibration_samples(1, heads_q=hq, heads_kv=1, seq_len=L, sink=sink, local=local)[0]
    run = Run(inp, mode="sale", sink=sink, local=local, tau=tau, block_k=32)
    heads = [(0, h) for h in range(hq)]
    res = compare_sale_masks(run, inp, heads)
    nqb = L // 128
    full = sum(max(0, (qb * 128 + 128 - local - sink)) // 32 for qb in range(nqb)) * hq
    assert res["kept"] < full, "the case must prune"
    # attention here sits on a few sink keys, so bf16 rounding of the
    # probabilities is not averaged away: the kernel's own error bound applies
    compare_outputs(run, inp, {hd: range(L) for hd in heads}, bound="bf16")
    dense = Run(inp, mode="dense", sink=sink, local=local)
    compare_outputs(dense, inp, {hd: range(L) for hd in heads}, dense=True, bound="bf16")


def test_sale_c2_full_size_pruning_tau():
    """SALE on the 128K layer at a threshold that skips key blocks (tau =
    0.1 keeps about 45 % of the candidate blocks on these inputs): sampled
    blocks bit-exact up to near-ties, sampled rows within the stated bound."""
    w = C2_LLAMA_128K
    inp = generate(w, kv_groups=[0, 7])
    run = Run(inp, mode="sale", sink=w.sink, local=w.local, tau=0.1, block_k=w.block_k)
    assert run.stats.kept_candidates < 0.8 * run.stats.candidates, "the case must prune"
    heads = [(0, 0), (0, 3), (0, 30)]
    compare_sale_masks(run, inp, heads, blocks_of=lambda b, h: edge_blocks(w.seq_len, 3, h))
    rows = {hd: sample_rows(w.seq_len, 10, hd[1], must=(w.seq_len - 1,)) for hd in heads}
    compare_outputs(run, inp, rows)
