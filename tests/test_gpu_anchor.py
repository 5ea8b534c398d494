"""GPU parity: anchor-mode selection and sparse attention vs the fp64 oracle.

Cases span several 128-row tiles and ragged tails (small L, all blocks and all
rows), the five layer shapes at full size (sampled blocks and rows, in the
launch configuration the benchmark times), the density extremes theta = +inf /
-inf, and the degenerate lengths L = 1, 127, 129.
"""

import math

import numpy as np
import pytest

import block_sparse_long_sm_b200 as spa
from workloads import (C0_TINY, C1_LLAMA_32K, C2_LLAMA_128K, C3_QWEN_64K, C4_B4_16K, generate)

from gpu_common import (Run, compare_anchor_masks, compare_outputs, edge_blocks, sample_rows)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("theta", [5.0, 3.0, 2.5, 2.0])
def test_c0_all_blocks_all_rows(theta):
    w = C0_TINY
    inp = generate(w)
    run = Run(inp, mode="anchor", sink=w.sink, local=w.local, theta=theta)
    compare_anchor_masks(run, inp, [(0, 0)])
    compare_outputs(run, inp, {(0, 0): range(w.seq_len)})


@pytest.mark.parametrize("L,sink,local,theta", [
    (1, 64, 128, 3.0), (127, 64, 128, 3.0), (129, 64, 128, 3.0), (1000, 64, 128, 2.5),
    (1500, 0, 128, 2.5), (1777, 200, 256, 2.5), (2300, 64, 384, 3.0), (3001, 128, 256, -math.inf),
    (2500, 100, 128, math.inf)])
def test_ragged_and_geometry(L, sink, local, theta):
    w = C0_TINY.with_(sink=sink, local=local)
    inp = generate(w, seq_len=L)
    run = Run(inp, mode="anchor", sink=sink, local=local, theta=theta)
    compare_anchor_masks(run, inp, [(0, 0)])
    compare_outputs(run, inp, {(0, 0): range(L)})


def test_c1_llama_32k_all_blocks():
    w = C1_LLAMA_32K
    inp = generate(w)
    run = Run(inp, mode="anchor", sink=w.sink, local=w.local, theta=w.theta)
    compare_anchor_masks(run, inp, [(0, h) for h in range(w.heads_q)])
    rows = {(0, h): sample_rows(w.seq_len, 24, h, must=(0, 127, 128, w.seq_len - 1))
            for h in (0, 5, 17, 31)}
    compare_outputs(run, inp, rows)


def test_c1_llama_32k_sparse_theta():
    w = C1_LLAMA_32K
    inp = generate(w)
    run = Run(inp, mode="anchor", sink=w.sink, local=w.local, theta=2.5)
    compare_anchor_masks(run, inp, [(0, h) for h in (0, 3, 9, 30)])
    rows = {(0, h): sample_rows(w.seq_len, 24, 100 + h, must=(w.seq_len - 1,)) for h in (3, 30)}
    compare_outputs(run, inp, rows)


@pytest.mark.parametrize("theta", [5.0, 3.0, 7.0])
def test_c2_llama_128k_sampled(theta):
    w = C2_LLAMA_128K
    inp = generate(w)
    run = Run(inp, mode="anchor", sink=w.sink, local=w.local, theta=theta)
    heads = [(0, 0), (0, 13), (0, 31)]
    compare_anchor_masks(run, inp, heads, blocks_of=lambda b, h: edge_blocks(w.seq_len, 5, h))
    rows = {hd: sample_rows(w.seq_len, 16, hd[1], must=(w.seq_len - 1, 65536)) for hd in heads}
    compare_outputs(run, inp, rows)


def test_c3_qwen_64k_half_diffuse_sampled():
    w = C3_QWEN_64K
    inp = generate(w)
    run = Run(inp, mode="anchor", sink=w.sink, local=w.local, theta=w.theta)
    heads = [(0, 0), (0, 31), (0, 32), (0, 63)]            # biased and diffuse kv groups
    compare_anchor_masks(run, inp, heads, blocks_of=lambda b, h: edge_blocks(w.seq_len, 5, h))
    rows = {hd: sample_rows(w.seq_len, 12, hd[1], must=(w.seq_len - 1,)) for hd in heads}
    compare_outputs(run, inp, rows)


def test_c4_batch4_16k():
    w = C4_B4_16K
    inp = generate(w)
    run = Run(inp, mode="anchor", sink=w.sink, local=w.local, theta=3.0)
    heads = [(0, 0), (1, 9), (2, 20), (3, 31)]
    compare_anchor_masks(run, inp, heads)
    rows = {hd: sample_rows(w.seq_len, 16, 7 * hd[0] + hd[1], must=(w.seq_len - 1,)) for hd in heads}
    compare_outputs(run, inp, rows)


def test_theta_inf_equals_dense_and_dense_mode():
    w = C1_LLAMA_32K
    L = 8192
    inp = generate(w, seq_len=L)
    run_inf = Run(inp, mode="anchor", sink=w.sink, local=w.local, theta=math.inf)
    run_dense = Run(inp, mode="dense", sink=w.sink, local=w.local,
                    dev=(run_inf.q, run_inf.k, run_inf.v))
    rows = {(0, h): sample_rows(L, 24, h, must=(0, 1, L - 1)) for h in (0, 7, 31)}
    compare_outputs(run_inf, inp, rows, dense=True)
    compare_outputs(run_dense, inp, rows, dense=True)
    assert run_inf.stats.kept_pairs == run_inf.stats.dense_pairs
    assert run_dense.stats.kept_pairs == run_dense.stats.dense_pairs


def test_stats_match_oracle_counts():
    from oracle import attention as oatt
    w = C0_TINY.with_(sink=64, local=256)
    L = 3000
    inp = generate(w, seq_len=L)
    run = Run(inp, mode="anchor", sink=w.sink, local=w.local, theta=2.5)
    nqb = (L + 127) // 128
    expect = sum(oatt.kept_pairs_block(qb, L, bq=128, sink=w.sink, local=w.local,
                                       n_selected=int(run.counts[qb])) for qb in range(nqb))
    assert run.stats.kept_pairs == expect
    assert run.stats.kept_candidates == int(run.counts.sum())
    assert run.stats.dense_pairs == L * (L + 1) // 2
    assert run.stats.query_blocks == nqb


@pytest.mark.parametrize("hq,hkv,mode", [(3, 1, "anchor"), (6, 2, "anchor"), (4, 2, "anchor"),
                                         (2, 1, "anchor"), (2, 2, "anchor"), (4, 1, "dense"),
                                         (3, 1, "dense"), (4, 2, "sale"), (3, 3, "sale")])
def test_gqa_group_sizes_single_and_paired_kernels(hq, hkv, mode):
    """Odd Hq/Hkv runs the one-head-per-CTA kernel, even Hq/Hkv the paired kernel
    (two q heads share every K/V tile; it merges the two heads' lists)."""
    from workloads import Workload
    L = 2100
    w = Workload(f"gqa-{hq}-{hkv}", 9, 1, hq, hkv, L, sink=64, local=256, theta=2.5,
                 needles_per_head=12)
    inp = generate(w)
    heads = [(0, h) for h in range(hq)]
    if mode == "sale":
        from gpu_common import compare_sale_masks
        run = Run(inp, mode="sale", sink=64, local=256, tau=0.02, block_k=32)
        compare_sale_masks(run, inp, heads)
    elif mode == "anchor":
        run = Run(inp, mode="anchor", sink=64, local=256, theta=2.5)
        compare_anchor_masks(run, inp, heads)
    else:
        run = Run(inp, mode="dense", sink=64, local=256)
    rows = {hd: sample_rows(L, 40, 3 * hd[1] + hq, must=(0, 127, 128, L - 1)) for hd in heads}
    compare_outputs(run, inp, rows, dense=(mode == "dense"))


@pytest.mark.parametrize("step,hq,hkv", [(2, 1, 1), (16, 1, 1), (4, 4, 2), (16, 8, 2), (32, 2, 1),
                                         (3, 4, 2), (5, 1, 1)])
def test_step_grouping(step, hq, hkv):
    """AnchorAttention's query-block grouping: a key kept by any block of a group
    of `step` blocks is kept by all of them (within each block's candidates).
    Powers of two up to 32 run the fused scan + compaction kernel, other steps
    the bitmask + compaction pair."""
    from workloads import Workload
    L = 6000
    w = Workload(f"step-{step}-{hq}", 12, 1, hq, hkv, L, sink=64, local=256, theta=2.6,
                 needles_per_head=16)
    inp = generate(w)
    run = Run(inp, mode="anchor", sink=64, local=256, theta=2.6, step=step)
    heads = [(0, h) for h in range(hq)]
    compare_anchor_masks(run, inp, heads)
    rows = {hd: sample_rows(L, 30, 5 * hd[1] + step, must=(L - 1, 2047, 2048)) for hd in heads}
    compare_outputs(run, inp, rows)


def test_c4_sweep_128k_operating_points():
    """The density sweep's layer at full size (its own seed), at the sweep's
    thresholds between the near-dense and the sparse ends: sampled blocks of
    three heads bit-exact up to near-ties, sampled rows within the stated
    bound, in the launch configuration the benchmark times."""
    from workloads import C4_SWEEP_128K
    w = C4_SWEEP_128K
    inp = generate(w)
    dev = None
    heads = [(0, 0), (0, 13), (0, 30)]
    for theta in (7.0, 4.0, 2.5, 2.0):
        run = Run(inp, mode="anchor", sink=w.sink, local=w.local, theta=theta, dev=dev)
        dev = (run.q, run.k, run.v)
        compare_anchor_masks(run, inp, heads,
                             blocks_of=lambda b, h: edge_blocks(w.seq_len, 3, h + int(theta)))
        rows = {hd: sample_rows(w.seq_len, 10, hd[1] + int(10 * theta), must=(w.seq_len - 1,))
                for hd in heads}
        compare_outputs(run, inp, rows)
        del run


def test_c4_sweep_128k_theta_inf_equals_dense_mode():
    from workloads import C4_SWEEP_128K
    w = C4_SWEEP_128K
    inp = generate(w, kv_groups=[0, 7])
    run_inf = Run(inp, mode="anchor", sink=w.sink, local=w.local, theta=math.inf)
    assert run_inf.stats.kept_pairs == run_inf.stats.dense_pairs
    rows = {(0, h): sample_rows(w.seq_len, 10, h, must=(0, w.seq_len - 1)) for h in (0, 3, 29)}
    compare_outputs(run_inf, inp, rows, dense=True)
    o_inf = run_inf.o.clone()
    run_dense = Run(inp, mode="dense", sink=w.sink, local=w.local,
                    dev=(run_inf.q, run_inf.k, run_inf.v))
    compare_outputs(run_dense, inp, rows, dense=True)
    # the same key sets through the two tile paths (candidate tiles vs
    # contiguous local tiles): outputs within bf16 rounding of each other
    d = (o_inf.float() - run_dense.o.float()).abs()
    assert float(d.max()) <= 2 * 2.0 ** -8 * float(run_dense.o.float().abs().max()) + 1e-3
