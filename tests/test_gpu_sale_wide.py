"""GPU parity of the SALE block scan with sixteen epilogue warps
(SPA_DEBUG_SALE_WIDE): the same key-block selection as the default scan,
checked against the fp64 oracle bit-exact up to near-ties, for one head,
for four heads of one kv head (every epilogue warp busy), for a group of six
(two CTAs per kv head, the second with two inactive heads) and with
per-head thresholds.

These tests carry the ``gpu_pending`` marker until their first passing run
on a B200 (``pytest -m gpu_pending``).
"""

import pytest

import block_sparse_long_sm_b200 as spa
from workloads import C0_TINY, C2_LLAMA_128K, generate

from gpu_common import Run, compare_outputs, compare_sale_masks

pytestmark = pytest.mark.gpu_pending

WIDE = spa.SPA_DEBUG_SALE_WIDE


@pytest.mark.parametrize("L,tau,bk,sink", [(2048, 1e-3, 32, 64), (1900, 0.02, 16, 32),
                                           (3000, 0.01, 64, 128), (2500, 0.03, 128, 128)])
def test_sale_wide_one_head(L, tau, bk, sink):
    w = C0_TINY.with_(sink=sink, local=256)
    inp = generate(w, seq_len=L)
    run = Run(inp, mode="sale", sink=sink, local=256, tau=tau, block_k=bk, debug_flags=WIDE)
    compare_sale_masks(run, inp, [(0, 0)])
    compare_outputs(run, inp, {(0, 0): range(L)})


@pytest.mark.parametrize("hq,hkv", [(4, 1), (6, 1), (8, 2)])
def test_sale_wide_head_groups(hq, hkv):
    w = C0_TINY.with_(heads_q=hq, heads_kv=hkv, sink=64, local=256)
    inp = generate(w, seq_len=2300)
    run = Run(inp, mode="sale", sink=64, local=256, tau=1e-2, block_k=32, do_attn=False,
              debug_flags=WIDE)
    compare_sale_masks(run, inp, [(0, h) for h in range(hq)])


def test_sale_wide_16k_layer_shape():
    w = C2_LLAMA_128K
    inp = generate(w, seq_len=16384)
    run = Run(inp, mode="sale", sink=w.sink, local=w.local, tau=w.tau, block_k=w.block_k,
              do_attn=False, debug_flags=WIDE)
    compare_sale_masks(run, inp, [(0, 0), (0, 5), (0, 22)])
