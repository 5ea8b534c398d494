"""GPU parity of the paired attention with window tiles for the selected keys
(SPA_DEBUG_WINDOW_TILES): 128-key windows holding at least 96 selected keys
are loaded contiguously with the absent keys masked, the rest gathered.  The
attention is over the same kept sets as the default paired kernel, so the
same stated bounds hold against the oracle on the GPU's own kept sets.

Densities from every candidate kept by both heads (the contiguous fast
path, no list read) and near-dense (window tiles) through mixed to sparse
(every tile gathered), ragged lengths, SALE key blocks and step groups.

These tests carry the ``gpu_pending`` marker until their first passing run
on a B200 (``pytest -m gpu_pending``).
"""

import pytest

import block_sparse_long_sm_b200 as spa
from workloads import C0_TINY, C1_LLAMA_32K, generate

from gpu_common import Run, compare_outputs, sample_rows

pytestmark = pytest.mark.gpu_pending

WIN = spa.SPA_DEBUG_WINDOW_TILES


@pytest.mark.parametrize("theta", [float("inf"), 7.0, 5.0, 4.0, 3.0, 2.0])
def test_window_tiles_all_rows(theta):
    w = C0_TINY.with_(heads_q=2, heads_kv=1)
    inp = generate(w)
    run = Run(inp, mode="anchor", sink=w.sink, local=w.local, theta=theta, debug_flags=WIN)
    compare_outputs(run, inp, {(0, 0): range(w.seq_len), (0, 1): range(w.seq_len)})


@pytest.mark.parametrize("L,sink,local,theta,step", [(129, 64, 128, 3.0, 1), (1777, 200, 256, 4.0, 1),
                                                    (3001, 128, 256, 4.5, 4)])
def test_window_tiles_ragged_and_steps(L, sink, local, theta, step):
    w = C0_TINY.with_(heads_q=4, heads_kv=2, sink=sink, local=local)
    inp = generate(w, seq_len=L)
    run = Run(inp, mode="anchor", sink=sink, local=local, theta=theta, step=step,
              debug_flags=WIN)
    compare_outputs(run, inp, {(0, h): range(L) for h in range(4)})


def test_window_tiles_sale_blocks():
    w = C0_TINY.with_(heads_q=2, heads_kv=1, block_k=32)
    inp = generate(w, seq_len=2500)
    run = Run(inp, mode="sale", sink=64, local=256, tau=1e-3, block_k=32, debug_flags=WIN)
    compare_outputs(run, inp, {(0, 0): range(2500), (0, 1): range(2500)})


def test_window_tiles_llama_32k():
    w = C1_LLAMA_32K
    inp = generate(w)
    run = Run(inp, mode="anchor", sink=w.sink, local=w.local, theta=4.0, debug_flags=WIN)
    rows = {(0, h): sample_rows(w.seq_len, 24, h, must=(0, 127, 128, w.seq_len - 1))
            for h in (0, 1, 17, 30)}
    compare_outputs(run, inp, rows)


def test_window_tiles_batch_of_two():
    w = C0_TINY.with_(batch=2, heads_q=4, heads_kv=2)
    inp = generate(w, seq_len=1500)
    run = Run(inp, mode="anchor", sink=w.sink, local=w.local, theta=4.0, debug_flags=WIN)
    compare_outputs(run, inp, {(b, h): range(1500) for b in range(2) for h in (0, 3)})
