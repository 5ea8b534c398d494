"""The plan's candidate-tile masks hold exactly the keys of its index lists.

For every query block the plan writes, beside the ascending list of kept
candidate keys, one 128-bit mask per candidate tile (keys 128 kt .. 128 kt +
127 for sink / 128 <= kt < ls / 128), which the paired attention kernel cuts
its tiles from, and three bitmaps over the candidate tiles (some key kept;
at least 64 kept, or all 128 for SALE's key blocks; all 128 kept).  All are
read back from the workspace here: the masks must spell out the list key
for key and the bitmaps must agree with the masks' counts, on fused
selection (steps 1 and 2), the
bitmask path (step 3), SALE key blocks of every size, a sink that is not a
multiple of 128, ragged lengths, one and two heads per kv head.
"""

import numpy as np
import pytest

import block_sparse_long_sm_b200 as spa

from workloads import C0_TINY, generate

from gpu_common import Run

pytestmark = pytest.mark.gpu


def _check(run: Run):
    p = run.params
    L, nqb = run.L, (run.L + 127) // 128
    c = 1 - p.local // 128 - p.sink // 128
    tiles = lambda q: max(0, q + c)
    prefix = lambda n: (n + c) * (n + c - 1) // 2 if n + c > 0 else 0
    per_head = prefix(nqb)
    nbytes = run.B * run.Hq * per_head * 16
    W = (tiles(nqb - 1) + 31) // 32                   # words of one tile bitmap
    bbytes = run.B * run.Hq * nqb * 3 * W * 4
    al = lambda x: (x + 255) // 256 * 256
    ws = run.ws.cpu().numpy()
    # the masks and then the bitmaps are the workspace's last two regions
    start = ws.size - al(bbytes) - al(nbytes)
    masks = ws[start:start + nbytes].view(np.uint32).reshape(run.B * run.Hq, per_head, 4)
    bstart = ws.size - al(bbytes)
    bitmaps = ws[bstart:bstart + bbytes].view(np.uint32).reshape(run.B * run.Hq, nqb, 3, W)
    kt0 = p.sink // 128
    # "dense": half the tile for keys selected one by one, the whole tile for
    # SALE's key blocks (which the attention gathers as whole boxes)
    dense_min = 128 if p.mode == spa.SPA_MODE_SALE else 64
    checked = 0
    for b in range(run.B):
        for h in range(run.Hq):
            for qb in range(nqb):
                n = tiles(qb)
                m = masks[b * run.Hq + h, prefix(qb):prefix(qb) + n]
                bits = np.unpackbits(m.view(np.uint8), bitorder="little").reshape(n, 128)
                keys = (np.nonzero(bits.reshape(-1))[0] + 128 * kt0).astype(np.int64)
                want = run.selected_keys(b, h, qb)
                assert np.array_equal(keys, want), (b, h, qb, keys[:8], want[:8])
                # the block's bitmaps: non-empty, dense, all 128 kept
                per_tile = bits.sum(axis=1)
                flags = np.unpackbits(bitmaps[b * run.Hq + h, qb].view(np.uint8),
                                      bitorder="little").reshape(3, -1)[:, :n]
                assert np.array_equal(flags[0], per_tile > 0), (b, h, qb)
                assert np.array_equal(flags[1], per_tile >= dense_min), (b, h, qb)
                assert np.array_equal(flags[2], per_tile == 128), (b, h, qb)
                checked += 1
    return checked


@pytest.mark.parametrize("hq,hkv,L,sink,local,theta,step", [
    (2, 1, 4096, 64, 128, 2.5, 1), (4, 2, 3001, 128, 256, 4.0, 2), (4, 2, 2500, 200, 256, 3.0, 3),
    (3, 1, 1777, 0, 384, 3.0, 1), (2, 1, 129, 64, 128, 3.0, 1)])
def test_anchor_tile_masks_match_lists(hq, hkv, L, sink, local, theta, step):
    w = C0_TINY.with_(heads_q=hq, heads_kv=hkv, sink=sink, local=local)
    inp = generate(w, seq_len=L)
    run = Run(inp, mode="anchor", sink=sink, local=local, theta=theta, step=step, do_attn=False)
    assert _check(run) > 0


@pytest.mark.parametrize("bk,sink,tau", [(16, 64, 0.02), (32, 128, 0.05), (64, 128, 0.01),
                                         (128, 256, 0.03)])
def test_sale_tile_masks_match_lists(bk, sink, tau):
    w = C0_TINY.with_(heads_q=4, heads_kv=2, sink=sink, local=256)
    inp = generate(w, seq_len=2300)
    run = Run(inp, mode="sale", sink=sink, local=256, tau=tau, block_k=bk, do_attn=False)
    assert _check(run) > 0
