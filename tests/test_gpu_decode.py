"""GPU parity of decode-shaped reuse of a plan (SpotAttention Fig. 2 / Sec. 3).

A decoding query at absolute position pos attends to the sink, the plan's
selection for the last prompt query block and that block's local window grown
up to pos.  As in the prefill output tests, the selection the GPU used is
first checked against the oracle (bit-exact up to near-ties), then the
outputs are compared with the oracle's decode attention over the GPU's own
kept set against fp64: |dLSE| <= 2e-3 always; on key sets of at least 128
keys max |dO| <= 1e-2 and mean <= 1e-3; on smaller key sets, where O is not
an average of many rows and its rounding to bf16 alone can exceed a mean of
1e-3 (half an ulp is 0.0078 at |O| in [2, 4)), every element obeys the bound
of the kernel's arithmetic, |dO| <= 2^-8 |O| + 1e-4 (the kernel keeps the
probabilities in fp32 and rounds only O).

Cases: GQA groups of 2, 3, 4 and 16 q heads (one to eight heads per CTA, two
head subgroups), ANCHOR, SALE and DENSE, positions from L - 1 (where the
decode key set is the last prompt row's prefill key set) to the end of the
cache, a prompt of one token, a sink that covers the whole candidate range,
repeated calls after one prepare, and the 128K Llama layer.
"""

import numpy as np
import pytest
import torch

import block_sparse_long_sm_b200 as spa
from oracle import decode as odec
from workloads import C0_TINY, C2_LLAMA_128K, bf16_bits_to_f32, generate, random_bf16

from gpu_common import (LSE_ABS, O_MAX_ABS, O_MEAN_ABS, Run, compare_anchor_masks,
                        compare_sale_masks, head_f64, to_dev)

SMALL_SET = 128      # key sets below this size get the element-wise bound


class Decode:
    """K/V cache (prompt rows + extra rows), prepare once, decode at positions."""

    def __init__(self, run: Run, inputs, cap: int, seed: int):
        B, Hkv, L = run.B, run.Hkv, run.L
        self.run, self.cap = run, cap
        k = np.zeros((B, Hkv, cap, 128), np.uint16)
        v = np.zeros((B, Hkv, cap, 128), np.uint16)
        k[:, :, :L] = inputs.k
        v[:, :, :L] = inputs.v
        if cap > L:
            k[:, :, L:] = random_bf16((B, Hkv, cap - L, 128), seed)
            v[:, :, L:] = random_bf16((B, Hkv, cap - L, 128), seed + 1)
        self.k_host, self.v_host = k, v
        self.k, self.v = to_dev(k), to_dev(v)
        nbytes = spa.sparse_decode_scratch_bytes(run.params, cap)
        assert nbytes > 0
        self.scratch = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        spa.check(spa.sparse_decode_prepare(run.params, cap, run.ws, self.scratch), "prepare")

    def attend(self, q_u16: np.ndarray, pos: int):
        B, Hq = self.run.B, self.run.Hq
        q = to_dev(q_u16)
        o = torch.empty((B, Hq, 128), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
        spa.check(spa.sparse_decode_attn(self.run.params, q, self.k, self.v, self.cap, pos,
                                         self.run.ws, self.scratch, o, lse), "decode")
        st, stats = spa.sparse_prefill_stats(self.run.params, self.run.ws)
        spa.check(st, "stats")
        return o.float().cpu().numpy(), lse.cpu().numpy()

    def compare(self, q_u16: np.ndarray, pos: int, heads=None):
        run, p = self.run, self.run.params
        o, lse = self.attend(q_u16, pos)
        qb = (run.L - 1) // 128
        errs, lse_err = [], 0.0
        heads = heads or [(b, h) for b in range(run.B) for h in range(run.Hq)]
        for b, h in heads:
            g = h // run.group
            kh = bf16_bits_to_f32(self.k_host[b, g]).astype(np.float64)
            vh = bf16_bits_to_f32(self.v_host[b, g]).astype(np.float64)
            if p.mode == spa.SPA_MODE_DENSE:
                keys = np.arange(pos + 1)
            else:
                keys = odec.decode_keys(pos, run.L, run.selected_keys(b, h, qb), bq=128,
                                        sink=p.sink, local=p.local)
            qv = bf16_bits_to_f32(q_u16[b, h]).astype(np.float64)
            o_ref, lse_ref = odec.decode_attend(qv, kh, vh, keys)
            d = np.abs(o[b, h] - o_ref)
            if keys.size >= SMALL_SET:
                errs.append(d)
            else:
                lim = 2.0 ** -8 * np.abs(o_ref) + 1e-4
                assert np.all(d <= lim), (b, h, pos, int(keys.size), float(np.max(d / lim)))
            lse_err = max(lse_err, abs(float(lse[b, h]) - lse_ref))
        assert lse_err <= LSE_ABS, lse_err
        if errs:
            e = np.concatenate(errs)
            res = dict(max_abs=float(e.max()), mean_abs=float(e.mean()), lse_max=lse_err)
            assert res["max_abs"] <= O_MAX_ABS, res
            assert res["mean_abs"] <= O_MEAN_ABS, res
        return o, lse


def _queries(B, Hq, seed, bias=0.0):
    return random_bf16((B, Hq, 128), seed, mean=bias)


@pytest.mark.gpu
@pytest.mark.parametrize("hq,hkv,theta", [(4, 2, 2.5), (6, 2, 3.0), (4, 1, 2.0), (16, 1, 2.5)])
def test_anchor_groups_and_positions(hq, hkv, theta):
    L, cap = 2000, 2100
    w = C0_TINY.with_(heads_q=hq, heads_kv=hkv, sink=64, local=256)
    inp = generate(w, seq_len=L)
    run = Run(inp, mode="anchor", sink=64, local=256, theta=theta, do_attn=False)
    qb = (L - 1) // 128
    compare_anchor_masks(run, inp, [(0, h) for h in range(hq)], blocks_of=lambda b, h: [qb])
    dec = Decode(run, inp, cap, seed=7)
    for i, pos in enumerate((L - 1, L + 37, cap - 1)):
        dec.compare(_queries(1, hq, 100 + i, bias=0.5), pos)


@pytest.mark.gpu
def test_last_prompt_row_matches_prefill():
    L, cap = 1500, 1600
    w = C0_TINY.with_(heads_q=4, heads_kv=2, sink=64, local=256)
    inp = generate(w, seq_len=L)
    run = Run(inp, mode="anchor", sink=64, local=256, theta=2.5)
    dec = Decode(run, inp, cap, seed=9)
    q_last = np.ascontiguousarray(inp.q[:, :, L - 1])
    o, lse = dec.compare(q_last, L - 1)
    o_pre = run.o.float().cpu().numpy()[:, :, L - 1]
    lse_pre = run.lse.cpu().numpy()[:, :, L - 1]
    # two kernels over the same key set: within the bf16 rounding of both outputs
    assert np.max(np.abs(o - o_pre)) <= 2 * O_MAX_ABS
    assert np.max(np.abs(lse - lse_pre)) <= 2 * LSE_ABS


@pytest.mark.gpu
@pytest.mark.parametrize("bk,tau", [(64, 1e-2), (32, 1e-3)])
def test_sale_blocks(bk, tau):
    L, cap = 1500, 1536
    w = C0_TINY.with_(heads_q=2, heads_kv=1, sink=128, local=256, block_k=bk)
    inp = generate(w, seq_len=L)
    run = Run(inp, mode="sale", sink=128, local=256, tau=tau, block_k=bk, do_attn=False)
    qb = (L - 1) // 128
    compare_sale_masks(run, inp, [(0, 0), (0, 1)], blocks_of=lambda b, h: [qb])
    dec = Decode(run, inp, cap, seed=11)
    for i, pos in enumerate((L - 1, L + 20)):
        dec.compare(_queries(1, 2, 200 + i), pos)


@pytest.mark.gpu
def test_dense_mode():
    L, cap = 700, 800
    w = C0_TINY.with_(heads_q=4, heads_kv=2)
    inp = generate(w, seq_len=L)
    run = Run(inp, mode="dense", sink=64, local=128, do_attn=False)
    dec = Decode(run, inp, cap, seed=13)
    dec.compare(_queries(1, 4, 300), L - 1)
    dec.compare(_queries(1, 4, 301), cap - 1)


@pytest.mark.gpu
@pytest.mark.parametrize("L,sink,local,positions", [
    (1, 64, 128, (0, 1, 3)),          # one-token prompt: no candidates
    (300, 256, 128, (299, 310)),      # sink covers the candidate range
    (129, 0, 128, (128, 200)),        # no sink
])
def test_degenerate_geometry(L, sink, local, positions):
    cap = max(positions) + 1
    w = C0_TINY.with_(heads_q=2, heads_kv=1, sink=sink, local=local)
    inp = generate(w, seq_len=L)
    run = Run(inp, mode="anchor", sink=sink, local=local, theta=3.0, do_attn=False)
    dec = Decode(run, inp, cap, seed=17)
    for i, pos in enumerate(positions):
        dec.compare(_queries(1, 2, 400 + i), pos)


@pytest.mark.gpu
def test_repeated_calls_are_identical():
    L, cap = 1200, 1300
    w = C0_TINY.with_(heads_q=4, heads_kv=2, sink=64, local=256)
    inp = generate(w, seq_len=L)
    run = Run(inp, mode="anchor", sink=64, local=256, theta=2.5, do_attn=False)
    dec = Decode(run, inp, cap, seed=19)
    q = _queries(1, 4, 500)
    o1, l1 = dec.attend(q, L + 3)
    for pos in (L - 1, cap - 1):
        dec.attend(_queries(1, 4, 501), pos)
    o2, l2 = dec.attend(q, L + 3)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


@pytest.mark.gpu
def test_llama_128k_layer():
    w = C2_LLAMA_128K
    L = w.seq_len
    groups = (0, 5)
    inp = generate(w, kv_groups=groups)
    run = Run(inp, mode="anchor", sink=w.sink, local=w.local, theta=w.theta, do_attn=False)
    heads = [(0, g * 4 + j) for g in groups for j in (0, 3)]
    compare_anchor_masks(run, inp, heads, blocks_of=lambda b, h: [(L - 1) // 128])
    dec = Decode(run, inp, L + 64, seed=23)
    for i, pos in enumerate((L - 1, L + 63)):
        dec.compare(_queries(1, w.heads_q, 600 + i, bias=0.5), pos, heads=heads)


@pytest.mark.gpu
def test_batch_of_two():
    L, cap = 1100, 1200
    w = C0_TINY.with_(batch=2, heads_q=4, heads_kv=2, sink=64, local=256)
    inp = generate(w, seq_len=L)
    run = Run(inp, mode="anchor", sink=64, local=256, theta=2.5, do_attn=False)
    dec = Decode(run, inp, cap, seed=29)
    for i, pos in enumerate((L - 1, cap - 1)):
        dec.compare(_queries(2, 4, 700 + i, bias=0.5), pos)
