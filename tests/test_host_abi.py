"""CPU-side checks of the C ABI: the library loads, exports every function that
include/spa.h declares, validates arguments before touching the device, and
sizes the workspace with the documented closed form.  No compute calls."""

import math
import os
import re

import pytest

import block_sparse_long_sm_b200 as spa
from block_sparse_long_sm_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"SPA_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)
    return names


def test_library_exports_every_declared_symbol():
    declared = _declared()
    assert set(declared) >= set(spa.EXPORTED)
    for name in declared:
        assert hasattr(binding._lib, name), name


def test_status_strings():
    for code in range(6):
        assert spa.sparse_prefill_status_string(code)
    assert spa.sparse_prefill_status_string(spa.SPA_ERR_WORKSPACE) == "workspace too small"


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=64), spa.SPA_ERR_UNSUPPORTED), (dict(causal=0), spa.SPA_ERR_UNSUPPORTED),
    (dict(block_q=64), spa.SPA_ERR_UNSUPPORTED), (dict(step=0), spa.SPA_ERR_INVALID),
    (dict(local=64), spa.SPA_ERR_INVALID), (dict(local=300), spa.SPA_ERR_INVALID),
    (dict(sink=-1), spa.SPA_ERR_INVALID), (dict(theta=math.nan), spa.SPA_ERR_INVALID),
    (dict(softmax_scale=-1.0), spa.SPA_ERR_INVALID), (dict(mode=7), spa.SPA_ERR_INVALID),
    (dict(heads_q=3, heads_kv=2), spa.SPA_ERR_INVALID),
    (dict(mode="sale", block_k=48), spa.SPA_ERR_UNSUPPORTED),
    (dict(mode="sale", sink=48, block_k=32), spa.SPA_ERR_UNSUPPORTED),
    (dict(mode="sale", tau=0.0), spa.SPA_ERR_INVALID),
    (dict(mode="sale", tau=1.5), spa.SPA_ERR_INVALID),
    (dict(mode="anchor", block_k=32), spa.SPA_ERR_UNSUPPORTED)])
def test_validation_before_any_launch(kw, code):
    base = dict(batch=1, heads_q=4, heads_kv=2, seq_len=1024, sink=64, local=128)
    base.update(kw)
    args = [base.pop(k) for k in ("batch", "heads_q", "heads_kv", "seq_len")]
    p = spa.make_params(*args, **base)
    assert spa.sparse_prefill_workspace_bytes(p) == 0
    assert spa.sparse_prefill_plan(p, 0, 0, 0, workspace_bytes=0, stream=0) == code
    assert spa.sparse_prefill_attn(p, 0, 0, 0, 0, 0, workspace_bytes=0, stream=0) == code


def test_workspace_too_small_and_null_pointers():
    p = spa.make_params(1, 4, 2, 1024, sink=64, local=128)
    n = spa.sparse_prefill_workspace_bytes(p)
    assert spa.sparse_prefill_plan(p, 0, 0, 0, workspace_bytes=n, stream=0) == spa.SPA_ERR_INVALID
    assert spa.sparse_prefill_plan(p, 0, 0, 4096, workspace_bytes=n - 1, stream=0) == spa.SPA_ERR_WORKSPACE
    assert spa.sparse_prefill_plan(p, 0, 0, 4104, workspace_bytes=n, stream=0) == spa.SPA_ERR_INVALID


@pytest.mark.parametrize("n,local,sink", [(0, 256, 128), (1, 128, 0), (5, 128, 64), (300, 256, 128),
                                          (1024, 256, 128), (77, 384, 200)])
def test_cap_prefix_closed_form(n, local, sink):
    assert binding.cap_prefix(n, local, sink) == sum(max(0, (q + 1) * 128 - local - sink)
                                                     for q in range(n))


def test_workspace_bytes_cover_documented_regions():
    for mode, bk in (("anchor", None), ("sale", 32), ("dense", None)):
        for L in (1, 127, 4096, 131072):
            p = spa.make_params(1, 32, 8, L, mode=mode, block_k=bk)
            n = spa.sparse_prefill_workspace_bytes(p)
            nqb = (L + 127) // 128
            nb = 32 * nqb
            lists_at = (256 + 4 * nb + 255) // 256 * 256
            unit = 32 if mode == "sale" else 1
            per_head = binding.cap_prefix(nqb, 256, 128) // unit if mode != "dense" else 0
            assert n >= lists_at + 4 * 32 * per_head
    # the 128K Llama layer: per-head lists (~8.55 GB), the candidate-tile
    # masks (16 B per candidate tile: ~0.27 GB) and small scratch; the bitmask
    # (0.54 GB) only when the selection groups do not fit a warp
    p = spa.make_params(1, 32, 8, 131072)
    assert 8.8e9 < spa.sparse_prefill_workspace_bytes(p) < 8.9e9
    p = spa.make_params(1, 32, 8, 131072, step=3)
    assert 9.35e9 < spa.sparse_prefill_workspace_bytes(p) < 9.45e9


def test_shard_units_partition():
    from block_sparse_long_sm_b200.shard import kv_head_slice, shard_units
    for B, H, world in ((1, 8, 1), (1, 8, 2), (1, 8, 8), (4, 8, 3), (2, 5, 4)):
        seen = []
        for r in range(world):
            seen += shard_units(B, H, world, r)
        assert seen == [(b, g) for b in range(B) for g in range(H)]
    assert kv_head_slice(8, 2, 1) == (4, 8)


def test_decode_scratch_bytes():
    p = spa.make_params(1, 32, 8, 131072)
    n = spa.sparse_decode_scratch_bytes(p, 131072 + 1024)
    # union of each kv head's selections (4 B per candidate), its tag words
    # (1 B per candidate) and the split partials: a few MB, independent of pos
    cand = 131072 - 256 - 128
    assert 8 * cand * 5 < n < 8 * cand * 5 + 4e6
    assert spa.sparse_decode_scratch_bytes(p, 131072) <= n
    assert spa.sparse_decode_scratch_bytes(p, 131071) == 0          # capacity below L
    assert spa.sparse_decode_scratch_bytes(p, (1 << 24) + 1) == 0   # beyond 2^24 rows
    assert spa.sparse_decode_scratch_bytes(spa.make_params(1, 4, 2, 0), 16) == 0
    assert spa.sparse_decode_scratch_bytes(spa.make_params(1, 4, 2, 100, head_dim=64), 128) == 0
    for mode, bk in (("anchor", None), ("sale", 32), ("dense", None)):
        for hq, hkv in ((4, 2), (6, 2), (16, 1), (24, 1)):
            assert spa.sparse_decode_scratch_bytes(
                spa.make_params(2, hq, hkv, 3000, mode=mode, block_k=bk), 4000) > 0


def test_decode_validation_before_any_launch():
    p = spa.make_params(1, 4, 2, 1024, sink=64, local=128)
    ws = spa.sparse_prefill_workspace_bytes(p)
    sc = spa.sparse_decode_scratch_bytes(p, 1100)
    A, S, Q = 1 << 20, 1 << 24, 1 << 28          # aligned stand-in addresses, never touched

    def attn(pos, cap=1100, ws_bytes=ws, sc_bytes=sc, scratch=S):
        return spa.sparse_decode_attn(p, Q, Q, Q, cap, pos, A, scratch, Q, None,
                                      workspace_bytes=ws_bytes, scratch_bytes=sc_bytes, stream=0)
    assert attn(1022) == spa.SPA_ERR_INVALID            # pos < L - 1
    assert attn(1100) == spa.SPA_ERR_INVALID            # pos >= capacity
    assert attn(1023, cap=1000) == spa.SPA_ERR_INVALID  # capacity < L
    assert attn(1023, cap=(1 << 24) + 1) == spa.SPA_ERR_UNSUPPORTED
    assert attn(1023, sc_bytes=sc - 1) == spa.SPA_ERR_WORKSPACE
    assert attn(1023, ws_bytes=ws - 1) == spa.SPA_ERR_WORKSPACE
    assert attn(1023, scratch=S + 8) == spa.SPA_ERR_INVALID
    assert spa.sparse_decode_attn(p, 0, Q, Q, 1100, 1023, A, S, Q, None, workspace_bytes=ws,
                                  scratch_bytes=sc, stream=0) == spa.SPA_ERR_INVALID
    assert spa.sparse_decode_prepare(p, 1100, A, S, workspace_bytes=ws, scratch_bytes=sc - 1,
                                     stream=0) == spa.SPA_ERR_WORKSPACE
    assert spa.sparse_decode_prepare(p, 1100, 0, S, workspace_bytes=ws, scratch_bytes=sc,
                                     stream=0) == spa.SPA_ERR_INVALID
    bad = spa.make_params(1, 4, 2, 1024, sink=64, local=100)
    assert spa.sparse_decode_prepare(bad, 1100, A, S, workspace_bytes=ws, scratch_bytes=sc,
                                     stream=0) == spa.SPA_ERR_INVALID


def test_fp8_sizes_and_validation_before_any_launch():
    p = spa.make_params(2, 8, 2, 1000, sink=64, local=128)
    nqb = 8
    assert spa.sparse_fp8_scales_floats(p) == 2 * 8 * nqb + 2 * 2 + 2 * (2 * 2 * 128)
    sc = spa.sparse_fp8_scratch_bytes(p)
    assert sc >= 2 * 2 * 64 * 128 * 8 + 4 * 2 * 2 * 128
    bad = spa.make_params(2, 8, 2, 1000, sink=64, local=100)
    assert spa.sparse_fp8_scales_floats(bad) == 0 and spa.sparse_fp8_scratch_bytes(bad) == 0
    A = 1 << 20
    assert spa.sparse_fp8_quantize(p, A, A, A, A, A, A, A, A, scratch_bytes=sc - 1,
                                   stream=0) == spa.SPA_ERR_WORKSPACE
    assert spa.sparse_fp8_quantize(p, 0, A, A, A, A, A, A, A, scratch_bytes=sc,
                                   stream=0) == spa.SPA_ERR_INVALID
    assert spa.sparse_fp8_quantize(p, A, A, A, A + 8, A, A, A, A, scratch_bytes=sc,
                                   stream=0) == spa.SPA_ERR_INVALID
    assert spa.sparse_fp8_quantize(bad, A, A, A, A, A, A, A, A, scratch_bytes=sc,
                                   stream=0) == spa.SPA_ERR_INVALID
    ws = spa.sparse_prefill_workspace_bytes(p)
    assert spa.sparse_prefill_attn_fp8(p, A, A, A, A, A, A, workspace_bytes=ws - 1,
                                       stream=0) == spa.SPA_ERR_WORKSPACE
    assert spa.sparse_prefill_attn_fp8(p, A, A, A, A + 2, A, A, workspace_bytes=ws,
                                       stream=0) == spa.SPA_ERR_INVALID
    assert spa.sparse_prefill_attn_fp8(p, A, 0, A, A, A, A, workspace_bytes=ws,
                                       stream=0) == spa.SPA_ERR_INVALID


def test_key_mass_validation_before_any_launch():
    p = spa.make_params(1, 4, 2, 1000, sink=64, local=256)
    ws = spa.sparse_prefill_workspace_bytes(p)
    A = 1 << 20

    def call(window, q=A, ws_bytes=ws, params=p):
        return spa.sparse_key_mass(params, q, A, A, window, A, A, workspace_bytes=ws_bytes,
                                   stream=0)
    assert call(-1) == spa.SPA_ERR_INVALID
    assert call(129) == spa.SPA_ERR_UNSUPPORTED             # beyond local - block_q
    assert call(0, ws_bytes=ws - 1) == spa.SPA_ERR_WORKSPACE
    assert call(0, q=0) == spa.SPA_ERR_INVALID
    assert call(0, q=A + 8) == spa.SPA_ERR_INVALID
