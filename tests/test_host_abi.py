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
    # the 128K Llama layer: per-head lists (~8.55 GB), the head pairs' tagged
    # union lists (~4.28 GB) and small scratch; the bitmask (0.54 GB) only when
    # the selection groups do not fit a warp
    p = spa.make_params(1, 32, 8, 131072)
    assert 12.8e9 < spa.sparse_prefill_workspace_bytes(p) < 12.9e9
    p = spa.make_params(1, 32, 8, 131072, step=3)
    assert 13.35e9 < spa.sparse_prefill_workspace_bytes(p) < 13.45e9


def test_shard_units_partition():
    from block_sparse_long_sm_b200.shard import kv_head_slice, shard_units
    for B, H, world in ((1, 8, 1), (1, 8, 2), (1, 8, 8), (4, 8, 3), (2, 5, 4)):
        seen = []
        for r in range(world):
            seen += shard_units(B, H, world, r)
        assert seen == [(b, g) for b in range(B) for g in range(H)]
    assert kv_head_slice(8, 2, 1) == (4, 8)
