"""Randomised checks of the C ABI's argument rules and size functions (no
launches): every size function returns 0 exactly when the parameters break a
rule that include/spa.h documents, and otherwise covers the documented
regions."""

import math

from hypothesis import given, settings, strategies as st

import block_sparse_long_sm_b200 as spa
from block_sparse_long_sm_b200 import binding


def _documented_ok(batch, hq, hkv, L, mode, sink, local, step, theta, tau, bk):
    """The rules as spa.h states them (head_dim, causal and block_q fixed)."""
    if batch < 0 or hq < 1 or hkv < 1 or L < 0 or hq % hkv:
        return False
    if step < 1 or sink < 0 or local < 128 or local % 128:
        return False
    if batch * max(hq, hkv) * L >= 2 ** 31 or batch * hq > 65535:
        return False
    if mode == "anchor":
        return bk == 1 and not math.isnan(theta)
    if mode == "sale":
        return (bk in (16, 32, 64, 128) and sink % bk == 0 and 0 < tau <= 1
                and L <= 262144)
    return True


params = st.tuples(
    st.integers(-1, 4), st.sampled_from([1, 2, 3, 4, 6, 8, 16, 32, 64]),
    st.sampled_from([1, 2, 3, 4, 8]), st.integers(-1, 300000),
    st.sampled_from(["anchor", "sale", "dense"]), st.integers(-2, 600),
    st.sampled_from([0, 64, 100, 128, 256, 384, 1000]), st.integers(0, 40),
    st.sampled_from([5.0, -1.0, float("inf"), float("nan")]),
    st.sampled_from([1e-3, 0.0, 1.0, 1.5]), st.sampled_from([1, 16, 32, 48, 64, 128]))


@settings(max_examples=400, deadline=None)
@given(params)
def test_size_functions_follow_the_documented_rules(args):
    batch, hq, hkv, L, mode, sink, local, step, theta, tau, bk = args
    p = spa.make_params(batch, hq, hkv, L, mode=mode, sink=sink, local=local, step=step,
                        theta=theta, tau=tau, block_k=bk)
    ok = _documented_ok(batch, hq, hkv, L, mode, sink, local, step, theta, tau, bk)
    ws = spa.sparse_prefill_workspace_bytes(p)
    assert (ws > 0) == ok, (args, ws)
    assert (spa.sparse_fp8_scratch_bytes(p) > 0) == ok
    if not ok:
        assert spa.sparse_fp8_scratch_bytes(p) == 0
        assert spa.sparse_decode_scratch_bytes(p, max(L, 1)) == 0
        return
    # documented regions: header, counts, lists (mode-dependent)
    nqb = (L + 127) // 128
    nb = batch * hq * nqb
    lists_at = (256 + 4 * nb + 255) // 256 * 256
    unit = bk if mode == "sale" else 1
    per_head = binding.cap_prefix(nqb, local, sink) // unit if mode != "dense" else 0
    assert ws >= lists_at + 4 * batch * hq * per_head
    # decode: defined for L >= 1 and L <= capacity <= 2^24
    if L >= 1:
        d1 = spa.sparse_decode_scratch_bytes(p, L)
        d2 = spa.sparse_decode_scratch_bytes(p, L + 4096) if L + 4096 <= 1 << 24 else d1
        assert d1 > 0 and d2 >= d1
        assert spa.sparse_decode_scratch_bytes(p, L - 1) == 0
    else:
        assert spa.sparse_decode_scratch_bytes(p, 16) == 0
    # FP8 scales: q scales per block, k scales per head, v scales and K means per channel
    bkv = batch * hkv
    assert spa.sparse_fp8_scales_floats(p) == batch * hq * nqb + bkv + 2 * bkv * 128
