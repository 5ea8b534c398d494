"""ctypes binding of the C ABI in ``include/spa.h`` (argument marshalling only).

Every function takes the same arguments as its C counterpart; device buffers
may be given as torch tensors (their ``data_ptr()``) or as raw integer
addresses, and ``stream`` as a ``torch.cuda.Stream``, a raw handle or ``None``
(the current torch stream).  All computation happens in ``lib/libspa.so``;
there is no fallback: importing this module fails loudly when the library has
not been built.
"""

from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libspa.so")

SPA_OK, SPA_ERR_INVALID, SPA_ERR_UNSUPPORTED, SPA_ERR_WORKSPACE, SPA_ERR_CUDA, SPA_ERR_TIMEOUT = range(6)
SPA_MODE_ANCHOR, SPA_MODE_SALE, SPA_MODE_DENSE = 0, 1, 2
SPA_DEBUG_STALL_ATTN = 0x1
MODES = {"anchor": SPA_MODE_ANCHOR, "sale": SPA_MODE_SALE, "dense": SPA_MODE_DENSE}

EXPORTED = ("sparse_prefill_workspace_bytes", "sparse_prefill_plan", "sparse_prefill_attn",
            "sparse_prefill_stats", "sparse_prefill_status_string", "sparse_prefill_plan_static",
            "sparse_decode_scratch_bytes", "sparse_decode_prepare", "sparse_decode_attn",
            "sparse_fp8_scales_floats", "sparse_fp8_scratch_bytes", "sparse_fp8_quantize",
            "sparse_prefill_attn_fp8", "sparse_key_mass")


class SpaParams(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("heads_q", ctypes.c_int32), ("heads_kv", ctypes.c_int32),
        ("seq_len", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("causal", ctypes.c_int32),
        ("block_q", ctypes.c_int32), ("block_k", ctypes.c_int32), ("sink", ctypes.c_int32),
        ("local", ctypes.c_int32), ("step", ctypes.c_int32), ("mode", ctypes.c_int32),
        ("theta", ctypes.c_float), ("tau", ctypes.c_float), ("softmax_scale", ctypes.c_float),
        ("wait_limit_us", ctypes.c_uint32), ("debug_flags", ctypes.c_uint32),
        ("tau_per_head", ctypes.POINTER(ctypes.c_float)),
    ]


class SpaStats(ctypes.Structure):
    _fields_ = [
        ("error_bits", ctypes.c_uint32), ("reserved", ctypes.c_uint32),
        ("query_blocks", ctypes.c_int64), ("candidates", ctypes.c_int64),
        ("kept_candidates", ctypes.c_int64), ("kept_pairs", ctypes.c_int64),
        ("dense_pairs", ctypes.c_int64),
    ]

    def as_dict(self):
        return {name: getattr(self, name) for name, _ in self._fields_ if name != "reserved"}


class SpaError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {sparse_prefill_status_string(status)} (status {status})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m block_sparse_long_sm_b200.build` "
            "(there is no fallback implementation)")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(SpaParams)
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    lib.sparse_prefill_workspace_bytes.argtypes = [P]
    lib.sparse_prefill_workspace_bytes.restype = sz
    lib.sparse_prefill_plan.argtypes = [P, vp, vp, vp, sz, vp]
    lib.sparse_prefill_plan.restype = ctypes.c_int
    lib.sparse_prefill_attn.argtypes = [P, vp, vp, vp, vp, sz, vp, vp, vp]
    lib.sparse_prefill_attn.restype = ctypes.c_int
    lib.sparse_prefill_stats.argtypes = [P, vp, sz, ctypes.POINTER(SpaStats), vp]
    lib.sparse_prefill_stats.restype = ctypes.c_int
    lib.sparse_prefill_plan_static.argtypes = [P, vp, vp, vp, vp, sz, vp, vp]
    lib.sparse_prefill_plan_static.restype = ctypes.c_int
    i32 = ctypes.c_int32
    lib.sparse_decode_scratch_bytes.argtypes = [P, i32]
    lib.sparse_decode_scratch_bytes.restype = sz
    lib.sparse_decode_prepare.argtypes = [P, i32, vp, sz, vp, sz, vp]
    lib.sparse_decode_prepare.restype = ctypes.c_int
    lib.sparse_decode_attn.argtypes = [P, vp, vp, vp, i32, i32, vp, sz, vp, sz, vp, vp, vp]
    lib.sparse_decode_attn.restype = ctypes.c_int
    lib.sparse_fp8_scales_floats.argtypes = [P]
    lib.sparse_fp8_scales_floats.restype = sz
    lib.sparse_fp8_scratch_bytes.argtypes = [P]
    lib.sparse_fp8_scratch_bytes.restype = sz
    lib.sparse_fp8_quantize.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.sparse_fp8_quantize.restype = ctypes.c_int
    lib.sparse_prefill_attn_fp8.argtypes = [P, vp, vp, vp, vp, vp, sz, vp, vp, vp]
    lib.sparse_prefill_attn_fp8.restype = ctypes.c_int
    lib.sparse_key_mass.argtypes = [P, vp, vp, vp, i32, vp, sz, vp, vp]
    lib.sparse_key_mass.restype = ctypes.c_int
    lib.sparse_prefill_status_string.argtypes = [ctypes.c_int]
    lib.sparse_prefill_status_string.restype = ctypes.c_char_p
    return lib


_lib = _load()


def make_params(batch: int, heads_q: int, heads_kv: int, seq_len: int, *, mode="anchor",
                sink: int = 128, local: int = 256, theta: float = 5.0, tau: float = 1e-3,
                block_k: Optional[int] = None, softmax_scale: float = 0.0,
                wait_limit_us: int = 0, debug_flags: int = 0, head_dim: int = 128,
                causal: int = 1, block_q: int = 128, step: int = 1,
                tau_per_head=None) -> SpaParams:
    m = MODES[mode] if isinstance(mode, str) else int(mode)
    if block_k is None:
        block_k = 32 if m == SPA_MODE_SALE else 1
    p = SpaParams(batch, heads_q, heads_kv, seq_len, head_dim, causal, block_q, block_k,
                  sink, local, step, m, float(theta), float(tau), float(softmax_scale),
                  int(wait_limit_us), int(debug_flags), None)
    if tau_per_head is not None:
        arr = (ctypes.c_float * len(tau_per_head))(*[float(t) for t in tau_per_head])
        p._tau_keepalive = arr          # the struct holds a raw pointer into this array
        p.tau_per_head = ctypes.cast(arr, ctypes.POINTER(ctypes.c_float))
    return p


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s) -> Optional[int]:
    if s is None:
        try:
            import torch
            return torch.cuda.current_stream().cuda_stream
        except Exception:  # pragma: no cover - no torch / no device
            return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _nbytes(x) -> int:
    if isinstance(x, int):
        raise TypeError("pass the workspace size explicitly when giving a raw pointer")
    return x.numel() * x.element_size()


def sparse_prefill_workspace_bytes(params: SpaParams) -> int:
    return int(_lib.sparse_prefill_workspace_bytes(ctypes.byref(params)))


def sparse_prefill_plan(params: SpaParams, q, k, workspace, workspace_bytes=None,
                        stream=None) -> int:
    wb = _nbytes(workspace) if workspace_bytes is None else int(workspace_bytes)
    return int(_lib.sparse_prefill_plan(ctypes.byref(params), _ptr(q), _ptr(k), _ptr(workspace),
                                        wb, _stream(stream)))


def sparse_prefill_attn(params: SpaParams, q, k, v, workspace, o, lse=None,
                        workspace_bytes=None, stream=None) -> int:
    wb = _nbytes(workspace) if workspace_bytes is None else int(workspace_bytes)
    return int(_lib.sparse_prefill_attn(ctypes.byref(params), _ptr(q), _ptr(k), _ptr(v),
                                        _ptr(workspace), wb, _ptr(o), _ptr(lse), _stream(stream)))


def sparse_prefill_stats(params: SpaParams, workspace, workspace_bytes=None, stream=None):
    """Returns (status, SpaStats)."""
    wb = _nbytes(workspace) if workspace_bytes is None else int(workspace_bytes)
    out = SpaStats()
    st = int(_lib.sparse_prefill_stats(ctypes.byref(params), _ptr(workspace), wb,
                                       ctypes.byref(out), _stream(stream)))
    return st, out


def sparse_prefill_plan_static(params: SpaParams, q, k, counts, lists, lists_elems=None,
                               error_word=None, stream=None) -> int:
    """Allocation-free ANCHOR plan: scratch in the library's fixed device array."""
    n = lists.numel() if lists_elems is None else int(lists_elems)
    return int(_lib.sparse_prefill_plan_static(ctypes.byref(params), _ptr(q), _ptr(k),
                                               _ptr(counts), _ptr(lists), n, _ptr(error_word),
                                               _stream(stream)))


def sparse_decode_scratch_bytes(params: SpaParams, kv_capacity: int) -> int:
    return int(_lib.sparse_decode_scratch_bytes(ctypes.byref(params), int(kv_capacity)))


def sparse_decode_prepare(params: SpaParams, kv_capacity: int, workspace, scratch,
                          workspace_bytes=None, scratch_bytes=None, stream=None) -> int:
    """Once per plan: the tagged union of each kv head's q-head selections."""
    wb = _nbytes(workspace) if workspace_bytes is None else int(workspace_bytes)
    sb = _nbytes(scratch) if scratch_bytes is None else int(scratch_bytes)
    return int(_lib.sparse_decode_prepare(ctypes.byref(params), int(kv_capacity), _ptr(workspace),
                                          wb, _ptr(scratch), sb, _stream(stream)))


def sparse_decode_attn(params: SpaParams, q, k_cache, v_cache, kv_capacity: int, pos: int,
                       workspace, scratch, o, lse=None, workspace_bytes=None,
                       scratch_bytes=None, stream=None) -> int:
    """One decoding query per (b, q head) at position ``pos`` over sink + selection + window."""
    wb = _nbytes(workspace) if workspace_bytes is None else int(workspace_bytes)
    sb = _nbytes(scratch) if scratch_bytes is None else int(scratch_bytes)
    return int(_lib.sparse_decode_attn(ctypes.byref(params), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                       int(kv_capacity), int(pos), _ptr(workspace), wb,
                                       _ptr(scratch), sb, _ptr(o), _ptr(lse), _stream(stream)))


def sparse_fp8_scales_floats(params: SpaParams) -> int:
    return int(_lib.sparse_fp8_scales_floats(ctypes.byref(params)))


def sparse_fp8_scratch_bytes(params: SpaParams) -> int:
    return int(_lib.sparse_fp8_scratch_bytes(ctypes.byref(params)))


def sparse_fp8_quantize(params: SpaParams, q, k, v, q8, k8, v8, scales, scratch,
                        scratch_bytes=None, stream=None) -> int:
    """E4M3 codes of q, k (mean-smoothed), v and their scales (layout in spa.h)."""
    sb = _nbytes(scratch) if scratch_bytes is None else int(scratch_bytes)
    return int(_lib.sparse_fp8_quantize(ctypes.byref(params), _ptr(q), _ptr(k), _ptr(v), _ptr(q8),
                                        _ptr(k8), _ptr(v8), _ptr(scales), _ptr(scratch), sb,
                                        _stream(stream)))


def sparse_prefill_attn_fp8(params: SpaParams, q8, k8, v8, scales, workspace, o, lse=None,
                            workspace_bytes=None, stream=None) -> int:
    """Attention over the plan's kept keys with E4M3 operands."""
    wb = _nbytes(workspace) if workspace_bytes is None else int(workspace_bytes)
    return int(_lib.sparse_prefill_attn_fp8(ctypes.byref(params), _ptr(q8), _ptr(k8), _ptr(v8),
                                            _ptr(scales), _ptr(workspace), wb, _ptr(o), _ptr(lse),
                                            _stream(stream)))


def sparse_key_mass(params: SpaParams, q, k, lse, window: int, workspace, mass,
                    workspace_bytes=None, stream=None) -> int:
    """Attention mass per key from the prefill rows, from the prefill LSE."""
    wb = _nbytes(workspace) if workspace_bytes is None else int(workspace_bytes)
    return int(_lib.sparse_key_mass(ctypes.byref(params), _ptr(q), _ptr(k), _ptr(lse), int(window),
                                    _ptr(workspace), wb, _ptr(mass), _stream(stream)))


def sparse_prefill_status_string(status: int) -> str:
    return _lib.sparse_prefill_status_string(int(status)).decode()


def check(status: int, what: str = "spa") -> None:
    if status != SPA_OK:
        raise SpaError(status, what)


def kept_flops(stats: SpaStats, head_dim: int = 128) -> int:
    """Executed attention FLOPs on kept entries: 4 * d * sum_i |K_i|."""
    return 4 * head_dim * int(stats.kept_pairs)


def default_scale(head_dim: int = 128) -> float:
    return 1.0 / math.sqrt(head_dim)


# ---------------------------------------------------------------------------
# workspace views (the layout documented in include/spa.h)
# ---------------------------------------------------------------------------
def _align256(x: int) -> int:
    return (x + 255) // 256 * 256


def cap_prefix(n: int, local: int, sink: int, bq: int = 128) -> int:
    """P(n) = sum_{q < n} max(0, (q + 1) * bq - local - sink), in closed form."""
    return _cap_prefix_closed(n, local + sink, bq)


def _cap_prefix_closed(n: int, a: int, bq: int) -> int:
    q0 = a // bq
    if n <= q0:
        return 0
    return bq * ((n * (n + 1) - q0 * (q0 + 1)) // 2) - (n - q0) * a


class WorkspaceView:
    """Host-side indexing of the counts and lists inside a workspace tensor."""

    def __init__(self, params: SpaParams, workspace):
        import torch
        self.p = params
        self.nqb = (params.seq_len + 127) // 128
        self.nb = params.batch * params.heads_q * self.nqb
        self.unit = params.block_k if params.mode == SPA_MODE_SALE else 1
        self.per_head = _cap_prefix_closed(self.nqb, params.local + params.sink, 128) // self.unit
        ws8 = workspace.view(torch.uint8)
        self.counts = ws8[256:256 + 4 * self.nb].view(torch.int32)
        lo = _align256(256 + 4 * self.nb)
        n_list = params.batch * params.heads_q * self.per_head
        self.lists = ws8[lo:lo + 4 * n_list].view(torch.int32)

    def block_index(self, b: int, h: int, qb: int) -> int:
        return (b * self.p.heads_q + h) * self.nqb + qb

    def list_offset(self, b: int, h: int, qb: int) -> int:
        return ((b * self.p.heads_q + h) * self.per_head +
                _cap_prefix_closed(qb, self.p.local + self.p.sink, 128) // self.unit)
