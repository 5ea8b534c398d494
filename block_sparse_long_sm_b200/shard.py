"""Host-side sharding of a prefill layer across ranks (one process per GPU).

The work units of the path are (batch element, kv-head group) pairs: a kv head
together with its Hq/Hkv q heads.  Units share nothing -- selection and
attention of one unit read only that unit's Q/K/V rows -- so ranks need no
collective on the data path.  Two uses:

* weak scaling: every rank runs a full layer of its own;
* strong scaling: the units of one layer are split contiguously across ranks
  and each rank runs the sub-layer made of its units.

Timing across ranks is reduced as the maximum (the job ends with its slowest
rank).
"""

from __future__ import annotations

from typing import List, Tuple


def shard_units(batch: int, heads_kv: int, world: int, rank: int) -> List[Tuple[int, int]]:
    """Contiguous, balanced split of the (b, kv head) units; rank r gets a slice."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    units = [(b, g) for b in range(batch) for g in range(heads_kv)]
    n = len(units)
    lo = rank * n // world
    hi = (rank + 1) * n // world
    return units[lo:hi]


def kv_head_slice(heads_kv: int, world: int, rank: int) -> Tuple[int, int]:
    """[lo, hi) kv heads of rank r when a B = 1 layer is split by kv head."""
    units = shard_units(1, heads_kv, world, rank)
    if not units:
        return 0, 0
    return units[0][1], units[-1][1] + 1


class SubLayer:
    """The kv heads [g0, g1) of a B = 1 layer as a layer of their own.

    A kv head and its q heads form a unit that shares nothing with the other
    units, so running the sub-layer of heads [g0, g1) through the same C ABI
    calls gives exactly the outputs (O, LSE) and the selection (counts,
    lists) that the whole layer gives for those heads.  With B = 1 the
    sub-layer's Q/K/V/O/LSE are contiguous slices of the layer's tensors, so
    it is addressed by byte offsets from the layer's base pointers (no copy).
    """

    def __init__(self, params, g0: int, g1: int):
        from . import binding
        if params.batch != 1:
            raise ValueError("kv-head sub-layers address B = 1 layers")
        if not 0 <= g0 < g1 <= params.heads_kv:
            raise ValueError("bad kv-head range")
        group = params.heads_q // params.heads_kv
        self.g0, self.g1 = g0, g1
        self.h0, self.h1 = g0 * group, g1 * group
        tau = None
        if params.tau_per_head:
            tau = [params.tau_per_head[h] for h in range(self.h0, self.h1)]
        self.params = binding.make_params(
            1, self.h1 - self.h0, g1 - g0, params.seq_len, mode=params.mode, sink=params.sink,
            local=params.local, theta=params.theta, tau=params.tau, block_k=params.block_k,
            softmax_scale=params.softmax_scale, wait_limit_us=params.wait_limit_us,
            debug_flags=params.debug_flags, head_dim=params.head_dim, causal=params.causal,
            block_q=params.block_q, step=params.step, tau_per_head=tau)
        row = params.seq_len * params.head_dim
        self.q_off = self.h0 * row * 2          # bf16 [B, Hq, L, d]
        self.kv_off = g0 * row * 2              # bf16 [B, Hkv, L, d]
        self.o_off = self.h0 * row * 2
        self.lse_off = self.h0 * params.seq_len * 4

    def pointers(self, q, k, v, o, lse=None):
        """Base addresses of the sub-layer inside the layer's tensors."""
        return (q.data_ptr() + self.q_off, k.data_ptr() + self.kv_off,
                v.data_ptr() + self.kv_off, o.data_ptr() + self.o_off,
                None if lse is None else lse.data_ptr() + self.lse_off)


def rank_sub_layer(params, world: int, rank: int) -> SubLayer:
    """The sub-layer rank r runs when a B = 1 layer is split by kv head."""
    g0, g1 = kv_head_slice(params.heads_kv, world, rank)
    return SubLayer(params, g0, g1)


def max_over_ranks(value: float, group=None) -> float:
    """Maximum of a per-rank float over the process group (identity when not initialised)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    backend = dist.get_backend(group)
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else torch.device("cpu")
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
