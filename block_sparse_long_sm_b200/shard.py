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
