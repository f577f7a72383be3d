"""Host-side plumbing for running the path on several GPUs of one node.

Two ways to shard the routed-attention step:

* samples (the default): samples are independent and routing is per sample,
  so each rank runs whole steps on its own samples and the ranks meet only at
  the barriers around the timed region and in one max-reduction of the
  elapsed time (weak scaling, no data-path collective);
* heads of one sample: attention heads are independent (Eq. (2)-(3) act per
  head), so rank r takes the contiguous head block ``head_range(H, G, r)``
  of Q/K/V and routes the sample's full u itself (routing is deterministic,
  so every rank gets the same lists); the uncertainty head's token rows are
  split the same way, and its output -- which every rank needs to route the
  next step -- is the one real exchange, an all-gather of equal slices
  (``all_gather_equal``), as is the optional all-gather of the output along
  heads.
"""
import dataclasses
import os
from datetime import timedelta

from . import workloads as W


@dataclasses.dataclass(frozen=True)
class RankInfo:
    rank: int
    local_rank: int
    world: int


def rank_info() -> RankInfo:
    return RankInfo(int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
                    int(os.environ.get("WORLD_SIZE", "1")))


def init(backend: str, info: RankInfo, timeout_s: float = 120.0):
    """Joins the process group (no-op for a single rank)."""
    import torch.distributed as dist
    if info.world == 1 or dist.is_initialized():
        return
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", "29517")
    kw = {}
    if backend == "nccl":
        import torch
        kw["device_id"] = torch.device("cuda", info.local_rank)
    dist.init_process_group(backend, rank=info.rank, world_size=info.world,
                            timeout=timedelta(seconds=timeout_s), **kw)


def rank_workload(w: W.Workload, rank: int) -> W.Workload:
    """The independent sample(s) rank `rank` processes: same shape, own seeds."""
    if rank == 0:
        return w
    off = 1000 * rank
    return dataclasses.replace(
        w, name="%s@rank%d" % (w.name, rank), qkv_seed=w.qkv_seed + off,
        u_seeds=tuple(s + off for s in w.u_seeds) if w.u_seeds else (w.qkv_seed + off + 1,),
        x_seed=w.x_seed + off)


def head_range(H: int, world: int, rank: int):
    """Contiguous head block [lo, hi) of rank `rank` when one sample's heads are split."""
    base, extra = divmod(H, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def row_range(n: int, world: int, rank: int):
    """Contiguous block [lo, hi) of n rows (tokens) for rank `rank`; equal blocks
    when world divides n (what ``all_gather_equal`` needs)."""
    return head_range(n, world, rank)


def all_gather_equal(local, info: RankInfo):
    """The ranks' equal-sized tensors concatenated in rank order, as one flat
    tensor on local's device (local itself, flattened, for one rank)."""
    if info.world == 1:
        return local.reshape(-1)
    import torch
    import torch.distributed as dist
    flat = local.contiguous().reshape(-1)
    out = torch.empty(info.world * flat.numel(), dtype=flat.dtype, device=flat.device)
    dist.all_gather_into_tensor(out, flat)
    return out


def max_over_ranks(x: float, info: RankInfo, device=None) -> float:
    """The largest x over all ranks (x itself for one rank)."""
    if info.world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(info: RankInfo, device=None):
    if info.world == 1:
        return
    import torch.distributed as dist
    if device is not None:
        dist.barrier(device_ids=[device.index])
    else:
        dist.barrier()
