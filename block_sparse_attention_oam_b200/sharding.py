"""One prefill layer split across ranks by KV-head group, and the output gathered.

Every step of the path works within one (kv-head, its q-heads) group: pooling reduces
inside a head, a q-head's scores, budget, selection and attention use only its own
kv-head's keys and values.  So rank r of N takes kv-heads [r*Hkv/N, (r+1)*Hkv/N) and
their q-heads [r*Hq/N, (r+1)*Hq/N), and runs the whole path on them as a problem of its
own (local q-head h - q0 reads local kv-head (h - q0) / g, the same kv-head as before).
The only cross-rank step is after the path: one all-gather of the ranks' output heads.

This module is plumbing (slicing host tensors, torch.distributed collectives); every
step of the path still runs in libstem's kernels on each rank.
"""
from __future__ import annotations

import dataclasses

import torch

from . import workloads as W


@dataclasses.dataclass(frozen=True)
class HeadShard:
    rank: int
    world: int
    q0: int        # first q-head of this rank
    q1: int        # one past its last q-head
    k0: int        # first kv-head
    k1: int

    @property
    def num_q_heads(self) -> int:
        return self.q1 - self.q0

    @property
    def num_kv_heads(self) -> int:
        return self.k1 - self.k0


def head_shard(num_q_heads: int, num_kv_heads: int, world: int, rank: int) -> HeadShard:
    """Rank `rank`'s contiguous share of the kv-heads and of their q-heads."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of {world}")
    if num_kv_heads % world != 0:
        raise ValueError(f"{num_kv_heads} kv-heads do not split evenly over {world} ranks")
    if num_q_heads % num_kv_heads != 0:
        raise ValueError(f"{num_q_heads} q-heads are not a multiple of {num_kv_heads} kv-heads")
    kpr = num_kv_heads // world
    g = num_q_heads // num_kv_heads
    return HeadShard(rank, world, rank * kpr * g, (rank + 1) * kpr * g, rank * kpr, (rank + 1) * kpr)


def shard_inputs(inp: W.Inputs, sh: HeadShard) -> W.Inputs:
    """The shard's heads of a workload's inputs, as contiguous tensors (the FP8 per-tensor
    scales stay those of the whole tensors, so every rank dequantises like one GPU would)."""
    wl = inp.wl.with_(num_q_heads=sh.num_q_heads, num_kv_heads=sh.num_kv_heads)
    out = W.Inputs(wl, inp.cu_seqlens, inp.q[:, sh.q0:sh.q1].contiguous(), inp.k[:, sh.k0:sh.k1].contiguous(),
                   inp.v[:, sh.k0:sh.k1].contiguous(), inp.q_scale, inp.k_scale, inp.v_scale)
    if inp.k_cache is not None:
        out.k_cache = inp.k_cache[:, :, sh.k0:sh.k1].contiguous()
        out.v_cache = inp.v_cache[:, :, sh.k0:sh.k1].contiguous()
        out.block_table = inp.block_table
    return out


def gather_heads(o_local: torch.Tensor, dist, out: torch.Tensor | None = None) -> torch.Tensor:
    """All-gather every rank's output heads: o_local [T, Hq/N, d] -> [N, T, Hq/N, d], rank r's
    heads at index r (NCCL: one all_gather_into_tensor into `out`; other backends: all_gather)."""
    world = dist.get_world_size()
    if out is None:
        out = torch.empty((world,) + tuple(o_local.shape), dtype=o_local.dtype, device=o_local.device)
    if dist.get_backend() == "nccl":
        dist.all_gather_into_tensor(out, o_local.contiguous())
    else:
        dist.all_gather(list(out.unbind(0)), o_local.contiguous())
    return out


def token_major(gathered: torch.Tensor) -> torch.Tensor:
    """[N, T, Hq/N, d] gathered heads as the [T, Hq, d] view of one GPU's output
    (a strided view: global q-head r*Hq/N + j is rank r's local head j)."""
    n, t, hl, d = gathered.shape
    return gathered.permute(1, 0, 2, 3).reshape(t, n * hl, d)
