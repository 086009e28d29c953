"""Tensor-parallel decode over a compressed KV cache.

The MLRA page ("moving the sum outside", first item) places the latent's
branches on different GPUs: each holds one branch of the cache plus the shared
rope key (1.5 d_h per token instead of MLA's 4.5 d_h, "key conclusions"),
attends it with every query head, and the branch outputs are summed only at
the end, by an all-reduce.  The GLA page splits the latent into groups that
serve disjoint query heads, so a group per GPU needs no reduction: the heads'
outputs are gathered (its deployment list runs GLA-2 with two-way tensor
parallelism and MLRA-4 with four-way).

A rank's shard is itself a decode problem the library covers: MLRA with
R / world branches (one for MLRA-4 on four GPUs), GLA with G / world groups
and the matching H / world heads, each with the shared rope key.  This module
slices a rank's inputs out of the full problem (the cache columns of its
branches or groups plus the rope key, its query slices), runs the library on
them, and assembles the result with one collective over the default process
group (NCCL between GPUs; any backend works).  Every rank computes MLRA branch
outputs in fp32 so the sum is rounded to the output type once, as on one GPU.
The arithmetic all happens in the library's kernels; this is data placement
and the collective.
"""

from __future__ import annotations

import numpy as np

from . import workloads as W


def units_per_rank(shape: W.Shape, world: int) -> int:
    """Branches (MLRA) or groups (GLA) each rank holds."""
    if shape.variant not in ("mlra", "gla"):
        raise ValueError(f"tensor parallelism splits MLRA branches or GLA groups, not {shape.variant}")
    if world < 1 or shape.num_kv % world:
        raise ValueError(f"{shape.num_kv} branches/groups do not split over {world} ranks")
    return shape.num_kv // world


def shard_shape(shape: W.Shape, world: int) -> W.Shape:
    """The decode problem one rank solves."""
    u = units_per_rank(shape, world)
    if shape.variant == "mlra":
        return shape.replace(num_kv=u, out_dtype="fp32")
    return shape.replace(num_kv=u, num_q_heads=shape.num_q_heads // world)


def shard_inputs(inputs: dict, rank: int, world: int) -> dict:
    """Rank `rank`'s inputs (numpy, as workloads.make_inputs returns them):
    the cache columns of its branches / groups followed by the rope key, and
    its query slices.  Block table, lengths and scale are shared."""
    s = inputs["shape"]
    u = units_per_rank(s, world)
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    dn, dr, nkv = s.d_nope, s.d_rope, s.num_kv
    lo, hi = rank * u * dn, (rank + 1) * u * dn
    kv = inputs["kv"]
    kv_r = np.ascontiguousarray(np.concatenate([kv[..., lo:hi], kv[..., nkv * dn:nkv * dn + dr]], axis=-1))
    if s.variant == "mlra":
        qn = np.ascontiguousarray(inputs["q_nope"][:, :, rank * u:(rank + 1) * u, :])
        qr = np.ascontiguousarray(inputs["q_rope"][:, :, rank * u:(rank + 1) * u, :])
    else:
        hr = s.num_q_heads // world
        qn = np.ascontiguousarray(inputs["q_nope"][:, rank * hr:(rank + 1) * hr, :])
        qr = np.ascontiguousarray(inputs["q_rope"][:, rank * hr:(rank + 1) * hr, :])
    out = dict(inputs)
    out.update(shape=shard_shape(s, world), kv=kv_r, q_nope=qn, q_rope=qr)
    return out


def library_compute(device):
    """Per-rank compute on the library (one decode call on `device`); returns
    (out, lse) as float64 numpy arrays."""

    def run(x):
        import torch

        from .device import DeviceProblem
        p = DeviceProblem(x, device)
        p.run()
        torch.cuda.synchronize(p.device)
        return p.results()

    return run


def assemble(variant: str, out_r, lse_r, group=None):
    """The collective step on torch tensors of one rank: MLRA sums the fp32
    branch outputs (all-reduce) and gathers the per-branch lse along the
    branch axis; GLA gathers heads.  Returns (out, lse) of the whole problem
    (MLRA out in fp32, to be rounded once by the caller)."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    if variant == "mlra":
        out = out_r.clone()
        dist.all_reduce(out, op=dist.ReduceOp.SUM, group=group)
        parts = [torch.empty_like(lse_r) for _ in range(world)]
        dist.all_gather(parts, lse_r.contiguous(), group=group)
        return out, torch.cat(parts, dim=-1)
    outs = [torch.empty_like(out_r) for _ in range(world)]
    lses = [torch.empty_like(lse_r) for _ in range(world)]
    dist.all_gather(outs, out_r.contiguous(), group=group)
    dist.all_gather(lses, lse_r.contiguous(), group=group)
    return torch.cat(outs, dim=1), torch.cat(lses, dim=1)


def tp_decode(inputs: dict, rank: int, world: int, compute=None, device=None, group=None):
    """Decode `inputs` with the branches / groups split over the `world`
    ranks of the default process group: this rank solves its shard with
    `compute` (default: the library on `device`) and the collective assembles
    the result.  Returns (out, lse) as float64 numpy arrays on every rank."""
    import torch

    compute = compute or library_compute(device)
    x = shard_inputs(inputs, rank, world)
    out_r, lse_r = compute(x)
    cpu = device is None or getattr(torch.device(device), "type", "cpu") == "cpu"
    dev = torch.device("cpu") if cpu else torch.device(device)
    dtype = torch.float64 if cpu else torch.float32
    out, lse = assemble(inputs["shape"].variant, torch.as_tensor(out_r, dtype=dtype, device=dev),
                        torch.as_tensor(lse_r, dtype=dtype, device=dev), group)
    return out.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def tp_decode_one_device(inputs: dict, world: int, device):
    """Every rank's shard solved in turn on one device and assembled with the
    same arithmetic as the collective (sum of branch outputs, or heads
    side by side): the single-GPU check of what each rank computes."""
    s = inputs["shape"]
    run = library_compute(device)
    outs, lses = zip(*(run(shard_inputs(inputs, r, world)) for r in range(world)))
    if s.variant == "mlra":
        return np.sum(outs, axis=0), np.concatenate(lses, axis=-1)
    return np.concatenate(outs, axis=1), np.concatenate(lses, axis=1)
