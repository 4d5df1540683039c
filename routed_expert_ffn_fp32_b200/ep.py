"""Expert parallelism: one routed MoE layer spread over the ranks of a
torch.distributed group, each rank holding a contiguous range of the routed
experts.

The pages run the layer on one device ("antirez ds4 DeepSeek Metal
inference", section 技术深度解析: only the activated experts' weights are
read); this is the same layer scaled out over several GPUs.  Per call, on every
rank, with the token rows x replicated:

1. router, softmax, top-k and renormalisation (identical on every rank);
2. the stable bucket of all T*k (token, slot) pairs by expert;
3. the expert FFNs of the pairs whose expert this rank holds -- its slice of
   the global buckets -- and, on rank 0 only, the shared expert;
4. the float32 combine of those pairs (moe_combine_range);
5. one all-reduce (sum) of the [T, H] float32 partial outputs;
6. rounding to bf16.

Steps 1-4 and 6 are the library's CUDA kernels through the C ABI (``lib``,
the ctypes binding); step 5 is the group's collective (NCCL over NVLink on
GPUs).  The sum over ranks adds float32 partial outputs, so the result equals
the single-device layer up to float32 rounding of that sum.
"""
from __future__ import annotations

import contextlib
import dataclasses

import torch

from . import moe

#: shard boundaries fall on multiples of this many experts, so the offsets
#: view a rank passes to the C ABI stays 16-byte aligned
ALIGN = 4


def expert_range(E: int, world: int, rank: int) -> tuple[int, int]:
    """[e_begin, e_end) of the routed experts rank ``rank`` of ``world`` holds:
    contiguous ranges whose boundaries are multiples of ALIGN, as equal as
    that allows (the last ranks may hold fewer, or none when E < ALIGN *
    world)."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    units = (E + ALIGN - 1) // ALIGN
    base, rem = divmod(units, world)
    u0 = rank * base + min(rank, rem)
    u1 = u0 + base + (1 if rank < rem else 0)
    return min(E, u0 * ALIGN), min(E, u1 * ALIGN)


@dataclasses.dataclass
class ExpertShard:
    """The experts one rank holds: routed experts [e_begin, e_end) (device
    tensors of those experts only) and, on the rank that runs it, the shared
    expert."""
    e_begin: int
    e_end: int
    experts: "moe.Experts | None"
    shared: "moe.Experts | None"

    @classmethod
    def from_full(cls, experts: "moe.Experts", shared, world: int, rank: int,
                  shared_rank: int = 0) -> "ExpertShard":
        """The shard of rank ``rank`` cut from a full set of experts (views)."""
        e0, e1 = expert_range(experts.n_experts, world, rank)
        local = None
        if e1 > e0:
            local = moe.Experts(**{f: getattr(experts, f)[e0:e1] for f in
                                   ("gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s")})
        return cls(e0, e1, local, shared if rank == shared_rank else None)


def _on(stream):
    """torch's current stream set to ``stream`` (when given), so the scratch
    tensors below are allocated, and freed, in the order of the library calls
    that use them."""
    return torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()


def ep_partial(x, w_router, bias, shard: ExpertShard, shape, ws, path=moe.MOE_PATH_AUTO,
               precision=moe.MOE_ACT_EXACT, stream=None, lib=moe):
    """Steps 1-4 on this rank: the float32 [T, H] partial output of the pairs
    whose expert this rank holds (plus the shared expert on its rank), and the
    routing (topk_idx, topk_w).  ``ws`` must cover moe_workspace_bytes of the
    full shape and of the local one (see ep_workspace_bytes)."""
    with _on(stream):
        return _ep_partial(x, w_router, bias, shard, shape, ws, path, precision, stream, lib)


def _ep_partial(x, w_router, bias, shard, shape, ws, path, precision, stream, lib):
    T, H, I, E, k = shape.T, shape.H, shape.I, shape.E, shape.k
    dev = x.device
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    w = torch.empty((T, k), dtype=torch.float32, device=dev)
    lib.moe_route_topk(x, w_router, bias, shape, idx, w, ws, stream=stream)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    entries = torch.empty(T * k, dtype=torch.int32, device=dev)
    lib.moe_bucket(idx, shape, counts, offsets, entries, ws, stream=stream)
    has_shared = shard.shared is not None
    partial = torch.empty((T * k + (T if has_shared else 0), H), dtype=torch.float32, device=dev)
    e0, e1 = shard.e_begin, shard.e_end
    if e1 > e0:
        # this rank's experts, their bucket starts (an aligned view of the
        # offsets) and the global entries; k keeps the full pair layout
        local_shape = moe.shape_of(T, H, I, e1 - e0, k)
        lib.moe_expert_ffn_mxfp4(shard.experts, shard.shared, x, offsets[e0:e1 + 1], entries,
                                 local_shape, partial, ws, path, precision, stream=stream)
    elif has_shared:
        raise ValueError("the shared expert must sit on a rank that holds routed experts")
    y32 = torch.empty((T, H), dtype=torch.float32, device=dev)
    lib.moe_combine_range(partial, w, idx, e0, e1, shape, has_shared, y32, stream=stream)
    return y32, idx, w


def ep_finish(y32, y, stream=None, lib=moe):
    """Step 6: the summed float32 output -> bf16 bits in y."""
    lib.moe_round_bf16(y32, y, stream=stream)


def ep_layer_forward(x, w_router, bias, shard: ExpertShard, shape, y, ws, group=None,
                     path=moe.MOE_PATH_AUTO, precision=moe.MOE_ACT_EXACT, stream=None, lib=moe,
                     dist=None):
    """The whole layer over an expert-parallel group: every rank calls it with
    the same x, router and shape and its own shard; every rank gets y."""
    if dist is None:
        import torch.distributed as dist
    y32, idx, w = ep_partial(x, w_router, bias, shard, shape, ws, path, precision, stream, lib)
    if dist.is_initialized() and dist.get_world_size(group) > 1:
        # the collective orders itself after the work of torch's current
        # stream: make it the stream the library calls ran on
        with _on(stream if y32.is_cuda else None):
            dist.all_reduce(y32, op=dist.ReduceOp.SUM, group=group)
    ep_finish(y32, y, stream, lib)
    return idx, w


def ep_workspace_bytes(shape, shard: ExpertShard, path=moe.MOE_PATH_AUTO,
                       precision=moe.MOE_ACT_EXACT, lib=moe) -> int:
    """Workspace bytes one rank's ep_layer_forward needs."""
    full = lib.moe_workspace_bytes(shape, moe.MOE_PATH_GEMV, moe.MOE_ACT_EXACT, False)
    n_local = shard.e_end - shard.e_begin
    local = 0
    if n_local > 0:
        ls = moe.shape_of(shape.T, shape.H, shape.I, n_local, shape.k)
        local = lib.moe_workspace_bytes(ls, path, precision, shard.shared is not None)
    return max(full, local)
