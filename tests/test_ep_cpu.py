"""Expert parallelism on the CPU: the shard ranges, and the orchestration of
ep_layer_forward over two and four gloo ranks on 127.0.0.1 (with four, one
rank holds no expert).

The per-rank compute steps are a CPU stand-in built from the fp64 oracle
(test code only, passed as ``lib``): this checks the host logic of the
expert-parallel layer -- which experts a rank holds, the slice of the
buckets it runs, the shared expert on one rank, the range-restricted combine
and the all-reduce -- against the single-device oracle.  The CUDA kernels of
the same steps are checked on the GPU (tests/test_gpu_ep.py).
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_expert_ranges_cover_every_expert_once():
    from routed_expert_ffn_fp32_b200 import ep
    for E in (1, 3, 4, 8, 64, 100, 256, 1024):
        for world in (1, 2, 3, 4, 8, 16):
            seen = []
            for r in range(world):
                e0, e1 = ep.expert_range(E, world, r)
                assert 0 <= e0 <= e1 <= E
                assert e0 % ep.ALIGN == 0 or e0 == e1
                seen += list(range(e0, e1))
            assert seen == list(range(E)), (E, world)
            sizes = [ep.expert_range(E, world, r)[1] - ep.expert_range(E, world, r)[0]
                     for r in range(world)]
            assert max(sizes) - min(sizes) <= ep.ALIGN or E < ep.ALIGN * world
    with pytest.raises(ValueError):
        ep.expert_range(8, 2, 2)


class CpuSteps:
    """The C-ABI steps ep_layer_forward calls, on CPU tensors, from the fp64
    oracle (a stand-in for the CUDA library in this host-logic test)."""

    FIELDS = ("gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s")

    def __init__(self, O):
        self.O = O

    def _x(self, x):
        return self.O.bf16_bits_to_f64(x.numpy().view(np.uint16))

    def moe_route_topk(self, x, w_router, bias, shape, idx, w, ws, logits_out=None, stream=None):
        logits = self.O.router_logits(self._x(x), w_router.numpy(),
                                      None if bias is None else bias.numpy())
        i, ww = self.O.route_topk(logits, shape.k)
        idx.copy_(torch.from_numpy(i))
        w.copy_(torch.from_numpy(ww.astype(np.float32)))

    def moe_bucket(self, idx, shape, counts, offsets, entries, ws, stream=None):
        c, o, e = self.O.bucket_by_expert(idx.numpy(), shape.E)
        counts.copy_(torch.from_numpy(c))
        offsets.copy_(torch.from_numpy(o))
        entries.copy_(torch.from_numpy(e))

    def moe_expert_ffn_mxfp4(self, experts, shared, x, offsets, entries, shape, partial, ws,
                             path, precision, stream=None):
        O, k, T = self.O, shape.k, shape.T
        xf = self._x(x)
        off, ent = offsets.numpy(), entries.numpy()
        ex = {f: getattr(experts, f).numpy() for f in self.FIELDS}
        assert ex["gate_q"].shape[0] == shape.E == off.size - 1
        for e in range(shape.E):
            rows = ent[off[e]:off[e + 1]]
            if rows.size:
                Wg, Wu, Wd = O.decode_expert(ex, e, shape.H, shape.I)
                partial[torch.from_numpy(rows.astype(np.int64))] = torch.from_numpy(
                    O.expert_ffn(Wg, Wu, Wd, xf[rows // k]).astype(np.float32))
        if shared is not None:
            sh = {f: getattr(shared, f).numpy() for f in self.FIELDS}
            Wg, Wu, Wd = O.decode_expert(sh, 0, shape.H, shape.I)
            partial[T * k:] = torch.from_numpy(O.expert_ffn(Wg, Wu, Wd, xf).astype(np.float32))

    def moe_combine_range(self, partial, w, idx, e0, e1, shape, has_shared, y32, stream=None):
        T, k = shape.T, shape.k
        p, wn, ix = partial.numpy(), w.numpy(), idx.numpy()
        out = np.zeros((T, shape.H), np.float32)
        for t in range(T):
            for j in range(k):
                if e0 <= ix[t, j] < e1:
                    out[t] += wn[t, j] * p[t * k + j]
            if has_shared:
                out[t] += p[T * k + t]
        y32.copy_(torch.from_numpy(out))

    def moe_round_bf16(self, y32, y, stream=None):
        bits = self.O.f64_to_bf16_bits(y32.numpy().astype(np.float64))
        y.copy_(torch.from_numpy(bits.view(np.int16)))

    def moe_workspace_bytes(self, *a, **k):
        return 256


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle as O
    from routed_expert_ffn_fp32_b200 import ep, moe, synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        cfg = synth.LayerConfig("ep", 128, 64, 12, 3, 6, 0.05, 1.0, True)
        L = synth.layer(cfg, 41)
        full = moe.Experts(**{f: torch.from_numpy(L["experts"][f]) for f in CpuSteps.FIELDS})
        shared = moe.Experts(**{f: torch.from_numpy(L["shared"][f]) for f in CpuSteps.FIELDS})
        shard = ep.ExpertShard.from_full(full, shared, world, rank)
        x = torch.from_numpy(L["x"].view(np.int16))
        shape = moe.shape_of(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k)
        y = torch.empty((cfg.T, cfg.H), dtype=torch.int16)
        idx, w = ep.ep_layer_forward(x, torch.from_numpy(L["W_r"]), torch.from_numpy(L["bias"]),
                                     shard, shape, y, ws=None, lib=CpuSteps(O), dist=dist)
        q.put((rank, shard.e_begin, shard.e_end, y.numpy().view(np.uint16).copy(),
               idx.numpy().copy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,ranges", [
    (2, [(0, 8), (8, 12)]),
    # the last rank holds no expert: its partial is zero, the sum unchanged
    (4, [(0, 4), (4, 8), (8, 12), (12, 12)]),
])
def test_gloo_ranks_match_single_device_oracle(world, ranges):
    sys.path.insert(0, ROOT)
    import oracle as O
    from helpers import check_y
    from routed_expert_ffn_fp32_b200 import synth
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=240) for _ in range(world))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert [(r[1], r[2]) for r in res] == ranges
    cfg = synth.LayerConfig("ep", 128, 64, 12, 3, 6, 0.05, 1.0, True)
    L = synth.layer(cfg, 41)
    ref = O.layer_forward(L["x"], L["W_r"], L["bias"], L["experts"], L["shared"], cfg.k)
    for r in res:
        np.testing.assert_array_equal(r[4], ref["idx"])
        check_y(r[3], ref)
    # the experts of both shards were used
    assert (ref["idx"] >= 8).any() and (ref["idx"] < 8).any()
