"""Slot bank (routed experts in pinned host memory, a bounded device bank of
them) against the fp64 oracle.

A sequence of banked layer calls with different token batches and a bank
smaller than the expert count, so experts are evicted and reloaded: every
call's output matches the oracle (routing bit-exact, the largest per-token
relative L2 within 2e-3), and the bank's hit / miss / eviction counts match a
model of its least-recently-used rule written here from its definition.
"""
import numpy as np
import pytest
import torch

import oracle as O
from routed_expert_ffn_fp32_b200 import build, moe, synth

from helpers import bits_np, check_routing, check_y, to_dev_bits

pytestmark = pytest.mark.gpu

FIELDS = ("gate_q", "gate_s", "up_q", "up_s", "down_q", "down_s")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    moe.load_library()


class LruModel:
    """Slots keep the call counter of their last use (-1: never); a call's
    experts already resident are hits; each missing expert, in order of first
    appearance, takes the slot with the smallest counter among those the call
    does not use (the lowest index among equals)."""

    def __init__(self, n_slots):
        self.last = [-1] * n_slots
        self.owner = [-1] * n_slots
        self.clock = 0
        self.hits = self.misses = self.evictions = 0

    def acquire(self, ids):
        self.clock += 1
        order = list(dict.fromkeys(int(e) for e in ids))
        need = []
        for e in order:
            if e in self.owner:
                self.last[self.owner.index(e)] = self.clock
                self.hits += 1
            else:
                need.append(e)
        for e in need:
            cand = [s for s in range(len(self.last)) if self.last[s] != self.clock]
            v = min(cand, key=lambda s: (self.last[s], s))
            if self.owner[v] >= 0:
                self.evictions += 1
            self.owner[v] = e
            self.last[v] = self.clock
            self.misses += 1


@pytest.mark.parametrize("cfg,T,n_slots,calls", [
    (synth.LayerConfig("bank", 256, 128, 16, 2, 3, 0.05, None, True), 3, 6, 8),
    (synth.DECODE64, 5, 16, 6),
])
def test_banked_layer_matches_oracle_and_lru(cfg, T, n_slots, calls):
    L = synth.layer(cfg, 61, T)
    host = moe.Experts(**{f: torch.from_numpy(L["experts"][f]) for f in FIELDS})
    shared = None if L["shared"] is None else moe.Experts.from_numpy(L["shared"])
    bank = moe.SlotBank(host, cfg.H, cfg.I, n_slots)
    W_r = torch.from_numpy(L["W_r"]).cuda()
    bias = None if L["bias"] is None else torch.from_numpy(L["bias"]).cuda()
    shape = moe.shape_of(T, cfg.H, cfg.I, cfg.E, cfg.k)
    ws = moe.banked_workspace(shape, n_slots, has_shared=shared is not None)
    model = LruModel(n_slots)
    y = torch.empty((T, cfg.H), dtype=torch.int16, device="cuda")
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, cfg.k), dtype=torch.float32, device="cuda")
    for c in range(calls):
        xb = synth.activations(cfg, 700 + c, T)
        moe.moe_layer_forward_banked(to_dev_bits(xb), W_r, bias, bank, shared, shape, y, ws, idx, w)
        torch.cuda.synchronize()
        assert moe.moe_get_error(ws) == 0
        ref = O.layer_forward(xb, L["W_r"], L["bias"], L["experts"], L["shared"], cfg.k)
        check_routing({"x": xb, "W_r": L["W_r"], "bias": L["bias"]}, ref, idx.cpu().numpy(),
                      w.cpu().numpy(), cfg.k, cfg.H)
        check_y(bits_np(y), ref)
        model.acquire(idx.cpu().numpy().reshape(-1))
        assert bank.stats() == (model.hits, model.misses, model.evictions), c
    assert model.evictions > 0          # the bank was too small to keep everything
    bank.close()


def test_bank_rejects_more_experts_than_slots():
    cfg = synth.LayerConfig("bank", 256, 128, 16, 2, 4, 0.05, None, False)
    L = synth.layer(cfg, 62)
    host = moe.Experts(**{f: torch.from_numpy(L["experts"][f]) for f in FIELDS})
    bank = moe.SlotBank(host, cfg.H, cfg.I, 3)
    with pytest.raises(moe.MoeError) as ei:
        bank.acquire([0, 1, 2, 3])
    assert ei.value.status == moe.MOE_ERR_WORKSPACE
    assert bank.acquire([5, 5, 7]) == [bank.acquire([5])[0]] * 2 + [bank.acquire([7])[0]]
    bank.close()
