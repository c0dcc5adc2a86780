"""Replica weight prefetch and replica gradient reduction on the GPU against
the oracle, on the VMM-aliased [E+B, H, Hp] views (the fp8 workload's sizes:
R=16, E=128, B=8, H=4096, Hp=1536) and on small views."""
import numpy as np
import pytest
import torch

import oracle
from dispatch_moonep_plan_b200 import workloads as wl
from gpu_helpers import me

pytestmark = pytest.mark.gpu


def _plan(cfgd, seed=0, rule=0):
    m = me()
    cfg = m.config_from(cfgd, rule)
    idx, _ = wl.routing(cfgd, seed=seed)
    bufs = m.PlanBuffers(cfg)
    m.plan(cfg, torch.from_numpy(idx).cuda(), bufs)
    o = oracle.plan(cfgd["R"], cfgd["S"], cfgd["E"], cfgd["K"], cfgd["B"], idx, rule=rule)
    h = bufs.host()
    assert h["status"] == o["status"] == 0
    assert np.array_equal(h["slot_expert"], o["slot_expert"])
    return cfg, bufs, o


def test_views_alias_home_rows():
    m = me()
    cfgd = wl.cfg_with("fp8", R=4, E=8, B=2, H=1024, Hp=1024, S=64)
    cfg = m.config_from(cfgd)
    wv = m.WeightViews(cfg, elem_bytes=2)
    try:
        v0 = m.weight_view_tensor(wv, 0, cfg, torch.bfloat16)
        v3 = m.weight_view_tensor(wv, 3, cfg, torch.bfloat16)
        v0[5].fill_(1.5)
        v3[cfg.E + 1].fill_(-2.0)
        torch.cuda.synchronize()
        assert bool((v3[5] == 1.5).all())           # home rows are shared
        assert not bool((v0[cfg.E + 1] == -2.0).any())  # slots are private
    finally:
        wv.close()


@pytest.mark.parametrize("full", [False, True])
def test_prefetch_and_grad_reduce(full):
    m = me()
    cfgd = wl.WORKLOADS["fp8"] if full else wl.cfg_with("fp8", R=4, S=512, E=16, B=4, H=1024,
                                                       Hp=1024, alpha=1.5)
    cfg, bufs, o = _plan(cfgd)
    R, E, B, H, Hp = cfg.R, cfg.E, cfg.B, cfg.H, cfg.Hp
    se = o["slot_expert"]
    assert (se >= 0).any()

    # ---- prefetch (bf16 weights) ----
    wv = m.WeightViews(cfg, elem_bytes=2)
    try:
        views = [m.weight_view_tensor(wv, r, cfg, torch.bfloat16) for r in range(R)]
        g = torch.Generator(device="cuda").manual_seed(5)
        views[0][:E].copy_(torch.randn((E, H, Hp), generator=g, device="cuda")
                           .to(torch.bfloat16))
        for r in range(R):
            views[r][E:].fill_(0)
        torch.cuda.synchronize()
        m.prefetch(cfg, bufs, wv.ptrs, elem_bytes=2)
        torch.cuda.synchronize()
        for r in range(R):
            for j in range(B):
                e = int(se[r, j])
                if e >= 0:
                    assert torch.equal(views[r][E + j].view(torch.int16),
                                       views[0][e].view(torch.int16)), (r, j, e)
                else:
                    assert not bool(views[r][E + j].view(torch.int16).any())
        # oracle on a sampled column set
        cols = torch.from_numpy(np.random.default_rng(0).choice(H * Hp, 4096, replace=False)).cuda()
        home = np.stack([views[0][e].reshape(-1)[cols].view(torch.int16).cpu().numpy()
                         for e in range(E)]).view(np.uint16)
        slots = np.zeros((R, B, cols.numel()), np.uint16)
        oracle.prefetch(R, B, se, home, slots)
        got = np.stack([np.stack([views[r][E + j].reshape(-1)[cols].view(torch.int16).cpu()
                                  .numpy() for j in range(B)]) for r in range(R)]).view(np.uint16)
        assert np.array_equal(got, slots)
        del views
    finally:
        wv.close()

    # ---- grad-reduce (fp32 grads) ----
    gv = m.WeightViews(cfg, elem_bytes=4)
    try:
        views = [m.weight_view_tensor(gv, r, cfg, torch.float32) for r in range(R)]
        g = torch.Generator(device="cuda").manual_seed(9)
        views[0][:E].copy_(torch.randn((E, H, Hp), generator=g, device="cuda"))
        for r in range(R):
            views[r][E:].copy_(torch.randn((B, H, Hp), generator=g, device="cuda"))
        torch.cuda.synchronize()
        cols = torch.from_numpy(np.random.default_rng(1).choice(H * Hp, 4096, replace=False)).cuda()
        home0 = np.stack([views[0][e].reshape(-1)[cols].cpu().numpy() for e in range(E)])
        slots0 = np.stack([np.stack([views[r][E + j].reshape(-1)[cols].cpu().numpy()
                                     for j in range(B)]) for r in range(R)])
        # full-size expectation with torch binary32 adds in the same order
        expect = {}
        for e in sorted(set(int(v) for v in se.reshape(-1) if v >= 0)):
            acc = views[0][e].clone()
            for r in range(R):
                for j in range(B):
                    if int(se[r, j]) == e:
                        acc = acc + views[r][E + j]
            expect[e] = acc
        m.grad_reduce(cfg, bufs, gv.ptrs)
        torch.cuda.synchronize()
        oracle.grad_reduce(R, B, E, se, home0, slots0)
        got = np.stack([views[0][e].reshape(-1)[cols].cpu().numpy() for e in range(E)])
        assert np.array_equal(got.view(np.uint32), home0.view(np.uint32))
        for e, acc in expect.items():
            assert torch.equal(views[0][e].view(torch.int32), acc.view(torch.int32)), e
        del views, expect
    finally:
        gv.close()
