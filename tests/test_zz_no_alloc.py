"""moonep_plan_noalloc, the planner for callers that cannot give it a
workspace buffer (a plugin whose host framework owns all device memory, a
serving loop that must not allocate once it runs): it must produce exactly
what moonep_plan produces, call after call, although every call reuses the
same static scratch array inside the library.

Collected last on purpose (file name), so that a run stopping at its first
failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from dispatch_moonep_plan_b200 import workloads as wl
from gpu_helpers import compare_plans

pytestmark = pytest.mark.gpu

KEYS = ("status", "fail_rank", "fail_slots", "max_count", "maxvio", "expert_count",
        "rank_load", "slot_expert", "cu_seqlens", "dst_row", "src_of_row")


def _plan_both(m, cfgd, seed, rule, alpha=None):
    cfg = m.config_from(cfgd, rule)
    idx, _ = wl.routing(cfgd, seed=seed, alpha=alpha)
    idx_d = torch.from_numpy(idx).cuda()
    ref = m.PlanBuffers(cfg)
    m.plan(cfg, idx_d, ref)
    got = m.PlanBuffers(cfg)
    got.c.workspace = None  # the allocation-free call must not need one
    got.c.workspace_bytes = 0
    stream = torch.cuda.current_stream()
    rc = m.lib.moonep_plan_noalloc(ctypes.byref(cfg), ctypes.c_void_p(idx_d.data_ptr()),
                                   ctypes.byref(got.c), ctypes.c_void_p(stream.cuda_stream))
    assert rc == m.OK, m.lib.moonep_last_error()
    torch.cuda.synchronize()
    # the plan stands on its own against the CPU oracle, as well as against
    # the workspace planner
    o = oracle.plan(cfgd["R"], cfgd["S"], cfgd["E"], cfgd["K"], cfgd["B"], idx, rule=rule)
    compare_plans(got.host(), o)
    return ref.host(), got.host()


def _same(ref, got):
    # plans are integer results: the bar is bit-exact
    for k in KEYS:
        if ref["status"] == 3 and k in ("slot_expert", "cu_seqlens", "dst_row", "src_of_row"):
            continue  # undefined after a failed plan
        a, b = ref[k], got[k]
        if isinstance(a, np.ndarray):
            assert np.array_equal(a, b), k
        else:
            assert a == b, k


def test_noalloc_matches_plan_on_consecutive_calls():
    from dispatch_moonep_plan_b200 import moonep as m
    # first call: a large E (256) leaves its tables in the shared array;
    # the second call, with a smaller E (64) and another routing, must not be
    # affected by them; a third call fails the slot budget like moonep_plan
    r1, g1 = _plan_both(m, wl.WORKLOADS["zipf"], seed=3, rule=1, alpha=1.0)
    _same(r1, g1)
    assert r1["status"] == 0
    r2, g2 = _plan_both(m, wl.WORKLOADS["uniform"], seed=4, rule=0)
    _same(r2, g2)
    assert r2["status"] == 0
    r3, g3 = _plan_both(m, wl.WORKLOADS["zipf"], seed=0, rule=0, alpha=1.5)
    _same(r3, g3)
    assert r3["status"] == m.STATUS_SLOT_BUDGET


def test_noalloc_at_its_largest_E():
    """E = MOONEP_NOALLOC_MAX_E fills the static scratch to its last word
    (per-block tables of E columns for every planner block); E = 384 is the
    hot-expert workload's expert count.  Both bit-exact, twice in a row."""
    from dispatch_moonep_plan_b200 import moonep as m
    assert m.NOALLOC_MAX_E == 512
    big = dict(name="noalloc512", R=4, S=512, E=512, K=4, B=16, H=64, Hp=0, routing="zipf",
               alpha=1.0, payload="bf16")
    mid = dict(big, name="noalloc384", R=32, S=256, E=384, K=8, B=16)
    for cfgd, rule in ((big, 2), (mid, 1), (big, 0)):
        r, g = _plan_both(m, cfgd, seed=5, rule=rule)
        _same(r, g)


def test_noalloc_rejects_E_above_its_limit():
    from dispatch_moonep_plan_b200 import moonep as m
    cfg = m.config(4, 8, 1024, 2, 2, 64)
    bufs = m.PlanBuffers(cfg)
    idx = torch.zeros((32, 2), dtype=torch.int32, device="cuda")
    with pytest.raises(m.MoonEPError, match="MOONEP_NOALLOC_MAX_E"):
        m.plan_noalloc(cfg, idx, bufs)
