"""Edge cases and failure reporting on the GPU, through the C ABI: degenerate
sizes, ragged rows, the largest E and R the planner takes, failed plans that
must move no data, a bad expert index, and a device wait that runs out."""
import numpy as np
import pytest
import torch

import oracle
from dispatch_moonep_plan_b200 import workloads as wl
from gpu_helpers import bits16, compare_plans, gpu_path, me

pytestmark = pytest.mark.gpu


def _cfg(R, S, E, K, B, H, routing="zipf", alpha=1.0, payload="bf16"):
    return dict(name="edge", R=R, S=S, E=E, K=K, B=B, H=H, Hp=0, routing=routing,
                alpha=alpha, payload=payload)


def _full_check(cfgd, idx, w, seed=0, rule=0, expert="scale"):
    x = wl.hidden(cfgd["R"] * cfgd["S"], cfgd["H"], seed=seed).cuda()
    out = gpu_path(cfgd, idx, w, x, rule=rule, expert=expert)
    o = oracle.plan(cfgd["R"], cfgd["S"], cfgd["E"], cfgd["K"], cfgd["B"], idx, rule=rule)
    compare_plans(out["bufs"].host(), o)
    if o["status"] == 0:
        T = idx.shape[0]
        y, _ = oracle.path_tokens(cfgd, bits16(x), w, o, np.arange(T), expert=expert,
                                  payload=cfgd["payload"])
        assert np.array_equal(bits16(out["y"]), y)
    return out, o


@pytest.mark.parametrize("shape", [
    (1, 1, 1, 1, 0, 8),        # one rank, one token, one expert
    (1, 7, 4, 3, 2, 24),       # single rank: never any overflow
    (4, 1, 4, 1, 1, 8),        # one token per rank, Er = 1
    (3, 5, 6, 6, 4, 136),      # K = E: every token picks every expert
    (2, 33, 8, 2, 3, 264),     # ragged: H/8 = 33 chunks, not a multiple of 32
    (5, 17, 10, 3, 5, 40),
])
def test_degenerate_and_ragged(shape):
    R, S, E, K, B, H = shape
    cfgd = _cfg(R, S, E, K, B, H)
    for seed in range(3):
        idx, w = wl.routing(cfgd, seed=seed)
        for rule in (0, 1, 2):
            _full_check(cfgd, idx, w, seed=seed, rule=rule)


@pytest.mark.parametrize("shape", [
    (2, 48, 16, 8, 8, 256),     # K = 8: the all-K-first combine with every pick slot used
    (2, 40, 16, 12, 8, 512),    # K = 12: the double-buffered combine and backward kernels
    (4, 16, 32, 32, 16, 64),    # K = 32 = the largest K, every token picks every expert
])
def test_many_picks_per_token(shape):
    """Above K = 8, combine and both backward kernels switch to the forms that
    keep two picks in flight; both sides of that switch, bit-exact."""
    R, S, E, K, B, H = shape
    cfgd = _cfg(R, S, E, K, B, H, alpha=0.5)
    for seed in range(2):
        idx, w = wl.routing(cfgd, seed=seed)
        for rule in (0, 2):
            _full_check(cfgd, idx, w, seed=seed, rule=rule, expert="scale")


@pytest.mark.parametrize("shape", [
    (2, 37, 8, 3, 4, 4096),     # 8 chunks of 512 per row, ragged token count
    (3, 50, 9, 8, 3, 4608),     # K = 8, 9 chunks
    (1, 5, 4, 1, 0, 4096),      # one rank, one pick per token, fewer tokens than warps
    (4, 23, 8, 5, 3, 7168),     # the hot workload's row length, K = 5
])
def test_combine_bulk_staged(shape):
    """Rows of at least 4096 elements (a multiple of 512) with K <= 8 take the
    combine that stages the rows in shared memory with bulk copies: every
    token against the oracle, bit for bit, under all rules and the scale
    expert."""
    R, S, E, K, B, H = shape
    cfgd = _cfg(R, S, E, K, B, H, alpha=1.2)
    for seed in range(2):
        idx, w = wl.routing(cfgd, seed=seed)
        for rule in (0, 1, 2):
            _full_check(cfgd, idx, w, seed=seed, rule=rule, expert="scale")


def test_largest_E_and_R():
    cfgd = _cfg(128, 16, 1024, 8, 16, 64, alpha=1.2)
    idx, w = wl.routing(cfgd, seed=0)
    for rule in (0, 1, 2):
        _full_check(cfgd, idx, w, rule=rule, expert="identity")


@pytest.mark.parametrize("R,S,E,K", [
    (8, 40000, 512, 8),  # 2.56 M picks: ranked by mask words; too many picks per
                         # block to keep in shared memory, so the walk reads and
                         # ranks them again in (t, k) order
    (8, 8192, 1024, 8),  # E = 1024 and 524 K picks: no room for the mask words
                         # (match.any) nor for the picks
])
def test_planner_picks_not_kept(R, S, E, K):
    cfgd = _cfg(R, S, E, K, 16, 64, alpha=0.8)
    idx, w = wl.routing(cfgd, seed=3)
    for rule in (0, 1, 2):  # rule 0 runs out of slots here; 1 and 2 place
        out, o = _full_check(cfgd, idx, w, rule=rule, expert="scale")
        assert (o["status"] == 0) == (rule > 0)


@pytest.mark.parametrize("alpha", [0.0, 3.0])
def test_planner_one_pick_per_token_few_experts(alpha):
    """K = 1 and E = 8 over 2.1 M picks: a row of 32 picks spans 32 tokens, so
    up to 32 lanes hold one expert (the mask words' worst case) in whole
    batches of rows, and the candidate expert keeps changing (alpha 0) or
    stays on the hot one (alpha 3)."""
    cfgd = _cfg(8, 262144, 8, 1, 8, 16, alpha=alpha)
    idx, _ = wl.routing(cfgd, seed=5)
    m = me()
    for rule in (1, 2):
        cfg = m.config_from(cfgd, rule)
        bufs = m.PlanBuffers(cfg)
        m.plan(cfg, torch.from_numpy(idx).cuda(), bufs)
        o = oracle.plan(cfgd["R"], cfgd["S"], cfgd["E"], cfgd["K"], cfgd["B"], idx, rule=rule)
        compare_plans(bufs.host(), o)


def test_duplicate_picks_and_all_to_one():
    cfgd = _cfg(4, 64, 8, 4, 8, 16)
    idx = np.full((256, 4), 5, np.int32)  # every pick on one expert
    w = np.full((256, 4), 0.25, np.float32)
    out, o = _full_check(cfgd, idx, w, rule=0)
    assert o["status"] == 0 and o["maxvio"] == 7.0


def test_round_robin_B0_balanced():
    cfgd = _cfg(4, 32, 16, 4, 0, 32, routing="round_robin")
    idx, w = wl.routing(cfgd)
    out, o = _full_check(cfgd, idx, w)
    assert o["status"] == 0


def test_slot_budget_moves_no_data():
    cfgd = _cfg(4, 64, 16, 2, 0, 64, alpha=2.0)  # B = 0 and skewed: must fail
    idx, w = wl.routing(cfgd, seed=0)
    x = wl.hidden(256, 64).cuda()
    out = gpu_path(cfgd, idx, w, x, expert="scale")
    g = out["bufs"].host()
    assert g["status"] == me().STATUS_SLOT_BUDGET
    o = oracle.plan(4, 64, 16, 2, 0, idx)
    compare_plans(g, o)
    assert not bool(out["recv"].any()) and not bool(out["eo"].any()) and not bool(out["y"].any())
    assert me().plan_status(out["bufs"])[:3] == [3, o["fail_rank"], o["fail_slots"]]


def test_bad_index_reported_and_no_data_moved():
    cfgd = _cfg(2, 8, 4, 2, 2, 16)
    idx, w = wl.routing(cfgd, seed=0)
    idx[5, 1] = 4  # == E
    x = wl.hidden(16, 16).cuda()
    out = gpu_path(cfgd, idx, w, x)
    assert me().plan_status(out["bufs"])[0] == me().STATUS_BAD_INDEX
    assert not bool(out["recv"].any()) and not bool(out["y"].any())
    idx[5, 1] = -3
    out = gpu_path(cfgd, idx, w, x)
    assert me().plan_status(out["bufs"])[0] == me().STATUS_BAD_INDEX


@pytest.fixture(scope="module")
def many_picks():
    cfgd = _cfg(8, 32768, 64, 8, 8, 16)  # 2.1 M picks: about 440 per warp
    idx, _ = wl.routing(cfgd, seed=1)
    return cfgd, idx


@pytest.mark.parametrize("q,bad", [(0, 64), (1000, -1), (777_777, 1 << 20), (2_097_151, -64)])
def test_bad_index_among_many_picks(many_picks, q, bad):
    """At this size every warp ranks whole batches of 8 rows (no per-row
    bounds checks) before its last, partial batch; an index outside [0, E) in
    either is still reported."""
    cfgd, idx = many_picks
    m = me()
    cfg = m.config_from(cfgd, 0)
    bufs = m.PlanBuffers(cfg)
    bad_idx = idx.copy()
    bad_idx.reshape(-1)[q] = bad
    m.plan(cfg, torch.from_numpy(bad_idx).cuda(), bufs)
    assert m.plan_status(bufs)[0] == m.STATUS_BAD_INDEX
    m.plan(cfg, torch.from_numpy(idx).cuda(), bufs)  # the same buffers, valid picks
    o = oracle.plan(cfgd["R"], cfgd["S"], cfgd["E"], cfgd["K"], cfgd["B"], idx)
    compare_plans(bufs.host(), o)


def test_wait_that_runs_out_reports_timeout():
    """The planner's first grid-wide wait is told to expect one block more
    than exists; it gives up after the (short) wait limit, the plan reports
    TIMEOUT, downstream kernels do nothing, and the context stays usable."""
    m = me()
    cfgd = _cfg(2, 64, 8, 2, 2, 32)
    idx, w = wl.routing(cfgd, seed=0)
    x = wl.hidden(128, 32).cuda()
    m.set_wait_limit_ns(20_000_000)
    m.debug_set_barrier_extra(1)
    try:
        out = gpu_path(cfgd, idx, w, x)
        assert m.plan_status(out["bufs"])[0] == m.STATUS_TIMEOUT
        assert not bool(out["recv"].any()) and not bool(out["y"].any())
    finally:
        m.debug_set_barrier_extra(0)
        m.set_wait_limit_ns(1_000_000_000)
    out, o = _full_check(cfgd, idx, w)
    assert o["status"] == 0


def test_invalid_arguments_rejected_before_launch():
    m = me()
    cfg = m.config(2, 8, 4, 2, 2, 100)  # H not a multiple of 8
    with pytest.raises(m.MoonEPError, match="multiple of 8"):
        m.sizes(cfg)
    cfg = m.config(2, 8, 4, 2, 2, 64, payload=m.PAYLOAD_FP8)  # fp8 needs H % 128 == 0
    with pytest.raises(m.MoonEPError, match="128"):
        m.sizes(cfg)
    cfg = m.config(2, 8, 4, 2, 2, 128)
    bufs = m.PlanBuffers(cfg)
    x = torch.zeros((16, 128), dtype=torch.bfloat16, device="cuda")
    recv = torch.zeros((32, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(m.MoonEPError, match="recv_scale"):
        m.dispatch(cfg, bufs, x, recv, recv_scale=torch.zeros(4, device="cuda"))
    with pytest.raises(m.MoonEPError, match="aligned"):
        m.dispatch(cfg, bufs, x.view(-1)[1:], recv)


@pytest.mark.parametrize("bad", [-1, 1 << 20])
def test_corrupted_plan_reported_as_internal(bad):
    """A plan whose dst_row (or slot map) the caller overwrote with an index
    outside the buffers: every kernel's range check skips or clamps the
    access and sets MOONEP_STATUS_INTERNAL instead of reporting OK.  The bad
    values are made on the host; no access leaves its buffer."""
    m = me()
    cfgd = wl.cfg_with("fp8", R=2, S=64, E=4, K=2, B=2, H=1024, Hp=1024, alpha=1.5,
                       payload="bf16")
    T, P, H = 128, 256, 1024
    idx, w = wl.routing(cfgd, seed=0)
    x = wl.hidden(T, H, seed=0).cuda()
    w_d = torch.from_numpy(w).cuda()
    idx_d = torch.from_numpy(idx).cuda()
    bad = bad if bad < 0 else P + bad

    def fresh(payload="bf16"):
        cfg = m.config_from(dict(cfgd, payload=payload))
        bufs = m.PlanBuffers(cfg)
        m.plan(cfg, idx_d, bufs)
        torch.cuda.synchronize()
        assert m.plan_status(bufs)[0] == m.STATUS_OK
        return cfg, bufs

    def corrupt_row(bufs):
        bufs.dst_row[37] = bad
        torch.cuda.synchronize()

    recv = torch.zeros((P, H), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((T, H), dtype=torch.bfloat16, device="cuda")
    calls = [
        lambda cfg, bufs: m.dispatch(cfg, bufs, x, recv),
        lambda cfg, bufs: m.combine(cfg, bufs, recv, w_d, y),
        lambda cfg, bufs: m.combine_backward(cfg, bufs, y, recv, w_d, torch.empty_like(recv),
                                             torch.empty_like(w_d)),
        lambda cfg, bufs: m.dispatch_backward(cfg, bufs, recv, torch.empty_like(y)),
    ]
    for call in calls:
        cfg, bufs = fresh()
        corrupt_row(bufs)
        call(cfg, bufs)
        assert m.plan_status(bufs)[0] == m.STATUS_INTERNAL
    # fp8 dispatch
    cfg, bufs = fresh("fp8")
    corrupt_row(bufs)
    q = torch.zeros((P, H), dtype=torch.uint8, device="cuda")
    sc = torch.zeros((P, H // 128), dtype=torch.float32, device="cuda")
    m.dispatch(cfg, bufs, x, q, sc)
    assert m.plan_status(bufs)[0] == m.STATUS_INTERNAL
    # a slot map entry >= E: prefetch and grad-reduce
    for kind in ("prefetch", "grad_reduce"):
        cfg, bufs = fresh()
        bufs.slot_expert[1] = cfg.E + (0 if bad < 0 else 7)
        torch.cuda.synchronize()
        eb = 2 if kind == "prefetch" else 4
        wv = m.WeightViews(cfg, elem_bytes=eb)
        try:
            if kind == "prefetch":
                m.prefetch(cfg, bufs, wv.ptrs, elem_bytes=2)
            else:
                m.grad_reduce(cfg, bufs, wv.ptrs)
            assert m.plan_status(bufs)[0] == m.STATUS_INTERNAL
        finally:
            wv.close()
    # and an intact plan still reports OK through every call
    cfg, bufs = fresh()
    for call in calls:
        call(cfg, bufs)
    assert m.plan_status(bufs)[0] == m.STATUS_OK
