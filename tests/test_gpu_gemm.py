"""The grouped expert GEMM on the GPU against the oracle, through the C ABI.

Bar (the arithmetic: bf16 products are exact in binary32; the tensor cores
add them in binary32 in an order the hardware picks; one round-to-nearest-even
to bf16 at the end):
  - integer-valued inputs whose every partial sum is an integer below 2^24:
    the binary32 sum is exact in any order, so the output is bit-exact;
  - general inputs: with s the oracle's binary64 sum and A = sum_h |x w|,
    |y - s| <= 2^-8 (|s| + d) + d with d = H 2^-23 A (each of the H binary32
    additions may round or truncate: relative error 2^-23 each).  A binary32
    sum only moves the bf16 rounding where s lies near a rounding boundary,
    so y must equal the oracle's rounding of s for at least 95 % of the
    outputs (a systematic error would fail that)."""
import numpy as np
import pytest
import torch

import oracle
from dispatch_moonep_plan_b200 import workloads as wl
from gpu_helpers import bits16, compare_plans, me

pytestmark = pytest.mark.gpu


def _gen(shape, seed, integer, scale=1.0):
    """Seeded bf16 tensor: integers in [-2, 2], or N(0, 1) * scale; drawn in
    slices along the first axis to bound the float32 intermediate."""
    g = torch.Generator(device="cuda")
    g.manual_seed(5_000_011 + seed)
    out = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    inner = int(np.prod(shape[1:]))
    step = max(1, (1 << 27) // inner)
    for i in range(0, shape[0], step):
        sl = out[i:i + step]
        if integer:
            sl.copy_(torch.randint(-2, 3, sl.shape, generator=g, device="cuda"))
        else:
            sl.copy_(torch.randn(sl.shape, generator=g, device="cuda") * scale)
    return out


def _experts_of(cfg, o, ranks, groups):
    if cfg.B == 0:
        return groups
    se = o["slot_expert"].reshape(cfg.R, cfg.B)
    return np.where(groups < cfg.E, groups, se[ranks, np.maximum(groups - cfg.E, 0)])


def _plan(cfgd, rule, seed):
    m = me()
    cfg = m.config_from(cfgd, rule)
    idx, _ = wl.routing(cfgd, seed=seed)
    bufs = m.PlanBuffers(cfg)
    m.plan(cfg, torch.from_numpy(idx).cuda(), bufs)
    torch.cuda.synchronize()
    o = oracle.plan(cfgd["R"], cfgd["S"], cfgd["E"], cfgd["K"], cfgd["B"], idx, rule=rule)
    compare_plans(bufs.host(), o)
    return cfg, bufs, o


def _plain_weights(cfg, o, home):
    """[R, E+B, H, Hp] with view r = home experts then rank r's replicas.
    Rows no plan of this routing can read (other ranks' experts, unused
    slots) hold NaN, so reading one shows up in the output."""
    R, E, B, Er = cfg.R, cfg.E, cfg.B, cfg.E // cfg.R
    w = torch.full((R, E + B, cfg.H, cfg.Hp), float("nan"), dtype=torch.bfloat16, device="cuda")
    se = o["slot_expert"].reshape(R, B)
    for r in range(R):
        w[r, r * Er:(r + 1) * Er] = home[r * Er:(r + 1) * Er]
        for j in range(B):
            if se[r, j] >= 0:
                w[r, E + j] = home[se[r, j]]
    return w


def _expected(cfg, o, recv, home, rows):
    """Oracle output for global rows: the row's matrix is its group's expert
    (home expert, or the expert the slot replicates)."""
    C = cfg.S * cfg.K
    ranks, groups = oracle.row_groups(cfg.E, cfg.B, C, o["cu_seqlens"], rows)
    experts = _experts_of(cfg, o, ranks, groups)
    uniq, mat = np.unique(experts, return_inverse=True)
    w_bits = bits16(home[torch.from_numpy(uniq).cuda()])
    x_bits = bits16(recv[torch.from_numpy(np.asarray(rows)).cuda()])
    return oracle.expert_gemm_rows(x_bits, mat.astype(np.int32), w_bits)


def _check(y_bits, ref, H, exact):
    yo, s, sabs = ref
    if exact:
        assert np.array_equal(y_bits, yo)
        return
    yv = oracle.bf16_to_f32(y_bits).astype(np.float64)
    d = H * 2.0 ** -23 * sabs
    assert np.all(np.abs(yv - s) <= 2.0 ** -8 * (np.abs(s) + d) + d)
    assert np.mean(y_bits != yo) <= 0.05


def _run(cfgd, rule=1, seed=0, integer=False, rows=None):
    m = me()
    cfg, bufs, o = _plan(cfgd, rule, seed)
    if o["status"] != 0:
        return None
    P = cfg.R * cfg.S * cfg.K
    recv = _gen((P, cfg.H), seed, integer)
    home = _gen((cfg.E, cfg.H, cfg.Hp), seed + 1, integer, scale=cfg.H ** -0.5)
    w = _plain_weights(cfg, o, home)
    y = torch.zeros((P, cfg.Hp), dtype=torch.bfloat16, device="cuda")
    m.expert_gemm(cfg, bufs, recv, w, y)
    torch.cuda.synchronize()
    assert m.plan_status(bufs)[0] == m.STATUS_OK
    rows = np.arange(P) if rows is None else rows
    ref = _expected(cfg, o, recv, home, rows)
    _check(bits16(y[torch.from_numpy(rows).cuda()]), ref, cfg.H, integer)
    return dict(cfg=cfg, bufs=bufs, o=o, recv=recv, home=home, w=w, y=y)


def _small(R, S, E, K, B, H, Hp, alpha=1.0):
    return dict(name="gemm", R=R, S=S, E=E, K=K, B=B, H=H, Hp=Hp, routing="zipf", alpha=alpha,
                payload="bf16")


@pytest.mark.parametrize("shape", [
    (2, 100, 4, 2, 2, 64, 128),      # one k-block, BN 128
    (4, 96, 8, 3, 4, 128, 256),      # BN 256
    (3, 150, 6, 2, 3, 192, 384),     # Hp 384: BN 128, three n-tiles
    (1, 300, 4, 2, 0, 64, 128),      # one rank, no slots
    (8, 40, 16, 4, 6, 256, 512),
])
@pytest.mark.parametrize("integer", [True, False])
def test_small_full(shape, integer):
    R, S, E, K, B, H, Hp = shape
    done = 0
    for seed in range(3):
        for rule in (0, 1, 2):
            if _run(_small(R, S, E, K, B, H, Hp, alpha=1.2), rule=rule, seed=seed,
                    integer=integer) is not None:
                done += 1
    assert done >= 3


def test_random_shapes_full():
    rng = np.random.default_rng(7)
    done = 0
    for it in range(12):
        c = wl.random_small_cfg(rng, H=64 * int(rng.integers(1, 5)))
        c["B"] = 16
        c["Hp"] = 128 * int(rng.integers(1, 4))
        if _run(c, rule=int(rng.integers(0, 3)), seed=it, integer=bool(it % 2)) is not None:
            done += 1
    assert done >= 8


def test_large_hot_ragged_groups():
    # many (rank, group) pairs, most groups ragged against 128-row tiles
    c = dict(name="gemm-hot", R=32, S=96, E=384, K=8, B=16, H=128, Hp=256, routing="hot_half",
             alpha=1.0, payload="bf16")
    assert _run(c, rule=2, seed=0, integer=True) is not None


def _sample_rows(o, cfg, n_random, seed):
    """First and last row of every non-empty group, plus random rows."""
    C = cfg.S * cfg.K
    cu = o["cu_seqlens"].reshape(cfg.R, cfg.E + cfg.B)
    rows = []
    for r in range(cfg.R):
        lo = 0
        for g in range(cfg.E + cfg.B):
            hi = int(cu[r, g])
            if hi > lo:
                rows += [r * C + lo, r * C + hi - 1]
                if hi - lo > 128:
                    rows += [r * C + lo + 127, r * C + lo + 128]
            lo = hi
    rng = np.random.default_rng(seed)
    rows += rng.integers(0, cfg.R * C, n_random).tolist()
    return np.unique(np.asarray(rows, np.int64))


def test_full_size_sampled_vmm_weights_and_prefetch():
    """The fp8 workload's sizes (R16 S16384 E128 K8 H4096, B8, H'=1536) with a
    bf16 payload: weights in VMM views filled by moonep_prefetch, sampled rows
    against the oracle, every row against torch's per-group matmul."""
    m = me()
    cfgd = wl.cfg_with("fp8", payload="bf16")
    cfg, bufs, o = _plan(cfgd, 0, 0)
    assert o["status"] == 0
    R, E, B, H, Hp = cfg.R, cfg.E, cfg.B, cfg.H, cfg.Hp
    C = cfg.S * cfg.K
    P = R * C
    recv = wl.hidden(P, H, seed=3, device="cuda")
    views = m.WeightViews(cfg, elem_bytes=2)
    try:
        v0 = m.weight_view_tensor(views, 0, cfg, torch.bfloat16)
        v0[:E] = _gen((E, H, Hp), 4, False, scale=H ** -0.5)
        m.prefetch(cfg, bufs, views.ptrs, 2)
        y = torch.zeros((P, Hp), dtype=torch.bfloat16, device="cuda")
        m.expert_gemm(cfg, bufs, recv, views.ptrs[0], y)
        torch.cuda.synchronize()
        assert m.plan_status(bufs)[0] == m.STATUS_OK
        home = v0[:E]
        rows = _sample_rows(o, cfg, 64, seed=1)
        # keep the oracle's work bounded: rows of 5 replicated experts (their
        # slot groups and home groups) and of 5 other experts
        ranks, groups = oracle.row_groups(E, B, C, o["cu_seqlens"], rows)
        ex = _experts_of(cfg, o, ranks, groups)
        chosen = np.unique(ex[groups >= E])[:5]
        rest = np.setdiff1d(np.unique(ex), chosen)
        chosen = np.concatenate([chosen, np.random.default_rng(2).choice(rest, 5, replace=False)])
        rows = rows[np.isin(ex, chosen)]
        assert len(rows) >= 40
        _check(bits16(y[torch.from_numpy(rows).cuda()]), _expected(cfg, o, recv, home, rows), H,
               False)
        # every row: torch's binary32 matmul of each group agrees with ours
        # within a bf16 ulp plus a summation term (H 2^-22 sum |x||w|)
        cu = o["cu_seqlens"].reshape(R, E + B)
        for r in range(R):
            vr = m.weight_view_tensor(views, r, cfg, torch.bfloat16)
            lo = 0
            for g in range(E + B):
                hi = int(cu[r, g])
                if hi > lo:
                    a = recv[r * C + lo:r * C + hi].float()
                    wg = vr[g].float()
                    ref = torch.matmul(a, wg)
                    got = y[r * C + lo:r * C + hi].float()
                    tol = 2.0 ** -7 * ref.abs() + H * 2.0 ** -22 * torch.matmul(a.abs(), wg.abs())
                    assert bool(((got - ref).abs() <= tol).all()), (r, g)
                lo = hi
        del v0, vr, home
    finally:
        views.close()


def test_vmm_and_plain_weights_agree_bitwise():
    m = me()
    c = dict(name="gemm-vmm", R=4, S=512, E=8, K=4, B=4, H=1024, Hp=1024, routing="zipf",
             alpha=1.5, payload="bf16")
    r = _run(c, rule=1, seed=2, integer=False, rows=np.arange(0, 4 * 2048, 7))
    assert r is not None
    cfg, bufs, o = r["cfg"], r["bufs"], r["o"]
    views = m.WeightViews(cfg, elem_bytes=2)
    try:
        v0 = m.weight_view_tensor(views, 0, cfg, torch.bfloat16)
        v0[:cfg.E] = r["home"]
        m.prefetch(cfg, bufs, views.ptrs, 2)
        y2 = torch.zeros_like(r["y"])
        m.expert_gemm(cfg, bufs, r["recv"], views.ptrs[0], y2)
        torch.cuda.synchronize()
        assert torch.equal(y2.view(torch.int16), r["y"].view(torch.int16))
        del v0
    finally:
        views.close()


def test_failed_plan_writes_nothing():
    m = me()
    c = _small(4, 64, 16, 2, 0, 64, 128, alpha=2.0)  # B = 0 and skewed: fails
    cfg, bufs, o = _plan(c, 0, 0)
    assert o["status"] == m.STATUS_SLOT_BUDGET
    P = cfg.R * cfg.S * cfg.K
    recv = _gen((P, cfg.H), 0, True)
    w = _gen((cfg.R, cfg.E + cfg.B, cfg.H, cfg.Hp), 1, True)
    y = torch.zeros((P, cfg.Hp), dtype=torch.bfloat16, device="cuda")
    m.expert_gemm(cfg, bufs, recv, w, y)
    torch.cuda.synchronize()
    assert not bool(y.any())
    assert m.plan_status(bufs)[0] == m.STATUS_SLOT_BUDGET


def test_wait_that_runs_out_reports_timeout():
    """The epilogue is told to wait on a barrier that nothing completes: the
    wait gives up after the (short) limit, every role stops and drains, the
    plan's status becomes TIMEOUT and the context stays usable."""
    m = me()
    c = _small(2, 512, 4, 2, 2, 256, 256)
    cfg, bufs, o = _plan(c, 1, 0)
    assert o["status"] == 0
    P = cfg.R * cfg.S * cfg.K
    recv = _gen((P, cfg.H), 0, True)
    home = _gen((cfg.E, cfg.H, cfg.Hp), 1, True)
    w = _plain_weights(cfg, o, home)
    y = torch.zeros((P, cfg.Hp), dtype=torch.bfloat16, device="cuda")
    m.set_wait_limit_ns(20_000_000)
    m.debug_set_barrier_extra(1)
    try:
        m.expert_gemm(cfg, bufs, recv, w, y)
        torch.cuda.synchronize()
        assert m.plan_status(bufs)[0] == m.STATUS_TIMEOUT
    finally:
        m.debug_set_barrier_extra(0)
        m.set_wait_limit_ns(1_000_000_000)
    assert _run(c, rule=1, seed=0, integer=True) is not None


def test_invalid_arguments_rejected_before_launch():
    m = me()
    cfg = m.config(2, 8, 4, 2, 2, 96, Hp=128)
    bufs = m.PlanBuffers(cfg)
    x = torch.zeros((32, 96), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((2, 6, 96, 128), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((32, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(m.MoonEPError, match="multiple of 64"):
        m.expert_gemm(cfg, bufs, x, w, y)
    cfg = m.config(2, 8, 4, 2, 2, 128, Hp=192)
    with pytest.raises(m.MoonEPError, match="multiple of 128"):
        m.expert_gemm(cfg, m.PlanBuffers(cfg), x, w, y)
    cfg = m.config(2, 8, 4, 2, 2, 128, Hp=128, payload=m.PAYLOAD_FP8)
    with pytest.raises(m.MoonEPError, match="recv_scale"):
        m.expert_gemm(cfg, m.PlanBuffers(cfg), x, w, y)


# ---------------------------------------------------------------- fp8 payload
# e4m3 codes of the integers -2..2 (sign bit 0x80; 1.0 = 0x38, 2.0 = 0x40)
_INT_CODES = np.array([0xC0, 0xB8, 0x00, 0x38, 0x40], np.uint8)


def _gen_fp8(P, H, seed, integer):
    """Seeded e4m3 rows and per-128 scales.  Integer mode: values -2..2 with
    power-of-two scales, so every dequantised value and partial sum is exact.
    Otherwise: any finite code and scales in [2^-8, 2^-4)."""
    rng = np.random.default_rng(1_234 + seed)
    if integer:
        q = _INT_CODES[rng.integers(0, 5, (P, H))]
        sc = (2.0 ** rng.integers(-1, 2, (P, H // 128))).astype(np.float32)
    else:
        q = rng.integers(0, 256, (P, H), dtype=np.uint8)
        q[(q & 0x7F) == 0x7F] = 0x3C  # no NaN codes
        sc = (2.0 ** rng.uniform(-8, -4, (P, H // 128))).astype(np.float32)
    return q, sc


def _run_fp8(cfgd, rule=1, seed=0, integer=False):
    m = me()
    cfgd = dict(cfgd, payload="fp8")
    cfg, bufs, o = _plan(cfgd, rule, seed)
    if o["status"] != 0:
        return None
    P, H = cfg.R * cfg.S * cfg.K, cfg.H
    q, sc = _gen_fp8(P, H, seed, integer)
    q_d, sc_d = torch.from_numpy(q).cuda(), torch.from_numpy(sc).cuda()
    home = _gen((cfg.E, H, cfg.Hp), seed + 1, integer, scale=H ** -0.5)
    w = _plain_weights(cfg, o, home)
    y = torch.zeros((P, cfg.Hp), dtype=torch.bfloat16, device="cuda")
    m.expert_gemm(cfg, bufs, q_d, w, y, recv_scale=sc_d)
    torch.cuda.synchronize()
    assert m.plan_status(bufs)[0] == m.STATUS_OK
    # oracle: the dequantised rows (the identity stand-in's values), then the GEMM
    C = cfg.S * cfg.K
    rows = np.arange(P)
    ranks, groups = oracle.row_groups(cfg.E, cfg.B, C, o["cu_seqlens"], rows)
    experts = _experts_of(cfg, o, ranks, groups)
    uniq, mat = np.unique(experts, return_inverse=True)
    a_bits = oracle.dequant_rows(q, sc)
    ref = oracle.expert_gemm_rows(a_bits, mat.astype(np.int32),
                                  bits16(home[torch.from_numpy(uniq).cuda()]))
    _check(bits16(y), ref, H, integer)
    # the fused path equals the stand-in followed by the bf16 GEMM, bit for bit
    a_dev = torch.zeros((P, H), dtype=torch.bfloat16, device="cuda")
    m.expert_standin(cfg, bufs, q_d, sc_d, m.EXPERT_IDENTITY, a_dev)
    cfg16 = m.config_from(dict(cfgd, payload="bf16"), rule)
    y16 = torch.zeros_like(y)
    m.expert_gemm(cfg16, bufs, a_dev, w, y16)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y16.view(torch.int16))
    return dict(cfg=cfg, y=y)


@pytest.mark.parametrize("shape", [
    (2, 100, 4, 2, 2, 128, 256),     # BN 256, two k-blocks
    (3, 150, 6, 2, 3, 256, 384),     # Hp 384: BN 128
    (4, 96, 8, 3, 4, 384, 512),      # odd number of 128-blocks per row
    (1, 300, 4, 2, 0, 128, 128),     # one rank, no slots
])
@pytest.mark.parametrize("integer", [True, False])
def test_fp8_small_full(shape, integer):
    R, S, E, K, B, H, Hp = shape
    done = 0
    for seed in range(2):
        for rule in (0, 1, 2):
            if _run_fp8(_small(R, S, E, K, B, H, Hp, alpha=1.2), rule=rule, seed=seed,
                        integer=integer) is not None:
                done += 1
    assert done >= 2


def test_fp8_random_shapes_and_ragged():
    rng = np.random.default_rng(17)
    done = 0
    for it in range(8):
        c = wl.random_small_cfg(rng, H=128 * int(rng.integers(1, 4)))
        c["B"] = 16
        c["Hp"] = 128 * int(rng.integers(1, 4))
        if _run_fp8(c, rule=int(rng.integers(0, 3)), seed=it, integer=bool(it % 2)) is not None:
            done += 1
    assert done >= 5


def test_fp8_many_pairs_without_epilogue_staging():
    """E + R*B = 128 + 128*64 = 8320 (rank, group) pairs: the m-tile prefix
    leaves no room for the epilogue's row staging next to the fp8 stages, so
    the kernel stores each lane's row directly; same results."""
    done = 0
    for rule in (1, 2):
        if _run_fp8(_small(128, 8, 128, 2, 64, 128, 128, alpha=1.2), rule=rule, seed=0,
                    integer=True) is not None:
            done += 1
    assert done >= 1


def test_fp8_wait_that_runs_out_reports_timeout():
    """The same stalled epilogue with the converter warps running: every role,
    converters included, stops at the wait limit and the status is TIMEOUT;
    the next launch is correct."""
    m = me()
    c = _small(2, 512, 4, 2, 2, 256, 256)
    cfgd = dict(c, payload="fp8")
    cfg, bufs, o = _plan(cfgd, 1, 0)
    assert o["status"] == 0
    P = cfg.R * cfg.S * cfg.K
    q, sc = _gen_fp8(P, cfg.H, 0, True)
    home = _gen((cfg.E, cfg.H, cfg.Hp), 1, True)
    w = _plain_weights(cfg, o, home)
    y = torch.zeros((P, cfg.Hp), dtype=torch.bfloat16, device="cuda")
    m.set_wait_limit_ns(20_000_000)
    m.debug_set_barrier_extra(1)
    try:
        m.expert_gemm(cfg, bufs, torch.from_numpy(q).cuda(), w, y,
                      recv_scale=torch.from_numpy(sc).cuda())
        torch.cuda.synchronize()
        assert m.plan_status(bufs)[0] == m.STATUS_TIMEOUT
    finally:
        m.debug_set_barrier_extra(0)
        m.set_wait_limit_ns(1_000_000_000)
    assert _run_fp8(c, rule=1, seed=0, integer=True) is not None


def test_fp8_full_size_sampled():
    """The fp8 workload at full size (R16 S16384 E128 K8 H4096, B8, H'=1536):
    seeded e4m3 codes and scales drawn on the device, weights in VMM views
    filled by the prefetch; sampled rows (every group's first and last rows,
    tile edges, random rows of ten experts) against the dequantisation and
    GEMM of the oracle."""
    m = me()
    cfgd = wl.WORKLOADS["fp8"]
    cfg, bufs, o = _plan(cfgd, 0, 0)
    assert o["status"] == 0
    R, E, B, H, Hp = cfg.R, cfg.E, cfg.B, cfg.H, cfg.Hp
    C = cfg.S * cfg.K
    P = R * C
    g = torch.Generator(device="cuda")
    g.manual_seed(77)
    q = torch.empty((P, H), dtype=torch.uint8, device="cuda")
    for i in range(0, P, 1 << 18):
        sl = q[i:i + (1 << 18)]
        sl.copy_(torch.randint(0, 256, sl.shape, generator=g, device="cuda", dtype=torch.int32))
        sl[(sl & 0x7F) == 0x7F] = 0x3C  # no NaN codes
    sc = torch.exp2(torch.rand((P, H // 128), generator=g, device="cuda") * 4 - 8)
    views = m.WeightViews(cfg, elem_bytes=2)
    try:
        v0 = m.weight_view_tensor(views, 0, cfg, torch.bfloat16)
        v0[:E] = _gen((E, H, Hp), 4, False, scale=H ** -0.5)
        m.prefetch(cfg, bufs, views.ptrs, 2)
        y = torch.zeros((P, Hp), dtype=torch.bfloat16, device="cuda")
        m.expert_gemm(cfg, bufs, q, views.ptrs[0], y, recv_scale=sc)
        torch.cuda.synchronize()
        assert m.plan_status(bufs)[0] == m.STATUS_OK
        rows = _sample_rows(o, cfg, 64, seed=3)
        ranks, groups = oracle.row_groups(E, B, C, o["cu_seqlens"], rows)
        ex = _experts_of(cfg, o, ranks, groups)
        chosen = np.unique(ex[groups >= E])[:5]
        rest = np.setdiff1d(np.unique(ex), chosen)
        chosen = np.concatenate([chosen, np.random.default_rng(4).choice(rest, 5, replace=False)])
        rows = rows[np.isin(ex, chosen)]
        assert len(rows) >= 40
        rows_d = torch.from_numpy(rows).cuda()
        q_rows = q[rows_d].cpu().numpy()
        s_rows = sc[rows_d].cpu().numpy()
        ranks, groups = oracle.row_groups(E, B, C, o["cu_seqlens"], rows)
        experts = _experts_of(cfg, o, ranks, groups)
        uniq, mat = np.unique(experts, return_inverse=True)
        ref = oracle.expert_gemm_rows(oracle.dequant_rows(q_rows, s_rows), mat.astype(np.int32),
                                      bits16(v0[torch.from_numpy(uniq).cuda()]))
        _check(bits16(y[rows_d]), ref, H, False)
        del v0
    finally:
        views.close()
