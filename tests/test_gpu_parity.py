"""GPU path vs the oracle, through the C ABI.

Bar: plans, placements, cu_seqlens, statuses and the bf16 / fp8 payloads are
bit-exact; combine is within max abs 1e-2 (it is bit-exact in practice: both
sides run the same binary32 fma chain and one bf16 rounding).
Small workloads are compared element by element; the full-size workloads are
compared on sampled tokens the oracle computes one by one, plus properties
that hold at any size checked over every element on the GPU."""
import numpy as np
import pytest
import torch

import oracle
from dispatch_moonep_plan_b200 import workloads as wl
from gpu_helpers import (bits16, check_combine_identity_property, check_dispatch_property,
                         compare_plans, gpu_path, routing_and_x, sample_tokens)
from plan_bruteforce import check_plan_invariants

pytestmark = pytest.mark.gpu

COMBINE_ABS_TOL = 1e-2


def _oracle_plan(cfgd, idx, rule):
    return oracle.plan(cfgd["R"], cfgd["S"], cfgd["E"], cfgd["K"], cfgd["B"], idx, rule=rule)


def _check_full_small(cfgd, idx, w, x_dev, rule, expert):
    out = gpu_path(cfgd, idx, w, x_dev, rule=rule, expert=expert)
    g = out["bufs"].host()
    o = _oracle_plan(cfgd, idx, rule)
    compare_plans(g, o)
    if o["status"] != 0:
        return out, o
    K, E, B, S = cfgd["K"], cfgd["E"], cfgd["B"], cfgd["S"]
    C = S * K
    x_bits = bits16(x_dev)
    P = idx.size
    rows = np.arange(P)
    if cfgd.get("payload") == "fp8":
        q, s = oracle.dispatch_rows_fp8(K, x_bits, o["src_of_row"], rows)
        assert np.array_equal(out["recv"].cpu().numpy(), q)
        assert np.array_equal(out["scale"].cpu().numpy(), s)
        eo = oracle.expert_rows(expert, E, B, C, o, rows, q=q, s=s)
    else:
        recv = oracle.dispatch_rows(K, x_bits, o["src_of_row"], rows)
        assert np.array_equal(bits16(out["recv"]), recv)
        eo = oracle.expert_rows(expert, E, B, C, o, rows, recv_bits=recv)
    assert np.array_equal(bits16(out["eo"]), eo)
    T = idx.shape[0]
    y, _ = oracle.path_tokens(cfgd, x_bits, w, o, np.arange(T), expert=expert,
                              payload=cfgd.get("payload", "bf16"))
    yg = bits16(out["y"])
    diff = np.abs(oracle.bf16_to_f32(yg).astype(np.float64) - oracle.bf16_to_f32(y))
    assert diff.max() <= COMBINE_ABS_TOL
    assert np.array_equal(yg, y)  # same chain, same rounding
    return out, o


@pytest.mark.parametrize("rule", [0, 1, 2])
def test_random_small_configs(rule):
    rng = np.random.default_rng(7 + rule)
    statuses = set()
    for it in range(60):
        cfgd = wl.random_small_cfg(rng, H=8 * int(rng.integers(1, 40)))
        idx, w = wl.routing(cfgd, seed=it)
        x = wl.hidden(cfgd["R"] * cfgd["S"], cfgd["H"], seed=it).cuda()
        out, o = _check_full_small(cfgd, idx, w, x, rule, "scale")
        statuses.add(o["status"])
    assert 0 in statuses and 3 in statuses


@pytest.mark.parametrize("expert", ["identity", "scale"])
def test_tiny_full(expert):
    cfgd = wl.WORKLOADS["tiny"]
    for seed in range(3):
        idx, w = wl.routing(cfgd, seed=seed)
        x = wl.hidden(cfgd["R"] * cfgd["S"], cfgd["H"], seed=seed).cuda()
        for rule in (0, 1, 2):
            _check_full_small(cfgd, idx, w, x, rule, expert)


def test_uniform_full():
    cfgd = wl.WORKLOADS["uniform"]
    idx, w = wl.routing(cfgd, seed=0)
    x = wl.hidden(cfgd["R"] * cfgd["S"], cfgd["H"], seed=0).cuda()
    out, o = _check_full_small(cfgd, idx, w, x, 0, "scale")
    assert o["status"] == 0
    check_plan_invariants(out["bufs"].host(), idx, cfgd["R"], cfgd["S"], cfgd["E"], cfgd["K"],
                          cfgd["B"])


def _check_large(cfgd, idx, w, x, rule, expert, n_sample=384):
    out = gpu_path(cfgd, idx, w, x, rule=rule, expert=expert)
    g = out["bufs"].host()
    o = _oracle_plan(cfgd, idx, rule)
    compare_plans(g, o)
    R, S, E, K, B, H = (cfgd[k] for k in ("R", "S", "E", "K", "B", "H"))
    T, C = R * S, S * K
    # per-rank shapes do not depend on the skew
    assert tuple(out["recv"].shape) == (R * C, H)
    assert tuple(out["bufs"].cu_seqlens.shape) == (R * (E + B),)
    if o["status"] != 0:
        # a failed plan moves no data: buffers stay as allocated (zero)
        assert not bool(out["recv"].any()) and not bool(out["y"].any())
        return out, o
    assert np.all(g["cu_seqlens"][:, -1] == C)
    tokens = sample_tokens(T, n_sample, seed=R + S)
    x_bits_rows = bits16(x[torch.from_numpy(tokens).cuda()])
    # the oracle only needs the sampled tokens' rows of x: give it a compact x
    # and a source map that points into it
    rows = o["dst_row"][tokens].reshape(-1).astype(np.int64)
    src_c = np.zeros(T * K, np.int32)
    for i, t in enumerate(tokens):
        src_c[o["dst_row"][t]] = i * K + np.arange(K)
    rows_gpu = torch.from_numpy(rows).cuda()
    payload = cfgd.get("payload", "bf16")
    if payload == "fp8":
        q, s = oracle.dispatch_rows_fp8(K, x_bits_rows, src_c, rows)
        assert np.array_equal(out["recv"][rows_gpu].cpu().numpy(), q)
        assert np.array_equal(out["scale"][rows_gpu].cpu().numpy(), s)
    else:
        r = oracle.dispatch_rows(K, x_bits_rows, src_c, rows)
        assert np.array_equal(bits16(out["recv"][rows_gpu]), r)
        check_dispatch_property(x, out["recv"], out["bufs"].dst_row, K)
    # combine on the sampled tokens, through the oracle's own dispatch/expert
    yo = _path_tokens_rows(cfgd, x_bits_rows, w[tokens], o, tokens, src_c, expert, payload)
    yg = bits16(out["y"][torch.from_numpy(tokens).cuda()])
    diff = np.abs(oracle.bf16_to_f32(yg).astype(np.float64) - oracle.bf16_to_f32(yo))
    assert diff.max() <= COMBINE_ABS_TOL
    assert np.array_equal(yg, yo)
    if expert == "identity" and payload == "bf16":
        check_combine_identity_property(x, out["w"], out["y"])
    return out, o


def _path_tokens_rows(cfgd, x_rows, w_rows, o, tokens, src_c, expert, payload):
    """Oracle y for the sampled tokens: dispatch through the oracle's plan
    (rows dst_row[t]), stand-in expert by the row's group, combine."""
    K, E, B, S = cfgd["K"], cfgd["E"], cfgd["B"], cfgd["S"]
    C = S * K
    rows = o["dst_row"][tokens].reshape(-1).astype(np.int64)
    if payload == "fp8":
        q, s = oracle.dispatch_rows_fp8(K, x_rows, src_c, rows)
        eo = oracle.expert_rows(expert, E, B, C, o, rows, q=q, s=s)
    else:
        r = oracle.dispatch_rows(K, x_rows, src_c, rows)
        eo = oracle.expert_rows(expert, E, B, C, o, rows, recv_bits=r)
    eo = eo.reshape(len(tokens), K, -1)
    return oracle.combine_tokens(w_rows, eo)


@pytest.mark.parametrize("alpha", [0.0, 0.5, 1.0, 1.5])
@pytest.mark.parametrize("rule", [0, 1, 2])
def test_zipf_sweep(alpha, rule):
    cfgd = wl.WORKLOADS["zipf"]
    idx, w, x = routing_and_x(cfgd, seed=0, alpha=alpha)
    out, o = _check_large(cfgd, idx, w, x, rule, "scale")
    if rule >= 1:
        assert o["status"] == 0  # keep-lightest fits the slot budget at every skew


@pytest.mark.parametrize("name,rule,expert", [
    ("hot", 0, "identity"), ("hot", 0, "scale"), ("hot", 2, "identity"),
    ("hot_tokens", 0, "identity"), ("hot_tokens", 1, "scale")])
def test_hot_adversarial(name, rule, expert):
    """The largest workload.  With the identity expert all K rows of a token
    hold the same vector, so a combine that gathered the wrong one of them
    would still agree; the scale expert (1 + e/E per row group) makes every
    row of a token differ, so the sampled tokens' y also pins which row each
    (t, k) was gathered from and which weight it was paired with."""
    cfgd = wl.WORKLOADS[name]
    idx, w, x = routing_and_x(cfgd, seed=0)
    out, o = _check_large(cfgd, idx, w, x, rule, expert, n_sample=256)
    assert o["status"] == 0
    if name == "hot":
        assert o["maxvio"] > 100  # half of all picks on one expert
    else:
        assert o["expert_count"].max() >= cfgd["R"] * cfgd["S"] // 2  # half the tokens
    del out
    torch.cuda.empty_cache()


def test_fp8_workload_scale_expert():
    """The fp8 workload with the scale expert applied to the dequantised
    rows: sampled tokens' y bit-exact, so each of a token's K rows is the one
    its (t, k) was dispatched to."""
    cfgd = wl.WORKLOADS["fp8"]
    idx, w, x = routing_and_x(cfgd, seed=0)
    for rule in (0, 2):
        out, o = _check_large(cfgd, idx, w, x, rule, "scale", n_sample=256)
        assert o["status"] == 0
        del out
        torch.cuda.empty_cache()


def test_fp8_workload():
    cfgd = wl.WORKLOADS["fp8"]
    idx, w, x = routing_and_x(cfgd, seed=0)
    out, o = _check_large(cfgd, idx, w, x, 0, "identity", n_sample=256)
    assert o["status"] == 0
    # all K copies of a token are identical and dequantise within 2^-4
    K, H = cfgd["K"], cfgd["H"]
    T = x.shape[0]
    d = out["bufs"].dst_row.view(T, K).long()
    for t0 in range(0, T, 8192):
        t1 = min(T, t0 + 8192)
        q = out["recv"][d[t0:t1].reshape(-1)].view(t1 - t0, K, H)
        s = out["scale"][d[t0:t1].reshape(-1)].view(t1 - t0, K, H // 128)
        assert torch.equal(q, q[:, :1].expand_as(q)) and torch.equal(s, s[:, :1].expand_as(s))
        deq = q[:, 0].view(torch.float8_e4m3fn).float() * s[:, 0].repeat_interleave(128, 1)
        xf = x[t0:t1].float()
        err = (deq - xf).abs()
        normal = xf.abs() >= s[:, 0].repeat_interleave(128, 1) * 2.0 ** -6
        assert bool((err[normal] <= xf.abs()[normal] * 2.0 ** -4 * 1.0001).all())
        sub_bound = s[:, 0].repeat_interleave(128, 1) * 2.0 ** -10 * 1.0001
        assert bool((err[~normal] <= sub_bound[~normal]).all())


def test_determinism_zipf():
    cfgd = wl.WORKLOADS["zipf"]
    idx, w, x = routing_and_x(cfgd, seed=1, alpha=0.5)
    a = gpu_path(cfgd, idx, w, x, rule=1, expert="scale")
    ha = a["bufs"].host()
    ya = a["y"].clone()
    del a
    b = gpu_path(cfgd, idx, w, x, rule=1, expert="scale")
    hb = b["bufs"].host()
    for k in ("dst_row", "src_of_row", "cu_seqlens", "slot_expert"):
        assert np.array_equal(ha[k], hb[k])
    assert torch.equal(ya.view(torch.int16), b["y"].view(torch.int16))


@pytest.mark.parametrize("H", [128, 384, 1152, 2176, 4224])
def test_small_fp8_full(H):
    """fp8 payload element by element: codes, scales, dequantised expert and
    combine, over several hidden sizes (odd numbers of 128-blocks and of
    32-lane passes; each of the dispatch kernel's three shapes, and a row
    longer than one 4096-element chunk), all rules, identity and scale
    experts."""
    rng = np.random.default_rng(H)
    for it in range(6):
        cfgd = wl.random_small_cfg(rng, H=H)
        cfgd["payload"] = "fp8"
        idx, w = wl.routing(cfgd, seed=it)
        x = wl.hidden(cfgd["R"] * cfgd["S"], H, seed=it).cuda()
        if it == 0:
            x[0].zero_()  # a zero row: scale 1, zero codes
        for rule in (0, 1, 2):
            _check_full_small(cfgd, idx, w, x, rule, "scale" if it % 2 else "identity")
