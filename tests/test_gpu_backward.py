"""Backward of combine and dispatch on the GPU against the oracle, through
the C ABI.

Bar: d_expert_out (one binary32 product, one bf16 rounding) and dx (binary32
additions in k order, one bf16 rounding) are bit-exact.  d_topk_w is a
binary32 dot product of length H; the GPU sums each lane's elements with an
fma chain of length L = 8 * ceil(H / 256), then adds 32 lane sums with a
5-level tree, so |d_w - exact| <= gamma(L + 5) * sum_h |dy * eo| with
gamma(n) = n u / (1 - n u), u = 2^-24 (recursive summation bound)."""
import math

import numpy as np
import pytest
import torch

import oracle
from dispatch_moonep_plan_b200 import workloads as wl
from gpu_helpers import bits16, compare_plans, me, sample_tokens

pytestmark = pytest.mark.gpu


def _gamma(n):
    u = 2.0 ** -24
    return n * u / (1 - n * u)


def _dw_bound(H, dy_bits, eo_bits):
    L = 8 * math.ceil(H / 256)
    absdot = np.einsum("nh,nkh->nk", np.abs(oracle.bf16_to_f32(dy_bits).astype(np.float64)),
                       np.abs(oracle.bf16_to_f32(eo_bits).astype(np.float64)))
    return _gamma(L + 5) * absdot + 1e-30


def _setup(cfgd, seed, rule=0):
    m = me()
    cfg = m.config_from(cfgd, rule)
    s = m.sizes(cfg)
    T, P, H, K = s.tokens, s.picks, cfg.H, cfg.K
    idx, w = wl.routing(cfgd, seed=seed)
    bufs = m.PlanBuffers(cfg)
    m.plan(cfg, torch.from_numpy(idx).cuda(), bufs)
    torch.cuda.synchronize()
    o = oracle.plan(cfgd["R"], cfgd["S"], cfgd["E"], cfgd["K"], cfgd["B"], idx, rule=rule)
    compare_plans(bufs.host(), o)
    dy = wl.hidden(T, H, seed=seed + 7, device="cuda")
    eo = wl.hidden(P, H, seed=seed + 11, device="cuda")
    d_recv = wl.hidden(P, H, seed=seed + 13, device="cuda")
    w_d = torch.from_numpy(w).cuda()
    d_eo = torch.zeros((P, H), dtype=torch.bfloat16, device="cuda")
    d_w = torch.zeros((T, K), dtype=torch.float32, device="cuda")
    dx = torch.zeros((T, H), dtype=torch.bfloat16, device="cuda")
    m.combine_backward(cfg, bufs, dy, eo, w_d, d_eo, d_w)
    m.dispatch_backward(cfg, bufs, d_recv, dx)
    torch.cuda.synchronize()
    return dict(cfg=cfg, o=o, w=w, w_d=w_d, dy=dy, eo=eo, d_recv=d_recv, d_eo=d_eo, d_w=d_w,
                dx=dx, bufs=bufs)


def _check_tokens(r, tokens):
    cfg, o = r["cfg"], r["o"]
    K, H = cfg.K, cfg.H
    tt = torch.from_numpy(tokens).cuda()
    rows = o["dst_row"][tokens].reshape(-1)
    rows_d = torch.from_numpy(rows.astype(np.int64)).cuda()
    dy_b = bits16(r["dy"][tt])
    eo_b = bits16(r["eo"][rows_d]).reshape(len(tokens), K, H)
    d_eo_o, d_w_o = oracle.combine_backward_tokens(r["w"][tokens], dy_b, eo_b)
    assert np.array_equal(bits16(r["d_eo"][rows_d]).reshape(len(tokens), K, H), d_eo_o)
    d_w_g = r["d_w"][tt].cpu().numpy().astype(np.float64)
    assert np.all(np.abs(d_w_g - d_w_o) <= _dw_bound(H, dy_b, eo_b))
    dr_b = bits16(r["d_recv"][rows_d]).reshape(len(tokens), K, H)
    assert np.array_equal(bits16(r["dx"][tt]), oracle.dispatch_backward_tokens(dr_b))


@pytest.mark.parametrize("rule", [0, 1])
def test_backward_small_full(rule):
    rng = np.random.default_rng(31 + rule)
    for it in range(30):
        cfgd = wl.random_small_cfg(rng, H=8 * int(rng.integers(1, 60)))
        cfgd["B"] = 64  # no slot budget failure: every routing plans
        r = _setup(cfgd, seed=it, rule=rule)
        if r["o"]["status"] != 0:
            continue
        _check_tokens(r, np.arange(cfgd["R"] * cfgd["S"]))


@pytest.mark.parametrize("K,H", [(8, 256), (12, 512), (32, 64)])
def test_backward_many_picks(K, H):
    """Both sides of the K = 8 switch in the backward kernels, every token."""
    cfgd = dict(name="bwd-k", R=2, S=40, E=32, K=K, B=16, H=H, Hp=0, routing="zipf",
                alpha=0.5, expert="identity", payload="bf16")
    r = _setup(cfgd, seed=1, rule=1)
    assert r["o"]["status"] == 0
    _check_tokens(r, np.arange(cfgd["R"] * cfgd["S"]))


def test_backward_tiny_and_uniform_full():
    for name in ("tiny", "uniform"):
        cfgd = wl.WORKLOADS[name]
        r = _setup(cfgd, seed=0)
        assert r["o"]["status"] == 0
        _check_tokens(r, np.arange(cfgd["R"] * cfgd["S"]))


@pytest.mark.parametrize("name,alpha,rule", [("zipf", 0.5, 1), ("hot", None, 0)])
def test_backward_large_sampled_and_properties(name, alpha, rule):
    cfgd = wl.cfg_with(name, **({"alpha": alpha} if alpha is not None else {}))
    r = _setup(cfgd, seed=0, rule=rule)
    assert r["o"]["status"] == 0
    T, K = cfgd["R"] * cfgd["S"], cfgd["K"]
    _check_tokens(r, sample_tokens(T, 128, seed=5))
    # every row of d_expert_out is w * dy of its token (torch binary32 product,
    # bf16 cast); dx is the k-ordered binary32 sum of the token's rows
    d = r["bufs"].dst_row.view(T, K).long()
    for t0 in range(0, T, 2048):
        t1 = min(T, t0 + 2048)
        dyf = r["dy"][t0:t1].float()
        ref = (r["w_d"][t0:t1, :, None] * dyf[:, None, :]).to(torch.bfloat16)
        got = r["d_eo"][d[t0:t1].reshape(-1)].view(t1 - t0, K, -1)
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
        acc = torch.zeros_like(dyf)
        for k in range(K):
            acc = acc + r["d_recv"][d[t0:t1, k]].float()
        assert torch.equal(r["dx"][t0:t1].view(torch.int16), acc.to(torch.bfloat16).view(torch.int16))
