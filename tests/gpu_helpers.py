"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
compare it with the oracle."""
import numpy as np
import torch

from dispatch_moonep_plan_b200 import workloads as wl

PLAN_KEYS = ("expert_count", "rank_load", "max_count", "maxvio")


def me():
    from dispatch_moonep_plan_b200 import moonep
    return moonep


def gpu_path(cfgd, idx, w, x_dev, rule=0, expert="identity", run_combine=True):
    """Plan, dispatch, stand-in expert and combine on the GPU.  Returns a dict
    of device tensors plus the plan buffers."""
    m = me()
    cfg = m.config_from(cfgd, rule)
    s = m.sizes(cfg)
    P, T, H = s.picks, s.tokens, cfg.H
    bufs = m.PlanBuffers(cfg)
    idx_d = torch.from_numpy(np.ascontiguousarray(idx, np.int32)).cuda()
    w_d = torch.from_numpy(np.ascontiguousarray(w, np.float32)).cuda()
    fp8 = cfg.payload == m.PAYLOAD_FP8
    if fp8:
        recv = torch.zeros((P, H), dtype=torch.uint8, device="cuda")
        scale = torch.zeros((P, H // 128), dtype=torch.float32, device="cuda")
    else:
        recv = torch.zeros((P, H), dtype=torch.bfloat16, device="cuda")
        scale = None
    m.plan(cfg, idx_d, bufs)
    m.dispatch(cfg, bufs, x_dev, recv, scale)
    out = dict(cfg=cfg, bufs=bufs, recv=recv, scale=scale, idx=idx_d, w=w_d)
    if run_combine:
        if expert == "identity" and not fp8:
            eo = recv
        else:
            eo = torch.zeros((P, H), dtype=torch.bfloat16, device="cuda")
            mode = m.EXPERT_SCALE if expert == "scale" else m.EXPERT_IDENTITY
            m.expert_standin(cfg, bufs, recv, scale, mode, eo)
        y = torch.zeros((T, H), dtype=torch.bfloat16, device="cuda")
        m.combine(cfg, bufs, eo, w_d, y)
        out.update(eo=eo, y=y)
    torch.cuda.synchronize()
    return out


def compare_plans(gpu, ora):
    assert gpu["status"] == ora["status"], (gpu["status"], ora["status"])
    if ora["status"] == 4:
        return
    for k in ("expert_count", "rank_load"):
        assert np.array_equal(gpu[k], ora[k]), k
    assert gpu["max_count"] == ora["max_count"]
    assert gpu["maxvio"] == ora["maxvio"]  # binary64, same operations
    if ora["status"] == 3:
        assert gpu["fail_rank"] == ora["fail_rank"]
        assert gpu["fail_slots"] == ora["fail_slots"]
        return
    for k in ("slot_expert", "cu_seqlens", "dst_row", "src_of_row"):
        assert np.array_equal(gpu[k], ora[k]), k


def bits16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def check_dispatch_property(x_dev, recv, dst_row_dev, K, chunk=4096):
    """Every pick's row holds its token exactly (bf16 payload), full size."""
    T = x_dev.shape[0]
    d = dst_row_dev.view(T, K).long()
    for t0 in range(0, T, chunk):
        t1 = min(T, t0 + chunk)
        got = recv[d[t0:t1].reshape(-1)].view(t1 - t0, K, -1)
        assert torch.equal(got.view(torch.int16), x_dev[t0:t1].unsqueeze(1).expand_as(got)
                           .view(torch.int16)), (t0, t1)


def check_combine_identity_property(x_dev, w_d, y, chunk=4096):
    """Identity expert: y = bf16(sum_k w_k x) within one bf16 rounding (2^-8
    relative) plus the binary32 chain's K roundings."""
    T = x_dev.shape[0]
    K = w_d.shape[1]
    worst = 0.0
    for t0 in range(0, T, chunk):
        t1 = min(T, t0 + chunk)
        ref = w_d[t0:t1].double().sum(1, keepdim=True) * x_dev[t0:t1].double()
        err = (y[t0:t1].double() - ref).abs()
        bound = ref.abs() * (2.0 ** -8 + K * 2.0 ** -23) * 1.0001 + 1e-30
        assert bool((err <= bound).all()), (t0, float((err - bound).max()))
        worst = max(worst, float(err.max()))
    return worst


def sample_tokens(T, n, seed=0):
    rng = np.random.default_rng(seed)
    pick = rng.choice(T, size=min(n, T), replace=False)
    return np.unique(np.concatenate([pick, [0, T - 1]])).astype(np.int64)


def routing_and_x(cfgd, seed=0, alpha=None, x_device="cuda"):
    idx, w = wl.routing(cfgd, seed=seed, alpha=alpha)
    x = wl.hidden(cfgd["R"] * cfgd["S"], cfgd["H"], seed=seed, device=x_device)
    return idx, w, x.cuda()
