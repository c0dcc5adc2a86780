"""Pins for the oracle's dispatch, fp8 quantisation, stand-in experts,
combine, replica prefetch and replica gradient reduction."""
import numpy as np
import torch

from dispatch_moonep_plan_b200 import workloads as wl


def _small(oracle, name="tiny", seed=0, **kw):
    cfg = wl.cfg_with(name, **kw)
    R, S, E, K, B, H = (cfg[k] for k in ("R", "S", "E", "K", "B", "H"))
    idx, w = wl.routing(cfg, seed=seed)
    x = wl.bf16_bits(wl.hidden(R * S, H, seed=seed))
    pl = oracle.plan(R, S, E, K, B, idx)
    assert pl["status"] == 0
    return cfg, idx, w, x, pl


def test_dispatch_is_gather_through_dst_row(oracle_mod):
    cfg, idx, w, x, pl = _small(oracle_mod)
    K = cfg["K"]
    P = idx.size
    recv = oracle_mod.dispatch_rows(K, x, pl["src_of_row"], np.arange(P))
    # the other direction: the row a pick was sent to holds its token
    T = idx.shape[0]
    for t in range(T):
        for k in range(K):
            assert np.array_equal(recv[pl["dst_row"][t, k]], x[t])


def test_quant_row_bounds_and_torch(oracle_mod):
    rng = np.random.default_rng(7)
    H = 1024
    xf = (rng.standard_normal(H) * np.repeat(2.0 ** rng.uniform(-8, 8, H // 128), 128))
    x = oracle_mod.bf16_from_f32(xf.astype(np.float32))
    x[128:256] = 0  # a zero block: scale 1, all-zero codes
    q, s = oracle_mod.quant_row_e4m3(x)
    xv = oracle_mod.bf16_to_f32(x)
    assert s[1] == 1.0 and np.all(q[128:256] == 0)
    deq = oracle_mod.e4m3_to_f32(q) * np.repeat(s, 128)
    for b in range(H // 128):
        blk = xv[b * 128:(b + 1) * 128]
        amax = np.float32(np.abs(blk).max())
        if amax == 0:
            continue
        assert s[b] == np.float32(amax / np.float32(448.0))
        inv = np.float32(np.float32(448.0) / amax)
        scaled = (blk * inv).astype(np.float32)
        ref = torch.from_numpy(scaled).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(q[b * 128:(b + 1) * 128], ref)
        d = deq[b * 128:(b + 1) * 128].astype(np.float64)
        err = np.abs(d - blk)
        # e4m3 normals (scaled magnitude >= 2^-6) keep 3 mantissa bits:
        # relative error <= 2^-4; below that the step is 2^-9 in the scaled
        # domain, i.e. an absolute error <= scale * 2^-10
        normal = np.abs(blk) >= s[b] * 2.0 ** -6
        assert np.all(err[normal] <= 2.0 ** -4 * np.abs(blk[normal]) * 1.0001)
        assert np.all(err[~normal] <= s[b] * 2.0 ** -10 * 1.0001)


def test_fp8_rows_identical_across_copies(oracle_mod):
    cfg, idx, w, x, pl = _small(oracle_mod, "tiny", H=256)
    K = cfg["K"]
    rows = pl["dst_row"].reshape(-1).astype(np.int64)
    q, s = oracle_mod.dispatch_rows_fp8(K, x, pl["src_of_row"], rows)
    q = q.reshape(-1, K, 256)
    s = s.reshape(-1, K, 2)
    for k in range(1, K):
        assert np.array_equal(q[:, 0], q[:, k]) and np.array_equal(s[:, 0], s[:, k])


def test_scale_expert_uses_row_group(oracle_mod):
    cfg, idx, w, x, pl = _small(oracle_mod, "tiny")
    R, S, E, K, B = (cfg[k] for k in ("R", "S", "E", "K", "B"))
    C = S * K
    P = idx.size
    rows = np.arange(P)
    recv = oracle_mod.dispatch_rows(K, x, pl["src_of_row"], rows)
    out = oracle_mod.expert_scale_rows(E, B, C, pl["cu_seqlens"], pl["slot_expert"], rows, recv)
    # expert of each row straight from the routing it came from
    e_of_row = idx.reshape(-1)[pl["src_of_row"]]
    s = (1.0 + torch.from_numpy(e_of_row.astype(np.float32)) / float(E)).to(torch.float32)
    ref = (torch.from_numpy(oracle_mod.bf16_to_f32(recv)) * s[:, None]).to(torch.bfloat16)
    assert np.array_equal(out, ref.view(torch.int16).numpy().view(np.uint16))


def test_combine_identity_closed_form(oracle_mod):
    """Identity expert: every row of token t is x[t], so y = bf16(sum_k w_k x).
    The binary32 chain then sits within one bf16 rounding (unit roundoff 2^-8)
    plus K binary32 roundings of the exact sum."""
    cfg, idx, w, x, pl = _small(oracle_mod, "tiny")
    T = idx.shape[0]
    y, y64 = oracle_mod.path_tokens(cfg, x, w, pl, np.arange(T), expert="identity")
    xv = oracle_mod.bf16_to_f32(x).astype(np.float64)
    exact = w.astype(np.float64).sum(1)[:, None] * xv
    assert np.allclose(y64, exact, rtol=1e-15, atol=0)
    yv = oracle_mod.bf16_to_f32(y).astype(np.float64)
    bound = np.abs(exact) * (2.0 ** -8 + cfg["K"] * 2.0 ** -23) * 1.0001
    assert np.all(np.abs(yv - exact) <= bound)
    small = np.abs(exact) < 2.0
    assert np.max(np.abs(yv - exact)[small]) <= 1e-2


def test_combine_matches_torch_chain(oracle_mod):
    """The chain acc = fma(w_k, v_k, acc) from zero in k order, then one bf16
    rounding, against torch binary32 arithmetic.  With weights of at most 13
    significant bits and bf16 values (8 bits) every product is exact in
    binary32, so fma and torch's multiply-then-add agree bit for bit."""
    rng = np.random.default_rng(11)
    n, K, H = 64, 8, 96
    w = rng.random((n, K)).astype(np.float32)
    w = (np.round(w * 2 ** 12) / 2 ** 12).astype(np.float32)
    eo = oracle_mod.bf16_from_f32(rng.standard_normal((n, K, H)).astype(np.float32))
    y = oracle_mod.combine_tokens(w, eo)
    acc = torch.zeros((n, H), dtype=torch.float32)
    ev = torch.from_numpy(oracle_mod.bf16_to_f32(eo))
    wt = torch.from_numpy(w)
    for k in range(K):
        acc = acc + wt[:, k:k + 1] * ev[:, k]
    ref = acc.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(y, ref)


def test_combine_scale_expert_against_routing(oracle_mod):
    """Scale expert through the plan equals the same expert applied straight
    from the routing (torch bf16 rounding), so a wrong gather or a wrong
    group expert shows up."""
    cfg, idx, w, x, pl = _small(oracle_mod, "tiny")
    T, K, E = idx.shape[0], cfg["K"], cfg["E"]
    y, y64 = oracle_mod.path_tokens(cfg, x, w, pl, np.arange(T), expert="scale")
    xs = torch.from_numpy(oracle_mod.bf16_to_f32(x))
    ref = np.zeros(y64.shape, np.float64)
    for k in range(K):
        s = 1.0 + torch.from_numpy(idx[:, k].astype(np.float32)) / float(E)
        eo = (xs * s[:, None]).to(torch.bfloat16).to(torch.float64).numpy()
        ref = ref + w[:, k:k + 1].astype(np.float64) * eo
    assert np.array_equal(y64, ref)
    yv = oracle_mod.bf16_to_f32(y).astype(np.float64)
    bound = np.abs(y64) * (2.0 ** -8 + K * 2.0 ** -23) * 1.0001
    assert np.all(np.abs(yv - y64) <= bound)


def test_prefetch_copies_home_rows(oracle_mod):
    rng = np.random.default_rng(2)
    R, B, E = 3, 2, 6
    home = rng.integers(0, 65535, (E, 5, 7)).astype(np.uint16)
    slots = np.zeros((R, B, 5, 7), np.uint16)
    se = np.array([[-1, -1], [4, 1], [2, -1]], np.int32)
    oracle_mod.prefetch(R, B, se, home, slots)
    assert np.array_equal(slots[1, 0], home[4]) and np.array_equal(slots[1, 1], home[1])
    assert np.array_equal(slots[2, 0], home[2])
    assert not slots[0].any() and not slots[2, 1].any()


def test_grad_reduce_order_and_single_replica(oracle_mod):
    R, B, E, n = 3, 2, 4, 4
    home = np.zeros((E, n), np.float32)
    slots = np.zeros((R, B, n), np.float32)
    se = np.array([[2, -1], [2, 0], [2, -1]], np.int32)
    # expert 2 has replicas (0,0), (1,0), (2,0) in that order; the order is
    # visible in binary32: ((1e8 + 1) + 1) - 1e8 = 0 but 1e8 - 1e8 + 1 + 1 = 2
    home[2] = 1e8
    slots[0, 0] = 1.0
    slots[1, 0] = 1.0
    slots[2, 0] = -1e8
    # expert 0 has the single replica (1,1): dW + s
    home[0] = np.float32(0.1)
    slots[1, 1] = np.float32(0.2)
    oracle_mod.grad_reduce(R, B, E, se, home, slots)
    assert np.all(home[2] == 0.0)
    assert np.all(home[0] == np.float32(0.1) + np.float32(0.2))
    assert np.all(home[1] == 0) and np.all(home[3] == 0)


def test_combine_backward_against_library(oracle_mod):
    """d_eo = bf16(w * dy) (torch binary32 product, bf16 cast); d_w is the
    dot product (numpy binary64)."""
    rng = np.random.default_rng(21)
    n, K, H = 40, 6, 72
    w = rng.random((n, K)).astype(np.float32)
    dy = oracle_mod.bf16_from_f32(rng.standard_normal((n, H)).astype(np.float32))
    eo = oracle_mod.bf16_from_f32(rng.standard_normal((n, K, H)).astype(np.float32))
    d_eo, d_w = oracle_mod.combine_backward_tokens(w, dy, eo)
    dyf = torch.from_numpy(oracle_mod.bf16_to_f32(dy))
    ref = (torch.from_numpy(w)[:, :, None] * dyf[:, None, :]).to(torch.bfloat16)
    assert np.array_equal(d_eo, ref.view(torch.int16).numpy().view(np.uint16))
    dot = np.einsum("nh,nkh->nk", oracle_mod.bf16_to_f32(dy).astype(np.float64),
                    oracle_mod.bf16_to_f32(eo).astype(np.float64))
    assert np.allclose(d_w, dot, rtol=1e-12, atol=1e-12)


def test_dispatch_backward_closed_form(oracle_mod):
    """If every row of token t holds the same bf16 vector v, the binary32 sum
    of K copies is exact (K <= 8, 8 significant bits), so dx = bf16(K * v)."""
    rng = np.random.default_rng(22)
    n, K, H = 30, 8, 40
    v = oracle_mod.bf16_from_f32(rng.standard_normal((n, H)).astype(np.float32))
    rows = np.repeat(v[:, None, :], K, axis=1)
    dx = oracle_mod.dispatch_backward_tokens(rows)
    ref = torch.from_numpy(oracle_mod.bf16_to_f32(v) * K).to(torch.bfloat16)
    assert np.array_equal(dx, ref.view(torch.int16).numpy().view(np.uint16))
    # k order is visible in binary32: (2^24 + 1) - 2^24 + 1 ... with bf16 rows
    big = oracle_mod.bf16_from_f32(np.array([2.0 ** 24], np.float32))[0]
    one = oracle_mod.bf16_from_f32(np.array([1.0], np.float32))[0]
    mbig = oracle_mod.bf16_from_f32(np.array([-(2.0 ** 24)], np.float32))[0]
    seq = np.array([[[big], [one], [mbig], [one]]], np.uint16)  # ((2^24 + 1) - 2^24) + 1 = 1
    assert oracle_mod.bf16_to_f32(oracle_mod.dispatch_backward_tokens(seq))[0, 0] == 1.0


def test_combine_fp8_identity_closed_form(oracle_mod):
    """fp8 payload, identity expert, through the whole oracle path: every row
    of token t dequantises to the same a[t] = bf16(float(q) * s), so y =
    bf16(sum_k w_k a[t]).  a[t] is rebuilt here from torch alone (its e4m3
    cast of x * (448/amax), its decode, binary32 multiply, bf16 cast), so the
    quantisation, the dequantisation and the combine are all pinned from
    outside the oracle."""
    cfg, idx, w, x, pl = _small(oracle_mod, "tiny", H=384)
    T, K, H = idx.shape[0], cfg["K"], 384
    y, y64 = oracle_mod.path_tokens(cfg, x, w, pl, np.arange(T), expert="identity",
                                    payload="fp8")
    xv = torch.from_numpy(oracle_mod.bf16_to_f32(x)).view(T, H // 128, 128)
    amax = xv.abs().amax(dim=2, keepdim=True)
    inv = torch.where(amax > 0, torch.tensor(448.0) / amax, torch.ones_like(amax))
    sc = torch.where(amax > 0, amax / torch.tensor(448.0), torch.ones_like(amax))
    q = (xv * inv).to(torch.float8_e4m3fn).to(torch.float32)
    a = (q * sc).view(T, H).to(torch.bfloat16).to(torch.float64).numpy()
    exact = w.astype(np.float64).sum(1)[:, None] * a
    assert np.allclose(y64, exact, rtol=1e-15, atol=0)
    yv = oracle_mod.bf16_to_f32(y).astype(np.float64)
    bound = np.abs(exact) * (2.0 ** -8 + K * 2.0 ** -23) * 1.0001
    assert np.all(np.abs(yv - exact) <= bound)
