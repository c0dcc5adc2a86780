"""Seeded synthetic inputs for the MoonEP path: router top-K picks, combine
weights and hidden states.

This module is shared by the CUDA-path tests, the oracle tests and the
benchmark.  It holds none of the method's arithmetic: it only draws routings
and activations with the shapes, sizes and skew of the five workloads below.

Routing recipes
  zipf(alpha)   p_e proportional to (pi(e)+1)^-alpha for a seeded permutation pi;
                K picks without replacement, drawn as the top-K of
                log p_e + Gumbel noise (the same law as sequential sampling
                without replacement), ordered by decreasing key.
  logits(sigma) router logits ~ N(0, sigma) over E experts, top-K by value
                (ties toward the lower index); weights = softmax of the
                K picked logits.
  hot_half      one seeded hot expert h; every pick is first drawn zipf(1.0)
                over the experts other than h, then exactly floor(P/2) seeded
                pick positions are overwritten with h (a token may then hold h
                more than once).
  hot_tokens    the reading of "50% of the traffic to one expert" that keeps a
                token's K picks distinct: every token draws K picks zipf(1.0)
                over the experts other than a seeded hot expert h, then the
                first pick of exactly floor(T/2) seeded tokens becomes h.
Combine weights are the softmax of K N(0,1) logits per token unless the
recipe says otherwise.  Hidden states are N(0,1) rounded to bf16.
"""
import numpy as np

# The five workloads: sizes, routing recipe and the stand-in expert.
WORKLOADS = {
    "tiny": dict(name="R4-S256-E16-K2-H128-zipf1.0", R=4, S=256, E=16, K=2, H=128, B=4,
               Hp=0, routing="zipf", alpha=1.0, expert="identity", payload="bf16"),
    "uniform": dict(name="R8-S4096-E64-K6-H2048-uniform", R=8, S=4096, E=64, K=6, H=2048, B=8,
               Hp=0, routing="logits", sigma=0.1, expert="scale", payload="bf16"),
    "zipf": dict(name="R8-S4096-E256-K8-H7168-zipf", R=8, S=4096, E=256, K=8, H=7168, B=16,
               Hp=0, routing="zipf", alpha=1.0, alphas=(0.0, 0.5, 1.0, 1.5),
               expert="scale", payload="bf16"),
    "hot": dict(name="R32-S8192-E384-K8-H7168-hot50", R=32, S=8192, E=384, K=8, H=7168,
               B=16, Hp=0, routing="hot_half", alpha=1.0, expert="identity",
               payload="bf16"),
    "hot_tokens": dict(name="R32-S8192-E384-K8-H7168-hot50tok", R=32, S=8192, E=384, K=8,
               H=7168, B=16, Hp=0, routing="hot_tokens", alpha=1.0, expert="identity",
               payload="bf16"),
    "fp8": dict(name="R16-S16384-E128-K8-H4096-zipf1.2-fp8", R=16, S=16384, E=128, K=8,
               H=4096, B=8, Hp=1536, routing="zipf", alpha=1.2, expert="identity",
               payload="fp8"),
}


def cfg_with(base, **kw):
    c = dict(WORKLOADS[base]) if isinstance(base, str) else dict(base)
    c.update(kw)
    return c


def _softmax_rows(logits):
    m = logits.max(axis=1, keepdims=True)
    z = np.exp(logits - m)
    return (z / z.sum(axis=1, keepdims=True)).astype(np.float32)


def zipf_topk(rng, T, E, K, alpha, exclude=None, chunk=8192):
    """Top-K picks without replacement under p_e ~ (pi(e)+1)^-alpha."""
    perm = rng.permutation(E)
    logp = -alpha * np.log(perm.astype(np.float64) + 1.0)
    if exclude is not None:
        logp[exclude] = -np.inf
    out = np.empty((T, K), np.int32)
    for i in range(0, T, chunk):
        n = min(chunk, T - i)
        u = rng.random((n, E))
        key = logp[None, :] - np.log(-np.log(u))
        part = np.argpartition(-key, K - 1, axis=1)[:, :K]
        pk = np.take_along_axis(key, part, axis=1)
        order = np.argsort(-pk, axis=1, kind="stable")
        out[i:i + n] = np.take_along_axis(part, order, axis=1)
    return out


def routing(cfg, seed=0, alpha=None):
    """Return (topk_idx int32 [T,K], topk_w float32 [T,K])."""
    R, S, E, K = cfg["R"], cfg["S"], cfg["E"], cfg["K"]
    T = R * S
    rng = np.random.default_rng(seed)
    kind = cfg["routing"]
    if kind == "zipf":
        a = cfg["alpha"] if alpha is None else alpha
        idx = zipf_topk(rng, T, E, K, a)
        w = _softmax_rows(rng.standard_normal((T, K)))
    elif kind == "logits":
        idx = np.empty((T, K), np.int32)
        w = np.empty((T, K), np.float32)
        for i in range(0, T, 8192):
            n = min(8192, T - i)
            lg = rng.normal(0.0, cfg["sigma"], (n, E))
            order = np.argsort(-lg, axis=1, kind="stable")[:, :K]
            idx[i:i + n] = order
            w[i:i + n] = _softmax_rows(np.take_along_axis(lg, order, axis=1))
    elif kind == "hot_half":
        hot = int(rng.integers(E))
        idx = zipf_topk(rng, T, E, K, cfg["alpha"] if alpha is None else alpha, exclude=hot)
        flat = idx.reshape(-1)
        pos = rng.permutation(T * K)[: (T * K) // 2]
        flat[pos] = hot
        w = _softmax_rows(rng.standard_normal((T, K)))
    elif kind == "hot_tokens":
        hot = int(rng.integers(E))
        idx = zipf_topk(rng, T, E, K, cfg["alpha"] if alpha is None else alpha, exclude=hot)
        tok = rng.permutation(T)[: T // 2]
        idx[tok, 0] = hot
        w = _softmax_rows(rng.standard_normal((T, K)))
    elif kind == "round_robin":
        p = np.arange(T * K, dtype=np.int64)
        idx = (p % E).astype(np.int32).reshape(T, K)
        w = _softmax_rows(rng.standard_normal((T, K)))
    else:
        raise ValueError(kind)
    return np.ascontiguousarray(idx, np.int32), np.ascontiguousarray(w, np.float32)


def hidden(T, H, seed=0, device="cpu"):
    """N(0,1) hidden states as a bf16 torch tensor [T, H] on ``device``,
    drawn from torch's generator for that device."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(1_000_003 + seed)
    x = torch.empty((T, H), dtype=torch.bfloat16, device=device)
    step = max(1, (1 << 28) // max(H, 1))
    for i in range(0, T, step):
        n = min(step, T - i)
        x[i:i + n] = torch.randn((n, H), generator=g, device=device,
                                 dtype=torch.float32).to(torch.bfloat16)
    return x


def bf16_bits(t):
    """bf16 torch tensor -> numpy uint16 bit array (host copy)."""
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def random_small_cfg(rng, max_R=6, max_Er=4, max_S=24, max_K=4, max_B=6, H=16):
    """A random tiny configuration for property sweeps."""
    R = int(rng.integers(1, max_R + 1))
    Er = int(rng.integers(1, max_Er + 1))
    E = R * Er
    K = int(rng.integers(1, min(max_K, E) + 1))
    S = int(rng.integers(1, max_S + 1))
    B = int(rng.integers(0, max_B + 1))
    return dict(name="rand", R=R, S=S, E=E, K=K, H=H, B=B, Hp=0, routing="zipf",
                alpha=float(rng.choice([0.0, 0.8, 1.5, 3.0])), expert="scale",
                payload="bf16")
