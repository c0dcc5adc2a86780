"""CPU oracle for the MoonEP plan -> dispatch -> combine path (test infrastructure).

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import
this package.  The library under ``dispatch_moonep_plan_b200`` never imports it,
and this package imports nothing from there.  The arithmetic lives in
``moonep_oracle.c`` (plain, single-threaded C); this module only marshals numpy
arrays through ctypes and strings the C steps together.

Sources: the web pages on MoonEP ("Moonshot AI Open-Sources MoonEP: A Perfectly
Balanced Expert Parallelism Library for MoE Training" on ainovat.com; the
"MoonEP" repository card on findrepo.work; the "MoonEP" post on
moses-y.github.io, sections "What This Does" and "Real-World Use").  Which
passage each step follows is written beside each C function.

Every function here is pinned by the ``-m "not gpu"`` tests (brute-force planner,
exhaustive tiny routings, hand-worked golden cases, closed forms, library
cross-checks of the number formats); none is "parity unpinned".
"""
import ctypes
import os

import numpy as np

from . import build as _build

STATUS_OK = 0
STATUS_INVALID = 1
STATUS_SLOT_BUDGET = 3
STATUS_BAD_INDEX = 4

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
        i64p = np.ctypeslib.ndpointer(np.int64, flags="C_CONTIGUOUS")
        u16p = np.ctypeslib.ndpointer(np.uint16, flags="C_CONTIGUOUS")
        u8p = np.ctypeslib.ndpointer(np.uint8, flags="C_CONTIGUOUS")
        f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
        f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
        ci, cl = ctypes.c_int, ctypes.c_int64
        L.oracle_plan.argtypes = [ci, ci, ci, ci, ci, ci, i32p, i32p, i32p, i32p, f64p,
                                  i32p, i32p, i32p, i32p, i32p, i32p]
        L.oracle_plan.restype = ci
        L.oracle_bf16_from_f32_array.argtypes = [f32p, u16p, cl]
        L.oracle_e4m3_from_f32_array.argtypes = [f32p, u8p, cl]
        L.oracle_e4m3_to_f32.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_to_f32.restype = ctypes.c_float
        L.oracle_dispatch_rows.argtypes = [ci, ci, u16p, i32p, i64p, cl, u16p]
        L.oracle_quant_row_e4m3.argtypes = [ci, u16p, u8p, f32p]
        L.oracle_dispatch_rows_fp8.argtypes = [ci, ci, u16p, i32p, i64p, cl, u8p, f32p]
        L.oracle_expert_scale_rows.argtypes = [ci, ci, cl, ci, i32p, i32p, i64p, cl, u16p, u16p]
        L.oracle_dequant_rows.argtypes = [ci, cl, u8p, f32p, u16p]
        L.oracle_combine_tokens.argtypes = [ci, ci, cl, f32p, u16p, u16p]
        L.oracle_combine_tokens_f64.argtypes = [ci, ci, cl, f32p, u16p, f64p]
        L.oracle_prefetch.argtypes = [ci, ci, cl, ci, i32p, u8p, u8p]
        L.oracle_grad_reduce.argtypes = [ci, ci, ci, cl, i32p, f32p, f32p]
        L.oracle_combine_backward_tokens.argtypes = [ci, ci, cl, f32p, u16p, u16p, u16p, f64p]
        L.oracle_dispatch_backward_tokens.argtypes = [ci, ci, cl, u16p, u16p]
        L.oracle_bf16_from_f64_array.argtypes = [f64p, u16p, cl]
        L.oracle_row_group.argtypes = [ci, ci, i32p, cl]
        L.oracle_row_group.restype = ci
        L.oracle_expert_gemm_rows.argtypes = [ci, ci, cl, u16p, i32p, u16p, u16p, f64p, f64p]
        _lib = L
    return _lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- formats
def bf16_from_f32(v):
    v = _c(v, np.float32)
    out = np.empty(v.shape, np.uint16)
    lib().oracle_bf16_from_f32_array(v.reshape(-1), out.reshape(-1), v.size)
    return out


def bf16_to_f32(bits):
    bits = np.asarray(bits, np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32)


def e4m3_from_f32(v):
    v = _c(v, np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().oracle_e4m3_from_f32_array(v.reshape(-1), out.reshape(-1), v.size)
    return out


def e4m3_to_f32(codes):
    codes = np.asarray(codes, np.uint8)
    table = np.array([lib().oracle_e4m3_to_f32(c) for c in range(256)], np.float32)
    return table[codes]


# ---------------------------------------------------------------- plan
def plan(R, S, E, K, B, idx, rule=0):
    """Run the oracle planner.  Returns a dict of numpy arrays plus 'status'."""
    idx = _c(idx, np.int32).reshape(-1)
    T = R * S
    P = T * K
    assert idx.size == P
    out = dict(
        expert_count=np.zeros(E, np.int32), rank_load=np.zeros(R, np.int32),
        max_count=np.zeros(1, np.int32), maxvio=np.zeros(1, np.float64),
        slot_expert=np.full(R * B if B > 0 else 1, -1, np.int32),
        cu_seqlens=np.zeros(R * (E + B), np.int32), dst_row=np.zeros(P, np.int32),
        src_of_row=np.zeros(P, np.int32), fail_rank=np.zeros(1, np.int32),
        fail_slots=np.zeros(1, np.int32))
    st = lib().oracle_plan(R, S, E, K, B, rule, idx, out["expert_count"], out["rank_load"],
                           out["max_count"], out["maxvio"], out["slot_expert"],
                           out["cu_seqlens"], out["dst_row"], out["src_of_row"],
                           out["fail_rank"], out["fail_slots"])
    res = dict(status=int(st), max_count=int(out["max_count"][0]),
               maxvio=float(out["maxvio"][0]), fail_rank=int(out["fail_rank"][0]),
               fail_slots=int(out["fail_slots"][0]),
               expert_count=out["expert_count"], rank_load=out["rank_load"],
               slot_expert=out["slot_expert"][:R * B].reshape(R, B),
               cu_seqlens=out["cu_seqlens"].reshape(R, E + B),
               dst_row=out["dst_row"].reshape(T, K), src_of_row=out["src_of_row"])
    return res


# ---------------------------------------------------------------- dispatch
def dispatch_rows(K, x_bits, src_of_row, rows):
    x_bits = _c(x_bits, np.uint16)
    H = x_bits.shape[-1]
    rows = _c(rows, np.int64)
    out = np.empty((rows.size, H), np.uint16)
    lib().oracle_dispatch_rows(K, H, x_bits.reshape(-1), _c(src_of_row, np.int32), rows,
                               rows.size, out.reshape(-1))
    return out


def quant_row_e4m3(x_row_bits):
    x_row_bits = _c(x_row_bits, np.uint16)
    H = x_row_bits.size
    q = np.empty(H, np.uint8)
    s = np.empty(H // 128, np.float32)
    lib().oracle_quant_row_e4m3(H, x_row_bits, q, s)
    return q, s


def dispatch_rows_fp8(K, x_bits, src_of_row, rows):
    x_bits = _c(x_bits, np.uint16)
    H = x_bits.shape[-1]
    rows = _c(rows, np.int64)
    q = np.empty((rows.size, H), np.uint8)
    s = np.empty((rows.size, H // 128), np.float32)
    lib().oracle_dispatch_rows_fp8(K, H, x_bits.reshape(-1), _c(src_of_row, np.int32), rows,
                                   rows.size, q.reshape(-1), s.reshape(-1))
    return q, s


# ---------------------------------------------------------------- expert stand-ins
def expert_scale_rows(E, B, C, cu_seqlens, slot_expert, rows, in_bits):
    rows = _c(rows, np.int64)
    in_bits = _c(in_bits, np.uint16)
    H = in_bits.shape[-1]
    out = np.empty_like(in_bits)
    lib().oracle_expert_scale_rows(E, B, C, H, _c(cu_seqlens, np.int32).reshape(-1),
                                   _c(slot_expert, np.int32).reshape(-1), rows, rows.size,
                                   in_bits.reshape(-1), out.reshape(-1))
    return out


def dequant_rows(q, s):
    q = _c(q, np.uint8)
    s = _c(s, np.float32)
    n, H = q.shape
    out = np.empty((n, H), np.uint16)
    lib().oracle_dequant_rows(H, n, q.reshape(-1), s.reshape(-1), out.reshape(-1))
    return out


# ---------------------------------------------------------------- combine
def combine_tokens(w, eo_bits):
    """w [n,K] fp32, eo_bits [n,K,H] bf16 bits -> y [n,H] bf16 bits."""
    w = _c(w, np.float32)
    eo_bits = _c(eo_bits, np.uint16)
    n, K, H = eo_bits.shape
    y = np.empty((n, H), np.uint16)
    lib().oracle_combine_tokens(K, H, n, w.reshape(-1), eo_bits.reshape(-1), y.reshape(-1))
    return y


def combine_tokens_f64(w, eo_bits):
    w = _c(w, np.float32)
    eo_bits = _c(eo_bits, np.uint16)
    n, K, H = eo_bits.shape
    y = np.empty((n, H), np.float64)
    lib().oracle_combine_tokens_f64(K, H, n, w.reshape(-1), eo_bits.reshape(-1), y.reshape(-1))
    return y


# ---------------------------------------------------------------- side steps
def prefetch(R, B, slot_expert, home, slots):
    """home [E, ...] any dtype; slots [R, B, ...] same dtype, updated in place."""
    assert home.flags.c_contiguous and slots.flags.c_contiguous
    elems = int(np.prod(home.shape[1:]))
    lib().oracle_prefetch(R, B, elems, home.dtype.itemsize, _c(slot_expert, np.int32).reshape(-1),
                          home.view(np.uint8).reshape(-1), slots.view(np.uint8).reshape(-1))


def grad_reduce(R, B, E, slot_expert, home, slots):
    """home [E, ...] fp32 updated in place; slots [R, B, ...] fp32."""
    assert home.dtype == np.float32 and slots.dtype == np.float32
    assert home.flags.c_contiguous and slots.flags.c_contiguous
    elems = int(np.prod(home.shape[1:]))
    lib().oracle_grad_reduce(R, B, E, elems, _c(slot_expert, np.int32).reshape(-1),
                             home.reshape(-1), slots.reshape(-1))


# ---------------------------------------------------------------- whole path
def expert_rows(mode, E, B, C, pl, rows, recv_bits=None, q=None, s=None):
    """The stand-in expert applied to the oracle's own dispatched rows.

    mode 'identity': bf16 rows unchanged, fp8 rows dequantised;
    mode 'scale': bf16(float(v) * (1 + e/E)) with e the row's expert."""
    if q is not None:
        base = dequant_rows(q, s)
    else:
        base = recv_bits
    if mode == "identity":
        return base
    if mode == "scale":
        return expert_scale_rows(E, B, C, pl["cu_seqlens"], pl["slot_expert"], rows, base)
    raise ValueError(mode)


def path_tokens(cfg, x_bits, w, pl, tokens, expert="identity", payload="bf16"):
    """Oracle output y for the given tokens: dispatch (its own plan), stand-in
    expert, combine.  Returns (y_bits [n,H], y_f64 [n,H])."""
    K, E, B, S = cfg["K"], cfg["E"], cfg["B"], cfg["S"]
    C = S * K
    tokens = np.asarray(tokens, np.int64)
    rows = pl["dst_row"][tokens].reshape(-1).astype(np.int64)
    if payload == "fp8":
        q, s = dispatch_rows_fp8(K, x_bits, pl["src_of_row"], rows)
        eo = expert_rows(expert, E, B, C, pl, rows, q=q, s=s)
    else:
        recv = dispatch_rows(K, x_bits, pl["src_of_row"], rows)
        eo = expert_rows(expert, E, B, C, pl, rows, recv_bits=recv)
    H = x_bits.shape[-1]
    eo = eo.reshape(tokens.size, K, H)
    wt = np.asarray(w, np.float32)[tokens]
    return combine_tokens(wt, eo), combine_tokens_f64(wt, eo)


# ---------------------------------------------------------------- backward
def combine_backward_tokens(w, dy_bits, eo_bits):
    """w [n,K] fp32, dy [n,H] bf16 bits, eo [n,K,H] bf16 bits ->
    (d_eo [n,K,H] bf16 bits, d_w [n,K] float64)."""
    w = _c(w, np.float32)
    dy_bits = _c(dy_bits, np.uint16)
    eo_bits = _c(eo_bits, np.uint16)
    n, K, H = eo_bits.shape
    d_eo = np.empty((n, K, H), np.uint16)
    d_w = np.empty((n, K), np.float64)
    lib().oracle_combine_backward_tokens(K, H, n, w.reshape(-1), dy_bits.reshape(-1),
                                         eo_bits.reshape(-1), d_eo.reshape(-1), d_w.reshape(-1))
    return d_eo, d_w


def dispatch_backward_tokens(d_recv_bits):
    """d_recv rows per token [n,K,H] bf16 bits -> dx [n,H] bf16 bits."""
    d_recv_bits = _c(d_recv_bits, np.uint16)
    n, K, H = d_recv_bits.shape
    dx = np.empty((n, H), np.uint16)
    lib().oracle_dispatch_backward_tokens(K, H, n, d_recv_bits.reshape(-1), dx.reshape(-1))
    return dx


# ---------------------------------------------------------------- expert GEMM
def bf16_from_f64(v):
    """double -> bf16 bits, one round-to-nearest-even on the double."""
    v = _c(v, np.float64)
    out = np.empty(v.shape, np.uint16)
    lib().oracle_bf16_from_f64_array(v.reshape(-1), out.reshape(-1), v.size)
    return out


def row_groups(E, B, C, cu_seqlens, rows):
    """(rank, group) of each global row index rank*C + i under a plan."""
    cu = _c(cu_seqlens, np.int32).reshape(-1, E + B)
    rows = np.asarray(rows, np.int64)
    ranks = rows // C
    groups = np.empty(rows.shape, np.int64)
    for n, (r, i) in enumerate(zip(ranks.tolist(), (rows % C).tolist())):
        groups[n] = lib().oracle_row_group(E, B, np.ascontiguousarray(cu[r]), i)
    return ranks, groups


def expert_gemm_rows(x_bits, mat, w_bits):
    """x [n,H] bf16 bits, mat [n] index into w [nmat,H,Hp] bf16 bits ->
    (y [n,Hp] bf16 bits, s [n,Hp] float64 sums, sabs [n,Hp] sum |x w|)."""
    x_bits = _c(x_bits, np.uint16)
    mat = _c(mat, np.int32)
    w_bits = _c(w_bits, np.uint16)
    n, H = x_bits.shape
    _, H2, Hp = w_bits.shape
    assert H2 == H and mat.shape == (n,)
    y = np.empty((n, Hp), np.uint16)
    s = np.empty((n, Hp), np.float64)
    sabs = np.empty((n, Hp), np.float64)
    lib().oracle_expert_gemm_rows(H, Hp, n, x_bits.reshape(-1), mat, w_bits.reshape(-1),
                                  y.reshape(-1), s.reshape(-1), sabs.reshape(-1))
    return y, s, sabs
