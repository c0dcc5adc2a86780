"""Pins for the oracle's grouped expert GEMM and its double -> bf16 rounding.

The GEMM's definition (a row of rank r in group g times row g of rank r's
[E+B, H, H'] view; [ainovat], the framework-contract paragraph) is pinned by
results that hold whatever the implementation: scaled identities and
permutations move inputs exactly, a rank-one weight factorises the product,
the row -> group map must return the expert each row was routed to, and the
single rounding from binary64 must agree with the (separately pinned) binary32
encoder wherever the two coincide and differ where a binary32 step would
round twice."""
import numpy as np
import pytest

import oracle
from dispatch_moonep_plan_b200 import workloads as wl


def _bits(v):
    return oracle.bf16_from_f32(np.asarray(v, np.float32))


def _vals(bits):
    return oracle.bf16_to_f32(bits).astype(np.float64)


def test_f64_rounding_matches_f32_encoder_on_floats():
    rng = np.random.default_rng(0)
    f = np.concatenate([rng.standard_normal(20000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 20000),
                        np.array([0.0, -0.0, 1.0, 3.0e38, 3.3e38, -3.4e38, 1e-40, 2 ** -133, 2 ** -134 * 3],
                                 np.float32)])
    f = f.astype(np.float32)
    assert np.array_equal(oracle.bf16_from_f64(f.astype(np.float64)), oracle.bf16_from_f32(f))


def test_f64_rounding_is_a_single_rounding():
    # 1 + 2^-8 + 2^-40 is above the midpoint between 1 and 1 + 2^-7: one
    # rounding goes up; a binary32 intermediate would lose 2^-40 and then
    # round the exact tie to even (down).
    v = np.array([1 + 2 ** -8 + 2 ** -40, 1 + 2 ** -8, -(1 + 2 ** -8 + 2 ** -40)])
    got = oracle.bf16_from_f64(v)
    assert _vals(got).tolist() == [1 + 2 ** -7, 1.0, -(1 + 2 ** -7)]
    assert _vals(oracle.bf16_from_f32(v.astype(np.float32)))[0] == 1.0
    # overflow threshold: the largest bf16 is (2 - 2^-7) 2^127; the midpoint
    # to 2^128 and above rounds to infinity
    big = (2 - 2 ** -7) * 2.0 ** 127
    mid = (2 - 2 ** -8) * 2.0 ** 127
    out = _vals(oracle.bf16_from_f64(np.array([big, mid - 2.0 ** 100, mid, 1e300, np.nan])))
    assert out[0] == big and out[1] == big and np.isinf(out[2]) and np.isinf(out[3])
    assert np.isnan(out[4])


def test_scaled_identity_and_permutation_move_inputs_exactly():
    rng = np.random.default_rng(1)
    H = 64
    x = _bits(rng.standard_normal((7, H)))
    eye = np.eye(H)
    perm = rng.permutation(H)
    P = np.zeros((H, H))
    P[np.arange(H), perm] = 1.0  # row h has its 1 in column perm[h]
    w = np.stack([_bits(eye * 4.0), _bits(P), _bits(eye * -0.5)])
    mat = np.array([0, 1, 2, 1, 0, 2, 1], np.int32)
    y, s, _ = oracle.expert_gemm_rows(x, mat, w)
    xv = _vals(x)
    for i, m in enumerate(mat):
        if m == 0:
            assert np.array_equal(_vals(y[i]), xv[i] * 4.0)
        elif m == 2:
            assert np.array_equal(_vals(y[i]), xv[i] * -0.5)
        else:
            out = np.empty(H)
            out[perm] = xv[i]  # column perm[h] receives x[h]
            assert np.array_equal(_vals(y[i]), out)
            assert np.array_equal(s[i], out)


def test_rank_one_weight_factorises():
    # W = v z^T with small integers: x W = (x . v) z^T, every partial sum an
    # exact integer; |result| < 256 so bf16 holds it exactly.
    rng = np.random.default_rng(2)
    H, Hp = 96, 40
    x = rng.integers(-2, 3, (9, H)).astype(np.float64)
    v = np.zeros(H)
    v[rng.choice(H, 5, replace=False)] = rng.integers(-2, 3, 5)
    z = rng.integers(-3, 4, Hp).astype(np.float64)
    w = _bits(np.outer(v, z))[None]
    y, s, sabs = oracle.expert_gemm_rows(_bits(x), np.zeros(9, np.int32), w)
    expect = np.outer(x @ v, z)
    assert np.abs(expect).max() < 256
    assert np.array_equal(_vals(y), expect)
    assert np.array_equal(s, expect)
    assert np.array_equal(sabs, np.outer(np.abs(x) @ np.abs(v), np.abs(z)))


def test_zero_rows_and_signed_zero():
    x = np.zeros((2, 64), np.uint16)
    w = _bits(np.ones((1, 64, 128)))
    y, s, _ = oracle.expert_gemm_rows(x, np.zeros(2, np.int32), w)
    assert not y.any() and not s.any()


@pytest.mark.parametrize("rule", [0, 1, 2])
def test_row_groups_return_the_routed_expert(rule):
    rng = np.random.default_rng(10 + rule)
    checked = 0
    for it in range(40):
        c = wl.random_small_cfg(rng, H=8)
        c["B"] = 16
        idx, _ = wl.routing(c, seed=it)
        pl = oracle.plan(c["R"], c["S"], c["E"], c["K"], c["B"], idx, rule=rule)
        if pl["status"] != 0:
            continue
        C = c["S"] * c["K"]
        rows = np.arange(c["R"] * C)
        ranks, groups = oracle.row_groups(c["E"], c["B"], C, pl["cu_seqlens"], rows)
        se = pl["slot_expert"].reshape(c["R"], c["B"])
        experts = np.where(groups < c["E"], groups, se[ranks, np.maximum(groups - c["E"], 0)])
        assert np.array_equal(experts, idx.reshape(-1)[pl["src_of_row"]])
        Er = c["E"] // c["R"]
        home = groups < c["E"]
        assert np.all(groups[home] // Er == ranks[home])  # home groups are the rank's experts
        checked += 1
    assert checked > 20
