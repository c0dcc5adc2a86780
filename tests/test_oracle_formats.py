"""Pins for the oracle's number formats against torch's CPU conversions and
against brute-force nearest-value search.

bf16: round to nearest even of the upper 16 bits of binary32.
e4m3: OCP FP8 E4M3 (bias 7, max 448, no infinity), round to nearest even,
saturating to +-448.
"""
import numpy as np
import torch


def _torch_bf16_bits(v):
    return torch.from_numpy(np.asarray(v, np.float32)).to(torch.bfloat16).view(torch.int16) \
        .numpy().view(np.uint16)


def test_bf16_matches_torch_random(oracle_mod):
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 2**32, 2_000_000, dtype=np.uint64).astype(np.uint32)
    v = bits.view(np.float32)
    v = v[np.isfinite(v)]
    assert np.array_equal(oracle_mod.bf16_from_f32(v), _torch_bf16_bits(v))
    g = rng.standard_normal(1_000_000).astype(np.float32) * 3
    assert np.array_equal(oracle_mod.bf16_from_f32(g), _torch_bf16_bits(g))


def test_bf16_ties_to_even(oracle_mod):
    # exact midpoints between consecutive bf16 values: low half = 0x8000
    hi = np.arange(0x3f00, 0x4100, dtype=np.uint32)
    v = ((hi << 16) | 0x8000).view(np.float32)
    got = oracle_mod.bf16_from_f32(v).astype(np.uint32)
    expect = np.where(hi % 2 == 0, hi, hi + 1)
    assert np.array_equal(got, expect)
    assert np.array_equal(got, _torch_bf16_bits(v))
    # largest finite rounds up to infinity only above the midpoint
    big = np.array([0x7f7f7fff, 0x7f7f8000, 0x7f7f8001], np.uint32).view(np.float32)
    assert oracle_mod.bf16_from_f32(big).tolist() == [0x7f7f, 0x7f80, 0x7f80]


def _torch_e4m3_decode_all():
    codes = torch.arange(256, dtype=torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float32).numpy()


def test_e4m3_decode_matches_torch(oracle_mod):
    ours = oracle_mod.e4m3_to_f32(np.arange(256))
    ref = _torch_e4m3_decode_all()
    finite = np.isfinite(ref)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    assert np.array_equal(ours[finite], ref[finite])
    assert ref[0x7e] == 448.0 and ref[0x01] == 2.0 ** -9 and ref[0x08] == 2.0 ** -6


def test_e4m3_roundtrip_all_codes(oracle_mod):
    vals = _torch_e4m3_decode_all()
    codes = np.arange(256)
    ok = np.isfinite(vals)
    got = oracle_mod.e4m3_from_f32(vals[ok])
    exp = codes[ok].astype(np.uint8)
    # -0 and +0 both round-trip to their own sign
    assert np.array_equal(got, exp)


def test_e4m3_nearest_brute_force(oracle_mod):
    """Every encoding equals the nearest finite code by exhaustive search,
    ties to the even code, values >= 448 in magnitude saturating."""
    table = _torch_e4m3_decode_all()
    pos_codes = np.array([c for c in range(0x7f)], np.int64)  # 0x00..0x7e finite, >= 0
    pos_vals = table[pos_codes].astype(np.float64)
    rng = np.random.default_rng(3)
    mags = np.concatenate([
        rng.uniform(0, 2 ** -6, 20000), rng.uniform(0, 1, 20000),
        2.0 ** rng.uniform(-12, 9.2, 60000),
        (pos_vals[:-1] + pos_vals[1:]) / 2,  # exact midpoints
        np.nextafter((pos_vals[:-1] + pos_vals[1:]) / 2, 0),
        np.nextafter((pos_vals[:-1] + pos_vals[1:]) / 2, 1e9),
        [448.0, 449.0, 463.9, 464.0, 500.0, 1e6, 0.0]]).astype(np.float32)
    signs = np.where(rng.random(mags.size) < 0.5, -1.0, 1.0).astype(np.float32)
    v = mags * signs
    got = oracle_mod.e4m3_from_f32(v)
    a = np.abs(v.astype(np.float64))
    dist = np.abs(a[:, None] - pos_vals[None, :])
    best = dist.min(axis=1, keepdims=True)
    cand = dist == best
    # ties: pick the candidate with an even code (even mantissa)
    even = cand & (pos_codes[None, :] % 2 == 0)
    pick = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    expect = pos_codes[pick]
    expect = np.where(a >= 448.0, 0x7e, expect)
    expect = expect | np.where(np.signbit(v), 0x80, 0)
    assert np.array_equal(got.astype(np.int64), expect)


def test_e4m3_matches_torch_in_range(oracle_mod):
    rng = np.random.default_rng(5)
    v = (rng.standard_normal(500_000) * 60).astype(np.float32)
    v = v[np.abs(v) <= 448]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle_mod.e4m3_from_f32(v), ref)
