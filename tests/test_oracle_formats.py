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


def _torch_dequant_bits(q, s):
    """bf16(float(e4m3 code) * scale of the code's 128-block), with torch's
    own e4m3 decode, binary32 multiply and round-to-nearest-even cast."""
    n, H = q.shape
    qt = torch.from_numpy(np.ascontiguousarray(q)).view(torch.float8_e4m3fn).to(torch.float32)
    st = torch.from_numpy(np.ascontiguousarray(s)).repeat_interleave(128, dim=1)
    return (qt * st).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16), (qt * st)


def test_dequant_rows_matches_torch_all_codes(oracle_mod):
    """The fp8 identity expert a = bf16(float(q) * s), one scale per 128
    codes of a row (the e4m3 + per-128 fp32 scale payload), against torch.
    Every one of the 256 codes meets every scale; the scales differ per
    block, so a wrong block index (h/128) changes the result, and they are
    chosen so that exact bf16 midpoints occur (ties to even) and the
    rounding goes up somewhere (round-to-nearest, not truncation)."""
    H = 384
    rng = np.random.default_rng(31)
    scales = np.concatenate([
        2.0 ** np.arange(-12, 9, dtype=np.float64),           # powers of two: exact
        1.0 + np.arange(1, 33) * 2.0 ** -8,                   # bf16 midpoints with small codes
        [1.0 + 2.0 ** -8, 3.0 * (1 + 2.0 ** -9), 0.1, 1.0 / 3.0, 448.0 / 3.0, 7e-5],
        rng.uniform(1e-4, 4.0, 60),
    ]).astype(np.float32)
    nblk = H // 128
    rows = []
    srows = []
    for i in range(0, scales.size, nblk):
        sc = scales[i:i + nblk]
        if sc.size < nblk:
            sc = np.concatenate([sc, scales[:nblk - sc.size]])
        for shift in range(nblk):  # each code block meets each scale
            code_row = np.concatenate([np.arange(256), np.arange(128)]).astype(np.uint8)
            code_row = np.roll(code_row, 128 * shift)
            rows.append(code_row)
            srows.append(np.roll(sc, shift))
    q = np.stack(rows)
    s = np.stack(srows).astype(np.float32)
    got = oracle_mod.dequant_rows(q, s)
    ref, prod = _torch_dequant_bits(q, s)
    prod = prod.numpy()
    nan = np.isnan(prod)
    assert nan.sum() == (q == 0x7f).sum() + (q == 0xff).sum()  # the two NaN codes
    assert np.all(np.isnan(oracle_mod.bf16_to_f32(got)[nan]))
    assert np.array_equal(got[~nan], ref[~nan])
    # the cases the scales were picked for did occur
    pbits = prod[~nan].astype(np.float32).view(np.uint32)
    assert np.count_nonzero((pbits & 0xffff) == 0x8000) > 100     # exact ties
    assert np.count_nonzero((pbits & 0xffff) > 0x8000) > 1000      # rounds up
    # the scale of a neighbouring block, or one scale for the whole row, gives
    # other values: the test can tell the block index apart
    qf = torch.from_numpy(q).view(torch.float8_e4m3fn).float().numpy()
    for s_wrong in (np.roll(s, 1, axis=1), np.tile(s[:, :1], (1, nblk))):
        wrong = oracle_mod.bf16_from_f32((qf * np.repeat(s_wrong, 128, axis=1)).astype(np.float32))
        assert not np.array_equal(wrong[~nan], got[~nan])


def test_dequant_rows_inverts_quantisation_within_bound(oracle_mod):
    """Quantise a row with the oracle (scale = amax/448, codes by RNE) and
    dequantise it: every element within 2^-4 relative for e4m3 normals and
    within scale * 2^-10 below them, plus one bf16 rounding (2^-8)."""
    rng = np.random.default_rng(32)
    H = 512
    for it in range(20):
        xf = rng.standard_normal(H) * np.repeat(2.0 ** rng.uniform(-10, 10, H // 128), 128)
        x = oracle_mod.bf16_from_f32(xf.astype(np.float32))
        q, s = oracle_mod.quant_row_e4m3(x)
        a = oracle_mod.bf16_to_f32(oracle_mod.dequant_rows(q[None], s[None])[0]).astype(np.float64)
        xv = oracle_mod.bf16_to_f32(x).astype(np.float64)
        sb = np.repeat(s.astype(np.float64), 128)
        err = np.abs(a - xv)
        normal = np.abs(xv) >= sb * 2.0 ** -6
        tol_n = np.abs(xv) * (2.0 ** -4 + 2.0 ** -8 * (1 + 2.0 ** -4)) * 1.0001
        tol_s = sb * 2.0 ** -10 * 1.0001 + np.abs(a) * 2.0 ** -8
        assert np.all(err[normal] <= tol_n[normal])
        assert np.all(err[~normal] <= tol_s[~normal])
