"""Pins for the oracle's E4M3, UE8M0 and bf16 codecs (CPU only).

Each check ties the oracle to something outside itself: the format facts the
pages state ("FP8 W8A8", "Two FP8 representations": E4M3 reaches +-448 and has
NaN, no infinity), torch's own float8_e4m3fn / float8_e8m0fnu / bfloat16
conversions (library routines), exhaustive brute force over the 256 codes, and
invariants that follow from the definitions.
"""
import numpy as np
import pytest
import torch


def torch_e4m3_values():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def torch_e4m3_encode(v: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.asarray(v, dtype=np.float32))
    t = t.clamp(-448.0, 448.0)      # saturation, then torch's RNE conversion
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_decode_matches_torch_all_256(orc):
    ours = orc.e4m3_table()
    ref = torch_e4m3_values()
    nan_ours = np.isnan(ours)
    assert (nan_ours == np.isnan(ref)).all()
    assert (ours[~nan_ours] == ref[~nan_ours]).all()
    # bit-level sign of zeros
    assert np.signbit(ours[0x80]) and not np.signbit(ours[0x00])


def test_decode_page_facts(orc):
    """+-448 is the largest magnitude, there are exactly two NaN codes and no
    infinity ("FP8 W8A8", "Two FP8 representations")."""
    t = orc.e4m3_table()
    finite = t[np.isfinite(t)]
    assert finite.max() == 448.0 and finite.min() == -448.0
    assert np.isnan(t).sum() == 2 and np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    assert not np.isinf(t).any()
    assert t[0x7E] == 448.0 and t[0xFE] == -448.0
    # the 127 non-negative finite codes are strictly increasing
    assert (np.diff(t[:0x7F]) > 0).all()
    # smallest subnormal / smallest normal / one (OCP FP8 E4M3: bias 7, 3 mantissa bits)
    assert t[0x01] == 2.0 ** -9 and t[0x08] == 2.0 ** -6 and t[0x38] == 1.0


def test_encode_roundtrip_all_finite_codes(orc):
    t = orc.e4m3_table()
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    enc = orc.e4m3_encode(t[codes].astype(np.float32))
    assert (enc == codes).all()


def _midpoints(t):
    pos = t[:0x7F]
    mids = (pos[:-1] + pos[1:]) / 2.0           # exact in fp64 and in fp32
    return mids.astype(np.float32)


def test_encode_ties_go_to_even_code(orc):
    t = orc.e4m3_table()
    mids = _midpoints(t)
    enc = orc.e4m3_encode(mids)
    lo = np.arange(0x7E)
    expect = np.where(lo % 2 == 0, lo, lo + 1)
    assert (enc == expect).all()
    # the same on the negative side
    enc_n = orc.e4m3_encode(-mids)
    assert (enc_n == (expect | 0x80)).all()


def test_encode_one_ulp_around_midpoints(orc):
    t = orc.e4m3_table()
    mids = _midpoints(t)
    below = np.nextafter(mids, np.float32(0))
    above = np.nextafter(mids, np.float32(np.inf))
    lo = np.arange(0x7E)
    assert (orc.e4m3_encode(below) == lo).all()
    assert (orc.e4m3_encode(above) == lo + 1).all()


def test_encode_saturation_and_specials(orc):
    vals = np.array([448, 449, 464, 480, 1e30, np.inf, -449, -np.inf, np.nan, 0.0, -0.0],
                    dtype=np.float32)
    enc = orc.e4m3_encode(vals)
    assert list(enc) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0x7F, 0x00, 0x80]


def test_encode_matches_torch_random(orc):
    rng = np.random.default_rng(1234)
    n = 1_000_000
    mag = np.exp2(rng.uniform(-16.0, 10.0, n))
    sign = np.where(rng.random(n) < 0.5, -1.0, 1.0)
    v = (mag * sign).astype(np.float32)
    t = orc.e4m3_table()
    mids = _midpoints(t)
    v = np.concatenate([v, mids, -mids, np.nextafter(mids, np.float32(0)),
                        np.nextafter(mids, np.float32(1e9)), np.float32([2.0 ** -10, 2.0 ** -11])])
    assert (orc.e4m3_encode(v) == torch_e4m3_encode(v)).all()


def test_encode_brute_force_nearest(orc):
    """Exhaustive nearest-value search over the 254 finite codes, independent
    of the oracle's bracketing: the chosen code is a nearest one and, on a tie,
    the even one."""
    t = orc.e4m3_table()
    rng = np.random.default_rng(7)
    v = (np.exp2(rng.uniform(-12.0, 9.0, 20000)) * np.where(rng.random(20000) < 0.5, -1, 1)).astype(np.float32)
    v = np.clip(v, -448, 448)
    enc = orc.e4m3_encode(v)
    finite_codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)])
    vals = t[finite_codes]
    d = np.abs(vals[None, :] - v.astype(np.float64)[:, None])
    best = d.min(axis=1)
    chosen = np.abs(t[enc] - v.astype(np.float64))
    assert (chosen == best).all()
    ties = (d == best[:, None]).sum(axis=1) > 1
    nonzero_tie = ties & (best > 0)
    # on a genuine tie between two magnitudes the low mantissa bit is 0
    assert ((enc[nonzero_tie] & 1) == 0).all()


# ---------------------------------------------------------------- scales
def _amax_sweep():
    base = []
    for e in range(-14, 120):
        p = np.float32(2.0 ** e)
        base += [p, np.nextafter(p, np.float32(0)), np.nextafter(p, np.float32(np.inf))]
        q = np.float32(448.0 * 2.0 ** e)
        base += [q, np.nextafter(q, np.float32(0)), np.nextafter(q, np.float32(np.inf))]
    rng = np.random.default_rng(3)
    base += list(np.exp2(rng.uniform(-13, 100, 20000)).astype(np.float32))
    a = np.array(base, dtype=np.float32)
    return a[(a >= np.float32(1e-4)) & np.isfinite(a)]


def test_scale_f32_is_ieee_division(orc):
    a = _amax_sweep()
    expect = (a / np.float32(448.0)).astype(np.float32)    # numpy IEEE fp32 division
    assert (orc.scale_f32(a).view(np.uint32) == expect.view(np.uint32)).all()


def test_ue8m0_invariants(orc):
    a = _amax_sweep()
    e = orc.scale_ue8m0(a).astype(np.int64)
    s = np.ldexp(1.0, e - 127)
    t = (a / np.float32(448.0)).astype(np.float64)        # the fp32-rounded ratio
    assert (e >= 1).all() and (e <= 254).all()
    assert (s >= t).all()                  # round up
    assert (s / 2 < t).all()               # smallest such power of two
    assert (a.astype(np.float64) / s <= 448.0 * (1 + 2.0 ** -23)).all()


def test_ue8m0_matches_torch_on_powers_of_two(orc):
    a = np.float32(448.0) * np.exp2(np.arange(-20, 100)).astype(np.float32)
    e = orc.scale_ue8m0(a)
    s = torch.from_numpy(np.exp2(np.arange(-20, 100)).astype(np.float32))
    ref = s.to(torch.float8_e8m0fnu).view(torch.uint8).numpy()
    assert (e == ref).all()
    # and the decode of every byte 0..254 matches torch's float8_e8m0fnu
    b = torch.arange(255, dtype=torch.int32).to(torch.uint8)
    ref_vals = b.view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    assert (orc.ue8m0_decode(np.arange(255)) == ref_vals).all()
    assert np.isnan(orc.ue8m0_decode([255])[0])


def test_ue8m0_floor_and_nonfinite(orc):
    assert orc.scale_ue8m0([1e-4])[0] == 105       # 1e-4/448 = 2^-22.03 -> 2^-22
    assert orc.scale_ue8m0([np.inf])[0] == 0xFF
    assert orc.scale_ue8m0([np.nan])[0] == 0xFF


# ---------------------------------------------------------------- bf16
def test_bf16_rne_matches_torch(orc):
    rng = np.random.default_rng(5)
    v = rng.standard_normal(200000).astype(np.float32) * np.exp2(rng.integers(-30, 30, 200000)).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert (orc.bf16_rne(v.astype(np.float64)) == ref).all()
