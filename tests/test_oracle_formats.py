"""Pins of the oracle's number formats against the OCP E4M3 definition and
against torch's independent casts."""
import numpy as np
import torch

import oracle as O


def test_e4m3_decode_golden(golden):
    g = golden("e4m3_codes.txt")
    for code, vals in g.items():
        v = O.e4m3_decode(np.array([int(code, 16)], np.uint8))[0]
        assert v == float(vals[0]), (code, v)
        if code == "0x80":
            assert np.signbit(v)


def test_e4m3_table_properties():
    pos = O.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    assert np.all(np.diff(pos) > 0)                  # strictly increasing codes 0..126
    assert pos[-1] == 448.0
    assert np.isnan(O.e4m3_decode(np.array([0x7F, 0xFF], np.uint8))).all()
    neg = O.e4m3_decode(np.arange(0x80, 0xFF, dtype=np.uint8))
    assert np.array_equal(neg, -pos)


def test_e4m3_decode_matches_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = O.e4m3_decode(codes.numpy())
    fin = ~np.isnan(ref)
    assert np.array_equal(np.isnan(ours), ~fin)
    assert np.array_equal(ours[fin], ref[fin])


def test_e4m3_encode_roundtrip_and_ties():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF, 0x80)], np.uint8)
    assert np.array_equal(O.e4m3_encode(O.e4m3_decode(codes)), codes)
    # midpoint between 1.0 (0x38, even) and 1.125 (0x39): ties to even -> 0x38
    assert O.e4m3_encode(np.array([1.0625]))[0] == 0x38
    # midpoint between 1.125 (0x39) and 1.25 (0x3A, even) -> 0x3A
    assert O.e4m3_encode(np.array([1.1875]))[0] == 0x3A
    assert O.e4m3_encode(np.array([1e6]))[0] == 0x7E      # saturates to 448
    assert O.e4m3_encode(np.array([-1e6]))[0] == 0xFE
    assert O.e4m3_encode(np.array([2.0 ** -11]))[0] == 0x00  # below half the smallest subnormal


def test_e4m3_encode_matches_torch_random():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(20000) * np.exp2(rng.integers(-12, 9, 20000))
    x = x[np.abs(x) < 448]
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = O.e4m3_encode(x.astype(np.float32).astype(np.float64))
    ref = np.where(ref == 0x80, 0, ref)   # torch keeps -0; the oracle canonicalises to +0
    assert np.array_equal(ours, ref)


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal(50000) * np.exp2(rng.integers(-20, 20, 50000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.bf16_round(x.astype(np.float64)), ref)
