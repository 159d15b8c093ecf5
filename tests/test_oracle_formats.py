"""Pins of the oracle's bit-level encoders (E2M1 elements, E4M3 block scales).

Each pin checks the oracle against something other than itself: the format
definitions written out as golden tables (tests/golden/), torch's own
float8_e4m3fn conversion (a library routine), and a second rounding algorithm
(scale-to-quantum then rint) that shares nothing with the oracle's
nearest-table-entry search.
"""
import math
import os

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_pairs(name):
    out = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            a, b = line.split()
            out.append((a, b))
    return out


def test_e2m1_decode_matches_spec_table():
    for code, val in _read_pairs("e2m1_codes.txt"):
        v = oracle.e2m1_value(int(code))
        assert v == float(val) and math.copysign(1, v) == math.copysign(1, float(val)), code


def test_e2m1_rne_tie_table():
    for x, code in _read_pairs("e2m1_rne_ties.txt"):
        assert oracle.e2m1_encode(float(x)) == int(code), x


def test_e2m1_grid_round_trips_exactly():
    # every code's value encodes back to the same code (P1 at unit scale)
    for code in range(16):
        assert oracle.e2m1_encode(oracle.e2m1_value(code)) == code


def _e2m1_by_quantum(q: float) -> float:
    """Independent E2M1 RNE: round |q| to a multiple of the binade's quantum
    (0.5 below 2, 1 in [2,4), 2 from 4) with rint (ties to even multiple),
    then saturate to 6."""
    a = abs(q)
    quantum = 0.5 if a < 2 else (1.0 if a < 4 else 2.0)
    r = float(np.rint(a / quantum)) * quantum
    return min(r, 6.0)


def test_e2m1_encoder_against_quantum_rounding():
    rng = np.random.default_rng(1)
    # every bf16 value in [-16, 16] plus random float32 values
    bits = np.arange(0, 1 << 16, dtype=np.uint32)
    vals = (bits << 16).view(np.float32)
    vals = vals[np.isfinite(vals) & (np.abs(vals) <= 16)]
    extra = rng.uniform(-8, 8, 20000).astype(np.float32)
    mag_table = {oracle.e2m1_value(c): c for c in range(8)}
    for q in np.concatenate([vals, extra]):
        q = float(q)
        code = oracle.e2m1_encode(q)
        want_mag = _e2m1_by_quantum(q)
        assert code & 7 == mag_table[want_mag], (q, code)
        assert (code >> 3) == (1 if math.copysign(1, q) < 0 else 0), q


def test_e4m3_decode_matches_spec_table():
    for hx, val in _read_pairs("e4m3_values.txt"):
        v = oracle.e4m3_value(int(hx, 16))
        assert v == float(val) and math.copysign(1, v) == math.copysign(1, float(val)), hx
    assert math.isnan(oracle.e4m3_value(0x7F)) and math.isnan(oracle.e4m3_value(0xFF))


def test_e4m3_decode_matches_torch_for_all_bytes():
    t = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).float()
    for b in range(256):
        tv = float(t[b])
        ov = oracle.e4m3_value(b)
        if math.isnan(tv):
            assert math.isnan(ov)
        else:
            assert ov == tv, b


def test_e4m3_rne_cases():
    for x, hx in _read_pairs("e4m3_rne_cases.txt"):
        assert oracle.e4m3_encode(float(x)) == int(hx, 16), x


def test_e4m3_encoder_against_torch_cast():
    # torch's float32 -> float8_e4m3fn conversion rounds to nearest even; it
    # does not saturate (>= 464 becomes NaN), so compare below 464 and check
    # saturation separately.
    rng = np.random.default_rng(2)
    bits = np.arange(0, 1 << 16, dtype=np.uint32)
    vals = (bits << 16).view(np.float32)
    vals = vals[np.isfinite(vals) & (vals >= 0) & (vals < 464)]
    extra = np.concatenate([rng.uniform(0, 464, 20000), np.exp(rng.uniform(-16, 6, 20000))])
    extra = extra[extra < 464].astype(np.float32)
    allv = np.concatenate([vals, extra])
    want = torch.from_numpy(allv).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v)) for v in allv], np.uint8)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(float(allv[i]), int(got[i]), int(want[i])) for i in bad[:10]]
    for v in [464.0, 465.0, 1e6, 3.0e38]:
        assert oracle.e4m3_encode(v) == 0x7E


def _e4m3_by_quantum(a: float) -> float:
    if a >= 448:
        return 448.0
    if a < 2.0 ** -6:
        quantum = 2.0 ** -9
    else:
        quantum = 2.0 ** (math.floor(math.log2(a)) - 3)
    return min(float(np.rint(a / quantum)) * quantum, 448.0)


def test_e4m3_encoder_against_quantum_rounding():
    rng = np.random.default_rng(3)
    vals = np.concatenate([np.exp(rng.uniform(-12, 7, 20000)), rng.uniform(0, 500, 5000)])
    for a in vals.astype(np.float32):
        a = float(a)
        got = oracle.e4m3_value(oracle.e4m3_encode(a))
        assert got == _e4m3_by_quantum(a), a


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(4)
    v = np.concatenate([rng.standard_normal(50000) * 10.0 ** rng.integers(-30, 30, 50000),
                        [0.0, -0.0, 1.0, 3.0e38, 1e-40]]).astype(np.float32)
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.bf16_from_f64(v.astype(np.float64))
    assert np.array_equal(got, want)
    # exact midpoints between bf16 neighbours (not float32-representable in
    # general when built in float64) resolve to the even pattern
    base = oracle.bf16_to_f64(np.array([0x3F80, 0x3F81, 0x4000], np.uint16))
    ulp = np.array([2.0 ** -7, 2.0 ** -7, 2.0 ** -6])
    mid = base + ulp / 2
    assert list(oracle.bf16_from_f64(mid)) == [0x3F80, 0x3F82, 0x4000]
