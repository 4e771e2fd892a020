"""The oracle against the hand-worked example in tests/golden/rrs_worked_example_k8.txt.

The fixture carries its derivation and the passages it follows.  Every stage is
compared on its own: rotation, reorder, group maxima, codes, packed bytes, fp32 scale
bit patterns, exact group products, and Y against its rational value.
"""
import pathlib
import struct
from fractions import Fraction

import numpy as np
import pytest

GOLDEN = pathlib.Path(__file__).parent / "golden" / "rrs_worked_example_k8.txt"


def _load():
    rows = {}
    for line in GOLDEN.read_text().splitlines():
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, _, val = line.partition(":")
        rows.setdefault(key.strip(), []).append(val.split())
    return rows


def _num(rows, key, dtype):
    return np.array([[dtype(v) for v in r] for r in rows[key]])


def _bits(rows, key):
    return np.array([int(v, 16) for v in rows[key][0]], dtype=np.uint32)


def _f32_bits(a):
    return np.asarray(a, np.float32).view(np.uint32)


@pytest.fixture(scope="module")
def ex():
    r = _load()
    d = {k: int(r[k][0][0]) for k in ("M", "K", "N", "G", "n")}
    d["perm"] = np.array([int(v) for v in r["perm"][0]], np.int32)
    d["X"] = _num(r, "X", float).astype(np.float16)
    d["W"] = _num(r, "W", float).astype(np.float16)
    d["rows"] = r
    return d


def test_fixture_inputs_are_exact_fp16(ex):
    r = ex["rows"]
    assert np.array_equal(ex["X"].astype(np.float64), _num(r, "X", float))
    assert np.array_equal(ex["W"].astype(np.float64), _num(r, "W", float))
    assert ex["X"].shape == (ex["M"], ex["K"]) and ex["W"].shape == (ex["N"], ex["K"])


def test_rotation_and_reorder(orc, ex):
    Xrot = orc.rotate(ex["X"], ex["n"])
    assert np.array_equal(Xrot, _num(ex["rows"], "X_rot", float).astype(np.float32))
    Xp = orc.reorder(Xrot, ex["perm"])
    assert np.array_equal(Xp, _num(ex["rows"], "X_prime", float).astype(np.float32))
    assert np.array_equal(orc.group_max(Xp, ex["G"]),
                          np.array([float(v) for v in ex["rows"]["s"][0]], np.float32))


def test_activation_codes_scales_and_bytes(orc, ex):
    codes, qX, s, st = orc.smooth_quant(ex["X"], ex["G"], ex["n"], ex["perm"])
    r = ex["rows"]
    assert np.array_equal(codes, _num(r, "codes_x", int).astype(np.int8))
    assert np.array_equal(qX, _num(r, "qX_hex", lambda v: int(v, 16)).astype(np.uint8))
    assert np.array_equal(s, np.array([float(v) for v in r["s"][0]], np.float32))
    assert np.array_equal(_f32_bits(st), _bits(r, "scale_t_bits"))
    assert np.array_equal(orc.unpack(qX, ex["K"]), codes)


def test_weight_codes_scales_and_bytes(orc, ex):
    codes, qW, sw = orc.prepare_weights(ex["W"], ex["n"], ex["perm"])
    r = ex["rows"]
    assert np.array_equal(codes, _num(r, "codes_w", int).astype(np.int8))
    assert np.array_equal(qW, _num(r, "qW_hex", lambda v: int(v, 16)).astype(np.uint8))
    assert np.array_equal(_f32_bits(sw), _bits(r, "scale_w_bits"))


def test_group_products_and_output(orc, ex):
    _, qX, s, st = orc.smooth_quant(ex["X"], ex["G"], ex["n"], ex["perm"])
    _, qW, sw = orc.prepare_weights(ex["W"], ex["n"], ex["perm"])
    r = ex["rows"]
    P = orc.group_partials(qX, qW, ex["G"])
    assert np.array_equal(P[0], _num(r, "P_0", int)) and np.array_equal(P[1], _num(r, "P_1", int))
    Y, _ = orc.linear_rows(qX, s, st, qW, sw, ex["G"])
    want = np.array([[float(Fraction(v)) for v in row] for row in r["Y_rational"]])
    # the fp32 scales are within 5e-8 relative of 1/7, 1/28 and 8/7
    assert np.allclose(Y.astype(np.float64), want, rtol=1e-6, atol=0.0)


def test_scale_bit_patterns_are_the_fp32_roundings(ex):
    """The stored hex words are the correctly rounded fp32 values of 1/7, 1/28, 8/7."""
    def rn32(q: Fraction) -> int:
        # round-to-nearest-even of a positive rational to fp32, by integer arithmetic
        e = q.numerator.bit_length() - q.denominator.bit_length()
        if Fraction(2) ** e > q:
            e -= 1
        m = q / Fraction(2) ** e * 2 ** 23          # in [2^23, 2^24)
        fl = m.numerator // m.denominator
        rem = m - fl
        if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2):
            fl += 1
        return ((e + 127) << 23) | (fl - (1 << 23))
    assert rn32(Fraction(1, 7)) == 0x3E124925
    assert rn32(Fraction(1, 28)) == 0x3D124925
    assert rn32(Fraction(8, 7)) == 0x3F924925
    assert struct.unpack("<I", struct.pack("<f", 1 / 7))[0] == 0x3E124925
