"""E4M3 input preparation (OCP 8-bit floating point, variant without
infinities: bias 7, 3 mantissa bits, max 448, S.1111.111 = NaN) pinned to the
format's definition, on CPU."""
import numpy as np
import pytest

import synth


def test_decode_known_codes():
    known = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0, 0x39: 1.125,
             0x3F: 1.875, 0x40: 2.0, 0x7E: 448.0, 0xB8: -1.0, 0xFE: -448.0, 0x80: -0.0}
    got = synth.e4m3_to_f32(np.array(list(known), dtype=np.uint8))
    assert got.tolist() == list(known.values())
    assert np.isnan(synth.e4m3_to_f32(np.array([0x7F, 0xFF], dtype=np.uint8))).all()


def test_every_finite_code_round_trips_and_is_exact_in_bf16():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = synth.e4m3_to_f32(codes)
    assert np.array_equal(synth.f32_to_e4m3(vals), codes)
    # exact in bf16: rounding to bf16 and back changes nothing
    assert np.array_equal(synth.bf16_to_f32(synth.f32_to_bf16(vals)), vals)
    pos = vals[(codes < 0x80)]
    assert np.all(np.diff(pos) > 0)  # codes 0..126 increase strictly


def test_rounding_ties_and_saturation():
    # ties go to the even code: 1.0625 halfway 1.0 (0x38) / 1.125 (0x39) -> 0x38;
    # 1.1875 halfway 1.125 / 1.25 (0x3A) -> 0x3A
    cases = {1.0625: 0x38, 1.1875: 0x3A, 1.06: 0x38, 1.07: 0x39, 448.0: 0x7E, 460.0: 0x7E, 1e6: 0x7E,
             -1e6: 0xFE, 2.0 ** -10: 0x00, 3 * 2.0 ** -11: 0x01, 2.0 ** -10 * 1.0001: 0x01, -2.0 ** -12: 0x80,
             0.0: 0x00}
    got = synth.f32_to_e4m3(np.array(list(cases), dtype=np.float32))
    assert got.tolist() == list(cases.values())


def test_brute_force_nearest_on_random_values():
    rng = np.random.default_rng(5)
    x = (rng.standard_normal(20000) * np.exp2(rng.uniform(-12, 10, 20000))).astype(np.float32)
    codes = synth.f32_to_e4m3(x)
    table = synth.e4m3_to_f32(np.arange(127, dtype=np.uint8)).astype(np.float64)
    a = np.minimum(np.abs(x.astype(np.float64)), 448.0)
    err = np.abs(synth.e4m3_to_f32(codes).astype(np.float64) - np.sign(x) * a)
    best = np.min(np.abs(table[None, :] - a[:, None]), axis=1)
    assert np.array_equal(err, best)


def test_per_tensor_quantisation_uses_the_full_range():
    q, k, v = synth.generate(synth.TINY)
    codes, inv, descale = synth.quantize_e4m3(q)
    x = synth.bf16_to_f32(q)
    assert np.max(np.abs(synth.e4m3_to_f32(codes))) == pytest.approx(448.0, rel=0.07)
    rel = np.abs(synth.e4m3_to_f32(codes) * descale - x) / np.maximum(np.abs(x), 1e-3)
    assert np.median(rel[np.abs(x) > 0.1]) < 2 ** -4
