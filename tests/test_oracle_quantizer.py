"""Pins of the oracle's number formats and the eq. 1 group quantiser.

Each test checks the oracle against something other than itself: exact
rational arithmetic (fractions.Fraction), torch's own bf16 conversion, the
scalar and group error bounds of eqs. 1 and 9 of the SVDQuant technical
review (sections 2.2 and 4.3), and literal nibble layouts.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from synth import f64_to_bf16_bits

HERE = os.path.dirname(os.path.abspath(__file__))


def _rne_fraction(q: Fraction) -> int:
    """Round-half-even of an exact rational (pure Python)."""
    fl = q.numerator // q.denominator
    rem = q - fl
    if rem > Fraction(1, 2):
        return fl + 1
    if rem < Fraction(1, 2):
        return fl
    return fl if fl % 2 == 0 else fl + 1


def _fraction_quantize(group):
    """Eq. 1 on exact rationals: s = fl32(max|z|/7) (the scale is stored in
    fp32), q = clamp(rne(z/s), -8, 7)."""
    m = max(abs(Fraction(float(v))) for v in group)
    s = float(np.float32(float(m / 7)))  # m/7 -> fp64 -> fp32
    # fl32 of the exact quotient, computed independently: fp64 of a rational
    # is correctly rounded by Fraction.__float__, and double rounding m/7 is
    # innocuous (53 >= 2*24+2).
    if s == 0.0:
        return [0] * len(group), 0.0
    S = Fraction(s)
    return [max(-8, min(7, _rne_fraction(Fraction(float(v)) / S))) for v in group], s


def test_round_bf16_matches_torch():
    rng = np.random.default_rng(11)
    x = rng.standard_normal(200000).astype(np.float32) * np.float32(3.7)
    x = np.concatenate([x, rng.standard_normal(1000).astype(np.float32) * np.float32(1e-39),
                        np.array([65504.0, 1e38, 3.3895e38, -3.3895e38], dtype=np.float32)])
    ours = oracle.round_bf16_bits(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_round_bf16_single_rounding_from_f64():
    # 1 + 2^-8 + 2^-40 lies just above the tie between two bf16 values:
    # a single rounding goes up, a detour through fp32 (which drops the
    # 2^-40) lands on the tie and rounds to even (down).
    x = 1.0 + 2.0 ** -8 + 2.0 ** -40
    assert oracle.round_bf16(np.array([x]))[0] == 1.0 + 2.0 ** -7
    # exact ties go to even
    assert oracle.round_bf16(np.array([1.0 + 2.0 ** -8]))[0] == 1.0
    assert oracle.round_bf16(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 1.0 + 2.0 ** -6


def test_quantizer_matches_exact_rationals_on_random_groups():
    rng = np.random.default_rng(3)
    bits = rng.integers(0, 1 << 16, size=(300, 64), dtype=np.uint32).astype(np.uint16)
    vals = oracle.bf16_bits_to_f64(bits)
    vals[~np.isfinite(vals)] = 0.0
    codes, s = oracle.quantize_groups(vals)
    for gi in range(vals.shape[0]):
        ref_codes, ref_s = _fraction_quantize(list(vals[gi]))
        assert s[gi] == ref_s
        assert list(codes[gi]) == ref_codes


def test_quantizer_exhaustive_bf16_patterns():
    """Every finite bf16 bit pattern, placed in groups whose scale comes from
    a planted maximum, quantised by the oracle and by exact rationals."""
    allbits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    v = oracle.bf16_bits_to_f64(allbits)
    v = v[np.isfinite(v)]
    rng = np.random.default_rng(5)
    rng.shuffle(v)
    n = (len(v) // 63) * 63
    body = v[:n].reshape(-1, 63)
    # planted group max: 7 * a power of two times a few mantissas
    plant = rng.choice([7.0, 7.5, 3.5, 0.4375, 1.0], size=(body.shape[0], 1))
    plant *= 2.0 ** rng.integers(-20, 20, size=(body.shape[0], 1))
    grp = np.hstack([body, plant])
    grp = np.clip(grp, -np.abs(plant), np.abs(plant))  # keep planted max
    codes, s = oracle.quantize_groups(grp)
    take = rng.choice(grp.shape[0], size=120, replace=False)
    for gi in take:
        ref_codes, ref_s = _fraction_quantize(list(grp[gi]))
        assert s[gi] == ref_s and list(codes[gi]) == ref_codes
    # whole-table invariants
    assert codes.min() >= -7 and codes.max() <= 7
    err = np.abs(grp - codes * s[:, None])
    assert np.all(err <= s[:, None] / 2)


def test_quantizer_ties_round_half_even():
    s = 0.25                      # m = 1.75 -> s = 1.75/7 = 0.25 exactly
    g = np.zeros(64)
    g[0] = 1.75
    g[1:6] = [0.375, 0.625, -0.375, -0.625, 0.125]   # 1.5s, 2.5s, -1.5s, -2.5s, 0.5s
    codes, sc = oracle.quantize_groups(g[None, :])
    assert sc[0] == s
    assert list(codes[0, :6]) == [7, 2, 2, -2, -2, 0]


def test_quantizer_element_and_group_bounds():
    """|z - q s| <= s/2 (eq. 1 with nearest rounding) and eq. 9:
    ||R - Q(R)||_F <= sqrt(N) / (2 q_max) max|R| per group, q_max = 7."""
    rng = np.random.default_rng(9)
    z = oracle.round_f32(rng.standard_normal((2000, 64)) * np.exp(rng.normal(0, 3, (2000, 1))))
    codes, s = oracle.quantize_groups(z)
    deq = codes * s[:, None]
    assert np.all(np.abs(z - deq) <= s[:, None] / 2)
    assert codes.min() >= -7 and codes.max() <= 7
    fro = np.sqrt(np.sum((z - deq) ** 2, axis=1))
    bound = np.sqrt(64) / (2 * 7) * np.max(np.abs(z), axis=1)
    assert np.all(fro <= bound * (1 + 1e-12))


def test_quantizer_zero_and_underflow_groups():
    codes, s = oracle.quantize_groups(np.zeros((1, 64)))
    assert s[0] == 0 and not codes.any()
    tiny = np.zeros((1, 64))
    tiny[0, 3] = 2.0 ** -149          # smallest fp32 subnormal: m/7 -> 0
    codes, s = oracle.quantize_groups(tiny)
    assert s[0] == 0 and not codes.any()
    # subnormal scale: clamp may act
    g = np.zeros((1, 64))
    g[0, 0] = 7.5 * 2.0 ** -149 * 2    # 15 * 2^-149, s = fl32(15/7 2^-149) = 2 * 2^-149
    g[0, 1] = -g[0, 0]
    codes, s = oracle.quantize_groups(g)
    assert s[0] == 2.0 ** -148
    assert codes[0, 0] == 7 and codes[0, 1] == -8   # 7.5 -> 8 -> clamp 7; -7.5 -> -8


def test_nibble_layout_literal():
    codes = np.array([[1, -1, 7, -8, 0, 3]])
    packed = oracle.pack_nibbles(codes)
    assert list(packed[0]) == [0xF1, 0x87, 0x30]
    assert np.array_equal(oracle.unpack_nibbles(packed), codes)


def test_golden_ratios():
    with open(os.path.join(HERE, "golden", "ratios.json")) as f:
        gold = json.load(f)
    for case in gold["cases"]:
        if "mac_ratio" in case:
            assert oracle.mac_ratio(case["m"], case["n"], case["r"]) == case["mac_ratio"]
        if "storage_ratio" in case:
            rho = oracle.storage_ratio(case["m"], case["n"], case["r"])
            assert rho == case["storage_ratio"]
            assert round(1 / rho, 2) == case["compression"]
    ts = gold["transformer_size"]
    assert round(ts["bf16_gib"] / ts["int4_gib"], 2) == ts["ratio"]


def test_input_generator_rounding_is_rne():
    x = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5e-3])
    ref = torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(f64_to_bf16_bits(x), ref)


@pytest.mark.parametrize("mutant", ["floor", "half_away", "scale_by_8"])
def test_planted_quantizer_mistakes_are_caught(mutant):
    """A wrong quantiser planted on the CPU fails the exact-rational pin."""
    s = 0.25
    g = np.zeros(64)
    g[0] = 1.75
    g[1:6] = [0.375, 0.625, -0.375, -0.65, 0.1]
    ref_codes, _ = _fraction_quantize(list(g))
    if mutant == "floor":
        bad = np.floor(g / s)
    elif mutant == "half_away":
        bad = np.sign(g) * np.floor(np.abs(g / s) + 0.5)
    else:
        bad = np.rint(g / (np.max(np.abs(g)) / 8))
    assert list(bad.astype(int)) != ref_codes
