"""Pins of the oracle's MXFP4 exponent rules (CPU only).

The rules are the floor(log2(x / 6)) family of "kirillbilchenko/Nex-N2.5-mini-
MXFP4-MxWave", Quantization method: the floor rule, the smallest exponent that
avoids clipping (ceil), the OCP MX shared-exponent rule, and the card's MSE
scale search (candidates floor(log2(p99.5 / 6)) - 4 ... + 1 plus the no-clip
exponent, lowest weight MSE wins).  Every pin here is computed independently
of the oracle's code: brute force over all bf16 magnitudes, numpy's own
percentile, and exact rational arithmetic.
"""
from fractions import Fraction

import numpy as np
import pytest

from conftest import parse_numbers
from oracle import moe_oracle as o

GRID = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3), Fraction(4),
        Fraction(6)]


def all_positive_bf16():
    bits = np.arange(1, 0x7F80, dtype=np.uint16)   # +subnormals .. largest finite
    return bits, o.bf16_to_f64(bits)


def pow2(e):
    return Fraction(2) ** e


def test_ceil_rule_is_the_smallest_non_clipping_exponent():
    _, amax = all_positive_bf16()
    e = o.mx_exponent_ceil(amax)
    for a, ei in zip(amax.tolist(), e.tolist()):
        fa = Fraction(a)
        assert fa <= 6 * pow2(ei)                       # nothing clips
        if ei > -127:
            assert fa > 6 * pow2(ei - 1)                # and one less would clip


def test_ocp_rule_is_floor_log2_minus_two():
    _, amax = all_positive_bf16()
    e = o.mx_exponent_ocp(amax)
    for a, ei in zip(amax.tolist(), e.tolist()):
        fa = Fraction(a)
        if ei > -127:
            assert pow2(ei + 2) <= fa < pow2(ei + 3)
        else:
            assert fa < pow2(-124)


def test_p995_is_numpy_linear_percentile():
    rng = np.random.default_rng(5)
    blocks = np.abs(o.bf16_round(rng.standard_normal((500, 32)) * rng.uniform(0.01, 10, (500, 1))))
    ours = o.mx_p995(blocks)
    ref = np.percentile(blocks, 99.5, axis=-1)          # default: linear interpolation
    assert np.allclose(ours, ref, rtol=1e-14, atol=0)


def exact_nearest(v):
    """E2M1 grid point nearest |v| (Fraction), ties to the even code index."""
    a = abs(v)
    best = min(range(8), key=lambda i: (abs(a - GRID[i]), i % 2))
    return GRID[best] if v >= 0 else -GRID[best]


def exact_sq_error(block, e):
    s = pow2(e)
    return sum((w - exact_nearest(w / s) * s) ** 2 for w in block)


def exact_candidates(block):
    """The card's candidate set, derived without the oracle: e0 from numpy's
    99.5th percentile (exact comparison of 6 * 2^e against it), the no-clip
    exponent by search."""
    mags = [abs(w) for w in block]
    amax = max(mags)
    p = Fraction(float(np.percentile(np.array([float(m) for m in mags]), 99.5)))
    e0 = 0
    while 6 * pow2(e0) > p:
        e0 -= 1
    while 6 * pow2(e0 + 1) <= p:
        e0 += 1
    enc = -200
    while amax > 6 * pow2(enc):
        enc += 1
    return sorted({min(127, max(-127, c)) for c in list(range(e0 - 4, e0 + 2)) + [enc]})


def test_mse_rule_is_the_exact_argmin_over_the_candidates():
    rng = np.random.default_rng(11)
    blocks = []
    for i in range(200):
        kind = i % 5
        if kind == 4:
            # the block max just past a power-of-two boundary 6 * 2^k and the
            # rest below it: the no-clip exponent is two above floor(log2(p99.5 / 6)),
            # so the search weighs a slight clip at e0 + 1 against a coarser grid
            k = int(rng.integers(-8, 4))
            b = rng.uniform(0.2, 0.7, 32) * 6 * 2.0 ** (k + 1)
            b[0] = 6 * 2.0 ** (k + 1) * rng.uniform(1.01, 1.15)
            b *= rng.choice([-1, 1], 32)
        elif kind == 0:
            b = rng.standard_normal(32) * 0.02
        elif kind == 1:
            b = rng.standard_t(2, 32) * 0.05              # heavy tails: outliers
        elif kind == 2:
            b = rng.integers(-12, 13, 32) * 0.125          # many exact ties
        else:
            b = np.zeros(32)
            b[rng.integers(0, 32, 3)] = rng.standard_normal(3)   # mostly zero
        blocks.append(b)
    for k in (-20, -3, 0, 5):
        # a max in (14, 14.2) * 2^k with p99.5 below 12 * 2^k: the no-clip
        # exponent k + 2 (grid point 16 * 2^k) beats every e0 - 4 .. e0 + 1
        b = np.zeros(32)
        b[7] = 14.125 * 2.0 ** k
        b[20:23] = np.array([0.25, -0.125, 0.0]) * 2.0 ** k
        blocks.append(b)
    bits = o.f64_to_bf16(np.stack(blocks))
    vals = o.bf16_to_f64(bits)
    got = o.mx_exponent_mse(vals)
    assert np.array_equal(got[-4:], np.array([-18, -1, 2, 7]))  # e = k + 2
    for row, e in zip(vals, got.tolist()):
        block = [Fraction(float(w)) for w in row]
        if max(abs(w) for w in block) == 0:
            assert e == -127
            continue
        cands = exact_candidates(block)
        errs = {c: exact_sq_error(block, c) for c in cands}
        best = min(errs.values())
        assert e == min(c for c in cands if errs[c] == best)
        # the search never does worse than the floor or the no-clip rule
        amax = max(abs(w) for w in block)
        ef = int(o.mx_exponent(np.float64(amax)))
        ec = int(o.mx_exponent_ceil(np.float64(amax)))
        assert errs[e] <= exact_sq_error(block, ef)
        assert errs[e] <= exact_sq_error(block, ec)


def test_mse_rule_hand_example(golden):
    g = golden("mxfp4_mse_hand_example.txt")
    block = np.array(parse_numbers(g["block"]), dtype=np.float64)
    block = np.concatenate([block, np.zeros(32 - block.size)])
    bits = o.f64_to_bf16(block[None, None, :])
    for rule, key in ((o.MX_RULE_FLOOR, "floor"), (o.MX_RULE_CEIL, "ceil"), (o.MX_RULE_MSE, "mse")):
        codes, scales = o.pack_mxfp4(bits, rule)
        assert int(scales[0, 0, 0]) == parse_numbers(g[f"{key}_scale_byte"])[0]
        deq = o.dequant_mxfp4(codes, scales)[0, 0, :len(parse_numbers(g[f"{key}_dequant"]))]
        assert np.array_equal(deq, np.array(parse_numbers(g[f"{key}_dequant"]), dtype=np.float64))


@pytest.mark.parametrize("rule", [o.MX_RULE_CEIL, o.MX_RULE_OCP, o.MX_RULE_MSE])
def test_rules_never_clip_less_accurately_than_floor_on_gaussian_weights(rule):
    """Relative Frobenius round-trip error on N(0, 0.02) weights: the floor rule
    clips every block maximum (about 21 %); the others stay near 11-12 %."""
    rng = np.random.default_rng(2)
    bits = o.f64_to_bf16(rng.standard_normal((64, 512)) * 0.02)
    w = o.bf16_to_f64(bits)
    def rel(r):
        return np.linalg.norm(o.dequant_mxfp4(*o.pack_mxfp4(bits, r)) - w) / np.linalg.norm(w)
    assert 0.19 < rel(o.MX_RULE_FLOOR) < 0.23
    assert rel(rule) < 0.125
    if rule == o.MX_RULE_MSE:
        assert rel(rule) <= min(rel(o.MX_RULE_CEIL), rel(o.MX_RULE_OCP))


def test_zero_block_and_codes_on_grid_for_every_rule():
    rng = np.random.default_rng(4)
    w = rng.standard_normal((3, 128)) * 0.3
    w[1, 32:64] = 0.0
    bits = o.f64_to_bf16(w)
    for rule in (o.MX_RULE_FLOOR, o.MX_RULE_CEIL, o.MX_RULE_OCP, o.MX_RULE_MSE):
        codes, scales = o.pack_mxfp4(bits, rule)
        assert scales[1, 1] == 0                         # e = -127 for the zero block
        nib = o.unpack_nibbles(codes)
        assert np.all(nib[1, 32:64] == 0)
        assert np.all(scales <= 254)                     # 0xFF (NaN scale) never produced


# ---------------------------------------------------------------- planted mistakes

_orig_p995 = o.mx_p995
_orig_ceil = o.mx_exponent_ceil
_orig_ocp = o.mx_exponent_ocp
_orig_sq = o.mx_block_sq_error


def _mse_variant(drop_noclip=False, ties_high=False, span=(-4, 2)):
    def rule(blocks):
        blocks = np.asarray(blocks, np.float64)
        mags = np.abs(blocks)
        amax = mags.max(-1)
        e0 = o.floor_log2_div6(np.where(amax > 0, o.mx_p995(mags), 6.0))
        cands = [np.clip(e0 + d, -127, 127) for d in range(*span)]
        if not drop_noclip:
            cands.append(o.mx_exponent_ceil(amax))
        best_e, best = cands[0], o.mx_block_sq_error(blocks, cands[0])
        for c in cands[1:]:
            err = o.mx_block_sq_error(blocks, c)
            better = (err <= best) if ties_high else (err < best)
            best_e, best = np.where(better, c, best_e), np.where(better, err, best)
        return np.where(amax > 0, best_e, -127)
    return rule


MX_MUTANTS = {
    "mse without the no-clip candidate": {"mx_exponent_mse": _mse_variant(drop_noclip=True)},
    "mse ties to the larger exponent": {"mx_exponent_mse": _mse_variant(ties_high=True)},
    "mse candidates without e0 + 1": {"mx_exponent_mse": _mse_variant(span=(-4, 1))},
    "p99.5 read as the block max": {"mx_p995": lambda m: np.max(np.asarray(m, np.float64), axis=-1)},
    "p99.5 interpolated the other way": {"mx_p995": lambda m: (lambda v: v[..., 31] + (v[..., 30] - v[..., 31])
                                                               * 0.845)(np.sort(np.asarray(m, np.float64), -1))},
    "ceil rule one too high": {"mx_exponent_ceil": lambda a: np.where(np.asarray(a) > 0, _orig_ceil(a) + 1, -127)},
    "ocp rule without the -2": {"mx_exponent_ocp": lambda a: np.where(np.asarray(a) > 0, _orig_ocp(a) + 2, -127)},
    "squared error drops clipped elements": {"mx_block_sq_error": lambda b, e: _orig_sq(
        np.where(np.abs(b) > 6 * np.ldexp(1.0, e)[..., None], 0.0, b), e)},
}


def _run_mx_pins():
    from conftest import read_golden
    failures = []
    for name, fn in sorted(globals().items()):
        if not name.startswith("test_") or name.startswith("test_planted") or name.startswith("test_unmutated"):
            continue
        runs = [[r] for r in (o.MX_RULE_CEIL, o.MX_RULE_OCP, o.MX_RULE_MSE)] \
            if name == "test_rules_never_clip_less_accurately_than_floor_on_gaussian_weights" else [[]]
        if name == "test_mse_rule_hand_example":
            runs = [[read_golden]]
        for a in runs:
            try:
                with np.errstate(all="ignore"):
                    fn(*a)
            except Exception:  # an assertion or a crash both count as caught
                failures.append(name)
    return failures


@pytest.mark.parametrize("mutant", sorted(MX_MUTANTS))
def test_planted_mx_rule_mistake_is_caught(mutant, monkeypatch):
    for attr, fn in MX_MUTANTS[mutant].items():
        monkeypatch.setattr(o, attr, fn)
    assert _run_mx_pins(), f"no pin noticed the planted mistake: {mutant}"


def test_unmutated_mx_rules_pass_the_same_pins():
    assert _run_mx_pins() == []
