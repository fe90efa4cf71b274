"""Pins of the oracle's NVFP4 (W4A16) packer and dequantiser (CPU only).

Format facts from "primitive-ai/Nex-N2.5-mini-mixed-NVFP4-FP8", What's
quantized to what: NVFP4 experts with group 16; gate and up share one
weight_global_scale per expert; weights-only round-to-nearest.  The E4M3
scale values are pinned to torch's float8_e4m3fn type (an independent
library conversion), the block maximum and global-scale relations by
invariants, the whole pipeline by a hand-worked fixture.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

from conftest import parse_numbers
from oracle import moe_oracle as o


def torch_e4m3(codes):
    return torch.tensor(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)


def test_e4m3_values_match_torch_float8():
    codes = np.arange(0x7F)
    assert np.array_equal(o.e4m3_value(codes), torch_e4m3(codes))


def test_e4m3_rounding_matches_torch_and_exact_nearest():
    rng = np.random.default_rng(3)
    t = np.concatenate([rng.uniform(0, 460, 4000), np.exp(rng.uniform(np.log(1e-4), np.log(448), 4000)),
                        o.e4m3_value(np.arange(0x7F)),                         # exact grid points
                        (o.e4m3_value(np.arange(1, 0x7F)) + o.e4m3_value(np.arange(0x7E))) / 2])  # exact ties
    t = t.astype(np.float32).astype(np.float64)
    got = o.e4m3_nearest(t)
    below = t <= 448
    ref = torch.tensor(t[below], dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got[below], ref)
    assert np.all(got[~below] == 0x7E)                      # saturation at 448
    grid = [Fraction(float(v)) for v in o.e4m3_value(np.arange(0x7F))]
    for x, c in list(zip(t.tolist(), got.tolist()))[::37]:
        fx = Fraction(x)
        best = min(range(0x7F), key=lambda i: (abs(fx - grid[i]), i % 2))
        assert c == (best if fx <= 448 else 0x7E)


def test_global_scale_puts_the_matrix_max_block_at_448():
    rng = np.random.default_rng(8)
    w = rng.standard_normal((4, 64, 256)) * rng.uniform(0.001, 10, (4, 1, 1))
    bits = o.f64_to_bf16(w)
    codes, (scales, g) = o.pack_nvfp4(bits)
    vals = o.bf16_to_f64(bits)
    for e in range(4):
        amax = np.max(np.abs(vals[e]))
        assert g[e] == np.float32(amax) / np.float32(2688.0)
        blocks = np.abs(vals[e]).reshape(64, 16, 16).max(-1)
        r, b = np.unravel_index(np.argmax(blocks), blocks.shape)
        assert scales[e, r, b] == 0x7E                        # E4M3 448


def test_codes_on_grid_and_error_band_on_gaussian_weights():
    rng = np.random.default_rng(2)
    bits = o.f64_to_bf16(rng.standard_normal((2, 64, 512)) * 0.02)
    codes, sg = o.pack_nvfp4(bits)
    w = o.bf16_to_f64(bits)
    deq = o.dequant_nvfp4(codes, sg)
    assert np.array_equal(o.bf16_round(deq), deq)
    rel = np.linalg.norm(deq - w) / np.linalg.norm(w)
    # group 16 with E4M3 scales: finer than MXFP4's group 32 (about 11-12 % there)
    assert 0.07 < rel < 0.11
    # each block's magnitude never exceeds 6 times its multiplier (rounded to bf16)
    d = o.nv_multiplier(sg[0], sg[1])
    assert np.all(np.abs(deq).reshape(2, 64, 32, 16).max(-1) <= o.bf16_round(6 * d))


def test_block_values_are_bf16_multiples_of_one_unit():
    """Within a block every dequantised value is bf16(code * u), u the value of
    a code-1 element of the same block: the block has one bf16 multiplier."""
    rng = np.random.default_rng(12)
    bits = o.f64_to_bf16(rng.standard_normal((1, 256, 256)) * rng.uniform(0.003, 3.0))
    codes, sg = o.pack_nvfp4(bits)
    nib = o.unpack_nibbles(codes).reshape(-1, 16)
    deq = o.dequant_nvfp4(codes, sg).reshape(-1, 16)
    mag = o.E2M1_GRID[nib & 7]
    checked = 0
    for b in range(nib.shape[0]):
        one = np.nonzero((nib[b] & 7) == 2)[0]          # magnitude code 2 = value 1.0
        if one.size == 0:
            continue
        u = abs(deq[b, one[0]])
        assert np.array_equal(np.abs(deq[b]), o.bf16_round(mag[b] * u))
        checked += 1
    assert checked > 1000


def test_gate_and_up_share_one_global_scale():
    """A fused gate_up matrix [2I, H] has one scale: the max of what its two
    halves would get on their own (the card: vLLM keeps the maximum)."""
    rng = np.random.default_rng(9)
    gate = rng.standard_normal((32, 128)) * 0.02
    up = rng.standard_normal((32, 128)) * 0.05
    bits = o.f64_to_bf16(np.concatenate([gate, up])[None])
    _, (_, g) = o.pack_nvfp4(bits)
    _, (_, g_gate) = o.pack_nvfp4(o.f64_to_bf16(gate))
    _, (_, g_up) = o.pack_nvfp4(o.f64_to_bf16(up))
    assert g[0] == max(g_gate, g_up)


def test_zero_matrix_packs_to_zero():
    codes, (scales, g) = o.pack_nvfp4(np.zeros((2, 16, 64), np.uint16))
    assert np.all(codes == 0) and np.all(scales == 0) and np.all(g == 0)
    assert np.all(o.dequant_nvfp4(codes, (scales, g)) == 0)


def test_hand_worked_example(golden):
    gd = golden("nvfp4_hand_example.txt")
    row = np.zeros(32)
    vals = parse_numbers(gd["block0"])
    row[:len(vals)] = vals
    row[16] = float(parse_numbers(gd["block1_first"])[0])
    bits = o.f64_to_bf16(row[None])
    codes, (scales, g) = o.pack_nvfp4(bits)
    assert float(g) == float(parse_numbers(gd["global_scale"])[0])
    assert list(scales[0]) == parse_numbers(gd["scale_bytes"])
    assert list(codes[0, :4]) == parse_numbers(gd["code_bytes"])
    deq = o.dequant_nvfp4(codes, (scales, g))[0]
    assert np.array_equal(deq[:len(vals)], np.array(parse_numbers(gd["block0_dequant"]), np.float64))
    assert deq[16] == float(parse_numbers(gd["block1_first_dequant"])[0])


# ---------------------------------------------------------------- planted mistakes

_orig = {n: getattr(o, n) for n in ("nv_global_scale", "e4m3_nearest", "nv_multiplier", "pack_nvfp4")}


def _mult_unrounded(scale_codes, g):
    v = o.e4m3_value(scale_codes).astype(np.float32)
    return (v * np.asarray(g, np.float32)[..., None, None]).astype(np.float64)


def _e4m3_ties_odd(t):
    t = np.asarray(t, np.float64)
    vals = o.e4m3_value(np.arange(0x7F))
    d = np.abs(t[..., None] - vals)
    best = d == d.min(-1, keepdims=True)
    return (0x7E - np.argmax(best[..., ::-1], axis=-1)).astype(np.uint8)


def _per_row_global(w_bits):
    w = o.bf16_to_f64(w_bits).astype(np.float32)
    amax = np.max(np.abs(w), axis=-1).max(-1) * 0 + np.max(np.abs(w[..., :1, :]), axis=(-1, -2))
    return (amax / np.float32(2688)).astype(np.float32)


NV_MUTANTS = {
    "global divisor 448": {"nv_global_scale": lambda wb: (_orig["nv_global_scale"](wb) * np.float32(6)).astype(np.float32)},
    "global scale from the first row only": {"nv_global_scale": _per_row_global},
    "e4m3 ties to odd": {"e4m3_nearest": _e4m3_ties_odd},
    "block multiplier not rounded to bf16": {"nv_multiplier": _mult_unrounded},
}


def _run_nv_pins():
    from conftest import read_golden
    failed = []
    for name, fn in sorted(globals().items()):
        if not name.startswith("test_") or "planted" in name or "unmutated" in name:
            continue
        try:
            with np.errstate(all="ignore"):
                fn(read_golden) if name == "test_hand_worked_example" else fn()
        except Exception:
            failed.append(name)
    return failed


@pytest.mark.parametrize("mutant", sorted(NV_MUTANTS))
def test_planted_nvfp4_mistake_is_caught(mutant, monkeypatch):
    for attr, fn in NV_MUTANTS[mutant].items():
        monkeypatch.setattr(o, attr, fn)
    assert _run_nv_pins(), f"no pin noticed the planted mistake: {mutant}"


def test_unmutated_nvfp4_passes_the_same_pins():
    assert _run_nv_pins() == []
