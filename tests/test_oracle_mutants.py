"""Planted mistakes in the oracle must be caught by its pins (CPU only).

Each mutant below swaps one oracle function for a version with one plausible
mistake (a wrong divisor, a tie rule, a dropped rounding, a swapped operand,
...), then runs the pin suite of test_oracle_pins.py against the patched
oracle.  The test passes only if at least one pin fails for every mutant, i.e.
the pins are strong enough to notice that kind of error.  The mistakes are
planted in the oracle, on the CPU; nothing here touches the CUDA path.
"""
import numpy as np
import pytest

import test_oracle_pins as pins
from oracle import moe_oracle as o

_orig = {name: getattr(o, name) for name in (
    "pack_int4_g128", "unpack_nibbles", "dequant_int4_g128", "mx_exponent", "e2m1_nearest",
    "route", "expert_mlp", "permute", "f64_to_bf16", "swiglu_exact", "expert_activations")}


def _int4_pack_variant(div=7.0, rnd=np.rint):
    def pack(w_bits):
        w32 = o.bf16_to_f64(np.asarray(w_bits, np.uint16)).astype(np.float32)
        K = w32.shape[-1]
        groups = o.int4_groups(K)
        q = np.zeros(w32.shape, np.int32)
        scales = np.zeros(w32.shape[:-1] + (len(groups),), np.uint16)
        for gi, (a, b) in enumerate(groups):
            amax = np.max(np.abs(w32[..., a:b]), axis=-1)
            sb = o.f64_to_bf16((amax / np.float32(div)).astype(np.float64))
            s = o.bf16_to_f64(sb).astype(np.float32)[..., None]
            safe = np.where(s == 0, np.float32(1), s)
            q[..., a:b] = np.where(s == 0, 0, np.clip(rnd(w32[..., a:b] / safe), -8, 7))
            scales[..., gi] = sb
        u = (q + 8).astype(np.uint8)
        return (u[..., 0::2] | (u[..., 1::2] << np.uint8(4))).astype(np.uint8), scales
    return pack


def _swap_nibbles(c):
    c = np.asarray(c, np.uint8)
    return ((c & np.uint8(15)) << np.uint8(4)) | (c >> np.uint8(4))


def _route_variant(tie_high=False, full_softmax=False, unit_weights=False):
    def route(logits32, bias32, k):
        L = np.asarray(logits32, np.float32)
        if bias32 is not None:
            L = (L + np.asarray(bias32, np.float32)[None]).astype(np.float32)
        if tie_high:
            E = L.shape[1]
            ids = (E - 1 - np.argsort(-L[:, ::-1], axis=1, kind="stable"))[:, :k].astype(np.int32)
        else:
            ids = np.argsort(-L, axis=1, kind="stable")[:, :k].astype(np.int32)
        sel = np.take_along_axis(L, ids, 1).astype(np.float64)
        if unit_weights:
            return ids, np.ones_like(sel)
        if full_softmax:
            allx = np.exp(L.astype(np.float64) - sel[:, :1])
            return ids, np.exp(sel - sel[:, :1]) / allx.sum(1, keepdims=True)
        ex = np.exp(sel - sel[:, :1])
        return ids, ex / ex.sum(1, keepdims=True)
    return route


def _swiglu_swapped(x_rows, w_gate_up):
    inter = w_gate_up.shape[0] // 2
    h = x_rows @ w_gate_up.T
    return o.silu(h[:, inter:]) * h[:, :inter]


def _activations_unrounded(x_bits, ids, gate_up, num_experts):
    a_exact, _ = _orig["expert_activations"](x_bits, ids, gate_up, num_experts)
    return a_exact, a_exact


def _unstable_permute(ids, E):
    offsets, sorted_rows, pos = _orig["permute"](ids, E)
    out = sorted_rows.copy()
    for e in range(E):                       # reverse the order inside each expert
        out[offsets[e]:offsets[e + 1]] = sorted_rows[offsets[e]:offsets[e + 1]][::-1]
    inv = np.empty_like(out)
    inv[out] = np.arange(out.size, dtype=out.dtype)
    return offsets, out, inv


def _e2m1_ties_odd(v):
    a = np.abs(np.asarray(v, np.float64))
    d = np.abs(a[..., None] - o.E2M1_GRID)
    best = d == d.min(-1, keepdims=True)
    return (7 - np.argmax(best[..., ::-1], axis=-1)).astype(np.uint8)   # highest index on ties


def _dequant_int4_unrounded(codes, scales):
    q = o.int4_codes(codes).astype(np.float64)
    s = o.bf16_to_f64(scales)
    full = np.concatenate([np.repeat(s[..., gi:gi + 1], b - a, -1)
                           for gi, (a, b) in enumerate(o.int4_groups(q.shape[-1]))], -1)
    return q * full


def _bf16_truncating(x):
    x = np.asarray(x, np.float64).astype(np.float32)
    return (x.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


MUTANTS = {
    "int4 scale amax/7.5": {"pack_int4_g128": _int4_pack_variant(div=7.5)},
    "int4 scale amax/8": {"pack_int4_g128": _int4_pack_variant(div=8.0)},
    "int4 ties away from zero": {"pack_int4_g128": _int4_pack_variant(rnd=lambda z: np.sign(z) * np.floor(np.abs(z) + 0.5))},
    "int4 truncation": {"pack_int4_g128": _int4_pack_variant(rnd=np.trunc)},
    "nibble order swapped": {"pack_int4_g128": lambda w: (lambda c, s: (_swap_nibbles(c), s))(*_orig["pack_int4_g128"](w)),
                             "unpack_nibbles": lambda c: _orig["unpack_nibbles"](_swap_nibbles(c))},
    "int4 weight not rounded to bf16": {"dequant_int4_g128": _dequant_int4_unrounded},
    "mx exponent ceil rule": {"mx_exponent": lambda a: np.where(np.asarray(a) > 0, _orig["mx_exponent"](a) + (
        ~np.isin(np.asarray(a, np.float64) / 6.0, [2.0 ** i for i in range(-140, 130)])), -127)},
    "e2m1 ties to odd": {"e2m1_nearest": _e2m1_ties_odd},
    "route ties to higher index": {"route": _route_variant(tie_high=True)},
    "route softmax over all experts": {"route": _route_variant(full_softmax=True)},
    "combine drops routing weight": {"route": _route_variant(unit_weights=True)},
    "gate and up swapped": {"swiglu_exact": _swiglu_swapped},
    "activation not rounded to bf16": {"expert_activations": _activations_unrounded},
    "unstable permutation": {"permute": _unstable_permute},
    "bf16 rounding truncates": {"f64_to_bf16": _bf16_truncating},
}

_SLOW = {"test_int4_group_max_maps_to_plus_minus_7"}


def _run_pins():
    failures = []
    for name in dir(pins):
        if not name.startswith("test_") or name in _SLOW:
            continue
        fn = getattr(pins, name)
        args = [[o.FMT_INT4], [o.FMT_MXFP4]] if name == "test_layer_bruteforce_tiny" else [[]]
        for a in args:
            try:
                with np.errstate(all="ignore"):
                    fn(*a)
            except Exception:  # an assertion or a crash both count as caught
                failures.append(name)
    return failures


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_planted_mistake_is_caught(mutant, monkeypatch):
    for attr, fn in MUTANTS[mutant].items():
        monkeypatch.setattr(o, attr, fn)
    caught = _run_pins()
    assert caught, f"no pin noticed the planted mistake: {mutant}"


def test_unmutated_oracle_passes_the_same_pins():
    assert _run_pins() == []
