"""Pins of the oracle's shared expert (CPU only).

The Qwen3.5-MoE block adds a dense SwiGLU expert, gated per token by a
sigmoid of x . w_gate, to the routed experts' combine ("Tech2wild/Nex-N2.5-
mini-Int4-Int8Mix", Recipe table: shared expert gate/up/down_proj and a
separate shared_expert_gate; "kirillbilchenko/Nex-N2.5-mini-MXFP4-MxWave",
What was quantized: shared experts stay bf16).  Its intermediate size is
pinned by the parameter count the NVFP4 card prints.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import moe_synth
from conftest import parse_numbers, read_golden
from oracle import moe_oracle as o


def exact_bf16(q: Fraction) -> Fraction:
    """Round a rational to bf16 (8 significant bits, half to even)."""
    if q == 0:
        return Fraction(0)
    s = -1 if q < 0 else 1
    a = abs(q)
    e = math.floor(math.log2(a))
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (e - 7)
    m = a / ulp
    r = math.floor(m)
    if m - r > Fraction(1, 2) or (m - r == Fraction(1, 2) and r % 2 == 1):
        r += 1
    return s * r * ulp


def shared_weights(H, I, seed):
    gu, dn, gate = moe_synth.shared_expert(moe_synth.LayerShape(H, I, 1, 1), I, seed)
    return moe_synth.bf16_bits(gu), moe_synth.bf16_bits(dn), moe_synth.bf16_bits(gate)


def test_shared_expert_against_naive_loops():
    H, I, T = 64, 32, 3
    gu, dn, gate = shared_weights(H, I, 4)
    x = moe_synth.bf16_bits(moe_synth.hidden_states(moe_synth.LayerShape(H, I, 1, 1), T, 4))
    g, y = o.shared_expert(x, gu, dn, gate)
    X, Wgu, Wd, wg = (o.bf16_to_f64(v) for v in (x, gu, dn, gate))
    for t in range(T):
        hg = [sum(Wgu[i, h] * X[t, h] for h in range(H)) for i in range(I)]
        hu = [sum(Wgu[I + i, h] * X[t, h] for h in range(H)) for i in range(I)]
        a = [float(exact_bf16(Fraction(gi * ui / (1 + math.exp(-gi))))) for gi, ui in zip(hg, hu)]
        yt = [sum(Wd[h, i] * a[i] for i in range(I)) for h in range(H)]
        z = sum(wg[h] * X[t, h] for h in range(H))
        assert math.isclose(g[t], 1 / (1 + math.exp(-z)), rel_tol=1e-12)
        assert np.allclose(y[t], yt, rtol=1e-12, atol=1e-15)


def test_gate_limits():
    H, I, T = 64, 32, 5
    gu, dn, _ = shared_weights(H, I, 5)
    x = moe_synth.bf16_bits(moe_synth.hidden_states(moe_synth.LayerShape(H, I, 1, 1), T, 5))
    g0, _ = o.shared_expert(x, gu, dn, np.zeros(H, np.uint16))
    assert np.all(g0 == 0.5)                                   # zero gate weights: sigmoid(0)
    big = o.f64_to_bf16(np.sign(o.bf16_to_f64(x[0])) * 100.0)  # aligned with token 0: z >> 0
    g1, _ = o.shared_expert(x[:1], gu, dn, big)
    assert g1[0] == 1.0


def test_layer_with_shared_expert_adds_the_gated_dense_mlp():
    shape = moe_synth.LayerShape(hidden=64, inter=32, num_experts=5, top_k=2)
    L = moe_synth.make_layer(shape, T=4, seed=22)
    xb, rb = moe_synth.bf16_bits(L.x), moe_synth.bf16_bits(L.router_w)
    gu = o.PackedBank.from_bf16(o.FMT_INT4, moe_synth.bf16_bits(L.gate_up))
    dn = o.PackedBank.from_bf16(o.FMT_INT4, moe_synth.bf16_bits(L.down))
    sh = shared_weights(64, 48, 22)
    with_shared = o.forward_with_shared(xb, rb, None, gu, dn, 2, sh)
    plain = o.forward(xb, rb, None, gu, dn, 2)
    # the dense expert as a routed one: a one-expert bank holding the shared weights in
    # bf16 is exactly what expert_mlp computes for that expert
    _, y = o.expert_mlp(o.bf16_to_f64(xb), o.bf16_to_f64(sh[0]), o.bf16_to_f64(sh[1]))
    z = o.bf16_to_f64(xb) @ o.bf16_to_f64(sh[2])
    assert np.allclose(with_shared["out"], plain["out"] + y / (1 + np.exp(-z))[:, None], rtol=1e-12, atol=1e-15)


def test_printed_parameter_count_fixes_the_intermediate_size():
    g = read_golden("shared_expert_size_fact.txt")
    L, E, H = int(g["layers"]), int(g["experts"]), int(g["hidden"])
    printed = float(g["shared_router_norm_params_billion"]) * 1e9
    routers = L * E * H
    norms_upper = L * 4 * H                  # a few hidden-sized norm vectors per layer
    def count(I):
        return L * (3 * H * I + H) + routers  # shared gate_up + down + gate vector, routers
    fits = [I for I in (128, 256, 384, 512, 640, 768, 1024)
            if abs(count(I) - printed) <= 0.005e9 + norms_upper]
    assert fits == [512]


# ---------------------------------------------------------------- planted mistakes

_orig = o.shared_expert


def _variant(gate_fn=None, round_act=True, swap=False):
    def shared(x_bits, gate_up_bits, down_bits, gate_bits):
        x = o.bf16_to_f64(x_bits)
        w = o.bf16_to_f64(gate_up_bits)
        if swap:
            I = w.shape[0] // 2
            w = np.concatenate([w[I:], w[:I]])
        a = o.swiglu_exact(x, w)
        a = o.bf16_round(a) if round_act else a
        y = a @ o.bf16_to_f64(down_bits).T
        z = x @ o.bf16_to_f64(gate_bits)
        return (gate_fn or (lambda v: 1 / (1 + np.exp(-v))))(z), y
    return shared


SH_MUTANTS = {
    "gate is tanh": _variant(gate_fn=np.tanh),
    "gate is one": _variant(gate_fn=lambda v: np.ones_like(v)),
    "activation not rounded to bf16": _variant(round_act=False),
    "gate and up swapped": _variant(swap=True),
}


def _run_shared_pins():
    failed = []
    for name, fn in sorted(globals().items()):
        if not name.startswith("test_") or "planted" in name or "unmutated" in name:
            continue
        try:
            with np.errstate(all="ignore"):
                fn()
        except Exception:
            failed.append(name)
    return failed


@pytest.mark.parametrize("mutant", sorted(SH_MUTANTS))
def test_planted_shared_expert_mistake_is_caught(mutant, monkeypatch):
    monkeypatch.setattr(o, "shared_expert", SH_MUTANTS[mutant])
    assert _run_shared_pins(), f"no pin noticed the planted mistake: {mutant}"


def test_unmutated_shared_expert_passes_the_same_pins():
    assert _run_shared_pins() == []
