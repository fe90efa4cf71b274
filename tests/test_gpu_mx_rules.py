"""MXFP4 exponent rules on the GPU vs the CPU oracle, through the C ABI.

moe_pack_mxfp4_rule must reproduce the oracle's codes and scale bytes bit for
bit under every rule (the MSE search included), and moe_forward must consume
banks packed under any rule: the layer output is checked against the oracle
with the same per-element tolerance as the other layer tests,
|gpu - ref| <= 1e-2 |ref| + 1e-3 rms(ref).
"""
import numpy as np
import pytest
import torch

import moe_synth
import weight_only_bit_router_b200 as moe
from oracle import moe_oracle as o
from parity_util import assert_out_close, flip_aware_activations
from test_gpu_parity import edge_bank, gpu_activations_in_oracle_order

pytestmark = pytest.mark.gpu
DEV = "cuda"
RULES = ["floor", "ceil", "ocp", "mse"]


def block_zoo():
    """[1, 40, 256] bank whose 32-element blocks stress the exponent rules:
    Gaussian, heavy-tailed, tie-rich, mostly-zero, a max just past a
    power-of-two boundary, a lone max in (14, 14.2) * 2^k, subnormal and
    near-overflow magnitudes."""
    rng = np.random.default_rng(21)
    rows = []
    for i in range(40):
        kind = i % 8
        if kind == 0:
            r = rng.standard_normal(256) * 0.02
        elif kind == 1:
            r = rng.standard_t(2, 256) * 0.05
        elif kind == 2:
            r = rng.integers(-12, 13, 256) * 0.125
        elif kind == 3:
            r = np.zeros(256)
            r[rng.integers(0, 256, 12)] = rng.standard_normal(12)
        elif kind == 4:
            k = int(rng.integers(-8, 4))
            r = rng.uniform(0.2, 0.7, 256) * 6 * 2.0 ** (k + 1) * rng.choice([-1, 1], 256)
            r[::32] = 6 * 2.0 ** (k + 1) * rng.uniform(1.01, 1.15, 8)
        elif kind == 5:
            k = int(rng.integers(-30, 30))
            r = np.zeros(256)
            r[3::32] = 14.125 * 2.0 ** k
            r[9::32] = 0.25 * 2.0 ** k
        elif kind == 6:
            r = rng.standard_normal(256) * 2.0 ** -128        # bf16 subnormals
        else:
            r = rng.standard_normal(256) * 1e37
        rows.append(r)
    bits = o.f64_to_bf16(np.stack(rows)[None])
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)


def gpu_codes_scales(packed, E, N, K):
    codes, scales = moe.split_bank(packed, "mxfp4", E, N, K)
    return codes.cpu().numpy(), scales.cpu().numpy()


@pytest.mark.parametrize("rule", RULES)
def test_pack_rule_bit_exact(rule):
    banks = (moe_synth.gate_up_bank(moe_synth.TINY, 0), moe_synth.down_bank(moe_synth.TINY, 0), edge_bank(),
             block_zoo())
    for w in banks:
        E, N, K = w.shape
        packed = moe.moe_pack_mxfp4_rule(w.to(DEV), rule)
        torch.cuda.synchronize()
        gc, gs = gpu_codes_scales(packed, E, N, K)
        rc, rs = o.pack_mxfp4(moe_synth.bf16_bits(w), rule)
        assert np.array_equal(gs, rs), f"{rule}: scale bytes differ"
        assert np.array_equal(gc, rc), f"{rule}: codes differ"


def test_floor_rule_equals_moe_pack_mxfp4():
    w = moe_synth.gate_up_bank(moe_synth.TINY, 3).to(DEV)
    assert torch.equal(moe.moe_pack_mxfp4_rule(w, "floor"), moe.moe_pack_mxfp4(w))


def test_pack_rule_mse_full_layer_sampled_experts():
    gu = moe_synth.gate_up_bank(moe_synth.NEX, seed=1000, device=DEV)
    packed = moe.moe_pack_mxfp4_rule(gu, "mse")
    torch.cuda.synchronize()
    E, N, K = gu.shape
    codes, scales = moe.split_bank(packed, "mxfp4", E, N, K)
    for e in (0, 77, 255):
        rc, rs = o.pack_mxfp4(moe_synth.bf16_bits(gu[e]), "mse")
        assert np.array_equal(scales[e].cpu().numpy(), rs)
        assert np.array_equal(codes[e].cpu().numpy(), rc)


def test_pack_rule_rejects_unknown_rule():
    w = moe_synth.gate_up_bank(moe_synth.TINY, 0).to(DEV)
    with pytest.raises(moe.MoeError):
        moe.moe_pack_mxfp4_rule(w, 7)


@pytest.mark.parametrize("rule", ["ceil", "mse"])
@pytest.mark.parametrize("path", [moe.MOE_PATH_DECODE, moe.MOE_PATH_PREFILL])
def test_forward_on_rule_packed_banks(rule, path):
    layer = moe_synth.make_layer(moe_synth.TINY, T=16, seed=moe_synth.SEED_TINY, device=DEV)
    s = layer.shape
    shape = moe.make_shape(s.hidden, s.inter, s.num_experts, s.top_k, "mxfp4")
    T = layer.x.shape[0]
    gu = moe.moe_pack_mxfp4_rule(layer.gate_up, rule)
    dn = moe.moe_pack_mxfp4_rule(layer.down, rule)
    ws = moe.alloc_workspace(shape, T)
    dbg = {
        "logits_out": torch.empty(T, s.num_experts, dtype=torch.float32, device=DEV),
        "topk_ids_out": torch.empty(T, s.top_k, dtype=torch.int32, device=DEV),
        "topk_w_out": torch.empty(T, s.top_k, dtype=torch.float32, device=DEV),
        "act_out": torch.empty(T * s.top_k, s.inter, dtype=torch.bfloat16, device=DEV),
        "offsets_out": torch.empty(s.num_experts + 1, dtype=torch.int32, device=DEV),
        "sorted_rows_out": torch.empty(T * s.top_k, dtype=torch.int32, device=DEV),
    }
    out = moe.moe_forward(shape, layer.x, layer.router_w, gu, dn, ws, path=path, debug=dbg)
    assert moe.moe_workspace_status(ws) == moe.MOE_OK
    rid, rw = o.route(dbg["logits_out"].cpu().numpy(), None, s.top_k)
    assert np.array_equal(rid, dbg["topk_ids_out"].cpu().numpy())
    xb = moe_synth.bf16_bits(layer.x)
    gu_o = o.PackedBank(o.FMT_MXFP4, *o.pack_mxfp4(moe_synth.bf16_bits(layer.gate_up), rule))
    dn_o = o.PackedBank(o.FMT_MXFP4, *o.pack_mxfp4(moe_synth.bf16_bits(layer.down), rule))
    a_exact, a_round = o.expert_activations(xb, rid, gu_o, s.num_experts)
    gpu_act = gpu_activations_in_oracle_order(dbg, np.arange(T), rid, s.num_experts, s.top_k)
    act_used, n_diff = flip_aware_activations(gpu_act, a_exact, a_round)
    ref = o.down_and_combine(act_used, rid, rw, dn_o, s.num_experts)
    assert_out_close(out, ref, f"mxfp4/{rule} path {path} ({n_diff} activations rounded the other way)")
