"""The layer with its bf16 shared expert (moe_forward_shared) against the CPU
oracle, through the C ABI (needs a B200).

Per element |gpu - ref| <= 1e-2 |ref| + 1e-3 rms(ref), ref = the oracle's
own layer: its routed combine plus its gated shared expert, each with the
oracle's own bf16 activation rounding.  Tokens where fp32 accumulation put a
routed or shared activation across a bf16 rounding boundary (both neighbours
are correct, parity_util.flip_aware_activations checks each against the exact
value) may exceed the bound by at most the flips' own effect on the output
(parity_util.flip_allowance, and the same bound for the shared expert's down
projection scaled by its gate); their output is also checked stage-wise
against the oracle's down projections of the GPU's own activations.  The
shared expert's bf16 activations are read from their place in the workspace,
right after the routed layer's part (at offset moe_workspace_bytes).
"""
import numpy as np
import pytest
import torch

import moe_synth
import weight_only_bit_router_b200 as moe
from oracle import moe_oracle as o
from parity_util import (LazyOracleBank, assert_layer_parity, assert_out_close, assert_routing_consistent,
                         bf16_ulp, flip_allowance, flip_aware_activations, record_parity)
from test_gpu_parity import DEV, gpu_activations_in_oracle_order, pack_gpu

pytestmark = pytest.mark.gpu


def check_shared(layer, fmt, inter_shared, path=None, sample=None, seed=0):
    s = layer.shape
    shape = moe.make_shape(s.hidden, s.inter, s.num_experts, s.top_k, fmt)
    T = layer.x.shape[0]
    shared = moe_synth.shared_expert(s, inter_shared, seed, DEV)
    gu, dn = pack_gpu(fmt, layer.gate_up), pack_gpu(fmt, layer.down)
    ws = moe.alloc_workspace_shared(shape, inter_shared, T)
    dbg = {
        "logits_out": torch.empty(T, s.num_experts, dtype=torch.float32, device=DEV),
        "topk_ids_out": torch.empty(T, s.top_k, dtype=torch.int32, device=DEV),
        "topk_w_out": torch.empty(T, s.top_k, dtype=torch.float32, device=DEV),
        "act_out": torch.empty(T * s.top_k, s.inter, dtype=torch.bfloat16, device=DEV),
        "offsets_out": torch.empty(s.num_experts + 1, dtype=torch.int32, device=DEV),
        "sorted_rows_out": torch.empty(T * s.top_k, dtype=torch.int32, device=DEV),
    }
    out = moe.moe_forward_shared(shape, shared, layer.x, layer.router_w, gu, dn, ws, bias=layer.bias, path=path,
                                 debug=dbg)
    assert moe.moe_workspace_status(ws) == moe.MOE_OK
    tok = np.arange(T) if sample is None else np.asarray(sample)
    tok_d = torch.as_tensor(tok, device=DEV)
    xb = moe_synth.bf16_bits(layer.x)[tok]
    bias = None if layer.bias is None else layer.bias.cpu().numpy()
    ref_logits = o.router_logits(xb, moe_synth.bf16_bits(layer.router_w))
    assert_routing_consistent(dbg["logits_out"][tok_d], ref_logits, dbg["topk_ids_out"][tok_d], bias, s.top_k)
    rid, rw = o.route(dbg["logits_out"][tok_d].cpu().numpy(), bias, s.top_k)
    assert np.array_equal(rid, dbg["topk_ids_out"][tok_d].cpu().numpy())
    gub, dnb = LazyOracleBank(fmt, layer.gate_up), LazyOracleBank(fmt, layer.down)
    gub.prefetch(rid)
    dnb.prefetch(rid)
    a_exact, a_round = o.expert_activations(xb, rid, gub, s.num_experts)
    gpu_act = gpu_activations_in_oracle_order(dbg, tok, rid, s.num_experts, s.top_k)
    act_used, n_diff = flip_aware_activations(gpu_act, a_exact, a_round)
    routed = o.down_and_combine(act_used, rid, rw, dnb, s.num_experts)
    sh_bits = [moe_synth.bf16_bits(t) for t in shared]
    g, _ = o.shared_expert(xb, *sh_bits)
    assert np.all((g > 0.01) & (g < 0.99))  # the gate is not saturated on these inputs
    # the GPU's shared-expert activations, checked like the routed ones
    off = moe.moe_workspace_bytes(shape, T)
    a_gpu = ws[off:off + T * inter_shared * 2].view(torch.bfloat16).view(T, inter_shared)[tok_d]
    a_gpu = o.bf16_to_f64(moe_synth.bf16_bits(a_gpu))
    a_s_exact = o.swiglu_exact(o.bf16_to_f64(xb), o.bf16_to_f64(sh_bits[0]))
    a_s_round = o.bf16_round(a_s_exact)
    a_s_used, n_sh = flip_aware_activations(a_gpu, a_s_exact, a_s_round)
    wd_s = o.bf16_to_f64(sh_bits[1])
    out_sel = out[tok_d]
    what = f"{fmt} shared T={T} ({n_diff} routed, {n_sh} shared activations rounded the other way)"
    # against the pure oracle: the oracle's own layer with its shared expert
    pure = o.down_and_combine(a_round, rid, rw, dnb, s.num_experts) + g[:, None] * (a_s_round @ wd_s.T)
    allow, flipped = flip_allowance(gpu_act, a_exact, a_round, rid, rw, dnb, s.num_experts)
    if allow is None:
        allow = np.zeros_like(pure)
    for t, i in zip(*np.nonzero(a_gpu != a_s_round)):
        allow[t] += abs(float(g[t])) * np.abs(wd_s[:, i]) * float(bf16_ulp(a_s_exact[t, i]))
        flipped[t] = True
    summary = assert_layer_parity(out_sel, pure, allow, flipped, what)
    # stage-wise: the oracle's down projections of the GPU's own activations
    ref = routed + g[:, None] * (a_s_used @ wd_s.T)
    assert_out_close(out_sel, ref, what + " stage-wise")
    record_parity(dict(case=f"shared_{fmt}_T{T}", fmt=fmt, T=T, path=int(path or 0),
                       shape=[s.hidden, s.inter, s.num_experts, s.top_k, inter_shared],
                       sampled_tokens=int(tok.size), activations_rounded_other_way=n_diff,
                       shared_activations_rounded_other_way=n_sh, **summary))
    # the shared expert changes the output: the routed-only oracle must not pass
    n_far = int(np.sum(np.abs(out[tok_d].float().cpu().numpy() - routed) > 1e-2 * np.abs(routed) +
                       1e-3 * np.sqrt(np.mean(routed ** 2))))
    assert n_far > out[tok_d].numel() // 4
    return out


@pytest.mark.parametrize("fmt", ["int4_g128", "nvfp4"])
@pytest.mark.parametrize("path", [moe.MOE_PATH_DECODE, moe.MOE_PATH_PREFILL])
def test_shared_tiny_layer(fmt, path):
    layer = moe_synth.make_layer(moe_synth.TINY, T=16, seed=moe_synth.SEED_TINY, device=DEV)
    check_shared(layer, fmt, 64, path, seed=3)


@pytest.mark.parametrize("T", [1, 4, 24, 32])
def test_shared_nex_decode(T):
    # folded: the shared expert rides the routing GEMV and the two decode kernels
    layer = moe_synth.make_layer(moe_synth.NEX, T=T, seed=100 + T, device=DEV)
    shape = moe.make_shape(2048, 512, 256, 8, "int4_g128")
    assert moe.moe_forward_shared_launch_count(shape, 512, T, moe.MOE_PATH_AUTO) == \
        moe.moe_forward_launch_count(shape, T, moe.MOE_PATH_AUTO, False)
    check_shared(layer, "int4_g128", 512, seed=100 + T)


@pytest.mark.parametrize("fmt,inter_shared,T", [("mxfp4", 448, 8), ("int4_g128", 640, 4)])
def test_shared_nex_decode_other_sizes(fmt, inter_shared, T):
    # 448: folded, its last 128-k sub-unit half past I_s; 640: too large for
    # the down kernel's sub-units, the shared expert's own kernels
    layer = moe_synth.make_layer(moe_synth.NEX, T=T, seed=300 + T, device=DEV)
    check_shared(layer, fmt, inter_shared, seed=300 + inter_shared)


def test_shared_decode_unfolded_odd_shape():
    # E % 4 != 0: no split-K routing, so the shared expert runs its own
    # split-K kernels beside the decode kernels (its output added in the
    # down kernel's combine)
    shp = moe_synth.LayerShape(hidden=320, inter=192, num_experts=6, top_k=3)
    shape = moe.make_shape(320, 192, 6, 3, "int4_g128")
    assert moe.moe_forward_shared_launch_count(shape, 64, 8, moe.MOE_PATH_DECODE) == \
        moe.moe_forward_launch_count(shape, 8, moe.MOE_PATH_DECODE, False) + 3
    layer = moe_synth.make_layer(shp, T=8, seed=77, device=DEV)
    check_shared(layer, "int4_g128", 64, moe.MOE_PATH_DECODE, seed=78)


def test_shared_nex_prefill_sampled():
    layer = moe_synth.make_layer(moe_synth.NEX, T=2048, seed=2048, device=DEV)
    sample = np.random.default_rng(9).choice(2048, 24, replace=False)
    check_shared(layer, "mxfp4", 512, sample=sample, seed=2048)


def test_shared_expert_rejects_bad_sizes():
    layer = moe_synth.make_layer(moe_synth.TINY, T=4, seed=1, device=DEV)
    s = layer.shape
    shape = moe.make_shape(s.hidden, s.inter, s.num_experts, s.top_k, "int4_g128")
    gu, dn = pack_gpu("int4_g128", layer.gate_up), pack_gpu("int4_g128", layer.down)
    small = torch.empty(moe.moe_workspace_bytes(shape, 4), dtype=torch.uint8, device=DEV)
    moe.moe_workspace_init(small)
    with pytest.raises(moe.MoeError):   # the routed layer's workspace is too small for the shared expert
        moe.moe_forward_shared(shape, moe_synth.shared_expert(s, 64, 1, DEV), layer.x, layer.router_w, gu, dn, small)
    assert moe.moe_workspace_bytes_shared(shape, 96, 4) == 0   # I_s not a multiple of 64
