"""The 40-layer MXFP4 expert stack against the CPU oracle (needs a B200).

"kirillbilchenko/Nex-N2.5-mini-MXFP4-MxWave", Model summary: 40 MoE layers of
256 routed experts, 30,720 expert matrices in MXFP4 (E2M1 codes, one E8M0
scale per 32 elements).  Layer l of the stack is drawn with seed 1000 + l
(router weight and both banks N(0, 0.02)); all 40 packed layers are resident
on the GPU together (17.1 GB), as in the benchmark's stack.  Every layer is
applied to the same tokens (no chaining, so a layer's parity does not depend
on another's) and checked with the rule of test_gpu_parity.check_layer:
bit-exact routing on the GPU's logits and, per element, the layer-output
tolerance against the pure oracle (plus the flip allowance for tokens whose
bf16 activations sit on a rounding boundary).  At 4 tokens every token of
every layer is checked; at 8192 tokens a seeded sample of tokens per layer.
"""
import numpy as np
import pytest
import torch

import moe_synth
import weight_only_bit_router_b200 as moe
from test_gpu_parity import DEV, run_forward, verify_layer

pytestmark = pytest.mark.gpu

LAYERS = 40
FMT = "mxfp4"


@pytest.fixture(scope="module")
def stack():
    s = moe_synth.NEX
    shape = moe.make_shape(s.hidden, s.inter, s.num_experts, s.top_k, FMT)
    gu = torch.empty(LAYERS, moe.moe_packed_bytes(shape, 0), dtype=torch.uint8, device=DEV)
    dn = torch.empty(LAYERS, moe.moe_packed_bytes(shape, 1), dtype=torch.uint8, device=DEV)
    for l in range(LAYERS):
        seed = moe_synth.SEED_STACK_BASE + l
        moe.moe_pack_mxfp4(moe_synth.gate_up_bank(s, seed, DEV), packed=gu[l])
        moe.moe_pack_mxfp4(moe_synth.down_bank(s, seed, DEV), packed=dn[l])
    torch.cuda.synchronize()
    yield gu, dn
    del gu, dn
    torch.cuda.empty_cache()


def stack_layer(l, x):
    """Layer l's bf16 source (regenerated from its seed, for the oracle) with tokens x."""
    s = moe_synth.NEX
    seed = moe_synth.SEED_STACK_BASE + l
    return moe_synth.Layer(shape=s, x=x, router_w=moe_synth.router_weight(s, seed, DEV),
                           gate_up=moe_synth.gate_up_bank(s, seed, DEV), down=moe_synth.down_bank(s, seed, DEV),
                           bias=None)


def test_stack40_mxfp4_decode4(stack):
    gu, dn = stack
    x = moe_synth.hidden_states(moe_synth.NEX, 4, 40_004, DEV)
    # every layer forward first, back to back on one stream, then the checks
    runs = []
    for l in range(LAYERS):
        layer = stack_layer(l, x)
        runs.append(run_forward(layer, FMT, packed=(gu[l], dn[l])))
        del layer
    for l, (out, dbg) in enumerate(runs):
        verify_layer(stack_layer(l, x), FMT, out, dbg, name=f"stack40_mxfp4_T4_layer{l}")


def test_stack40_mxfp4_prefill8192_sampled(stack):
    gu, dn = stack
    T = 8192
    x = moe_synth.hidden_states(moe_synth.NEX, T, 48_192, DEV)
    rng = np.random.default_rng(40)
    for l in range(LAYERS):
        layer = stack_layer(l, x)
        out, dbg = run_forward(layer, FMT, packed=(gu[l], dn[l]))
        sample = rng.choice(T, 2, replace=False)
        verify_layer(layer, FMT, out, dbg, sample=sample, name=f"stack40_mxfp4_T8192_layer{l}")
        del layer, out, dbg
