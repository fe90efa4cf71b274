"""Seeded synthetic inputs for the W4A16 routed-expert MoE layer.

This module is the one piece shared by the CPU oracle's tests and the CUDA
path's tests and benchmark.  It draws random numbers and rounds them to the
input dtypes; it holds none of the layer's arithmetic (no quantisation, no
routing, no matmul).

Layer shapes follow the Qwen3.5-MoE expert bank printed on
"Tech2wild/Nex-N2.5-mini-Int4-Int8Mix" (Recipe section: experts.gate_up_proj
[256, 1024, 2048], experts.down_proj [256, 2048, 512]) with top-8 routing
("cbert33/Nex-N2.5-mini-FP8-Calibrated", Artifact summary: 256 routed experts,
8 active per token).

Value recipe (the pages print no data, so these are synthetic stand-ins):
  * hidden states x ~ N(0, 1), rounded to bf16 (round-to-nearest-even by torch);
  * router weight and both expert banks ~ N(0, 0.02), rounded to bf16;
  * optional skewed routing: a per-expert logit bias b_e = -s * ln(rank_e),
    rank = a seeded random permutation of 1..E, s = 1.1 (a Zipf(1.1) prior on
    expert popularity added to the fp32 logits).

Every tensor is drawn from its own torch.Generator seeded with
``seed * 16 + tensor_id`` so that the CPU and the GPU copies of a layer are the
same bits when they are generated on the same device kind.  Large banks are
drawn on the GPU (torch's CUDA generator) and copied to the host for the oracle;
the bf16 bits are then the shared ground truth.
"""
from __future__ import annotations

import dataclasses
import math

import torch

# tensor ids for the per-tensor generator seeds
_X, _ROUTER, _GATE_UP, _DOWN, _BIAS = 0, 1, 2, 3, 4
_SH_GATE_UP, _SH_DOWN, _SH_GATE = 5, 6, 7

ZIPF_S = 1.1
WEIGHT_STD = 0.02


@dataclasses.dataclass(frozen=True)
class LayerShape:
    hidden: int       # H
    inter: int        # I (expert intermediate size)
    num_experts: int  # E
    top_k: int        # k

    @property
    def gate_up_shape(self):
        return (self.num_experts, 2 * self.inter, self.hidden)

    @property
    def down_shape(self):
        return (self.num_experts, self.hidden, self.inter)


TINY = LayerShape(hidden=256, inter=64, num_experts=8, top_k=2)
NEX = LayerShape(hidden=2048, inter=512, num_experts=256, top_k=8)


def _gen(seed: int, tensor_id: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 16 + tensor_id)
    return g


def normal_bf16(shape, std: float, seed: int, tensor_id: int, device="cpu") -> torch.Tensor:
    """N(0, std^2) samples rounded to bf16 by torch."""
    g = _gen(seed, tensor_id, device)
    t = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


def hidden_states(shape: LayerShape, T: int, seed: int, device="cpu") -> torch.Tensor:
    return normal_bf16((T, shape.hidden), 1.0, seed, _X, device)


def router_weight(shape: LayerShape, seed: int, device="cpu") -> torch.Tensor:
    return normal_bf16((shape.num_experts, shape.hidden), WEIGHT_STD, seed, _ROUTER, device)


def gate_up_bank(shape: LayerShape, seed: int, device="cpu") -> torch.Tensor:
    return normal_bf16(shape.gate_up_shape, WEIGHT_STD, seed, _GATE_UP, device)


def down_bank(shape: LayerShape, seed: int, device="cpu") -> torch.Tensor:
    return normal_bf16(shape.down_shape, WEIGHT_STD, seed, _DOWN, device)


def shared_expert(shape: LayerShape, inter_shared: int, seed: int, device="cpu"):
    """bf16 weights of the dense shared expert beside the routed ones: gate_up
    [2 I_s, H] (gate rows then up rows), down [H, I_s], and the shared-expert
    gate vector [H], all N(0, 0.02)."""
    H = shape.hidden
    return (normal_bf16((2 * inter_shared, H), WEIGHT_STD, seed, _SH_GATE_UP, device),
            normal_bf16((H, inter_shared), WEIGHT_STD, seed, _SH_DOWN, device),
            normal_bf16((H,), WEIGHT_STD, seed, _SH_GATE, device))


def zipf_bias(shape: LayerShape, seed: int, s: float = ZIPF_S) -> torch.Tensor:
    """fp32 per-expert logit bias -s*ln(rank), rank a seeded permutation of 1..E."""
    g = _gen(seed, _BIAS, "cpu")
    rank = torch.randperm(shape.num_experts, generator=g) + 1
    return torch.tensor([-s * math.log(int(r)) for r in rank], dtype=torch.float32)


@dataclasses.dataclass
class Layer:
    shape: LayerShape
    x: torch.Tensor            # [T, H] bf16
    router_w: torch.Tensor     # [E, H] bf16
    gate_up: torch.Tensor      # [E, 2I, H] bf16
    down: torch.Tensor         # [E, H, I] bf16
    bias: torch.Tensor | None  # [E] fp32 or None


def make_layer(shape: LayerShape, T: int, seed: int, zipf: bool = False, device="cpu") -> Layer:
    return Layer(
        shape=shape,
        x=hidden_states(shape, T, seed, device),
        router_w=router_weight(shape, seed, device),
        gate_up=gate_up_bank(shape, seed, device),
        down=down_bank(shape, seed, device),
        bias=zipf_bias(shape, seed).to(device) if zipf else None,
    )


def bf16_bits(t: torch.Tensor):
    """Host numpy uint16 view of a bf16 tensor (no rounding: a bit copy)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")


# seeds used by the tests and the benchmark
SEED_TINY = 0
SEED_STACK_BASE = 1000  # layer l of a stacked sweep uses seed 1000 + l
