"""Helpers shared by the GPU parity tests (the oracle side runs on the CPU)."""
import json
import os

import numpy as np
import torch

import moe_synth
from oracle import moe_oracle as o

FMT_NAMES = {"int4_g128": o.FMT_INT4, "mxfp4": o.FMT_MXFP4, "nvfp4": o.FMT_NVFP4}


class LazyOracleBank:
    """Oracle-packed, oracle-dequantised experts of a bf16 bank that lives on
    the GPU; each expert is copied to the host and packed by the oracle on
    first use (so big banks are only packed where a test needs them)."""

    def __init__(self, fmt: str, bank_bf16: torch.Tensor):
        self.fmt = FMT_NAMES[fmt]
        self.bank = bank_bf16
        self._cache = {}

    def packed(self, e: int):
        return o.pack(self.fmt, moe_synth.bf16_bits(self.bank[e]))

    def expert(self, e: int):
        if e not in self._cache:
            self._cache[e] = o.dequant(self.fmt, *self.packed(e))
        return self._cache[e]


def out_tolerance_report(gpu_out: torch.Tensor, ref: np.ndarray):
    """Element-wise |gpu - ref| <= 1e-2 |ref| + 1e-3 rms(ref) (the layer-output
    tolerance); returns (n_bad, worst excess ratio)."""
    g = gpu_out.float().cpu().numpy().astype(np.float64)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    bound = 1e-2 * np.abs(ref) + 1e-3 * rms
    err = np.abs(g - ref)
    bad = err > bound
    return int(bad.sum()), float(np.max(err / bound)) if err.size else 0.0


def assert_out_close(gpu_out, ref, what=""):
    n_bad, worst = out_tolerance_report(gpu_out, ref)
    assert n_bad == 0, f"{what}: {n_bad} of {ref.size} outputs outside tolerance (worst {worst:.2f}x bound)"


def assert_routing_consistent(gpu_logits, ref_logits, gpu_ids, bias, k):
    """GPU and oracle fp32 logits agree to fp32 accumulation error, and the
    oracle's routing of them picks the GPU's experts except on near-ties."""
    gl = gpu_logits.cpu().numpy()
    scale = np.maximum(1.0, np.abs(ref_logits))
    assert np.max(np.abs(gl - ref_logits) / scale) < 2e-5
    ref_ids, _ = o.route(ref_logits, bias, k)
    gids = gpu_ids.cpu().numpy()
    differ = np.any(ref_ids != gids, axis=1)
    if differ.any():
        margin = o.routing_margin(ref_logits, bias, k)[differ]
        lmag = np.max(np.abs(ref_logits[differ]), axis=1)
        assert np.all(margin < 1e-4 * (1 + lmag)), "routing differs on a token that is not a near-tie"
    return int(differ.sum())


def bf16_ulp(v):
    """Spacing of bf16 values at v (2^-133 in the subnormal range)."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    _, e = np.frexp(a)
    return np.where(a == 0, 2.0 ** -133, np.ldexp(1.0, np.maximum(e - 8, -133)))


def flip_aware_activations(gpu_act, a_exact, a_round, rel=1e-4, abs_frac=2e-5, max_frac_differing=0.01):
    """The GPU's bf16 activations must be correct roundings of the exact SwiGLU
    value up to the GPU's fp32 accumulation error: every GPU value g must
    satisfy |g - a_exact| <= ulp(g)/2 + rel*|a_exact| + abs_frac*rms(a), i.e. g
    is the bf16 rounding of some value within that error band.  The band's
    absolute part covers tensor-core fp32 accumulation over K (error ~1e-6 on
    activations of rms ~0.4 at K = 2048), far below what a wrong weight, scale
    or token would cause; at most `max_frac_differing` of the elements may
    differ from the oracle's own rounding at all.  Where they differ both are
    correct results and the reference continues with the GPU's.  Returns
    (activations for the reference, number of elements that differ)."""
    diff = gpu_act != a_round
    n = int(diff.sum())
    assert n <= max_frac_differing * gpu_act.size, f"{n} of {gpu_act.size} activations differ from the oracle"
    if n:
        g, r, x = gpu_act[diff], a_round[diff], a_exact[diff]
        tol = rel * np.abs(x) + abs_frac * float(np.sqrt(np.mean(a_round ** 2)))
        bad = np.abs(g - x) > 0.5 * bf16_ulp(g) + tol
        assert not bad.any(), (f"{int(bad.sum())} of {gpu_act.size} activations differ from the oracle beyond "
                               f"fp32 accumulation error; e.g. gpu={g[bad][:4]} oracle={r[bad][:4]} "
                               f"exact={x[bad][:4]}")
    return np.where(diff, gpu_act, a_round), n


def record_parity(rec: dict):
    """Append one parity record to $MOE_PARITY_REPORT (a JSON-lines file) if set."""
    path = os.environ.get("MOE_PARITY_REPORT")
    if path:
        rec = dict(rec, test=os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0])
        with open(path, "a") as f:
            f.write(json.dumps(rec) + "\n")
