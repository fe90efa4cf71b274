"""Helpers shared by the GPU parity tests (the oracle side runs on the CPU)."""
import concurrent.futures
import json
import multiprocessing
import os

import numpy as np
import torch

import moe_synth
from oracle import moe_oracle as o

FMT_NAMES = {"int4_g128": o.FMT_INT4, "mxfp4": o.FMT_MXFP4, "nvfp4": o.FMT_NVFP4}


_POOL = None


def oracle_pool():
    """Worker processes for the oracle's per-expert packing (started with
    spawn: the test process already holds a CUDA context)."""
    global _POOL
    if _POOL is None:
        workers = max(1, min(16, (os.cpu_count() or 2) - 1))
        _POOL = concurrent.futures.ProcessPoolExecutor(max_workers=workers,
                                                       mp_context=multiprocessing.get_context("spawn"))
    return _POOL


def _pack_dequant(fmt, bits):
    return o.dequant(fmt, *o.pack(fmt, bits))


class LazyOracleBank:
    """Oracle-packed, oracle-dequantised experts of a bf16 bank that lives on
    the GPU; each expert is copied to the host and packed by the oracle on
    first use (so big banks are only packed where a test needs them).
    prefetch() packs a set of experts in parallel worker processes."""

    def __init__(self, fmt: str, bank_bf16: torch.Tensor):
        self.fmt = FMT_NAMES[fmt]
        self.bank = bank_bf16
        self._cache = {}

    def packed(self, e: int):
        return o.pack(self.fmt, moe_synth.bf16_bits(self.bank[e]))

    def prefetch(self, experts):
        todo = sorted(set(int(e) for e in np.asarray(experts).ravel()) - set(self._cache))
        if len(todo) < 2:
            return
        futs = {e: oracle_pool().submit(_pack_dequant, self.fmt, moe_synth.bf16_bits(self.bank[e])) for e in todo}
        for e, f in futs.items():
            self._cache[e] = f.result()

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


def flip_allowance(gpu_act, a_exact, a_round, rid, rw, down, num_experts):
    """How far correct re-roundings can move each output element.

    Where the GPU's fp32 accumulation put an activation a = (token t, slot j,
    feature i) on the other side of a bf16 rounding boundary than the exact
    value, the GPU's bf16 a and the oracle's differ by the bf16 spacing at a.
    Through the down projection and the combine that moves out[t, h] by
    |w_tj| * |Wd_e[h, i]| * spacing(a) at most (e = ids[t, j]).  Returns
    (allowance [T, H]: that bound summed over each token's flipped
    activations, flipped [T]: tokens with at least one flipped activation).
    Everything but the set of flipped positions comes from the oracle."""
    offsets, sorted_rows, _ = o.permute(rid, num_experts)
    T, k = rid.shape
    flipped = np.zeros(T, dtype=bool)
    allow = None
    ps, fs = np.nonzero(gpu_act != a_round)
    for p, i in zip(ps, fs):
        t, j = divmod(int(sorted_rows[p]), k)
        wd = down.expert(int(rid[t, j]))
        if allow is None:
            allow = np.zeros((T, wd.shape[0]))
        allow[t] += abs(float(rw[t, j])) * np.abs(wd[:, i]) * float(bf16_ulp(a_exact[p, i]))
        flipped[t] = True
    return allow, flipped


def assert_layer_parity(gpu_out, pure, allowance, flipped, what=""):
    """The layer-output bound against the pure oracle (no GPU value in `pure`).

    Every element of a token without a flipped activation must satisfy
    |gpu - ref| <= 1e-2 |ref| + 1e-3 rms(ref).  A token with flipped
    activations may exceed that by at most its flip allowance (see
    flip_allowance) element by element.  Returns a summary for the report."""
    g = gpu_out.float().cpu().numpy().astype(np.float64) if isinstance(gpu_out, torch.Tensor) else gpu_out
    rms = float(np.sqrt(np.mean(pure ** 2)))
    tol = 1e-2 * np.abs(pure) + 1e-3 * rms
    err = np.abs(g - pure)
    outside = err > tol
    clean = ~flipped
    n_clean_bad = int(outside[clean].sum())
    assert n_clean_bad == 0, (f"{what}: {n_clean_bad} of {int(clean.sum()) * pure.shape[1]} outputs of tokens "
                              f"without flipped activations outside the tolerance (worst "
                              f"{float(np.max(err[clean] / tol[clean])):.2f}x)")
    n_flip_outside = int(outside[flipped].sum())
    worst_flip = 0.0
    if flipped.any():
        bound = tol[flipped] + allowance[flipped]
        over = err[flipped] > bound
        assert not over.any(), (f"{what}: {int(over.sum())} outputs of tokens with flipped activations exceed the "
                                f"tolerance plus their flip allowance (worst "
                                f"{float(np.max(err[flipped] / bound)):.2f}x)")
        worst_flip = float(np.max(err[flipped] / tol[flipped]))
    return dict(end_to_end_elements=int(pure.size), tokens=int(pure.shape[0]),
                tokens_with_flips=int(flipped.sum()), outside_tolerance=int(outside.sum()),
                outside_tolerance_in_flipped_tokens=n_flip_outside,
                worst_ratio_clean_tokens=float(np.max(err[clean] / tol[clean])) if clean.any() else 0.0,
                worst_ratio_flipped_tokens=worst_flip,
                max_allowance_over_tol=float(np.max(allowance[flipped] / tol[flipped])) if flipped.any() else 0.0)


def record_parity(rec: dict):
    """Append one parity record to $MOE_PARITY_REPORT (a JSON-lines file) if set."""
    path = os.environ.get("MOE_PARITY_REPORT")
    if path:
        rec = dict(rec, test=os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0])
        with open(path, "a") as f:
            f.write(json.dumps(rec) + "\n")
