"""Benchmark of the W4A16 routed-expert MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Workloads (Qwen3.5-MoE expert layer: hidden 2048, 256 experts, top-8, expert
intermediate 512; synthetic seeded inputs, random-init weights):
  decode4   (default) INT4 g128, 4 tokens per layer, a stack of 40 layers with
            independently seeded weights (16.6 GB packed); one step = one CUDA
            graph replay of moe_forward over all 40 layers on the same tokens
  decode1   the same with 1 token
  c32       INT4, 32 tokens with a Zipf(1.1) expert-popularity logit bias
  prefill   INT4, 8192 tokens, one step = one layer (rotating over 40 layers)
  prefill_zipf  the same with the Zipf logit bias
  mx_decode4 / mx_prefill   the MXFP4 stack (17.1 GB packed) at 4 / 8192 tokens
  nv_decode4 / nv_prefill   the NVFP4 stack (E4M3 scale per 16 elements) at 4 / 8192 tokens
  sh_decode4 / sh_prefill   the INT4 stack with each layer's bf16 shared expert (moe_forward_shared)

The metric is MoE-layer tokens per second: tokens x layers processed per
second of device time, whole job (all ranks).  With --gpus N > 1 (launched by
torch.distributed.run) every rank runs its own replica of the stack on its own
tokens (data parallel, weak scaling); the only collective is the max-over-ranks
reduction of the timed region.

The default run prints ONE JSON line for decode4 that also carries a
`prefill` record: the INT4 8192-token prefill on the same stack, timed the
same way with its own steps, clocks and roofline.

Roofline: the whole layer's algorithmic bytes (decode) or flops (prefill) over
the device-timed time per layer, and the same for the dominant kernel.  A
kernel's time is the per-layer time times its share of the layer, the share
measured live with CUDA events recorded around each stage in a replay of the
same graph (events inside a graph stop programmatic launch overlap, so their
raw durations, also reported, overstate the kernels).  `traffic` is DRAM read
+ write bytes of one ncu capture of the dominant kernel, reported only while
the kernel sources still match the capture's digest (null otherwise).
`e2e` times moe_forward_host (the C ABI call with the hidden states and the
output in pinned host memory, copies in the timed region), one call per layer.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import moe_synth  # noqa: E402

NUM_LAYERS = 40
PREFILL_T = 8192
WORKLOADS = {
    # name: (fmt, T, zipf, layers per step)
    "decode4": ("int4_g128", 4, False, NUM_LAYERS),
    "decode1": ("int4_g128", 1, False, NUM_LAYERS),
    "c32": ("int4_g128", 32, True, NUM_LAYERS),
    "prefill": ("int4_g128", PREFILL_T, False, 1),
    "prefill_zipf": ("int4_g128", PREFILL_T, True, 1),
    "mx_decode4": ("mxfp4", 4, False, NUM_LAYERS),
    "mx_prefill": ("mxfp4", PREFILL_T, False, 1),
    "nv_decode4": ("nvfp4", 4, False, NUM_LAYERS),
    "nv_prefill": ("nvfp4", PREFILL_T, False, 1),
    "sh_decode4": ("int4_g128", 4, False, NUM_LAYERS),
    "sh_prefill": ("int4_g128", PREFILL_T, False, 1),
}
# workloads whose layers carry the bf16 shared expert (intermediate 512)
SHARED_INTER = {"sh_decode4": 512, "sh_prefill": 512}
METRIC = "W4A16 MoE-layer tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
CSRC = os.path.join(ROOT, "weight_only_bit_router_b200", "csrc")
# the sources of each kernel family (their digest keys a traffic capture)
KERNEL_SOURCES = {
    "decode": ("decode.cu", "decode_common.cuh", "common.cuh", "internal.h"),
    "grouped": ("gemm_sm100.cu", "common.cuh", "internal.h"),
}
# DRAM bytes (read + write) per launch of a workload's dominant kernel from one
# ncu capture: (workload, kernel) -> (bytes, kernel family, digest of its sources).
# decode4 gate_up: 47.31 MB read + 0.04 MB written (2-layer stack, the same
# per-layer work): its 32.5 MB of packed gate_up rows and the 16.3 MB of down
# matrices it requests into L2 for the down kernel (moved earlier, not re-read).
# prefill gate_up: 377.57 MB read + 56.87 MB written (packed bank, x rows
# gathered per 128-row weight tile, activations out).
MEASURED_TRAFFIC = {
    ("decode4", "gate_up"): (47_347_968, "decode", "23db5b2d1058ea6c"),
    ("prefill", "gate_up"): (434_441_472, "grouped", "6957f73dd9f9e7fa"),
}


# ---------------------------------------------------------------- distributed plumbing

def dist_env():
    """(rank, local_rank, world_size) from the torchrun environment."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def dist_init(backend: str):
    rank, local, world = dist_env()
    if world > 1 and not torch.distributed.is_initialized():
        import datetime
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, local, world


def reduce_max(value: float, device) -> float:
    """Max of a per-rank scalar over all ranks (identity on one process)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier():
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.barrier()


def rank_token_seed(rank: int, T: int) -> int:
    """Each rank processes its own tokens (weak scaling): a distinct seed per rank."""
    return 500_000 + 1000 * rank + T


def source_digest(family: str) -> str:
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[family]:
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic(workload: str, kernel: str):
    """ncu DRAM bytes of the kernel, or None when no capture matches its current sources."""
    rec = MEASURED_TRAFFIC.get((workload, kernel))
    if rec is None:
        return None
    nbytes, family, digest = rec
    return nbytes if source_digest(family) == digest else None


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str, period_ms: int = 100):
        self.gpu_id, self.period_ms, self.proc = gpu_id, period_ms, None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_id}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(self.period_ms)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
        time.sleep(0.25)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- the layer stack

class Stack:
    """L layers of packed expert banks + bf16 router weights on one GPU."""

    def __init__(self, moe, fmt: str, layers: int, device):
        s = moe_synth.NEX
        self.moe, self.fmt, self.L = moe, fmt, layers
        self.shape = moe.make_shape(s.hidden, s.inter, s.num_experts, s.top_k, fmt)
        gu_b, dn_b = moe.moe_packed_bytes(self.shape, 0), moe.moe_packed_bytes(self.shape, 1)
        self.gate_up = torch.empty(layers, gu_b, dtype=torch.uint8, device=device)
        self.down = torch.empty(layers, dn_b, dtype=torch.uint8, device=device)
        self.router = torch.empty(layers, s.num_experts, s.hidden, dtype=torch.bfloat16, device=device)
        self.zipf_bias = [moe_synth.zipf_bias(s, moe_synth.SEED_STACK_BASE + l).to(device) for l in range(layers)]
        pack = {"int4_g128": moe.moe_pack_int4_g128, "mxfp4": moe.moe_pack_mxfp4, "nvfp4": moe.moe_pack_nvfp4}[fmt]
        for l in range(layers):
            seed = moe_synth.SEED_STACK_BASE + l
            w = moe_synth.gate_up_bank(s, seed, device)
            pack(w, packed=self.gate_up[l])
            del w
            w = moe_synth.down_bank(s, seed, device)
            pack(w, packed=self.down[l])
            del w
            self.router[l].copy_(moe_synth.router_weight(s, seed, device))
        torch.cuda.synchronize()
        self.packed_bytes = (gu_b + dn_b) * layers

    def bias(self, zipf: bool):
        return self.zipf_bias if zipf else [None] * self.L

    def layer_bf16(self, l: int):
        """The bf16 source of layer l (regenerated from its seed; for the oracle)."""
        s = moe_synth.NEX
        seed = moe_synth.SEED_STACK_BASE + l
        dev = self.gate_up.device
        return moe_synth.gate_up_bank(s, seed, dev), moe_synth.down_bank(s, seed, dev)


def capture_graph(fn):
    """Capture fn() (a sequence of enqueues on the current stream) into a CUDA graph."""
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()  # warm-up outside capture (also loads kernels)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    return g


# ---------------------------------------------------------------- algorithmic work

def layer_work(moe, shape, T: int, touched: float, inter_sh: int = 0, folded: bool = False):
    """Algorithmic bytes (decode) and flops (prefill) per layer of each kernel
    stage and of the whole layer.

    bytes: packed weights of the touched experts streamed once + the stage's
    inputs and outputs (intermediates that the method does not define, such as
    per-row fp32 partials, are not counted); flops: 2*T*E*H for the router,
    2*R*(2I)*H for gate_up, 2*R*H*I for down, R = T*k.  A bf16 shared expert
    of intermediate inter_sh adds its weights (gate_up, gate vector, down) and
    flops to the layer; folded into the decode kernels, its gate_up rows and
    gate to the router stage (the routing GEMV computes them) and its down
    rows to the down stage."""
    H, I, E, k = shape.hidden, shape.inter, shape.num_experts, shape.top_k
    R = T * k
    gu_e = moe.moe_packed_bytes(shape, 0) // E
    dn_e = moe.moe_packed_bytes(shape, 1) // E
    router = {"bytes": E * H * 2 + T * H * 2 + T * E * 4, "flops": 2 * T * E * H}
    gate_up = {"bytes": touched * gu_e + T * H * 2 + R * I * 2, "flops": 2 * R * 2 * I * H}
    down = {"bytes": touched * dn_e + R * I * 2 + T * H * 2, "flops": 2 * R * H * I}
    n_sh = 2 * inter_sh + 1 if inter_sh else 0  # gate_up rows and the gate vector
    sh_gu = {"bytes": n_sh * H * 2, "flops": 2 * T * n_sh * H}
    sh_dn = {"bytes": H * inter_sh * 2, "flops": 2 * T * H * inter_sh}
    if folded:
        for d, add in ((router, sh_gu), (down, sh_dn)):
            d["bytes"] += add["bytes"]
            d["flops"] += add["flops"]
    layer = {"bytes": E * H * 2 + T * H * 2 + touched * (gu_e + dn_e) + T * H * 2,
             "flops": 2 * T * E * H + 2 * R * 2 * I * H + 2 * R * H * I}
    layer["bytes"] += sh_gu["bytes"] + sh_dn["bytes"]
    layer["flops"] += sh_gu["flops"] + sh_dn["flops"]
    return {"router": router, "gate_up": gate_up, "down": down, "layer": layer}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def workload_config(name: str, world: int, stack_layers: int):
    """The `config` object of a workload's JSON line (identical in both arms)."""
    fmt, T, zipf, layers_per_step = WORKLOADS[name]
    layers_per_step = min(layers_per_step, stack_layers)
    inter_sh = SHARED_INTER.get(name)
    s = moe_synth.NEX
    return {
        "workload": (f"nex_moe_{fmt}_T{T}{'_zipf' if zipf else ''}{f'_shared{inter_sh}' if inter_sh else ''}"
                     f"_{layers_per_step}layer_step_of_{stack_layers}layer_stack"),
        "hidden": s.hidden, "experts": s.num_experts, "top_k": s.top_k, "inter": s.inter,
        "tokens_per_layer": T, "layers_per_step": layers_per_step, "stack_layers": stack_layers,
        "l2": "inputs larger than L2: steps rotate over a stack of packed layers larger than L2",
        "parallelism": f"dp{world} replicas (one stack per GPU)",
    }


# ---------------------------------------------------------------- CPU oracle timing

def oracle_sample(stack, x_bf16, bias, T, budget_s: float, max_layers: int = 3, shared=None):
    """Time the CPU oracle on a bounded sample of the workload.

    Inputs (bf16 weights of the touched experts, packed by the oracle's own
    packer) are prepared untimed; the timed part is the oracle's forward of
    the sampled tokens: router logits, top-k, dequantisation of every touched
    expert (cold), SwiGLU experts and the weighted combine.  Returns
    (layer-tokens per second, description, threads, seconds)."""
    from oracle import moe_oracle as o
    from threadpoolctl import threadpool_info
    fmt = {"int4_g128": o.FMT_INT4, "mxfp4": o.FMT_MXFP4, "nvfp4": o.FMT_NVFP4}[stack.fmt]
    k = stack.shape.top_k
    done_tokens, elapsed, used_layers = 0.0, 0.0, 0
    xb_all = moe_synth.bf16_bits(x_bf16)
    for l in range(min(max_layers, stack.L)):
        if elapsed >= budget_s:
            break
        router = moe_synth.bf16_bits(stack.router[l])
        b = None if bias[l] is None else bias[l].cpu().numpy()
        ntok = min(T, 16)  # the oracle runs at most 16 tokens of a layer per sample
        xb = xb_all[:ntok]
        ids, _ = o.route(o.router_logits(xb, router), b, k)
        touched = sorted(set(int(e) for e in ids.reshape(-1)))
        gu_bf16, dn_bf16 = stack.layer_bf16(l)
        gu_c, gu_s, dn_c, dn_s = {}, {}, {}, {}
        for e in touched:
            gu_c[e], gu_s[e] = o.pack(fmt, moe_synth.bf16_bits(gu_bf16[e]))
            dn_c[e], dn_s[e] = o.pack(fmt, moe_synth.bf16_bits(dn_bf16[e]))
        del gu_bf16, dn_bf16
        gu = o.PackedBank(fmt, gu_c, gu_s)
        dn = o.PackedBank(fmt, dn_c, dn_s)
        sh = None if shared is None else [moe_synth.bf16_bits(t) for t in shared[l]]
        t0 = time.perf_counter()
        if sh is None:
            o.forward(xb, router, b, gu, dn, k)
        else:
            o.forward_with_shared(xb, router, b, gu, dn, k, sh)
        elapsed += time.perf_counter() - t0
        done_tokens += ntok
        used_layers += 1
    threads = max((d.get("num_threads", 1) for d in threadpool_info()), default=1)
    desc = (f"CPU oracle (NumPy fp64) forward of {int(done_tokens)} token-layers "
            f"({used_layers} layer(s) x up to 16 tokens of this workload, cold dequantisation of every touched "
            f"expert{', the bf16 shared expert' if shared is not None else ''}; packing untimed)")
    return done_tokens / max(elapsed, 1e-9), desc, int(threads), elapsed


# ---------------------------------------------------------------- our arm

def time_replays(replay, steps: int, warmup: int, stream, device, gpu_id):
    """Device time of `steps` calls of replay(i) after `warmup` untimed ones:
    barrier + synchronize on both sides, CUDA events on the stream, max over
    ranks, nvidia-smi clocks sampled during the timed region."""
    for i in range(warmup):
        replay(i)
    torch.cuda.synchronize()
    barrier()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_id) as clk:
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        start.record(stream)
        for i in range(steps):
            replay(warmup + i)
        end.record(stream)
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
    return reduce_max(start.elapsed_time(end), device), clk.summary()


def measure(moe, stack, name: str, steps: int, warmup: int, path: int, rank: int, world: int, device,
            cpu_budget: float, with_cpu: bool):
    """One workload on a packed stack: the device-timed value, the roofline,
    the end-to-end number and (optionally) the CPU oracle beside it."""
    fmt, T, zipf, layers_per_step = WORKLOADS[name]
    L = stack.L
    layers_per_step = min(layers_per_step, L)
    shape = stack.shape
    bias = stack.bias(zipf)
    x = moe_synth.hidden_states(moe_synth.NEX, T, rank_token_seed(rank, T), device)
    inter_sh = SHARED_INTER.get(name)
    shared = ([moe_synth.shared_expert(moe_synth.NEX, inter_sh, moe_synth.SEED_STACK_BASE + l, device)
               for l in range(L)] if inter_sh else None)
    ws = moe.alloc_workspace_shared(shape, inter_sh, T, device) if inter_sh else moe.alloc_workspace(shape, T, device)
    outs = torch.empty(L, T, shape.hidden, dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream()

    def layer_call(l, events=None, debug=None):
        if shared:
            moe.moe_forward_shared(shape, shared[l], x, stack.router[l], stack.gate_up[l], stack.down[l], ws,
                                   out=outs[l], bias=bias[l], path=path, events=events, debug=debug,
                                   stream=torch.cuda.current_stream())
        else:
            moe.moe_forward(shape, x, stack.router[l], stack.gate_up[l], stack.down[l], ws, out=outs[l],
                            bias=bias[l], path=path, events=events, debug=debug,
                            stream=torch.cuda.current_stream())

    def step_layers(gi):
        return list(range(gi * layers_per_step, (gi + 1) * layers_per_step))

    # one step: layers_per_step consecutive layers; graphs rotate over the stack
    n_graphs = L // layers_per_step
    graphs = [capture_graph(lambda ls=step_layers(gi): [layer_call(l) for l in ls]) for gi in range(n_graphs)]
    assert moe.moe_workspace_status(ws) == moe.MOE_OK
    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    ms, clocks = time_replays(lambda i: graphs[i % n_graphs].replay(), steps, warmup, stream, device, gpu_id)
    value = world * T * layers_per_step * steps / (ms / 1e3)
    status = moe.moe_workspace_status(ws)
    layer_ms = ms / steps / layers_per_step
    del graphs

    # ---- stage shares: events around each stage in an instrumented replay
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * moe.MOE_NUM_STAGES)] for _ in range(L)]
    for evs in ev:
        for e in evs:
            e.record(stream)  # materialise the events before capture
    torch.cuda.synchronize()
    inst = [capture_graph(lambda ls=step_layers(gi): [layer_call(l, ev[l]) for l in ls]) for gi in range(n_graphs)]
    stage_ms = {n: [] for n in moe.STAGE_NAMES}
    for r in range(max(1, min(20, steps))):
        gi = r % n_graphs
        inst[gi].replay()
        torch.cuda.synchronize()
        for l in step_layers(gi):
            for si, n in enumerate(moe.STAGE_NAMES):
                stage_ms[n].append(ev[l][2 * si].elapsed_time(ev[l][2 * si + 1]))
    del inst
    stage_events = {n: float(np.mean(v)) for n, v in stage_ms.items()}
    total_events = sum(stage_events.values())
    stage_share = {n: v / total_events for n, v in stage_events.items()}

    # touched experts per layer (from the routing of each layer)
    touched = []
    ids_buf = torch.empty(T, shape.top_k, dtype=torch.int32, device=device)
    for l in range(L):
        layer_call(l, debug={"topk_ids_out": ids_buf})
        touched.append(len(torch.unique(ids_buf)))
    avg_touched = float(np.mean(touched))
    folded = bool(shared) and (moe.moe_forward_shared_launch_count(shape, inter_sh, T, path)
                               == moe.moe_forward_launch_count(shape, T, path, False))
    work = layer_work(moe, shape, T, avg_touched, inter_sh or 0, folded)
    peaks, peak_kind = load_peaks()
    decode = T <= 32 and path != moe.MOE_PATH_PREFILL
    dom = max(("router", "gate_up", "down"), key=lambda n: stage_share[n])
    dom_ms = layer_ms * stage_share[dom]
    if decode:
        peak, unit, key, scale = peaks["hbm_gbs"], "GB/s", "bytes", 1e9
        bound, pk = "hbm", f"{peak_kind} STREAM-copy HBM bandwidth"
    else:
        peak, unit, key, scale = peaks["bf16_tflops_sustained"], "TFLOP/s", "flops", 1e12
        bound, pk = "tensor", f"{peak_kind} sustained cuBLAS bf16 GEMM"
    achieved = work[dom][key] / (dom_ms / 1e3) / scale
    layer_ach = work["layer"][key] / (layer_ms / 1e3) / scale
    roof = {"bound": bound, "kernel": dom, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
            "traffic": measured_traffic(name, dom) if path == moe.MOE_PATH_AUTO else None,
            "peak_kind": pk, f"algorithmic_{key}_per_launch": work[dom][key], "avg_launch_ms": dom_ms,
            "avg_launch_ms_event_bracketed": stage_events[dom],
            "layer": {"achieved": layer_ach, "frac": layer_ach / peak, f"algorithmic_{key}": work["layer"][key],
                      "ms": layer_ms}}

    # ---- end to end through the C ABI with host buffers (one call per layer)
    e2e = None
    if not shared:
        ws_h = torch.empty(moe.moe_workspace_bytes_host(shape, T), dtype=torch.uint8, device=device)
        moe.moe_workspace_init(ws_h)
        x_host = x.cpu().pin_memory()
        out_host = torch.empty(layers_per_step, T, shape.hidden, dtype=torch.bfloat16).pin_memory()

        def host_step(i):
            for j, l in enumerate(step_layers(i % n_graphs)):
                moe.moe_forward_host(shape, x_host, stack.router[l], stack.gate_up[l], stack.down[l], ws_h,
                                     out_host[j], bias=bias[l], path=path, stream=stream)

        e2e_steps = max(3, min(steps, 50))
        e2e_ms, _ = time_replays(host_step, e2e_steps, 3, stream, device, gpu_id)
        assert moe.moe_workspace_status(ws_h) == moe.MOE_OK
        e2e = {"value": world * T * layers_per_step * e2e_steps / (e2e_ms / 1e3), "unit": "layer-tokens/s",
               "h2d_bytes_per_step": layers_per_step * T * shape.hidden * 2,
               "d2h_bytes_per_step": layers_per_step * T * shape.hidden * 2, "steps": e2e_steps,
               "call": "moe_forward_host per layer, pinned host buffers"}
        del ws_h

    per_layer = (moe.moe_forward_shared_launch_count(shape, inter_sh, T, path) if shared
                 else moe.moe_forward_launch_count(shape, T, path, False))
    cpu = None
    if with_cpu and rank == 0 and world == 1:
        v, desc, threads, secs = oracle_sample(stack, x, bias, T, budget_s=cpu_budget, shared=shared)
        cpu = {"value": v, "unit": "layer-tokens/s", "cores": threads, "kind": "oracle", "sample": desc,
               "seconds": secs}
    del ws, outs
    torch.cuda.empty_cache()
    return {
        "value": value, "ms_per_step": ms / steps, "steps": steps, "warmup": warmup,
        "roofline": roof, "stage_ms_event_bracketed": stage_events, "stage_share": stage_share,
        "e2e": e2e, "gpu_launches": per_layer * layers_per_step * steps, "clocks": clocks,
        "cpu_baseline": cpu, "device_status": moe.moe_status_str(status),
        "avg_touched_experts": avg_touched,
        "path": "decode GEMV kernels" if decode else "tcgen05 grouped GEMMs",
    }


def run_ours(args, rank, local, world):
    import weight_only_bit_router_b200 as moe
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    fmt = WORKLOADS[args.workload][0]
    stack = Stack(moe, fmt, args.stack_layers, device)
    path = {"auto": moe.MOE_PATH_AUTO, "decode": moe.MOE_PATH_DECODE, "prefill": moe.MOE_PATH_PREFILL}[args.path]
    m = measure(moe, stack, args.workload, args.steps, args.warmup, path, rank, world, device, args.cpu_budget,
                not args.no_cpu_baseline)
    details = {k: m[k] for k in ("stage_ms_event_bracketed", "stage_share", "device_status", "avg_touched_experts",
                                 "path")}
    details.update(packed_stack_bytes=stack.packed_bytes, path_option=args.path)
    line = {
        "metric": METRIC, "value": m["value"], "unit": "layer-tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": m["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic seeded N(0,1) tokens, N(0,0.02) random-init weights",
        "config": workload_config(args.workload, world, stack.L),
        "roofline": m["roofline"], "cpu_baseline": m["cpu_baseline"], "e2e": m["e2e"],
        "gpu_launches": m["gpu_launches"], "clocks": m["clocks"], "details": details,
    }
    if (args.prefill_record and WORKLOADS[args.workload][1] <= 32 and fmt == "int4_g128"
            and args.workload not in SHARED_INTER):
        # the INT4 8192-token prefill on the same stack: its own steps, clocks and roofline
        steps = max(3, min(args.steps, 40))
        p = measure(moe, stack, "prefill", steps, args.warmup, moe.MOE_PATH_AUTO, rank, world, device, 0.0, False)
        line["prefill"] = {
            "workload": workload_config("prefill", world, stack.L)["workload"], "value": p["value"],
            "unit": "layer-tokens/s", "ms_per_step": p["ms_per_step"], "steps": steps, "warmup": args.warmup,
            "roofline": p["roofline"], "e2e": p["e2e"], "gpu_launches": p["gpu_launches"], "clocks": p["clocks"],
            "details": {k: p[k] for k in ("stage_ms_event_bracketed", "stage_share", "device_status",
                                          "avg_touched_experts", "path")},
        }
        line["gpu_launches"] += p["gpu_launches"]
    return line


# ---------------------------------------------------------------- reference arm (the CPU oracle)

def run_reference(args, rank, world):
    """The oracle timed on the host cores, on this workload's config and metric.
    Each step is a bounded sample: one token of one layer (cold dequantisation
    of its k experts), so that the whole run ends within a few minutes."""
    if rank != 0:
        return None
    from oracle import moe_oracle as o
    from threadpoolctl import threadpool_info
    fmt_name, T, zipf, _ = WORKLOADS[args.workload]
    fmt = {"int4_g128": o.FMT_INT4, "mxfp4": o.FMT_MXFP4, "nvfp4": o.FMT_NVFP4}[fmt_name]
    inter_sh = SHARED_INTER.get(args.workload)
    s = moe_synth.NEX
    n_layers = 2
    prepared = []
    # inputs drawn with the same generator as our arm when a GPU is present
    gen_dev = "cuda" if torch.cuda.is_available() else "cpu"
    for l in range(n_layers):
        seed = moe_synth.SEED_STACK_BASE + l
        router = moe_synth.bf16_bits(moe_synth.router_weight(s, seed, gen_dev))
        b = moe_synth.zipf_bias(s, seed).numpy() if zipf else None
        x = moe_synth.bf16_bits(moe_synth.hidden_states(s, T, rank_token_seed(0, T), gen_dev))[:max(1, min(T, 64))]
        ids, _ = o.route(o.router_logits(x, router), b, s.top_k)
        touched = sorted(set(int(e) for e in ids.reshape(-1)))
        gu = moe_synth.gate_up_bank(s, seed, gen_dev)
        dn = moe_synth.down_bank(s, seed, gen_dev)
        gu_p = {e: o.pack(fmt, moe_synth.bf16_bits(gu[e])) for e in touched}
        dn_p = {e: o.pack(fmt, moe_synth.bf16_bits(dn[e])) for e in touched}
        del gu, dn
        sh = ([moe_synth.bf16_bits(t) for t in moe_synth.shared_expert(s, inter_sh, seed, gen_dev)]
              if inter_sh else None)
        prepared.append((router, b, x, gu_p, dn_p, sh))

    def one_step(i):
        router, b, x, gu_p, dn_p, sh = prepared[i % n_layers]
        t = i % x.shape[0]
        gu = o.PackedBank(fmt, {e: v[0] for e, v in gu_p.items()}, {e: v[1] for e, v in gu_p.items()})
        dn = o.PackedBank(fmt, {e: v[0] for e, v in dn_p.items()}, {e: v[1] for e, v in dn_p.items()})
        t0 = time.perf_counter()
        if sh is None:
            o.forward(x[t:t + 1], router, b, gu, dn, s.top_k)
        else:
            o.forward_with_shared(x[t:t + 1], router, b, gu, dn, s.top_k, sh)
        return time.perf_counter() - t0

    for i in range(args.warmup):
        one_step(i)
    total = 0.0
    steps_done = 0
    for i in range(args.steps):
        total += one_step(args.warmup + i)
        steps_done += 1
        if total > 170.0:
            break
    value = steps_done / total
    threads = max((d.get("num_threads", 1) for d in threadpool_info()), default=1)
    sample = ("CPU oracle (NumPy fp64) forward of one token of one layer per step (router, top-k, cold "
              f"dequantisation of its {s.top_k} experts, SwiGLU, combine"
              f"{', the bf16 shared expert' if inter_sh else ''}); packing untimed")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "layer-tokens/s", "n_gpus": world,
        "steps": steps_done, "warmup": args.warmup, "ms_per_step": 1e3 * total / max(1, steps_done),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic seeded N(0,1) tokens, N(0,0.02) random-init weights",
        "config": workload_config(args.workload, world, args.stack_layers),
        "cpu_baseline": {"value": value, "unit": "layer-tokens/s", "cores": int(threads), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "layer-tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="decode4")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill-record", dest="prefill_record", action="store_false",
                    help="leave out the 8192-token prefill record of the decode workloads")
    ap.add_argument("--path", choices=["auto", "decode", "prefill"], default="auto",
                    help="kernel path of moe_forward (auto: decode kernels up to 32 tokens, grouped GEMMs above)")
    ap.add_argument("--stack-layers", type=int, default=NUM_LAYERS,
                    help="layers in the packed stack (smaller only for profiling captures)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("at least 3 warm-up steps are required")
    rank, local, world = dist_env()
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0
    dist_init("nccl")
    line = run_ours(args, rank, local, world)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
