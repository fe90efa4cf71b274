"""Host-side pieces of bench.py (no GPU): the algorithmic work that its
roofline divides by, the workload config both arms print, and the rule that
a DRAM-traffic capture is reported only for the kernel sources it was taken
from."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
import weight_only_bit_router_b200 as moe  # noqa: E402

H, I, E, K = 2048, 512, 256, 8


def nex(fmt="int4_g128"):
    return moe.make_shape(H, I, E, K, fmt)


def test_layer_work_counts_each_touched_expert_once():
    T, touched = 4, 30.0
    w = bench.layer_work(moe, nex(), T, touched)
    gu_e, dn_e = 1_081_344, 540_672  # one INT4 expert's packed gate_up / down bytes (codes + bf16 scales)
    assert moe.moe_packed_bytes(nex(), 0) == E * gu_e
    assert moe.moe_packed_bytes(nex(), 1) == E * dn_e
    assert w["gate_up"]["bytes"] == touched * gu_e + T * H * 2 + T * K * I * 2
    assert w["down"]["bytes"] == touched * dn_e + T * K * I * 2 + T * H * 2
    assert w["router"]["bytes"] == E * H * 2 + T * H * 2 + T * E * 4
    assert w["layer"]["bytes"] == E * H * 2 + 2 * T * H * 2 + touched * (gu_e + dn_e)
    R = T * K
    assert w["layer"]["flops"] == 2 * T * E * H + 2 * R * 2 * I * H + 2 * R * H * I


@pytest.mark.parametrize("folded", [False, True])
def test_layer_work_adds_the_shared_expert(folded):
    T, touched, I_s = 4, 30.0, 512
    base = bench.layer_work(moe, nex(), T, touched)
    w = bench.layer_work(moe, nex(), T, touched, I_s, folded)
    sh_gu = (2 * I_s + 1) * H * 2  # gate_up rows and the gate vector, bf16
    sh_dn = H * I_s * 2
    assert w["layer"]["bytes"] - base["layer"]["bytes"] == sh_gu + sh_dn
    assert w["layer"]["flops"] - base["layer"]["flops"] == 2 * T * (2 * I_s + 1) * H + 2 * T * H * I_s
    # folded: the routing GEMV reads the shared gate_up rows, the down kernel its down rows
    assert w["router"]["bytes"] - base["router"]["bytes"] == (sh_gu if folded else 0)
    assert w["down"]["bytes"] - base["down"]["bytes"] == (sh_dn if folded else 0)
    assert w["gate_up"] == base["gate_up"]


def test_workload_config_is_the_same_for_both_arms_and_names_the_workload():
    for name in ("decode4", "c32", "prefill", "sh_decode4", "mx_decode4"):
        c = bench.workload_config(name, 1, bench.NUM_LAYERS)
        fmt, T, zipf, _ = bench.WORKLOADS[name]
        assert c["workload"].startswith(f"nex_moe_{fmt}_T{T}")
        assert ("_zipf" in c["workload"]) == zipf
        assert ("_shared512" in c["workload"]) == (name in bench.SHARED_INTER)
        assert (c["hidden"], c["experts"], c["top_k"], c["inter"]) == (H, E, K, I)
        assert bench.workload_config(name, 1, bench.NUM_LAYERS) == c


def test_traffic_is_reported_only_for_the_captured_sources(monkeypatch):
    for (workload, kernel), (nbytes, family, _) in list(bench.MEASURED_TRAFFIC.items()):
        assert family in bench.KERNEL_SOURCES
        # a record taken from the sources as they are is reported
        monkeypatch.setitem(bench.MEASURED_TRAFFIC, (workload, kernel),
                            (nbytes, family, bench.source_digest(family)))
        assert bench.measured_traffic(workload, kernel) == nbytes
        # after a source change the record is stale: traffic is not reported
        monkeypatch.setitem(bench.MEASURED_TRAFFIC, (workload, kernel), (nbytes, family, "0" * 16))
        assert bench.measured_traffic(workload, kernel) is None
        monkeypatch.undo()
    assert bench.measured_traffic("decode4", "down") is None  # never captured
