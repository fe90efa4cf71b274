"""CUDA path vs the CPU oracle, through the C ABI (needs a B200).

Bit-exact: packed bytes, dequantised weights, routing ids on identical
logits, permutations.  Tolerance: routing weights |dw| <= 1e-6 (1 + |w|);
layer outputs |gpu - ref| <= 1e-2 |ref| + 1e-3 rms(ref) per element.
"""
import numpy as np
import pytest
import torch

import moe_synth
import weight_only_bit_router_b200 as moe
from oracle import moe_oracle as o
from parity_util import (FMT_NAMES, LazyOracleBank, assert_layer_parity, assert_out_close,
                         assert_routing_consistent, flip_allowance, flip_aware_activations, out_tolerance_report,
                         record_parity)

pytestmark = pytest.mark.gpu
DEV = "cuda"
FMTS = ["int4_g128", "mxfp4", "nvfp4"]
PACKERS = {"int4_g128": moe.moe_pack_int4_g128, "mxfp4": moe.moe_pack_mxfp4, "nvfp4": moe.moe_pack_nvfp4}


def pack_gpu(fmt, w):
    return PACKERS[fmt](w)


def gpu_split(fmt, packed, E, N, K):
    codes, scales = moe.split_bank(packed, fmt, E, N, K)
    c = codes.cpu().numpy()
    if fmt == "nvfp4":
        return c, (scales[0].cpu().numpy(), scales[1].cpu().numpy())
    s = scales.cpu().numpy()
    return c, (s.view(np.uint16) if fmt == "int4_g128" else s)


def scales_equal(fmt, a, b):
    if fmt == "nvfp4":
        return np.array_equal(a[0], b[0]) and np.array_equal(a[1].view(np.uint32), np.asarray(b[1], np.float32).view(np.uint32))
    return np.array_equal(a, b)


# ---------------------------------------------------------------- packing

def edge_bank():
    """Rows that exercise the corners of both packers (K = 192: a short last
    INT4 group of 64; MXFP4 blocks of 32)."""
    rng = np.random.default_rng(0)
    K = 192
    rows = [
        np.zeros(K),                                               # all-zero groups
        rng.normal(size=K) * 0.02,
        rng.normal(size=K) * 1e3,
        np.concatenate([[1.75, -0.875, 0.125, 0.1875], np.zeros(K - 4)]),  # hand-worked ties
        np.concatenate([[3.0, -0.3125, 1.25, 0.625], np.zeros(K - 4)]),
        np.full(K, 2.0 ** -133),                                   # bf16 subnormals
        rng.normal(size=K) * 1e-38,
        np.concatenate([[3.0e38, -1.0], rng.normal(size=K - 2)]),  # near bf16 max
        (rng.integers(-8, 8, size=K) * 0.25),                      # many exact ties
        -np.abs(rng.normal(size=K)),
    ]
    w = np.stack(rows)[None]                                       # [1, 10, 192]
    bits = o.f64_to_bf16(w)
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)


@pytest.mark.parametrize("fmt", FMTS)
def test_pack_bit_exact_tiny_and_edges(fmt):
    for w in (moe_synth.gate_up_bank(moe_synth.TINY, 0), moe_synth.down_bank(moe_synth.TINY, 0), edge_bank()):
        E, N, K = w.shape
        packed = pack_gpu(fmt, w.to(DEV))
        torch.cuda.synchronize()
        gc, gs = gpu_split(fmt, packed, E, N, K)
        rc, rs = o.pack(FMT_NAMES[fmt], moe_synth.bf16_bits(w))
        assert np.array_equal(gc, rc)
        assert scales_equal(fmt, gs, rs)


@pytest.mark.parametrize("fmt", FMTS)
def test_dequant_bit_exact(fmt):
    for w in (moe_synth.gate_up_bank(moe_synth.TINY, 1), edge_bank()):
        E, N, K = w.shape
        packed = pack_gpu(fmt, w.to(DEV))
        deq = moe.moe_dequant(packed, fmt, E, N, K)
        torch.cuda.synchronize()
        ref = o.dequant(FMT_NAMES[fmt], *o.pack(FMT_NAMES[fmt], moe_synth.bf16_bits(w)))
        got = o.bf16_to_f64(moe_synth.bf16_bits(deq))
        assert np.array_equal(got, ref)


@pytest.mark.parametrize("fmt", FMTS)
def test_pack_bit_exact_full_layer_sampled_experts(fmt):
    gu = moe_synth.gate_up_bank(moe_synth.NEX, seed=1000, device=DEV)
    packed = pack_gpu(fmt, gu)
    torch.cuda.synchronize()
    E, N, K = gu.shape
    codes, scales = moe.split_bank(packed, fmt, E, N, K)
    for e in (0, 131, 255):
        rc, rs = o.pack(FMT_NAMES[fmt], moe_synth.bf16_bits(gu[e]))
        assert np.array_equal(codes[e].cpu().numpy(), rc)
        if fmt == "nvfp4":
            s = (scales[0][e].cpu().numpy(), scales[1][e:e + 1].cpu().numpy()[0])
        else:
            s = scales[e].cpu().numpy()
            s = s.view(np.uint16) if fmt == "int4_g128" else s
        assert scales_equal(fmt, s, rs)


def test_pack_counts_nonfinite_inputs():
    w = moe_synth.gate_up_bank(moe_synth.TINY, 2).to(DEV)
    w[0, 0, 5] = float("nan")
    w[3, 7, 100] = float("inf")
    cnt = torch.zeros(1, dtype=torch.int32, device=DEV)
    moe.moe_pack_int4_g128(w, nonfinite=cnt)
    moe.moe_pack_mxfp4(w, nonfinite=cnt)
    moe.moe_pack_nvfp4(w, nonfinite=cnt)
    assert int(cnt.item()) == 6


# ---------------------------------------------------------------- routing

@pytest.mark.parametrize("T,E,k", [(1, 256, 8), (1000, 256, 8), (77, 8, 2), (64, 1024, 32), (5, 32, 32)])
def test_route_bit_exact_on_identical_logits(T, E, k):
    g = torch.Generator().manual_seed(T * 31 + E)
    logits = torch.randn(T, E, generator=g)
    logits[: T // 2] = torch.round(logits[: T // 2] * 2) / 2     # exact ties
    bias = moe_synth.zipf_bias(moe_synth.LayerShape(64, 64, E, k), seed=3) if E >= k else None
    for b in (None, bias):
        ids, w = moe.moe_route(logits.to(DEV), k, bias=None if b is None else b.to(DEV))
        torch.cuda.synchronize()
        rid, rw = o.route(logits.numpy(), None if b is None else b.numpy(), k)
        assert np.array_equal(ids.cpu().numpy(), rid)
        wg = w.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(wg - rw) <= 1e-6 * (1 + np.abs(rw)))
        assert np.all(np.abs(wg.sum(1) - 1) <= 8 * 2.0 ** -23 * k)


@pytest.mark.parametrize("T,E,k", [(1, 256, 8), (4, 256, 8), (32, 256, 8), (100, 8, 2), (8192, 256, 8),
                                   (3000, 1024, 32), (129, 3, 1)])
def test_permute_bit_exact(T, E, k):
    g = torch.Generator().manual_seed(T + E)
    ids = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32)
    if T >= 100:  # skew: most tokens on a few experts
        hot = torch.randperm(E, generator=g)[:k]
        ids[: T // 2] = hot.to(torch.int32)
    offsets, sorted_rows, pos = moe.moe_permute(ids.to(DEV), E)
    torch.cuda.synchronize()
    ro, rs, rp = o.permute(ids.numpy(), E)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(sorted_rows.cpu().numpy(), rs)
    assert np.array_equal(pos.cpu().numpy(), rp)


# ---------------------------------------------------------------- layer forward

def run_forward(layer, fmt, path=None, routed=None, packed=None, flags=0):
    """moe_forward (or moe_forward_routed) of a layer with every debug output;
    `packed` = (gate_up, down) banks already packed on the GPU, else they are
    packed here."""
    s = layer.shape
    shape = moe.make_shape(s.hidden, s.inter, s.num_experts, s.top_k, fmt)
    T = layer.x.shape[0]
    gu, dn = packed if packed is not None else (pack_gpu(fmt, layer.gate_up), pack_gpu(fmt, layer.down))
    ws = moe.alloc_workspace(shape, T, flags=flags)
    dbg = {
        "logits_out": torch.empty(T, s.num_experts, dtype=torch.float32, device=DEV),
        "topk_ids_out": torch.empty(T, s.top_k, dtype=torch.int32, device=DEV),
        "topk_w_out": torch.empty(T, s.top_k, dtype=torch.float32, device=DEV),
        "act_out": torch.empty(T * s.top_k, s.inter, dtype=torch.bfloat16, device=DEV),
        "offsets_out": torch.empty(s.num_experts + 1, dtype=torch.int32, device=DEV),
        "sorted_rows_out": torch.empty(T * s.top_k, dtype=torch.int32, device=DEV),
    }
    if routed is None:
        out = moe.moe_forward(shape, layer.x, layer.router_w, gu, dn, ws, bias=layer.bias, path=path, debug=dbg,
                              flags=flags)
    else:
        ids, w = routed
        for key in ("logits_out", "topk_ids_out", "topk_w_out"):
            dbg.pop(key)
        out = moe.moe_forward_routed(shape, layer.x, ids, w, gu, dn, ws, path=path, debug=dbg, flags=flags)
    assert moe.moe_workspace_status(ws) == moe.MOE_OK
    return out, dbg


def gpu_activations_in_oracle_order(dbg, tok, rid, E, k):
    """GPU expert-sorted activations of the sampled tokens, reordered to the
    oracle's expert-sorted order of that sample."""
    sorted_rows = dbg["sorted_rows_out"].cpu().numpy()
    pos = np.empty_like(sorted_rows)
    pos[sorted_rows] = np.arange(sorted_rows.size, dtype=sorted_rows.dtype)
    _, o_sorted, _ = o.permute(rid, E)                     # sample rows r' = i*k + j
    gpu_rows = tok[o_sorted // k] * k + (o_sorted % k)     # the same rows in the full batch
    act = o.bf16_to_f64(moe_synth.bf16_bits(dbg["act_out"]))
    return act[pos[gpu_rows]]


def check_layer(layer, fmt, path=None, sample=None, name="", packed=None):
    """Full forward on the GPU; the oracle recomputes the (sampled) tokens.

    Routing is checked bit-exact on the GPU's own fp32 logits, which must agree
    with the oracle's to fp32 accumulation error.  The layer output is held to
    |gpu - ref| <= 1e-2 |ref| + 1e-3 rms(ref) against the oracle's own layer
    (its own bf16 activation rounding, no GPU value): exactly for tokens whose
    bf16 SwiGLU activations all equal the oracle's, and up to the flip
    allowance (parity_util.flip_allowance) for tokens where fp32 accumulation
    put an activation across a bf16 rounding boundary.  Each such activation is
    itself checked to be a correct rounding (flip_aware_activations), and the
    output of those tokens is also checked stage-wise: against the oracle's down
    projection and combine of the activations the GPU chose."""
    out, dbg = run_forward(layer, fmt, path, packed=packed)
    return verify_layer(layer, fmt, out, dbg, path, sample, name)


def verify_layer(layer, fmt, out, dbg, path=None, sample=None, name=""):
    """The checks of check_layer on a forward's output and debug outputs."""
    s = layer.shape
    T = layer.x.shape[0]
    tok = np.arange(T) if sample is None else np.asarray(sample)
    tok_d = torch.as_tensor(tok, device=DEV)
    xb = moe_synth.bf16_bits(layer.x)[tok]
    bias = None if layer.bias is None else layer.bias.cpu().numpy()
    ref_logits = o.router_logits(xb, moe_synth.bf16_bits(layer.router_w))
    gpu_logits = dbg["logits_out"][tok_d]
    gpu_ids = dbg["topk_ids_out"][tok_d]
    n_near_ties = assert_routing_consistent(gpu_logits, ref_logits, gpu_ids, bias, s.top_k)
    rid, rw = o.route(gpu_logits.cpu().numpy(), bias, s.top_k)
    assert np.array_equal(rid, gpu_ids.cpu().numpy())
    gw = dbg["topk_w_out"][tok_d].cpu().numpy().astype(np.float64)
    assert np.all(np.abs(gw - rw) <= 1e-6 * (1 + np.abs(rw)))
    if sample is None:
        ro, rs, _ = o.permute(rid, s.num_experts)
        assert np.array_equal(dbg["offsets_out"].cpu().numpy(), ro)
        assert np.array_equal(dbg["sorted_rows_out"].cpu().numpy(), rs)
    gu = LazyOracleBank(fmt, layer.gate_up)
    dn = LazyOracleBank(fmt, layer.down)
    gu.prefetch(rid)
    dn.prefetch(rid)
    a_exact, a_round = o.expert_activations(xb, rid, gu, s.num_experts)
    gpu_act = gpu_activations_in_oracle_order(dbg, tok, rid, s.num_experts, s.top_k)
    act_used, n_diff = flip_aware_activations(gpu_act, a_exact, a_round)
    out_sel = out[tok_d]
    # the layer against the pure oracle
    pure = o.down_and_combine(a_round, rid, rw, dn, s.num_experts)
    allow, flipped = flip_allowance(gpu_act, a_exact, a_round, rid, rw, dn, s.num_experts)
    what = f"{fmt} T={T} path={int(path or 0)} ({n_diff} activations rounded the other way)"
    summary = assert_layer_parity(out_sel, pure, allow, flipped, what)
    # stage-wise: the down projection and combine of the GPU's own activations
    ref_stage = o.down_and_combine(act_used, rid, rw, dn, s.num_experts)
    assert_out_close(out_sel, ref_stage, what + " stage-wise")
    _, worst_stage = out_tolerance_report(out_sel, ref_stage)
    record_parity(dict(case=name or f"{fmt}_T{T}", fmt=fmt, T=T, path=int(path or 0),
                       shape=[s.hidden, s.inter, s.num_experts, s.top_k], sampled_tokens=int(tok.size),
                       routing_near_ties=n_near_ties, activations=int(gpu_act.size),
                       activations_rounded_other_way=n_diff, stagewise_worst_ratio=worst_stage, **summary))
    return out


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("path", [moe.MOE_PATH_DECODE, moe.MOE_PATH_PREFILL])
def test_forward_tiny_layer(fmt, path):
    layer = moe_synth.make_layer(moe_synth.TINY, T=16, seed=moe_synth.SEED_TINY, device=DEV)
    check_layer(layer, fmt, path)


@pytest.mark.parametrize("T", [1, 3, 29, 32, 33, 130, 300])
def test_forward_tiny_shape_ragged_token_counts(T):
    layer = moe_synth.make_layer(moe_synth.TINY, T=T, seed=40 + T, zipf=True, device=DEV)
    check_layer(layer, "int4_g128", moe.MOE_PATH_PREFILL)
    if T <= 32:
        check_layer(layer, "mxfp4", moe.MOE_PATH_DECODE)
    else:
        # the decode kernels take at most 32 tokens
        with pytest.raises(moe.MoeError):
            run_forward(layer, "mxfp4", moe.MOE_PATH_DECODE)


def test_forward_odd_shapes_and_partial_tiles():
    """I = 192 and H = 320: weight-row tiles of 128 end part-way, one INT4 group
    of 64 closes every row of the down bank and of gate_up."""
    shape = moe_synth.LayerShape(hidden=320, inter=192, num_experts=6, top_k=3)
    layer = moe_synth.make_layer(shape, T=45, seed=77, device=DEV)
    small = moe_synth.make_layer(shape, T=30, seed=76, device=DEV)
    for fmt in FMTS:
        check_layer(layer, fmt, moe.MOE_PATH_PREFILL)
        check_layer(small, fmt, moe.MOE_PATH_DECODE)


def test_forward_odd_shapes_small_batch():
    """H = 320, I = 192 at 5 tokens: a k-block of the gate_up rows ends
    part-way and four rows of scales are not a whole number of 16-byte units."""
    shape = moe_synth.LayerShape(hidden=320, inter=192, num_experts=6, top_k=3)
    layer = moe_synth.make_layer(shape, T=5, seed=78, device=DEV)
    for fmt in FMTS:
        check_layer(layer, fmt, moe.MOE_PATH_DECODE)


@pytest.mark.parametrize("T", [1, 4])
def test_forward_nex_decode_int4(T):
    layer = moe_synth.make_layer(moe_synth.NEX, T=T, seed=100 + T, device=DEV)
    check_layer(layer, "int4_g128")


def test_forward_nex_concurrency32_zipf_int4():
    layer = moe_synth.make_layer(moe_synth.NEX, T=32, seed=132, zipf=True, device=DEV)
    check_layer(layer, "int4_g128")


@pytest.mark.parametrize("zipf", [False, True])
def test_forward_nex_prefill_8192_int4(zipf):
    layer = moe_synth.make_layer(moe_synth.NEX, T=8192, seed=8192 + zipf, zipf=zipf, device=DEV)
    sample = np.random.default_rng(5).choice(8192, 24, replace=False)
    sample = np.concatenate([sample, [0, 8191]])
    check_layer(layer, "int4_g128", sample=sample)


@pytest.mark.parametrize("T", [4, 8192])
def test_forward_nex_mxfp4(T):
    layer = moe_synth.make_layer(moe_synth.NEX, T=T, seed=4000 + T, device=DEV)
    sample = None if T <= 32 else np.random.default_rng(6).choice(T, 24, replace=False)
    check_layer(layer, "mxfp4", sample=sample)


@pytest.mark.parametrize("T", [4, 8192])
def test_forward_nex_nvfp4(T):
    layer = moe_synth.make_layer(moe_synth.NEX, T=T, seed=5000 + T, device=DEV)
    sample = None if T <= 32 else np.random.default_rng(7).choice(T, 24, replace=False)
    check_layer(layer, "nvfp4", sample=sample)


def test_decode_and_grouped_paths_on_one_nex_layer():
    layer = moe_synth.make_layer(moe_synth.NEX, T=24, seed=7, device=DEV)
    check_layer(layer, "int4_g128", moe.MOE_PATH_DECODE)
    check_layer(layer, "int4_g128", moe.MOE_PATH_PREFILL)


def test_forward_routed_matches_forward():
    layer = moe_synth.make_layer(moe_synth.NEX, T=40, seed=9, device=DEV)
    out, dbg = run_forward(layer, "int4_g128")
    out2, _ = run_forward(layer, "int4_g128", routed=(dbg["topk_ids_out"], dbg["topk_w_out"]))
    # the grouped path sums expert outputs with fp32 atomics: equal up to order
    assert_out_close(out2, out.float().cpu().numpy().astype(np.float64), "routed vs forward")
    small = moe_synth.make_layer(moe_synth.NEX, T=24, seed=10, device=DEV)
    d1, dbg1 = run_forward(small, "int4_g128", moe.MOE_PATH_DECODE)
    d2, _ = run_forward(small, "int4_g128", moe.MOE_PATH_DECODE,
                        routed=(dbg1["topk_ids_out"], dbg1["topk_w_out"]))
    assert torch.equal(d1, d2)  # the decode path is deterministic
    d3, _ = run_forward(small, "int4_g128", moe.MOE_PATH_DECODE)
    assert torch.equal(d1, d3)


@pytest.mark.parametrize("fmt,T,zipf", [("int4_g128", 300, True), ("nvfp4", 2048, False)])
def test_deterministic_grouped_combine(fmt, T, zipf):
    """MOE_FLAG_DETERMINISTIC: the grouped path's output is bit-identical from run
    to run (each token's slot rows summed in slot order) and meets the oracle."""
    layer = moe_synth.make_layer(moe_synth.NEX, T=T, seed=6000 + T, zipf=zipf, device=DEV)
    packed = (pack_gpu(fmt, layer.gate_up), pack_gpu(fmt, layer.down))
    det = moe.MOE_FLAG_DETERMINISTIC
    s = layer.shape
    shape = moe.make_shape(s.hidden, s.inter, s.num_experts, s.top_k, fmt)
    assert moe.moe_workspace_bytes_flags(shape, T, det) == moe.moe_workspace_bytes(shape, T) + T * 8 * 2048 * 4
    out1, dbg = run_forward(layer, fmt, packed=packed, flags=det)
    for _ in range(3):
        out2, _ = run_forward(layer, fmt, packed=packed, flags=det)
        assert torch.equal(out1, out2)
    sample = np.random.default_rng(T).choice(T, 16, replace=False)
    verify_layer(layer, fmt, out1, dbg, sample=sample, name=f"deterministic_{fmt}_T{T}")
    # the default (arrival-order) combine agrees within the tolerance
    out3, _ = run_forward(layer, fmt, packed=packed)
    assert_out_close(out3, out1.float().cpu().numpy().astype(np.float64), "default vs deterministic combine")


def test_deterministic_flag_needs_its_workspace():
    layer = moe_synth.make_layer(moe_synth.TINY, T=40, seed=12, device=DEV)
    s = layer.shape
    shape = moe.make_shape(s.hidden, s.inter, s.num_experts, s.top_k, "int4_g128")
    gu, dn = pack_gpu("int4_g128", layer.gate_up), pack_gpu("int4_g128", layer.down)
    small = moe.alloc_workspace(shape, 40)
    with pytest.raises(moe.MoeError):
        moe.moe_forward(shape, layer.x, layer.router_w, gu, dn, small, flags=moe.MOE_FLAG_DETERMINISTIC)
    with pytest.raises(moe.MoeError):
        moe.moe_forward(shape, layer.x, layer.router_w, gu, dn, small, flags=2)   # unknown flag


def scaled_layer(shape, T, seed, gate_up_scale=1.0, down_scale=1.0, x_scale=1.0):
    """A layer whose banks and tokens are multiplied by powers of two, rounded
    to bf16 again (exact unless the scaled value leaves bf16's normal range);
    the router weight takes the inverse of the tokens' factor, so the logits
    keep their size."""
    layer = moe_synth.make_layer(shape, T=T, seed=seed, device=DEV)
    scale = lambda t, f: (t.float() * f).to(torch.bfloat16) if f != 1.0 else t
    return moe_synth.Layer(shape=shape, x=scale(layer.x, x_scale), router_w=scale(layer.router_w, 1.0 / x_scale),
                           gate_up=scale(layer.gate_up, gate_up_scale), down=scale(layer.down, down_scale),
                           bias=None)


@pytest.mark.parametrize("path", [moe.MOE_PATH_DECODE, moe.MOE_PATH_PREFILL])
def test_forward_int4_scales_outside_the_single_fma_range(path):
    """INT4 scales at or above 2^-5 (weights x 16) and subnormal scales (gate_up
    weights x 2^-122, tokens x 2^100 to keep the activations representable)
    take the kernels' two-step dequantisation; zero groups too."""
    s = moe_synth.TINY
    big = scaled_layer(s, 32, 301, gate_up_scale=16.0, down_scale=16.0)
    big.gate_up[1, :4, :128] = 0  # whole zero groups: scale 0
    check_layer(big, "int4_g128", path, name="int4_scales_ge_2^-5")
    tiny = scaled_layer(s, 32, 302, gate_up_scale=2.0 ** -122, x_scale=2.0 ** 100)
    gu = LazyOracleBank("int4_g128", tiny.gate_up)
    scales = np.concatenate([gu.packed(e)[1].ravel() for e in range(s.num_experts)])
    assert np.mean((scales > 0) & (scales < 0x0080)) > 0.5   # most scales are subnormal bf16
    check_layer(tiny, "int4_g128", path, name="int4_subnormal_scales")


def test_zero_tokens_is_a_no_op():
    s = moe.make_shape(256, 64, 8, 2, "int4_g128")
    ws = moe.alloc_workspace(s, 0)
    x = torch.empty(0, 256, dtype=torch.bfloat16, device=DEV)
    r = torch.zeros(8, 256, dtype=torch.bfloat16, device=DEV)
    gu = torch.zeros(moe.moe_packed_bytes(s, 0), dtype=torch.uint8, device=DEV)
    dn = torch.zeros(moe.moe_packed_bytes(s, 1), dtype=torch.uint8, device=DEV)
    out = moe.moe_forward(s, x, r, gu, dn, ws)
    assert out.shape == (0, 256)


# ---------------------------------------------------------------- failure reporting

def test_bounded_wait_reports_timeout_and_context_survives():
    s = moe.make_shape(256, 64, 8, 2, "int4_g128")
    ws = moe.alloc_workspace(s, 16)
    moe.moe_selftest_bounded_wait(ws, 20_000_000)  # 20 ms
    assert moe.moe_workspace_status(ws) == moe.MOE_ERR_TIMEOUT
    assert moe.moe_workspace_status(ws) == moe.MOE_OK  # reading clears it
    layer = moe_synth.make_layer(moe_synth.TINY, T=16, seed=0, device=DEV)
    check_layer(layer, "int4_g128")
