"""CPU oracle for the weight-only 4-bit routed-expert MoE layer (W4A16).

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the CPU
baseline leg of bench.py may import this module.  The product path (the CUDA
library and its Python binding) never calls it and shares no code with it.

Plain, slow and meant to be checked by eye: NumPy, fp64 arithmetic unless a
step's definition fixes another precision, no blocking or fusion.

Sources, cited by page title and section:
  [INT4]   "Tech2wild/Nex-N2.5-mini-Int4-Int8Mix", Recipe: routed experts are
           INT4, symmetric, group 128, round-to-nearest per group with min-max
           scales, no calibration; the fused banks experts.gate_up_proj
           [256, 1024, 2048] and experts.down_proj [256, 2048, 512].
  [MXFP4]  "kirillbilchenko/Nex-N2.5-mini-MXFP4-MxWave", Model summary / What
           was quantized / Quantization method: MXFP4 W4A16 experts (E2M1
           codes, one shared power-of-two scale per 32 elements, one packed and
           one scale tensor per matrix), scale exponents of the
           floor(log2(x / 6)) family.
  [ROUTE]  "cbert33/Nex-N2.5-mini-FP8-Calibrated", Artifact summary: 256
           routed experts, 8 active per token; routers kept in bf16
           ("Tech2wild/...", Recipe table).
  [LAYOUT] "primitive-ai/Nex-N2.5-mini-mixed-NVFP4-FP8", What's quantized to
           what: experts shipped as two batched 3-D tensors per layer; gate and
           up are the two halves of the fused gate_up bank.
  [NVFP4]  the same section: NVFP4 experts, group 16, one global scale per
           expert shared by gate and up, round-to-nearest.
  [SHARED] the dense shared expert and its sigmoid gate (Int4-Int8Mix Recipe
           table; MxWave What was quantized: kept in bf16).

Readings where the pages are silent (each also listed in the design notes):
  * INT4 scale s = bf16(fp32(amax) / 7): the group max maps to code +-7, code
    -8 is never produced; q = clamp(round_half_even(fp32(w / s)), -8, 7);
    stored as offset-binary nibbles q + 8, element 2j in the low nibble of
    byte j.  Scales are bf16 in their own plane.  An all-zero group has s = 0
    and codes 0.  The last group of a row holds K mod 128 elements.
  * MXFP4 exponent e = floor(log2(amax / 6)), i.e. the largest integer with
    6 * 2^e <= amax, clamped to [-127, 127]; e = -127 for an all-zero block.
    Scale byte e + 127 (E8M0).  Codes: nearest point of the E2M1 magnitude
    grid {0, .5, 1, 1.5, 2, 3, 4, 6} to w / 2^e, ties to the even code index,
    values past 6 saturate to 6; nibble = sign << 3 | code, zero is +0.
  * Router: fp32 logits (+ optional fp32 bias), top-k by value with ties to
    the lower expert index, ids in descending-logit order; weights are the
    softmax restricted to the selected k (= full softmax renormalised over
    the top-k), in fp64.
  * Expert MLP is SwiGLU: a = silu(gate) * up with gate = rows [0, I) of the
    fused bank and up = rows [I, 2I); y = W_down a.
  * Two bf16 roundings belong to the W4A16 method itself and are modelled:
    the dequantised weight (bf16(q * s) for INT4; exact for MXFP4) and the
    activation a that feeds the down projection.  Expert outputs y and the
    routing-weighted sum stay in fp64 here.
"""
from __future__ import annotations

import numpy as np

INT4_GROUP = 128
MX_BLOCK = 32
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)

FMT_INT4 = "int4_g128"
FMT_MXFP4 = "mxfp4"
FMT_NVFP4 = "nvfp4"
NV_BLOCK = 16
E4M3_MAX = 448.0
NV_GLOBAL_DIVISOR = 6.0 * E4M3_MAX   # largest E2M1 magnitude x largest E4M3 value


# --------------------------------------------------------------------------
# bf16 <-> float helpers (bit-level, no casts that could flush or double-round)
# --------------------------------------------------------------------------

def bf16_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact fp64 values."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def f64_to_bf16(x) -> np.ndarray:
    """Round fp64 values to bf16 with round-half-to-even; returns uint16 bits.

    bf16 keeps 8 significant bits and the fp32 exponent range: normal numbers
    down to 2^-126 and subnormals on the 2^-133 grid below that.  Rounding is
    done exactly in fp64 (scaling by powers of two is exact, np.rint is
    half-to-even), then the already-representable value is narrowed.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                       # x = m * 2^e, 0.5 <= |m| < 1
    normal = e >= -125                        # |x| >= 2^-126
    r_norm = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)
    r_sub = np.ldexp(np.rint(np.ldexp(x, 133)), -133)
    r = np.where(normal, r_norm, r_sub)
    r = np.where(np.abs(r) >= 2.0 ** 128, np.copysign(np.inf, x), r)
    return (r.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_round(x) -> np.ndarray:
    """fp64 -> nearest bf16 value, returned as fp64."""
    return bf16_to_f64(f64_to_bf16(x))


# --------------------------------------------------------------------------
# INT4 symmetric round-to-nearest, group 128, bf16 min-max scales   [INT4]
# --------------------------------------------------------------------------

def int4_groups(K: int):
    """Column ranges of the 128-element groups of a row of length K."""
    return [(g0, min(g0 + INT4_GROUP, K)) for g0 in range(0, K, INT4_GROUP)]


def pack_int4_g128(w_bits):
    """Quantise a bf16 bank [E, N, K] (or [N, K]) row by row, group by group.

    Returns (codes uint8 [..., N, K/2], scales uint16 bf16 bits [..., N, G]).
    """
    w_bits = np.asarray(w_bits, dtype=np.uint16)
    K = w_bits.shape[-1]
    assert K % 2 == 0
    w32 = bf16_to_f64(w_bits).astype(np.float32)        # exact
    groups = int4_groups(K)
    q = np.zeros(w32.shape, dtype=np.int32)
    scales = np.zeros(w32.shape[:-1] + (len(groups),), dtype=np.uint16)
    for gi, (a, b) in enumerate(groups):
        wg = w32[..., a:b]
        amax = np.max(np.abs(wg), axis=-1)               # fp32, exact
        s32 = amax / np.float32(7.0)                      # fp32 correctly rounded quotient
        s_bits = f64_to_bf16(s32.astype(np.float64))
        s = bf16_to_f64(s_bits).astype(np.float32)[..., None]
        safe = np.where(s == 0, np.float32(1.0), s)
        quot = wg / safe                                  # fp32 correctly rounded quotient
        qg = np.clip(np.rint(quot), -8, 7).astype(np.int32)
        q[..., a:b] = np.where(s == 0, 0, qg)
        scales[..., gi] = s_bits
    u = (q + 8).astype(np.uint8)                          # offset binary 0..15
    codes = (u[..., 0::2] | (u[..., 1::2] << np.uint8(4))).astype(np.uint8)
    return codes, scales


def unpack_nibbles(codes) -> np.ndarray:
    """uint8 [..., K/2] -> uint8 nibbles [..., K], element 2j = low nibble of byte j."""
    codes = np.asarray(codes, dtype=np.uint8)
    out = np.empty(codes.shape[:-1] + (codes.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = codes & np.uint8(0x0F)
    out[..., 1::2] = codes >> np.uint8(4)
    return out


def int4_codes(codes) -> np.ndarray:
    """Signed INT4 values q in [-8, 7] from packed offset-binary nibbles."""
    return unpack_nibbles(codes).astype(np.int32) - 8


def dequant_int4_g128(codes, scales) -> np.ndarray:
    """w_hat = bf16(q * s) per element (q * s is exact in fp64), as fp64."""
    q = int4_codes(codes).astype(np.float64)
    K = q.shape[-1]
    s = bf16_to_f64(scales)
    s_full = np.empty_like(q)
    for gi, (a, b) in enumerate(int4_groups(K)):
        s_full[..., a:b] = s[..., gi:gi + 1]
    return bf16_round(q * s_full)


# --------------------------------------------------------------------------
# MXFP4: E2M1 codes, E8M0 scale per 32 elements                      [MXFP4]
# --------------------------------------------------------------------------

def floor_log2_div6(x) -> np.ndarray:
    """Largest integer e with 6 * 2^e <= x, for x > 0 (no clamping)."""
    x = np.asarray(x, dtype=np.float64)
    e = np.floor(np.log2(x / 6.0)).astype(np.int64)
    # fix up the fp64 log2 estimate with exact power-of-two comparisons
    e = np.where(6.0 * np.ldexp(1.0, e + 1) <= x, e + 1, e)
    return np.where(6.0 * np.ldexp(1.0, e) > x, e - 1, e)


def mx_exponent(amax) -> np.ndarray:
    """Largest integer e with 6 * 2^e <= amax (= floor(log2(amax/6))), clamped
    to [-127, 127]; -127 for amax == 0."""
    amax = np.asarray(amax, dtype=np.float64)
    pos = amax > 0
    e = np.clip(floor_log2_div6(np.where(pos, amax, 6.0)), -127, 127)
    return np.where(pos, e, -127)


def e2m1_nearest(v) -> np.ndarray:
    """Magnitude code 0..7 of the E2M1 grid point nearest |v|; ties go to the
    even code index (the grid point whose mantissa bit is 0)."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    d = np.abs(a[..., None] - E2M1_GRID)                  # distance to each grid point
    best = np.min(d, axis=-1, keepdims=True)
    is_best = d == best
    # among equally near points prefer an even index; there is never more than one
    even_best = is_best & (np.arange(8) % 2 == 0)
    pick = np.where(even_best.any(axis=-1), np.argmax(even_best, axis=-1), np.argmax(is_best, axis=-1))
    return pick.astype(np.uint8)


# Exponent rules of the MXFP4 packer.  FLOOR is the one above; the others are
# the members of the same family that the MxWave card compares against or
# searches over ("kirillbilchenko/Nex-N2.5-mini-MXFP4-MxWave", Quantization
# method: the "smallest exponent that avoids clipping", and the MSE search).
MX_RULE_FLOOR = "floor"   # largest e with 6 * 2^e <= amax (block max may clip)
MX_RULE_CEIL = "ceil"     # smallest e with amax <= 6 * 2^e (nothing clips)
MX_RULE_OCP = "ocp"       # floor(log2(amax)) - 2: the OCP MX shared-exponent rule for E2M1
MX_RULE_MSE = "mse"       # MxWave: lowest-MSE exponent among the candidates below
MX_P995_FRACTION = 0.845  # 99.5th percentile of 32 values: index 0.995 * 31 = 30.845


def mx_exponent_ceil(amax) -> np.ndarray:
    """Smallest integer e with amax <= 6 * 2^e (= ceil(log2(amax/6))), clamped
    to [-127, 127]; -127 for amax == 0."""
    amax = np.asarray(amax, dtype=np.float64)
    pos = amax > 0
    safe = np.where(pos, amax, 6.0)
    e = np.ceil(np.log2(safe / 6.0)).astype(np.int64)
    e = np.where(6.0 * np.ldexp(1.0, e - 1) >= safe, e - 1, e)
    e = np.where(6.0 * np.ldexp(1.0, e) < safe, e + 1, e)
    e = np.clip(e, -127, 127)
    return np.where(pos, e, -127)


def mx_exponent_ocp(amax) -> np.ndarray:
    """floor(log2(amax)) - 2 (2 = the largest exponent of an E2M1 value), clamped
    to [-127, 127]; -127 for amax == 0."""
    amax = np.asarray(amax, dtype=np.float64)
    pos = amax > 0
    _, ex = np.frexp(np.where(pos, amax, 1.0))            # amax = m * 2^ex, 0.5 <= m < 1
    e = np.clip(ex.astype(np.int64) - 1 - 2, -127, 127)
    return np.where(pos, e, -127)


def mx_p995(mag_blocks) -> np.ndarray:
    """99.5th percentile of each block's 32 magnitudes, linear interpolation
    between order statistics: v30 + 0.845 * (v31 - v30) of the sorted values,
    in fp64 with the multiply rounded before the add."""
    v = np.sort(np.asarray(mag_blocks, dtype=np.float64), axis=-1)
    v30, v31 = v[..., 30], v[..., 31]
    return v30 + (v31 - v30) * MX_P995_FRACTION


def mx_block_sq_error(blocks, e) -> np.ndarray:
    """Squared reconstruction error of each block quantised with exponent e
    (array over blocks), summed over the 32 elements pairwise in halving order
    (element i with i + 16, then with i + 8, ...), in fp64."""
    v = blocks / np.ldexp(1.0, e)[..., None]
    mag = e2m1_nearest(v)
    w_hat = np.where(blocks < 0, -1.0, 1.0) * E2M1_GRID[mag] * np.ldexp(1.0, e)[..., None]
    sq = (blocks - w_hat) * (blocks - w_hat)                 # both exact in fp64
    n = sq.shape[-1]
    while n > 1:
        n //= 2
        sq = sq[..., :n] + sq[..., n:2 * n]
    return sq[..., 0]


def mx_exponent_mse(blocks) -> np.ndarray:
    """MxWave's scale search per block of 32: the candidates are
    floor(log2(p995 / 6)) - 4 ... + 1 and the smallest exponent that avoids
    clipping, each clamped to [-127, 127]; the one with the lowest squared
    error wins, ties to the smaller exponent.  An all-zero block gets -127."""
    blocks = np.asarray(blocks, dtype=np.float64)
    mags = np.abs(blocks)
    amax = np.max(mags, axis=-1)
    p = mx_p995(mags)
    e0 = floor_log2_div6(np.where(amax > 0, p, 6.0))      # largest e with 6 * 2^e <= p995
    cands = [np.clip(e0 + d, -127, 127) for d in range(-4, 2)] + [mx_exponent_ceil(amax)]
    best_e = cands[0]
    best_err = mx_block_sq_error(blocks, best_e)
    for c in cands[1:]:                                    # ascending exponents
        err = mx_block_sq_error(blocks, c)
        better = err < best_err
        best_e = np.where(better, c, best_e)
        best_err = np.where(better, err, best_err)
    return np.where(amax > 0, best_e, -127)


def pack_mxfp4(w_bits, rule: str = MX_RULE_FLOOR):
    """Quantise a bf16 bank [..., N, K] in blocks of 32 along K with the given
    exponent rule.

    Returns (codes uint8 [..., N, K/2], scales uint8 E8M0 [..., N, K/32]).
    """
    w_bits = np.asarray(w_bits, dtype=np.uint16)
    K = w_bits.shape[-1]
    assert K % MX_BLOCK == 0
    w = bf16_to_f64(w_bits)
    blocks = w.reshape(w.shape[:-1] + (K // MX_BLOCK, MX_BLOCK))
    amax = np.max(np.abs(blocks), axis=-1)
    if rule == MX_RULE_FLOOR:
        e = mx_exponent(amax)
    elif rule == MX_RULE_CEIL:
        e = mx_exponent_ceil(amax)
    elif rule == MX_RULE_OCP:
        e = mx_exponent_ocp(amax)
    elif rule == MX_RULE_MSE:
        e = mx_exponent_mse(blocks)
    else:
        raise ValueError(f"unknown MXFP4 exponent rule {rule!r}")
    v = blocks / np.ldexp(1.0, e)[..., None]              # exact power-of-two scaling
    mag = e2m1_nearest(v)
    sign = ((blocks < 0) & (mag > 0)).astype(np.uint8)
    nib = ((sign << np.uint8(3)) | mag).reshape(w.shape).astype(np.uint8)
    codes = (nib[..., 0::2] | (nib[..., 1::2] << np.uint8(4))).astype(np.uint8)
    scales = (e + 127).astype(np.uint8)
    return codes, scales


def e2m1_value(nibbles) -> np.ndarray:
    nib = np.asarray(nibbles, dtype=np.uint8)
    mag = E2M1_GRID[nib & np.uint8(7)]
    return np.where(nib & np.uint8(8), -mag, mag)


def dequant_mxfp4(codes, scales) -> np.ndarray:
    """w_hat = e2m1(c) * 2^(scale - 127), exact (asserted representable in bf16)."""
    vals = e2m1_value(unpack_nibbles(codes))
    K = vals.shape[-1]
    e = np.asarray(scales, dtype=np.int64) - 127
    full = vals * np.repeat(np.ldexp(1.0, e), MX_BLOCK, axis=-1)[..., :K]
    assert np.array_equal(bf16_round(full), full), "MXFP4 dequant not exact in bf16"
    return full


# --------------------------------------------------------------------------
# NVFP4 as W4A16: E2M1 codes, E4M3 scale per 16 elements, one fp32 global
# scale per expert matrix                                              [NVFP4]
# ("primitive-ai/Nex-N2.5-mini-mixed-NVFP4-FP8", What's quantized to what:
# NVFP4 experts with group 16; gate and up share one weight_global_scale per
# expert; weights-only round-to-nearest, no calibration)
# --------------------------------------------------------------------------

def e4m3_value(code) -> np.ndarray:
    """Value of an E4M3 (fn) byte without its sign bit: 4 exponent bits (bias 7),
    3 mantissa bits, subnormals m * 2^-9."""
    c = np.asarray(code, dtype=np.int64) & 0x7F
    e, m = c >> 3, c & 7
    return np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.ldexp(1.0, e - 7))


_E4M3_CODES = np.arange(0x7F)                      # 0x7F is NaN in E4M3fn: never produced
_E4M3_VALUES = e4m3_value(_E4M3_CODES)             # increasing


def e4m3_nearest(t) -> np.ndarray:
    """Code of the E4M3 value nearest t >= 0, ties to the even code (mantissa
    bit 0), saturating at 448."""
    t = np.asarray(t, dtype=np.float64)
    d = np.abs(t[..., None] - _E4M3_VALUES)
    best = d == d.min(axis=-1, keepdims=True)
    even_best = best & (_E4M3_CODES % 2 == 0)
    pick = np.where(even_best.any(axis=-1), np.argmax(even_best, axis=-1), np.argmax(best, axis=-1))
    return pick.astype(np.uint8)


def nv_global_scale(w_bits) -> np.ndarray:
    """Per matrix (leading dims kept): g = fp32(amax / 2688), so that the block
    with the matrix's largest magnitude gets the E4M3 scale 448."""
    w = bf16_to_f64(w_bits).astype(np.float32)
    amax = np.max(np.abs(w.reshape(w.shape[:-2] + (-1,))), axis=-1)
    return (amax / np.float32(NV_GLOBAL_DIVISOR)).astype(np.float32)


def nv_multiplier(scale_codes, g) -> np.ndarray:
    """Per block: bf16(fp32(e4m3(code) * g)), the bf16 multiplier of the block's
    E2M1 codes, as fp64."""
    v = e4m3_value(scale_codes).astype(np.float32)
    prod = (v * np.asarray(g, dtype=np.float32)[..., None, None]).astype(np.float32)
    return bf16_round(prod.astype(np.float64))


def pack_nvfp4(w_bits):
    """Quantise a bf16 bank [E, N, K] (or one matrix [N, K]) to NVFP4:
    g = fp32(amax / 2688) per matrix; per block of 16 along K the scale code
    e4m3_nearest(fp32(amax_b / fp32(6 g))); the block multiplier
    d = bf16(fp32(e4m3(code) g)); codes = nearest E2M1 magnitude of
    fp32(w / d) (ties to the even code, saturating at 6), sign bit set only
    for nonzero codes; all zero when d == 0.

    Returns (codes uint8 [..., N, K/2], (scales uint8 [..., N, K/16], g fp32 [...])).
    """
    w_bits = np.asarray(w_bits, dtype=np.uint16)
    K = w_bits.shape[-1]
    assert K % NV_BLOCK == 0
    w32 = bf16_to_f64(w_bits).astype(np.float32)
    g = nv_global_scale(w_bits)
    blocks = w32.reshape(w32.shape[:-1] + (K // NV_BLOCK, NV_BLOCK))
    amax_b = np.max(np.abs(blocks), axis=-1)
    six_g = (np.float32(6.0) * g).astype(np.float32)[..., None, None]
    safe = np.where(six_g == 0, np.float32(1.0), six_g)
    t = np.where(six_g == 0, np.float32(0.0), (amax_b / safe).astype(np.float32))
    scales = e4m3_nearest(t.astype(np.float64))
    d = nv_multiplier(scales, g)                                   # fp64, bf16 values
    d32 = d.astype(np.float32)[..., None]
    quot = np.where(d32 == 0, np.float32(0.0), blocks / np.where(d32 == 0, np.float32(1.0), d32))
    mag = np.where(d32 == 0, 0, e2m1_nearest(quot.astype(np.float32).astype(np.float64))).astype(np.uint8)
    sign = ((blocks < 0) & (mag > 0)).astype(np.uint8)
    nib = ((sign << np.uint8(3)) | mag).reshape(w32.shape).astype(np.uint8)
    codes = (nib[..., 0::2] | (nib[..., 1::2] << np.uint8(4))).astype(np.uint8)
    return codes, (scales, g)


def dequant_nvfp4(codes, scales_g) -> np.ndarray:
    """w_hat = bf16(e2m1(c) * d), d the block's bf16 multiplier (one rounding of
    an exact product), as fp64."""
    scales, g = scales_g
    vals = e2m1_value(unpack_nibbles(codes))
    d = nv_multiplier(scales, g)
    return bf16_round(vals * np.repeat(d, NV_BLOCK, axis=-1))


def pack(fmt: str, w_bits):
    if fmt == FMT_INT4:
        return pack_int4_g128(w_bits)
    return pack_mxfp4(w_bits) if fmt == FMT_MXFP4 else pack_nvfp4(w_bits)


def dequant(fmt: str, codes, scales):
    if fmt == FMT_INT4:
        return dequant_int4_g128(codes, scales)
    return dequant_mxfp4(codes, scales) if fmt == FMT_MXFP4 else dequant_nvfp4(codes, scales)


def packed_bytes_per_expert(fmt: str, hidden: int, inter: int) -> int:
    """Bytes of codes + scales for one expert's gate_up [2I, H] and down [H, I]."""
    def mat(N, K):
        if fmt == FMT_INT4:
            return N * K // 2 + N * len(int4_groups(K)) * 2
        if fmt == FMT_NVFP4:
            return N * K // 2 + N * (K // NV_BLOCK) + 4
        return N * K // 2 + N * (K // MX_BLOCK)
    return mat(2 * inter, hidden) + mat(hidden, inter)


# --------------------------------------------------------------------------
# Router: logits -> top-k -> softmax over the selected k             [ROUTE]
# --------------------------------------------------------------------------

def router_logits(x_bits, router_bits) -> np.ndarray:
    """fp32 logits = fp32(x . Wr^T) with the dot products taken in fp64."""
    return (bf16_to_f64(x_bits) @ bf16_to_f64(router_bits).T).astype(np.float32)


def route(logits32, bias32, k: int):
    """Top-k of the fp32 logits (+ fp32 bias), ties to the lower expert index.

    Returns (ids int32 [T, k] in descending-logit order, weights fp64 [T, k]).
    """
    L = np.asarray(logits32, dtype=np.float32)
    if bias32 is not None:
        L = (L + np.asarray(bias32, dtype=np.float32)[None, :]).astype(np.float32)
    # a stable sort of -L keeps the lower index first among equal logits
    ids = np.argsort(-L, axis=1, kind="stable")[:, :k].astype(np.int32)
    sel = np.take_along_axis(L, ids, axis=1).astype(np.float64)
    ex = np.exp(sel - sel[:, :1])                         # sel[:, 0] is the row max
    return ids, ex / ex.sum(axis=1, keepdims=True)


def permute(ids, num_experts: int):
    """Stable counting sort of the flat (token, slot) index r = t*k + j by expert.

    Returns (offsets int32 [E+1], sorted_rows int32 [T*k], pos int32 [T*k]) with
    sorted_rows[offsets[e]:offsets[e+1]] the rows routed to expert e in
    ascending r, and pos the inverse permutation.
    """
    flat = np.asarray(ids, dtype=np.int64).reshape(-1)
    counts = np.bincount(flat, minlength=num_experts)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    sorted_rows = np.argsort(flat, kind="stable").astype(np.int32)
    pos = np.empty_like(sorted_rows)
    pos[sorted_rows] = np.arange(flat.size, dtype=np.int32)
    return offsets, sorted_rows, pos


# --------------------------------------------------------------------------
# Expert MLP and combine                                         [INT4][LAYOUT]
# --------------------------------------------------------------------------

def silu(z):
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


class PackedBank:
    """Codes + scales of one fused bank, dequantised lazily per expert."""

    def __init__(self, fmt: str, codes, scales):
        self.fmt, self.codes, self.scales = fmt, codes, scales
        self._cache = {}

    @classmethod
    def from_bf16(cls, fmt: str, w_bits):
        return cls(fmt, *pack(fmt, w_bits))

    def expert(self, e: int) -> np.ndarray:
        if e not in self._cache:
            if isinstance(self.scales, dict) or self.fmt != FMT_NVFP4:
                sc = self.scales[e]                             # per-expert entries
            else:
                sc = (self.scales[0][e], self.scales[1][e])     # (block scales, global scales)
            self._cache[e] = dequant(self.fmt, self.codes[e], sc)
        return self._cache[e]


def swiglu_exact(x_rows, w_gate_up):
    """silu(h_gate) * h_up in fp64, before the activation's bf16 rounding."""
    inter = w_gate_up.shape[0] // 2
    h = x_rows @ w_gate_up.T
    return silu(h[:, :inter]) * h[:, inter:]


def expert_mlp(x_rows, w_gate_up, w_down):
    """SwiGLU expert on fp64 rows: a = bf16(silu(h_gate) * h_up), y = W_down a."""
    a = bf16_round(swiglu_exact(x_rows, w_gate_up))
    return a, a @ w_down.T


def expert_activations(x_bits, ids, gate_up: PackedBank, num_experts: int):
    """Expert-sorted activations of every (token, slot) row.

    Returns (a_exact fp64 [T*k, I] before rounding, a = bf16(a_exact)) with
    row q holding sorted_rows[q] of permute(ids).
    """
    x = bf16_to_f64(x_bits)
    T, k = ids.shape
    offsets, sorted_rows, _ = permute(ids, num_experts)
    a_exact = None
    for e in range(num_experts):
        rows = sorted_rows[offsets[e]:offsets[e + 1]]
        if rows.size == 0:
            continue
        ae = swiglu_exact(x[rows // k], gate_up.expert(e))
        if a_exact is None:
            a_exact = np.zeros((T * k, ae.shape[1]), dtype=np.float64)
        a_exact[offsets[e]:offsets[e + 1]] = ae
    return a_exact, bf16_round(a_exact)


def down_and_combine(a_sorted, ids, weights, down: PackedBank, num_experts: int):
    """out_t = sum_j w_tj * W_down[ids_tj] a_(t,j), from expert-sorted activations."""
    T, k = ids.shape
    offsets, sorted_rows, _ = permute(ids, num_experts)
    wflat = np.asarray(weights, dtype=np.float64).reshape(-1)
    out = None
    for e in range(num_experts):
        rows = sorted_rows[offsets[e]:offsets[e + 1]]
        if rows.size == 0:
            continue
        y = a_sorted[offsets[e]:offsets[e + 1]] @ down.expert(e).T
        if out is None:
            out = np.zeros((T, y.shape[1]), dtype=np.float64)
        out[rows // k] += wflat[rows][:, None] * y      # each token at most once per expert
    return out


def forward_routed(x_bits, ids, weights, gate_up: PackedBank, down: PackedBank, num_experts: int):
    """Layer output for given routing: out_t = sum_j w_tj * y(expert ids_tj, x_t).

    Returns (out fp64 [T, H], a fp64 [T*k, I] in expert-sorted row order).
    """
    _, a_sorted = expert_activations(x_bits, ids, gate_up, num_experts)
    return down_and_combine(a_sorted, ids, weights, down, num_experts), a_sorted


def forward(x_bits, router_bits, bias32, gate_up: PackedBank, down: PackedBank, top_k: int):
    """The whole layer: router logits -> route -> experts -> weighted combine."""
    E = np.asarray(router_bits).shape[0]
    logits = router_logits(x_bits, router_bits)
    ids, w = route(logits, bias32, top_k)
    out, a_sorted = forward_routed(x_bits, ids, w, gate_up, down, E)
    return {"logits": logits, "ids": ids, "weights": w, "out": out, "a_sorted": a_sorted}


# --------------------------------------------------------------------------
# Shared expert beside the routed ones                              [SHARED]
# ("Tech2wild/Nex-N2.5-mini-Int4-Int8Mix", Recipe table: shared expert
# gate/up/down_proj and a separate shared_expert_gate; "kirillbilchenko/Nex-
# N2.5-mini-MXFP4-MxWave", What was quantized: shared experts stay bf16;
# "primitive-ai/Nex-N2.5-mini-mixed-NVFP4-FP8": shared experts, routers and
# norms hold 0.15 B parameters, i.e. an intermediate size of 512)
# --------------------------------------------------------------------------

def shared_expert(x_bits, gate_up_bits, down_bits, gate_bits):
    """Dense SwiGLU expert on every token, scaled by its gate:
    g_t = sigmoid(x_t . w_gate), a = bf16(silu(h_gate) * h_up) (the same bf16
    activation rounding as the routed experts), y = W_down a; in fp64 on the
    bf16 weights.  Returns (g [T], y [T, H])."""
    x = bf16_to_f64(x_bits)
    a = bf16_round(swiglu_exact(x, bf16_to_f64(gate_up_bits)))
    y = a @ bf16_to_f64(down_bits).T
    z = x @ bf16_to_f64(gate_bits)
    return 1.0 / (1.0 + np.exp(-z)), y


def forward_with_shared(x_bits, router_bits, bias32, gate_up: PackedBank, down: PackedBank, top_k: int,
                        shared_bits):
    """The layer with its shared expert: out_t = sum_j w_tj y_tj + g_t y_shared,t."""
    r = forward(x_bits, router_bits, bias32, gate_up, down, top_k)
    g, ys = shared_expert(x_bits, *shared_bits)
    r["shared_gate"], r["shared_y"] = g, ys
    r["out"] = r["out"] + g[:, None] * ys
    return r


def routing_margin(logits32, bias32, k: int) -> np.ndarray:
    """Per token, the gap between the k-th and (k+1)-th largest (biased) logit."""
    L = np.asarray(logits32, dtype=np.float64)
    if bias32 is not None:
        L = L + np.asarray(bias32, dtype=np.float64)[None, :]
    s = -np.sort(-L, axis=1)
    if s.shape[1] <= k:
        return np.full(s.shape[0], np.inf)
    return s[:, k - 1] - s[:, k]
