"""CPU oracle of the MXFP8 (block-scaled 8-bit float) variant of the expert
FFN (test infrastructure only; the product path never imports it).

Source: "Dropless MoE Is a Runtime Problem as Much as a Model Design" -- its
MXFP8 paragraph: block-scaled low precision raises arithmetic throughput and
cuts data movement, and the scaling must be checked for overflow, underflow
and accumulation precision. The pages name MXFP8 without defining it; the
definition used here is the public OCP Microscaling (MX) format, read as:

  * a block is 32 consecutive elements along the reduction (K) axis of one
    row; every block shares one scale X = 2^E, stored as an E8M0 byte
    (E + 127), with E = floor(log2(max |v|)) - 8 clamped to [-127, 127]
    (8 is the exponent of the largest power of two in FP8 E4M3);
  * every element is stored as FP8 E4M3 (1 sign, 4 exponent bits with bias 7,
    3 mantissa bits, no infinities; largest finite value 448, smallest
    subnormal 2^-9) of v / X, rounded to nearest with ties to even, and
    clamped to +-448 when |v / X| exceeds it ("saturated");
  * an all-zero block gets E = -127;
  * a non-zero element whose quantised value is 0 has underflowed.

Readings where the pages leave a step open (also listed in the design notes):
  * the expert FFN in MXFP8: the token rows and all three expert weight
    matrices are quantised along their reduction axis (d for the gate and up
    projections, F for the down projection); the SwiGLU product silu(a) * u is
    formed from the exact products of the dequantised operands and quantised
    again, along F, before the down projection; the down projection's result
    and the combine are as in the bf16 layer. Routing is unchanged: the
    router reads the unquantised token rows.
  * overflow is counted as saturated elements, underflow as non-zero elements
    that quantise to zero.

Everything is fp64; numpy is the one library primitive.
"""
from __future__ import annotations

import numpy as np

from . import moe_oracle as O

F64 = np.float64
BLOCK = 32
E4M3_MAX = 448.0
E4M3_EMAX = 8            # exponent of the largest power of two below E4M3_MAX
E4M3_MIN_NORMAL_EXP = -6
E4M3_MANTISSA_BITS = 3
SCALE_EXP_MIN, SCALE_EXP_MAX = -127, 127


def e4m3_round(v):
    """Round to the nearest FP8 E4M3 value (ties to even), clamping to +-448.
    Returns (values on the E4M3 grid as fp64, saturated mask |v| > 448)."""
    v = np.asarray(v, F64)
    a = np.abs(v)
    # binade of each magnitude; the subnormal range shares the spacing of the
    # lowest normal binade
    with np.errstate(divide="ignore"):
        _, e = np.frexp(a)                      # a = m 2^e, m in [0.5, 1)
    exp = np.maximum(e - 1, E4M3_MIN_NORMAL_EXP)
    ulp = np.ldexp(1.0, exp - E4M3_MANTISSA_BITS)
    q = np.rint(a / ulp) * ulp                  # numpy rint: half to even
    sat = a > E4M3_MAX
    q = np.minimum(q, E4M3_MAX)
    return np.copysign(q, v), sat


def scale_exponent(amax):
    """E of the shared block scale X = 2^E: floor(log2 amax) - 8, clamped to
    [-127, 127]; -127 for an all-zero block."""
    amax = np.asarray(amax, F64)
    _, e = np.frexp(amax)
    E = (e - 1) - E4M3_EMAX
    E = np.where(amax > 0, E, SCALE_EXP_MIN)
    return np.clip(E, SCALE_EXP_MIN, SCALE_EXP_MAX).astype(np.int64)


def mx_quantize(x, block=BLOCK):
    """MX-quantise along the last axis in blocks of 32.

    Returns dict:
      q      -- the E4M3 element values (fp64, on the E4M3 grid), x's shape
      exp    -- the block scale exponents E, shape [..., n / 32]
      scale_byte -- E + 127 (the E8M0 encoding)
      saturated, underflow -- element counts
    """
    x = np.asarray(x, F64)
    n = x.shape[-1]
    if n % block:
        raise ValueError("the reduction length must be a multiple of the block size")
    xb = x.reshape(x.shape[:-1] + (n // block, block))
    E = scale_exponent(np.abs(xb).max(axis=-1))
    scaled = xb * np.ldexp(1.0, -E)[..., None]           # exact: a power of two
    q, sat = e4m3_round(scaled)
    under = (xb != 0) & (q == 0)
    return dict(q=q.reshape(x.shape), exp=E, scale_byte=(E + 127).astype(np.uint8),
                saturated=int(sat.sum()), underflow=int(under.sum()))


def mx_dequantize(q, exp, block=BLOCK):
    """v = q * 2^E per block of 32 along the last axis."""
    q = np.asarray(q, F64)
    n = q.shape[-1]
    qb = q.reshape(q.shape[:-1] + (n // block, block))
    return (qb * np.ldexp(1.0, np.asarray(exp))[..., None]).reshape(q.shape)


def mx_roundtrip(x):
    """dequantize(quantize(x)) and the quantisation's counts."""
    m = mx_quantize(x)
    return mx_dequantize(m["q"], m["exp"]), m["saturated"], m["underflow"]


def mx_swiglu_expert(x, w_gate, w_up, w_down):
    """f_e(x) in MXFP8: x, W_gate and W_up quantised along d, W_down along F,
    the SwiGLU product quantised along F before the down projection. Products
    and sums are exact (fp64). Returns (rows, counts of the h_mid
    quantisation: saturated, underflow)."""
    xq, _, _ = mx_roundtrip(x)
    gq, _, _ = mx_roundtrip(w_gate)
    uq, _, _ = mx_roundtrip(w_up)
    dq, _, _ = mx_roundtrip(w_down)
    a = xq @ gq.T
    u = xq @ uq.T
    m = O.silu(a) * u
    mq, sat, under = mx_roundtrip(m)
    return mq @ dq.T, sat, under


def mx_combine(h, idx, gate, dest_row, weights, tokens=None):
    """y_t = sum over kept slots j of g_{t,j} f^MX_{e_j}(h_t), as O.combine
    with the MXFP8 expert; tokens: optional subset."""
    h = np.asarray(h, F64)
    T, d = h.shape
    tok = np.arange(T) if tokens is None else np.asarray(tokens)
    idx = np.asarray(idx)[tok]
    gate = np.asarray(gate, F64)[tok]
    kept = np.asarray(dest_row)[tok] >= 0
    y = np.zeros((len(tok), d), F64)
    for e in (np.unique(idx[kept]) if kept.any() else []):
        rows, js = np.nonzero(kept & (idx == e))
        out, _, _ = mx_swiglu_expert(h[tok[rows]], *weights(int(e)))
        y[rows] += gate[rows, js, None] * out
    return y


def mx_layer_forward(h, w_r, bias, k, weights, cap=-1, tokens=None):
    """Whole layer with MXFP8 experts: routing and dispatch as in the bf16
    layer (O.route, O.dispatch_meta), experts in MXFP8, combine in order."""
    idx, g, s, nan_row = O.route(h, w_r, bias, k)
    meta = O.dispatch_meta(idx, np.asarray(w_r).shape[0], cap)
    y = mx_combine(h, idx, g, meta["dest_row"], weights, tokens)
    return dict(idx=idx, gate=g, logits=s, nan_row=nan_row, y=y, **meta)
