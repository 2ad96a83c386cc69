"""Pins of the MXFP8 oracle (oracle/mxfp8.py) to things outside it (CPU).

* the E4M3 grid: every finite E4M3 value decoded by torch's float8_e4m3fn
  type maps to itself, and rounding of in-range values (including every
  midpoint between neighbours) agrees with torch's float8 conversion;
* saturation and underflow edges, counted;
* the shared scale at amax a power of two, just below it, zero and clamped;
* blocks built from exact E4M3 values and a chosen scale quantise back to
  exactly those values and that scale;
* the element error bound of the format (half a unit in the last place);
* a down projection by the identity reduces the MXFP8 expert to the
  quantisation of its SwiGLU product, computed here with torch's float8
  conversion as the element quantiser.
"""
import numpy as np
import torch

import oracle as O
from oracle import mxfp8 as X


def e4m3_values():
    v = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().double().numpy()
    return v[np.isfinite(v)]


def test_every_e4m3_value_is_a_fixed_point():
    v = e4m3_values()
    assert len(v) == 254 and v.max() == 448.0 and v[v > 0].min() == 2.0 ** -9
    q, sat = X.e4m3_round(v)
    assert np.array_equal(q, v) and not sat.any()


def test_rounding_matches_torch_float8_in_range():
    r = np.random.default_rng(0)
    v = (r.uniform(-448, 448, 100000) * np.exp2(r.integers(-14, 1, 100000))).astype(np.float32).astype(np.float64)
    g = np.unique(np.abs(e4m3_values()))
    mids = (g[:-1] + g[1:]) / 2                      # exact ties: must go to the even neighbour
    for x in (v, mids, -mids):
        q, _ = X.e4m3_round(x)
        t = torch.from_numpy(x).float().to(torch.float8_e4m3fn).double().numpy()
        assert np.array_equal(q, t)


def test_saturation_and_underflow_edges():
    q, sat = X.e4m3_round(np.array([448.0, 449.0, 470.0, 1e9, -500.0, 2.0 ** -10, 2.0 ** -10 * (1 + 2.0 ** -20),
                                    -(2.0 ** -10) * 3]))
    assert q.tolist() == [448.0, 448.0, 448.0, 448.0, -448.0, 0.0, 2.0 ** -9, -(2.0 ** -8)]
    assert sat.tolist() == [False, True, True, True, True, False, False, False]
    E = -3
    blk = np.zeros(32)
    blk[0] = 256.0 * 2.0 ** E                         # amax: scale exponent E exactly
    blk[1] = 2.0 ** -10 * 2.0 ** E                    # a tie at half the smallest subnormal: rounds to 0
    blk[2] = 500.0 * 2.0 ** E / 2                     # 250 after scaling: representable range
    blk[3] = -(2.0 ** -12) * 2.0 ** E                 # below it: 0
    m = X.mx_quantize(blk[None, :])
    assert m["exp"].tolist() == [[E]]
    assert m["underflow"] == 2 and m["saturated"] == 0
    over = np.full((1, 32), 1.0)
    over[0, 0] = 1.99                                 # amax mantissa above 1.75: saturates (OCP rule)
    mo = X.mx_quantize(over)
    assert mo["exp"].tolist() == [[-8]] and mo["saturated"] == 1
    assert mo["q"][0, 0] == 448.0


def test_scale_exponent_rule():
    p = np.arange(-20, 21)
    assert X.scale_exponent(np.exp2(p.astype(float))).tolist() == (p - 8).tolist()
    assert X.scale_exponent(1.5 * np.exp2(p.astype(float))).tolist() == (p - 8).tolist()
    assert X.scale_exponent(np.nextafter(np.exp2(p.astype(float)), 0)).tolist() == (p - 9).tolist()
    assert X.scale_exponent(np.array([0.0, 2.0 ** 200, 2.0 ** -200])).tolist() == [-127, 127, -127]


def test_exact_blocks_round_trip():
    r = np.random.default_rng(1)
    v = e4m3_values()
    big = v[(np.abs(v) >= 256)]
    rows = []
    exps = r.integers(-30, 30, size=(5, 4))
    for i in range(5):
        row = []
        for b in range(4):
            q = r.choice(v, 32)
            q[r.integers(32)] = r.choice(big)           # block max in [256, 448]: its scale is exps[i, b]
            row.append(q * 2.0 ** exps[i, b])
        rows.append(np.concatenate(row))
    x = np.array(rows)
    m = X.mx_quantize(x)
    assert np.array_equal(m["exp"], exps)
    assert np.array_equal(X.mx_dequantize(m["q"], m["exp"]), x)
    assert m["saturated"] == 0
    assert np.array_equal(m["scale_byte"], (exps + 127).astype(np.uint8))
    z = X.mx_quantize(np.zeros((2, 64)))
    assert (z["exp"] == -127).all() and not z["q"].any()


def test_element_error_bound():
    r = np.random.default_rng(2)
    x = r.standard_normal((64, 256)) * np.exp2(r.integers(-10, 10, size=(64, 1)))
    m = X.mx_quantize(x)
    deq = X.mx_dequantize(m["q"], m["exp"])
    scale = np.repeat(np.exp2(m["exp"].astype(float)), 32, axis=1)
    s = np.abs(x) / scale
    ok = s <= 448.0
    normal = ok & (s >= 2.0 ** -6)
    assert np.all(np.abs(deq - x)[normal] <= 2.0 ** -4 * np.abs(x)[normal])
    assert np.all(np.abs(deq - x)[ok & ~normal] <= 2.0 ** -10 * scale[ok & ~normal])
    assert m["saturated"] == int((~ok).sum())


def test_identity_down_projection_reduces_to_quantised_swiglu():
    """W_down = I (exact in MXFP8): the expert returns the MX quantisation of
    silu(a) * u, re-derived here with torch's float8 conversion."""
    r = np.random.default_rng(3)
    d = F = 64
    x = r.standard_normal((16, d))
    wg = r.standard_normal((F, d)) / 8
    wu = r.standard_normal((F, d)) / 8
    got, _, _ = X.mx_swiglu_expert(x, wg, wu, np.eye(F))
    xq, _, _ = X.mx_roundtrip(x)
    gq, _, _ = X.mx_roundtrip(wg)
    uq, _, _ = X.mx_roundtrip(wu)
    a = torch.from_numpy(xq @ gq.T)
    u = torch.from_numpy(xq @ uq.T)
    m = torch.nn.functional.silu(a) * u
    blocks = m.reshape(16, F // 32, 32)
    _, e = torch.frexp(blocks.abs().amax(dim=-1))
    scale = torch.exp2((e - 1 - 8).double())[..., None]
    s = (blocks / scale).clamp(-448.0, 448.0)         # saturation (pinned above); torch gives NaN past 464
    want = (s.float().to(torch.float8_e4m3fn).double() * scale).reshape(16, F).numpy()
    assert np.allclose(got, want, rtol=0, atol=1e-12)


def test_mx_expert_is_close_to_the_exact_expert():
    """The MXFP8 expert differs from the exact one by the format's rounding
    only: E4M3 keeps 3 mantissa bits (up to 6.25% per element, about 2.5%
    rms), applied to x, both weights and the SwiGLU product, so each output
    row moves by several per cent of its magnitude, never zero and well
    under 20%."""
    r = np.random.default_rng(4)
    d, F = 256, 128
    x = r.standard_normal((32, d))
    wg, wu = r.standard_normal((F, d)) / 16, r.standard_normal((F, d)) / 16
    wd = r.standard_normal((d, F)) / np.sqrt(F)
    got, _, _ = X.mx_swiglu_expert(x, wg, wu, wd)
    want = O.swiglu_expert(x, wg, wu, wd)
    err = np.abs(got - want).max(axis=1) / np.abs(want).max(axis=1)
    assert 1e-3 < err.max() < 0.2
