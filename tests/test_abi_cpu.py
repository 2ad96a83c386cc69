"""The C ABI library loads and exports what include/moe.h declares (CPU only).

No compute call is made here: the argument checks below all fail before the
library touches CUDA.
"""
import ctypes
import os
import re

import pytest

import combine_router_gemm_softmax_b200 as M
from combine_router_gemm_softmax_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def L():
    from combine_router_gemm_softmax_b200 import build
    build.build()
    return M.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("moe_route", "moe_permute", "moe_grouped_ffn", "moe_unpermute_combine", "moe_layer_forward",
              "moe_workspace_size", "moe_pack_weights"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for n in declared_functions():
        assert hasattr(L, n), n
    assert set(declared_functions()) <= set(_lib.EXPORTED)


def test_header_constants_match_binding():
    src = open(HEADER).read()
    consts = dict(re.findall(r"#define\s+(MOE_[A-Z0-9_]+)\s+(-?\d+)", src))
    for name, val in consts.items():
        assert getattr(_lib, name) == int(val), name


def test_version_and_status_strings(L):
    assert L.moe_version() >> 16 == 1
    assert L.moe_status_string(0) == b"ok"
    assert b"workspace" in L.moe_status_string(3)
    assert L.moe_status_string(99) == b"unknown status"


def test_workspace_sizes(L):
    cfg = M.config(4096, 1024, 8, 2, 3584)
    assert M.moe_workspace_size(cfg, M.MOE_OP_ROUTE) == 0
    nc = 4096 // 128
    assert M.moe_workspace_size(cfg, M.MOE_OP_PERMUTE) == 2 * ((nc * 8 * 4 + 255) // 256 * 256)
    assert M.moe_workspace_size(cfg, M.MOE_OP_GROUPED_FFN) == 4096 * 2 * 3584 * 2
    # the default layer materialises x_perm; with GATHER, GEMM1 reads h directly
    layer = M.moe_workspace_size(cfg, M.MOE_OP_LAYER)
    assert layer > 2 * 4096 * 2 * 1024 * 2 + 4096 * 2 * 3584 * 2
    assert M.moe_workspace_size(M.config(4096, 1024, 8, 2, 3584, dispatch="copy"), M.MOE_OP_LAYER) == layer
    gather = M.moe_workspace_size(M.config(4096, 1024, 8, 2, 3584, dispatch="gather"), M.MOE_OP_LAYER)
    assert gather == layer - 4096 * 2 * 1024 * 2
    ident = M.config(4096, 1024, 8, 2, 3584, expert_kind="identity")
    assert M.moe_workspace_size(ident, M.MOE_OP_GROUPED_FFN) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(E=300), M.MOE_ERR_UNSUPPORTED),
    (dict(k=9, E=16), M.MOE_ERR_UNSUPPORTED),
    (dict(k=5, E=4), M.MOE_ERR_UNSUPPORTED),
    (dict(d=96), M.MOE_ERR_UNSUPPORTED),
    (dict(d_ff=200), M.MOE_ERR_UNSUPPORTED),
    (dict(T=-1), M.MOE_ERR_INVALID_ARG),
    (dict(capacity=-2), M.MOE_ERR_INVALID_ARG),
])
def test_config_rejected_before_any_cuda_call(L, kw, code):
    base = dict(T=64, d=128, E=8, k=2, d_ff=256)
    base.update(kw)
    cfg = M.config(**base)
    assert M.moe_workspace_size(cfg, M.MOE_OP_LAYER) == 0
    rc = L.moe_route(ctypes.byref(cfg), None, None, None, None, None, None, None, 0, None, None)
    assert rc == code


def test_gemm_tiles_value_checked(L):
    cfg = M.config(64, 128, 8, 2, 256)
    cfg.gemm_tiles = 7
    assert L.moe_route(ctypes.byref(cfg), None, None, None, None, None, None, None, 0, None, None) \
        == M.MOE_ERR_INVALID_ARG
    for tiles in ("auto", "single", "pair"):
        assert M.moe_workspace_size(M.config(64, 128, 8, 2, 256, gemm_tiles=tiles), M.MOE_OP_LAYER) > 0


def test_gemm_tiles_auto_rule(L):
    """AUTO resolves to CTA-pair tiles only for bf16 SwiGLU experts of at
    least 1024 rows on average (T*k/E, capped by a compact capacity; the
    capacity itself in the padded layout) and at most 128 MiB of weights each,
    and never when an option that needs single tiles is set. Host only."""
    used = M.moe_gemm_tiles_used
    S, P = M.MOE_GEMM_TILES_SINGLE, M.MOE_GEMM_TILES_PAIR
    # the layers this rule was measured on
    assert used(M.config(4096, 1024, 8, 2, 3584)) == P                      # 1024 rows, 22 MB
    assert used(M.config(16384, 2048, 64, 6, 1408)) == P                    # 1536 rows, 17 MB
    assert used(M.config(16384, 2048, 64, 6, 1408, capacity=1920)) == P
    assert used(M.config(16384, 2048, 64, 6, 1408, capacity=1920, layout="padded")) == P
    assert used(M.config(32768, 4096, 8, 2, 14336)) == S                    # 352 MB an expert
    assert used(M.config(8192, 2048, 128, 8, 768)) == S                     # 512 rows
    # the edges of the rule
    assert used(M.config(4095, 1024, 8, 2, 3584)) == S                      # 1023 rows
    assert used(M.config(16384, 2048, 64, 6, 1408, capacity=1000)) == S     # capped below 1024
    assert used(M.config(1024, 2048, 64, 6, 1408, capacity=1024, layout="padded")) == P
    assert used(M.config(16384, 2048, 8, 2, 7168)) == P                     # 88 MB, measured faster
    assert used(M.config(8192, 4096, 8, 1, 5376)) == P                      # 3 d F 2 = 132 MB <= 128 MiB
    assert used(M.config(8192, 4096, 8, 1, 5504)) == S                      # 135 MB > 128 MiB
    # options that need single tiles, other dtypes and expert kinds
    for kw in (dict(dispatch="gather"), dict(combine="fused"), dict(preact="save"), dict(precision="mxfp8"),
               dict(dtype="f32"), dict(expert_kind="identity"), dict(gemm_tiles="single")):
        assert used(M.config(4096, 1024, 8, 2, 3584, **kw)) == S, kw
    # an explicit request is kept
    assert used(M.config(64, 128, 8, 2, 256, gemm_tiles="pair")) == P
    assert used(M.config(64, 128, 8, 2, 256)) == S
    # errors come back as the return code and leave the output alone
    out = ctypes.c_int32(-1)
    bad = M.config(64, 128, 8, 2, 256)
    bad.gemm_tiles = 7
    assert L.moe_gemm_tiles_used(ctypes.byref(bad), ctypes.byref(out)) == M.MOE_ERR_INVALID_ARG
    odd = M.config(64, 128, 8, 2, 200)                                      # d_ff not a multiple of 128
    assert L.moe_gemm_tiles_used(ctypes.byref(odd), ctypes.byref(out)) == M.MOE_ERR_UNSUPPORTED
    assert L.moe_gemm_tiles_used(ctypes.byref(M.config(64, 128, 8, 2, 256)), None) == M.MOE_ERR_INVALID_ARG
    assert out.value == -1
    with pytest.raises(M.MoeError):
        used(odd)


def test_null_pointers_rejected(L):
    cfg = M.config(64, 128, 8, 2, 256)
    assert L.moe_route(ctypes.byref(cfg), None, None, None, None, None, None, None, 0, None, None) \
        == M.MOE_ERR_INVALID_ARG
    assert L.moe_unpermute_combine(ctypes.byref(cfg), None, None, None, None, None, None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_layer_forward(ctypes.byref(cfg), None, None, None, None, None, None, None, None, None, None, None,
                               0, None, None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_pack_weights(None, None, None, None, None) == M.MOE_ERR_INVALID_ARG


def test_misaligned_pointer_rejected(L):
    cfg = M.config(64, 128, 8, 2, 256)
    p = ctypes.c_void_p(0x1000)
    odd = ctypes.c_void_p(0x1008)
    rc = L.moe_route(ctypes.byref(cfg), odd, p, None, None, p, p, None, 0, None, None)
    assert rc == M.MOE_ERR_UNSUPPORTED


def test_small_workspace_rejected(L):
    cfg = M.config(4096, 1024, 8, 2, 3584)
    p = ctypes.c_void_p(0x1000)
    rc = L.moe_permute(ctypes.byref(cfg), p, p, p, p, p, p, p, p, p, 16, None, None)
    assert rc == M.MOE_ERR_WORKSPACE


def test_layout_checked_and_sized(L):
    """The padded layout needs a capacity and sizes the permuted buffers at
    E*capacity rows; an unknown layout value is rejected."""
    bad = M.config(64, 128, 8, 2, 256, layout="padded")          # no capacity
    assert L.moe_route(ctypes.byref(bad), None, None, None, None, None, None, None, 0, None, None) \
        == M.MOE_ERR_INVALID_ARG
    odd = M.config(64, 128, 8, 2, 256, capacity=20)
    odd.layout = 9
    assert M.moe_workspace_size(odd, M.MOE_OP_LAYER) == 0
    compact = M.config(64, 128, 8, 2, 256, capacity=40)
    padded = M.config(64, 128, 8, 2, 256, capacity=40, layout="padded")
    assert M.perm_rows(compact) == 128 and M.perm_rows(padded) == 320
    # h_mid [P, F] bf16 is the whole grouped-FFN workspace
    assert M.moe_workspace_size(padded, M.MOE_OP_GROUPED_FFN) == 320 * 256 * 2
    assert M.moe_workspace_size(compact, M.MOE_OP_GROUPED_FFN) == 128 * 256 * 2
    assert M.moe_workspace_size(padded, M.MOE_OP_LAYER) > M.moe_workspace_size(compact, M.MOE_OP_LAYER)


def test_dispatch_mode_checked(L):
    """GATHER is only for bf16 SwiGLU experts in the compact layout with
    single-CTA tiles; other values are rejected before any CUDA call."""
    ok = M.config(64, 128, 8, 2, 256, dispatch="gather")
    assert M.moe_workspace_size(ok, M.MOE_OP_LAYER) > 0
    for kw in (dict(dtype="f32"), dict(expert_kind="identity"), dict(gemm_tiles="pair"),
               dict(capacity=20, layout="padded")):
        cfg = M.config(64, 128, 8, 2, 256, dispatch="gather", **kw)
        assert L.moe_route(ctypes.byref(cfg), None, None, None, None, None, None, None, 0, None, None) \
            == M.MOE_ERR_UNSUPPORTED, kw
    bad = M.config(64, 128, 8, 2, 256)
    bad.dispatch = 3
    assert L.moe_route(ctypes.byref(bad), None, None, None, None, None, None, None, 0, None, None) \
        == M.MOE_ERR_INVALID_ARG


def test_backward_checked_before_any_cuda_call(L):
    """The backward needs bf16 SwiGLU experts, the compact layout and x_perm
    from the forward; its scratch is sized by MOE_OP_BACKWARD."""
    cfg = M.config(4096, 1024, 8, 2, 3584)
    need = M.moe_workspace_size(cfg, M.MOE_OP_BACKWARD)
    P, d, F = 4096 * 2, 1024, 3584
    assert need >= P * (d + F + 2 * F + d) * 2          # dy_perm, dh_mid, dgu, dx_perm
    for kw in (dict(dtype="f32"), dict(expert_kind="identity"), dict(dispatch="gather")):
        bad = M.config(4096, 1024, 8, 2, 3584, **kw)
        assert M.moe_workspace_size(bad, M.MOE_OP_BACKWARD) == 0, kw
        p = ctypes.c_void_p(0x1000)
        rc = L.moe_layer_backward(ctypes.byref(bad), p, p, p, p, p, p, p, p, p, p, p, p, 1 << 40, p, 1 << 40,
                                  None, None)
        assert rc == M.MOE_ERR_UNSUPPORTED, kw
    p = ctypes.c_void_p(0x1000)
    assert L.moe_layer_backward(ctypes.byref(cfg), p, p, p, p, p, p, p, p, p, p, p, p, 16, p, 1 << 40, None,
                                None) == M.MOE_ERR_WORKSPACE
    assert L.moe_pack_weights_backward(ctypes.byref(cfg), None, None, None, None, None) == M.MOE_ERR_INVALID_ARG
    padded = M.config(4096, 1024, 8, 2, 3584, capacity=2000, layout="padded")
    assert M.moe_workspace_size(padded, M.MOE_OP_BACKWARD) > 0


def test_backward_workspace_formula(L):
    """MOE_OP_BACKWARD scratch: four row buffers, ds, the column offsets, four
    transposed operands over P' = roundup64(P) + 64 E columns, and the router
    gradient's per-512-token partial sums, each piece 256-byte aligned."""
    def up(n):
        return (n + 255) // 256 * 256
    for T, d, E, k, F in ((4096, 1024, 8, 2, 3584), (777, 256, 40, 4, 384), (8192, 2048, 128, 8, 768)):
        P = T * k
        pp = (P + 63) // 64 * 64 + 64 * E
        chunks = (T + 511) // 512
        want = (up(P * d * 2) + up(P * F * 2) + up(P * 2 * F * 2) + up(P * d * 2) + up(T * k * 4) + up((E + 1) * 4)
                + up(d * pp * 2) + up(F * pp * 2) + up(2 * F * pp * 2) + up(d * pp * 2) + up(chunks * E * (d + 1) * 4))
        assert M.moe_workspace_size(M.config(T, d, E, k, F), M.MOE_OP_BACKWARD) == want
