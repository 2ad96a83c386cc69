"""ctypes binding of libmoe_b200.so (argument marshalling only).

Every function here checks shapes, dtypes and devices of torch tensors, passes
their device pointers and the current CUDA stream to the C ABI of the same
name, and turns a non-zero return code into MoeError. All computation happens
in the library's CUDA kernels; there is no other implementation to fall back
to, so a missing library is an error.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_NO_DEVICE = range(6)
MOE_STATUS_NAN_LOGIT, MOE_STATUS_BAD_ROUTE, MOE_STATUS_TIMEOUT = 1, 2, 4
MOE_STATUS_MX_SATURATED, MOE_STATUS_MX_UNDERFLOW = 8, 16
MOE_PRECISION_BF16, MOE_PRECISION_MXFP8 = 0, 1
MOE_COMBINE_AUTO, MOE_COMBINE_SEPARATE, MOE_COMBINE_FUSED = 0, 1, 2
MOE_PREACT_RECOMPUTE, MOE_PREACT_SAVE = 0, 1
MOE_DTYPE_BF16, MOE_DTYPE_F32 = 0, 1
MOE_EXPERT_SWIGLU, MOE_EXPERT_IDENTITY, MOE_EXPERT_SCALE = 0, 1, 2
MOE_OP_ROUTE, MOE_OP_PERMUTE, MOE_OP_GROUPED_FFN, MOE_OP_LAYER, MOE_OP_BACKWARD = 0, 1, 2, 3, 4
MOE_GEMM_TILES_AUTO, MOE_GEMM_TILES_SINGLE, MOE_GEMM_TILES_PAIR = 0, 1, 2
MOE_LAYOUT_COMPACT, MOE_LAYOUT_PADDED = 0, 1
MOE_DISPATCH_AUTO, MOE_DISPATCH_COPY, MOE_DISPATCH_GATHER = 0, 1, 2
MOE_MAX_E, MOE_MAX_K, MOE_PACK_BLOCK = 256, 8, 128

EXPORTED = ("moe_workspace_size", "moe_status_string", "moe_version", "moe_pack_weights", "moe_route",
            "moe_permute", "moe_grouped_ffn", "moe_unpermute_combine", "moe_layer_forward",
            "moe_permute_static_scratch", "moe_layer_forward_timed", "moe_pack_weights_backward",
            "moe_layer_backward", "moe_mxfp8_quantize", "moe_mxfp8_weights_size", "moe_pack_weights_mxfp8",
            "moe_debug_stall_next_gemms", "moe_gemm_tiles_used")


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int, text: str):
        super().__init__(f"{fn} failed: {text} (code {code})")
        self.code = code


class MoeConfig(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("E", ctypes.c_int32), ("k", ctypes.c_int32),
                ("d_ff", ctypes.c_int32), ("dtype", ctypes.c_int32), ("expert_kind", ctypes.c_int32),
                ("capacity", ctypes.c_int32), ("gemm_tiles", ctypes.c_int32), ("layout", ctypes.c_int32),
                ("dispatch", ctypes.c_int32), ("precision", ctypes.c_int32), ("combine", ctypes.c_int32),
                ("preact", ctypes.c_int32)]

    def __repr__(self):
        return "MoeConfig(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == MOE_DTYPE_BF16 else torch.float32


_lib = None
_lock = threading.Lock()

P = ctypes.c_void_p
I32 = ctypes.c_int32
SZ = ctypes.c_size_t
CFG = ctypes.POINTER(MoeConfig)

_SIGS = {
    "moe_workspace_size": (SZ, [CFG, I32]),
    "moe_status_string": (ctypes.c_char_p, [I32]),
    "moe_version": (I32, []),
    "moe_gemm_tiles_used": (I32, [CFG, P]),
    "moe_pack_weights": (I32, [CFG, P, P, P, P]),
    "moe_route": (I32, [CFG, P, P, P, P, P, P, P, SZ, P, P]),
    "moe_permute": (I32, [CFG, P, P, P, P, P, P, P, P, P, SZ, P, P]),
    "moe_grouped_ffn": (I32, [CFG, P, P, P, P, P, P, SZ, P, P]),
    "moe_unpermute_combine": (I32, [CFG, P, P, P, P, P, P]),
    "moe_layer_forward": (I32, [CFG, P, P, P, P, P, P, P, P, P, P, P, SZ, P, P]),
    "moe_permute_static_scratch": (I32, [CFG, P, P, P, P, P, P, P, P, P, P]),
    "moe_layer_forward_timed": (I32, [CFG, P, P, P, P, P, P, P, P, P, P, P, SZ, P, P, P]),
    "moe_pack_weights_backward": (I32, [CFG, P, P, P, P, P]),
    "moe_layer_backward": (I32, [CFG, P, P, P, P, P, P, P, P, P, P, P, P, SZ, P, SZ, P, P]),
    "moe_mxfp8_quantize": (I32, [P, I32, I32, P, P, P, P, P]),
    "moe_mxfp8_weights_size": (SZ, [CFG, I32]),
    "moe_pack_weights_mxfp8": (I32, [CFG, P, P, P, P, P, P]),
    "moe_debug_stall_next_gemms": (I32, [I32]),
}


def lib() -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                                   "`python -m combine_router_gemm_softmax_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in _SIGS.items():
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            _lib = L
    return _lib


def config(T, d, E, k, d_ff, dtype="bf16", expert_kind="swiglu", capacity=-1, gemm_tiles="auto",
           layout="compact", dispatch="auto", precision="bf16", combine="auto", preact="recompute") -> MoeConfig:
    dt = {"bf16": MOE_DTYPE_BF16, "f32": MOE_DTYPE_F32, torch.bfloat16: MOE_DTYPE_BF16,
          torch.float32: MOE_DTYPE_F32}[dtype]
    kind = {"swiglu": MOE_EXPERT_SWIGLU, "identity": MOE_EXPERT_IDENTITY, "scale": MOE_EXPERT_SCALE}[expert_kind]
    tiles = {"auto": MOE_GEMM_TILES_AUTO, "single": MOE_GEMM_TILES_SINGLE, "pair": MOE_GEMM_TILES_PAIR}[gemm_tiles]
    lay = {"compact": MOE_LAYOUT_COMPACT, "padded": MOE_LAYOUT_PADDED}[layout]
    disp = {"auto": MOE_DISPATCH_AUTO, "copy": MOE_DISPATCH_COPY, "gather": MOE_DISPATCH_GATHER}[dispatch]
    prec = {"bf16": MOE_PRECISION_BF16, "mxfp8": MOE_PRECISION_MXFP8}[precision]
    comb = {"auto": MOE_COMBINE_AUTO, "separate": MOE_COMBINE_SEPARATE, "fused": MOE_COMBINE_FUSED}[combine]
    pre = {"recompute": MOE_PREACT_RECOMPUTE, "save": MOE_PREACT_SAVE}[preact]
    return MoeConfig(T, d, E, k, d_ff, dt, kind, capacity, tiles, lay, disp, prec, comb, pre)


def perm_rows(cfg) -> int:
    """Rows P of x_perm, y_perm and perm_src: T*k, or E*capacity in the padded layout."""
    return cfg.E * cfg.capacity if cfg.layout == MOE_LAYOUT_PADDED else cfg.T * cfg.k


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _check(t, shape, dtype, name):
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)} != {tuple(shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype} != {dtype}")


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _rc(fn, code):
    if code != MOE_OK:
        raise MoeError(fn, code, lib().moe_status_string(code).decode())


def _dev(ref):
    return ref.device


def _check_expert_weights(cfg, w13, w_down):
    """bf16: w13_packed [E, 2F, d] and w_down [E, d, F]; MXFP8: the two uint8
    blobs of moe_pack_weights_mxfp8."""
    if cfg.precision == MOE_PRECISION_MXFP8:
        _check(w13, (moe_mxfp8_weights_size(cfg, 0),), torch.uint8, "w13 MXFP8 blob")
        _check(w_down, (moe_mxfp8_weights_size(cfg, 1),), torch.uint8, "w_down MXFP8 blob")
    else:
        _check(w13, (cfg.E, 2 * cfg.d_ff, cfg.d), cfg.torch_dtype, "w13_packed")
        _check(w_down, (cfg.E, cfg.d, cfg.d_ff), cfg.torch_dtype, "w_down")


def moe_workspace_size(cfg: MoeConfig, op: int) -> int:
    return int(lib().moe_workspace_size(ctypes.byref(cfg), op))


def moe_gemm_tiles_used(cfg: MoeConfig) -> int:
    """MOE_GEMM_TILES_SINGLE or MOE_GEMM_TILES_PAIR: the grouped GEMMs' tile
    shape for cfg with AUTO resolved (host only)."""
    tiles = ctypes.c_int32(-1)
    _rc("moe_gemm_tiles_used", lib().moe_gemm_tiles_used(ctypes.byref(cfg), ctypes.byref(tiles)))
    return tiles.value


def workspace(cfg: MoeConfig, op: int, device) -> torch.Tensor:
    n = moe_workspace_size(cfg, op)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def moe_pack_weights(cfg, w_gate, w_up, w13_packed=None, stream=None):
    dt = cfg.torch_dtype
    _check(w_gate, (cfg.E, cfg.d_ff, cfg.d), dt, "w_gate")
    _check(w_up, (cfg.E, cfg.d_ff, cfg.d), dt, "w_up")
    if w13_packed is None:
        w13_packed = torch.empty((cfg.E, 2 * cfg.d_ff, cfg.d), dtype=dt, device=_dev(w_gate))
    _check(w13_packed, (cfg.E, 2 * cfg.d_ff, cfg.d), dt, "w13_packed")
    _rc("moe_pack_weights", lib().moe_pack_weights(ctypes.byref(cfg), _ptr(w_gate), _ptr(w_up), _ptr(w13_packed),
                                                   _stream(stream)))
    return w13_packed


def moe_route(cfg, h, w_router, bias=None, logits_out=None, topk_idx=None, topk_gate=None, status=None,
              stream=None):
    dt = cfg.torch_dtype
    dev = _dev(h)
    _check(h, (cfg.T, cfg.d), dt, "h")
    _check(w_router, (cfg.E, cfg.d), dt, "w_router")
    _check(bias, (cfg.E,), torch.float32, "bias")
    _check(logits_out, (cfg.T, cfg.E), torch.float32, "logits_out")
    if topk_idx is None:
        topk_idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=dev)
    if topk_gate is None:
        topk_gate = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device=dev)
    _check(topk_idx, (cfg.T, cfg.k), torch.int32, "topk_idx")
    _check(topk_gate, (cfg.T, cfg.k), torch.float32, "topk_gate")
    _rc("moe_route", lib().moe_route(ctypes.byref(cfg), _ptr(h), _ptr(w_router), _ptr(bias), _ptr(logits_out),
                                     _ptr(topk_idx), _ptr(topk_gate), None, 0, _ptr(status), _stream(stream)))
    return topk_idx, topk_gate


def moe_permute(cfg, h, topk_idx, out=None, ws=None, status=None, stream=None):
    """Returns dict routed_counts, counts, offsets, dest_row, perm_src, x_perm."""
    dt = cfg.torch_dtype
    dev = _dev(h)
    A = perm_rows(cfg)
    _check(h, (cfg.T, cfg.d), dt, "h")
    _check(topk_idx, (cfg.T, cfg.k), torch.int32, "topk_idx")
    if out is None:
        out = dict(routed_counts=torch.empty(cfg.E, dtype=torch.int32, device=dev),
                   counts=torch.empty(cfg.E, dtype=torch.int32, device=dev),
                   offsets=torch.empty(cfg.E + 1, dtype=torch.int32, device=dev),
                   dest_row=torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=dev),
                   perm_src=torch.empty(max(A, 1), dtype=torch.int32, device=dev),
                   x_perm=torch.empty((max(A, 1), cfg.d), dtype=dt, device=dev))
    if ws is None:
        ws = workspace(cfg, MOE_OP_PERMUTE, dev)
    _rc("moe_permute", lib().moe_permute(
        ctypes.byref(cfg), _ptr(h), _ptr(topk_idx), _ptr(out["routed_counts"]), _ptr(out["counts"]),
        _ptr(out["offsets"]), _ptr(out["dest_row"]), _ptr(out["perm_src"]), _ptr(out["x_perm"]), _ptr(ws),
        ws.numel(), _ptr(status), _stream(stream)))
    return out


def moe_grouped_ffn(cfg, x_perm, offsets, w13_packed=None, w_down=None, y_perm=None, ws=None, status=None,
                    stream=None):
    dt = cfg.torch_dtype
    dev = _dev(x_perm)
    rows = x_perm.shape[0]
    if rows < max(perm_rows(cfg), 1):
        raise ValueError("x_perm needs perm_rows(cfg) rows")
    _check(offsets, (cfg.E + 1,), torch.int32, "offsets")
    if cfg.expert_kind == MOE_EXPERT_SWIGLU:
        _check_expert_weights(cfg, w13_packed, w_down)
    if y_perm is None:
        y_perm = torch.empty((rows, cfg.d), dtype=dt, device=dev)
    if ws is None:
        ws = workspace(cfg, MOE_OP_GROUPED_FFN, dev)
    _rc("moe_grouped_ffn", lib().moe_grouped_ffn(
        ctypes.byref(cfg), _ptr(x_perm), _ptr(offsets), _ptr(w13_packed), _ptr(w_down), _ptr(y_perm), _ptr(ws),
        ws.numel(), _ptr(status), _stream(stream)))
    return y_perm


def moe_unpermute_combine(cfg, y_perm, dest_row, topk_gate, y=None, status=None, stream=None):
    dt = cfg.torch_dtype
    _check(dest_row, (cfg.T, cfg.k), torch.int32, "dest_row")
    _check(topk_gate, (cfg.T, cfg.k), torch.float32, "topk_gate")
    if y is None:
        y = torch.empty((cfg.T, cfg.d), dtype=dt, device=_dev(y_perm))
    _check(y, (cfg.T, cfg.d), dt, "y")
    _rc("moe_unpermute_combine", lib().moe_unpermute_combine(
        ctypes.byref(cfg), _ptr(y_perm), _ptr(dest_row), _ptr(topk_gate), _ptr(y), _ptr(status), _stream(stream)))
    return y


def moe_layer_forward(cfg, h, w_router, bias=None, w13_packed=None, w_down=None, y=None, topk_idx=None,
                      topk_gate=None, routed_counts=None, counts=None, ws=None, status=None, stream=None,
                      stage_events=None):
    """The whole layer; returns y. stage_events: None, or 5 torch.cuda.Event
    (or None) recorded before the router and after the router, the dispatch,
    the expert stage and the combine (moe_layer_forward_timed)."""
    dt = cfg.torch_dtype
    dev = _dev(h)
    _check(h, (cfg.T, cfg.d), dt, "h")
    _check(w_router, (cfg.E, cfg.d), dt, "w_router")
    _check(bias, (cfg.E,), torch.float32, "bias")
    if cfg.expert_kind == MOE_EXPERT_SWIGLU:
        _check_expert_weights(cfg, w13_packed, w_down)
    _check(topk_idx, (cfg.T, cfg.k), torch.int32, "topk_idx")
    _check(topk_gate, (cfg.T, cfg.k), torch.float32, "topk_gate")
    _check(routed_counts, (cfg.E,), torch.int32, "routed_counts")
    _check(counts, (cfg.E,), torch.int32, "counts")
    if y is None:
        y = torch.empty((cfg.T, cfg.d), dtype=dt, device=dev)
    _check(y, (cfg.T, cfg.d), dt, "y")
    if ws is None:
        ws = workspace(cfg, MOE_OP_LAYER, dev)
    args = (ctypes.byref(cfg), _ptr(h), _ptr(w_router), _ptr(bias), _ptr(w13_packed), _ptr(w_down), _ptr(y),
            _ptr(topk_idx), _ptr(topk_gate), _ptr(routed_counts), _ptr(counts), _ptr(ws), ws.numel(), _ptr(status),
            _stream(stream))
    if stage_events is None:
        _rc("moe_layer_forward", lib().moe_layer_forward(*args))
        return y
    if len(stage_events) != 5:
        raise ValueError("stage_events needs 5 entries")
    handles = (ctypes.c_void_p * 5)(*[None if e is None else _event_handle(e) for e in stage_events])
    _rc("moe_layer_forward_timed", lib().moe_layer_forward_timed(*args, handles))
    return y


def _event_handle(ev):
    """Raw cudaEvent_t of a torch.cuda.Event; torch creates the event on its
    first record, so an event that was never recorded is recorded once here."""
    if not ev.cuda_event:
        ev.record()
    return ctypes.c_void_p(ev.cuda_event)


def moe_permute_static_scratch(cfg, h, topk_idx, out=None, status=None, stream=None):
    """moe_permute without a workspace argument, for callers that cannot
    allocate device memory; the library keeps the scratch in a fixed 1 MiB
    device array shared by all calls (calls that overlap on the GPU race).
    Returns the same dict as moe_permute."""
    dt = cfg.torch_dtype
    dev = _dev(h)
    A = perm_rows(cfg)
    _check(h, (cfg.T, cfg.d), dt, "h")
    _check(topk_idx, (cfg.T, cfg.k), torch.int32, "topk_idx")
    if out is None:
        out = dict(routed_counts=torch.empty(cfg.E, dtype=torch.int32, device=dev),
                   counts=torch.empty(cfg.E, dtype=torch.int32, device=dev),
                   offsets=torch.empty(cfg.E + 1, dtype=torch.int32, device=dev),
                   dest_row=torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=dev),
                   perm_src=torch.empty(max(A, 1), dtype=torch.int32, device=dev),
                   x_perm=torch.empty((max(A, 1), cfg.d), dtype=dt, device=dev))
    _rc("moe_permute_static_scratch", lib().moe_permute_static_scratch(
        ctypes.byref(cfg), _ptr(h), _ptr(topk_idx), _ptr(out["routed_counts"]), _ptr(out["counts"]),
        _ptr(out["offsets"]), _ptr(out["dest_row"]), _ptr(out["perm_src"]), _ptr(out["x_perm"]), _ptr(status),
        _stream(stream)))
    return out


def moe_pack_weights_backward(cfg, w13_packed, w_down, stream=None):
    """Per-expert transposes for the backward dgrad GEMMs: returns
    (w13_t [E, d, 2F], w_down_t [E, F, d])."""
    dt = cfg.torch_dtype
    dev = _dev(w13_packed)
    _check(w13_packed, (cfg.E, 2 * cfg.d_ff, cfg.d), dt, "w13_packed")
    _check(w_down, (cfg.E, cfg.d, cfg.d_ff), dt, "w_down")
    w13_t = torch.empty((cfg.E, cfg.d, 2 * cfg.d_ff), dtype=dt, device=dev)
    w_down_t = torch.empty((cfg.E, cfg.d_ff, cfg.d), dtype=dt, device=dev)
    _rc("moe_pack_weights_backward", lib().moe_pack_weights_backward(
        ctypes.byref(cfg), _ptr(w13_packed), _ptr(w_down), _ptr(w13_t), _ptr(w_down_t), _stream(stream)))
    return w13_t, w_down_t


def moe_layer_backward(cfg, h, w_router, w13_packed, w13_t, w_down_t, dy, fwd_ws, with_bias=True, ws=None,
                       status=None, stream=None):
    """Gradients of <dy, y> for the moe_layer_forward call that last used
    fwd_ws. Returns dict dh [T,d] (bf16), dw_router [E,d], dbias [E] (or None),
    dw13 [E,2F,d] (packed row order), dw_down [E,d,F] (fp32)."""
    dt = cfg.torch_dtype
    dev = _dev(h)
    _check(h, (cfg.T, cfg.d), dt, "h")
    _check(w_router, (cfg.E, cfg.d), dt, "w_router")
    _check(w13_packed, (cfg.E, 2 * cfg.d_ff, cfg.d), dt, "w13_packed")
    _check(w13_t, (cfg.E, cfg.d, 2 * cfg.d_ff), dt, "w13_t")
    _check(w_down_t, (cfg.E, cfg.d_ff, cfg.d), dt, "w_down_t")
    _check(dy, (cfg.T, cfg.d), dt, "dy")
    out = dict(dh=torch.empty((cfg.T, cfg.d), dtype=dt, device=dev),
               dw_router=torch.empty((cfg.E, cfg.d), dtype=torch.float32, device=dev),
               dbias=torch.empty(cfg.E, dtype=torch.float32, device=dev) if with_bias else None,
               dw13=torch.empty((cfg.E, 2 * cfg.d_ff, cfg.d), dtype=torch.float32, device=dev),
               dw_down=torch.empty((cfg.E, cfg.d, cfg.d_ff), dtype=torch.float32, device=dev))
    if ws is None:
        ws = workspace(cfg, MOE_OP_BACKWARD, dev)
    _rc("moe_layer_backward", lib().moe_layer_backward(
        ctypes.byref(cfg), _ptr(h), _ptr(w_router), _ptr(w13_packed), _ptr(w13_t), _ptr(w_down_t), _ptr(dy),
        _ptr(out["dh"]), _ptr(out["dw_router"]), _ptr(out["dbias"]), _ptr(out["dw13"]), _ptr(out["dw_down"]),
        _ptr(fwd_ws), fwd_ws.numel(), _ptr(ws), ws.numel(), _ptr(status), _stream(stream)))
    return out


def moe_mxfp8_weights_size(cfg, which: int) -> int:
    """Bytes of the MXFP8 weight blob: which 0 = w13, 1 = w_down."""
    return int(lib().moe_mxfp8_weights_size(ctypes.byref(cfg), which))


def mxfp8_scale_bytes(rows, cols) -> int:
    """Bytes of the scale atoms moe_mxfp8_quantize writes for [rows, cols]."""
    return (cols // 128) * ((rows + 127) // 128) * 512


def moe_mxfp8_quantize(x, q=None, sf=None, counts=None, status=None, stream=None):
    """MXFP8 quantisation of a bf16 matrix [rows, cols] along its rows.
    Returns (q [rows, cols] uint8 E4M3 bytes, sf uint8 scale atoms);
    counts (uint32 [2], may be None) receives the saturated and underflowed
    element counts added."""
    if x.dim() != 2 or x.dtype != torch.bfloat16:
        raise ValueError("x must be a 2-D bf16 tensor")
    rows, cols = x.shape
    dev = _dev(x)
    if q is None:
        q = torch.empty((rows, cols), dtype=torch.uint8, device=dev)
    if sf is None:
        sf = torch.zeros(max(mxfp8_scale_bytes(rows, cols), 1), dtype=torch.uint8, device=dev)
    _check(q, (rows, cols), torch.uint8, "q")
    if sf.numel() < mxfp8_scale_bytes(rows, cols) or sf.dtype != torch.uint8:
        raise ValueError("sf too small")
    if counts is not None and (counts.dtype != torch.int32 or counts.numel() < 2):
        raise ValueError("counts must be int32 with 2 entries (read as uint32)")
    _rc("moe_mxfp8_quantize", lib().moe_mxfp8_quantize(_ptr(x), rows, cols, _ptr(q), _ptr(sf), _ptr(counts),
                                                       _ptr(status), _stream(stream)))
    return q, sf


def moe_pack_weights_mxfp8(cfg, w13_packed, w_down, counts=None, stream=None):
    """Quantise the expert weights for MOE_PRECISION_MXFP8. Returns the two
    uint8 blobs (w13_mx, w_down_mx)."""
    _check(w13_packed, (cfg.E, 2 * cfg.d_ff, cfg.d), torch.bfloat16, "w13_packed")
    _check(w_down, (cfg.E, cfg.d, cfg.d_ff), torch.bfloat16, "w_down")
    dev = _dev(w13_packed)
    a = torch.empty(moe_mxfp8_weights_size(cfg, 0), dtype=torch.uint8, device=dev)
    b = torch.empty(moe_mxfp8_weights_size(cfg, 1), dtype=torch.uint8, device=dev)
    _rc("moe_pack_weights_mxfp8", lib().moe_pack_weights_mxfp8(ctypes.byref(cfg), _ptr(w13_packed), _ptr(w_down),
                                                               _ptr(a), _ptr(b), _ptr(counts), _stream(stream)))
    return a, b


def mx_counters(ws):
    """The four uint32 counters an MXFP8 call leaves at the start of its
    workspace: x saturated, x underflowed, h_mid saturated, h_mid underflowed."""
    return ws[:16].view(torch.int32).cpu().tolist()
