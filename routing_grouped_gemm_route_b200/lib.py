"""Thin ctypes binding of the C ABI in include/moe.h (argument marshalling only).

Every function here has the name of the C entry point it calls, takes torch tensors
(device memory owned by the caller) and the current CUDA stream, and raises
``MoEError`` on a non-zero status.  All arithmetic happens in the CUDA library; if
``libmoe.so`` is missing this module refuses to load rather than fall back to
anything else.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe.so")

MOE_OK, MOE_EINVAL, MOE_EALIGN, MOE_EWORKSPACE, MOE_EUNSUPPORTED, MOE_ECUDA, MOE_EDEVICE = \
    0, -1, -2, -3, -4, -5, -6
MOE_FP32, MOE_BF16, MOE_MXFP8 = 0, 1, 2
MOE_FLAG_ROUTER, MOE_FLAG_DW_FP32, MOE_FLAG_ACCUM_DW, MOE_FLAG_RECOMPUTE = 1, 2, 4, 8
MOE_FLAG_SHARED_EXPERT = 16
MOE_FLAG_MX_KEEP_WEIGHT_CODES = 32       # MXFP8: weight codes of the forward reused
MOE_FLAG_TEST_WAIT_TIMEOUT = 1 << 30      # test hook: the GEMMs' device waits run out
MOE_DEV_BAD_INDEX, MOE_DEV_BAD_OFFSETS, MOE_DEV_TIMEOUT, MOE_DEV_CHECK_FAILED = 1, 2, 4, 8
MOE_ROUTE_NOALLOC_SCRATCH_BYTES = 4 * 1024 * 1024

DTYPES = {"fp32": MOE_FP32, "bf16": MOE_BF16, "mxfp8": MOE_MXFP8}

# Every entry point that include/moe.h declares.
EXPORTS = ["moe_status_string", "moe_check_desc", "moe_workspace_size", "moe_saved_layout_get",
           "moe_workspace_init", "moe_read_device_status", "moe_router_logits", "moe_route",
           "moe_route_noalloc", "moe_mx_scale_bytes", "moe_mx_quantize",
           "moe_dispatch", "moe_grouped_gemm_fwd", "moe_combine", "moe_combine_bwd",
           "moe_grouped_gemm_bwd", "moe_dispatch_bwd", "moe_router_bwd", "moe_load_stats",
           "moe_layer_fwd", "moe_layer_bwd"]


class MoEError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


class moe_desc(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("d_ff", ctypes.c_int32),
                ("E", ctypes.c_int32), ("k", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("flags", ctypes.c_int32), ("capacity", ctypes.c_int32)]


class moe_saved_layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in
                ("topk_idx", "gates", "counts", "offsets", "slot", "row_token", "row_gate",
                 "logits", "x_perm", "H13", "a", "y_perm", "H13_shared", "a_shared",
                 "total")]


class moe_load_stats_t(ctypes.Structure):
    _fields_ = [("total", ctypes.c_int64), ("max_count", ctypes.c_int32),
                ("min_count", ctypes.c_int32), ("num_empty", ctypes.c_int32),
                ("num_experts", ctypes.c_int32), ("mean", ctypes.c_double),
                ("max_over_mean", ctypes.c_double), ("cv", ctypes.c_double)]


_lib = None
_P = ctypes.c_void_p
_S = ctypes.c_size_t
_I = ctypes.c_int32


def load():
    """Load libmoe.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m routing_grouped_gemm_route_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    lib.moe_status_string.restype = ctypes.c_char_p
    lib.moe_status_string.argtypes = [_I]
    sig = {
        "moe_check_desc": [_P],
        "moe_workspace_size": [_P, ctypes.POINTER(_S)],
        "moe_saved_layout_get": [_P, _P],
        "moe_workspace_init": [_P, _S, _P],
        "moe_read_device_status": [_P, _P, ctypes.POINTER(_I)],
        "moe_router_logits": [_P, _P, _P, _P, _P],
        "moe_route": [_P] + [_P] * 8 + [_P, _S, _P],
        "moe_route_noalloc": [_P] + [_P] * 8 + [_P],
        "moe_mx_scale_bytes": [ctypes.c_int64, _I, _I, ctypes.POINTER(_S)],
        "moe_mx_quantize": [_P, ctypes.c_int64, _I, _P, _I, _I, _P, _P, _P, _S, _P],
        "moe_dispatch": [_P, _P, _P, _P, _P, _P, _S, _P],
        "moe_grouped_gemm_fwd": [_P] + [_P] * 8 + [_P, _S, _P],
        "moe_combine": [_P, _P, _P, _P, _P, _P, _S, _P],
        "moe_combine_bwd": [_P] + [_P] * 7 + [_P, _S, _P],
        "moe_grouped_gemm_bwd": [_P] + [_P] * 11 + [_P, _S, _P],
        "moe_dispatch_bwd": [_P, _P, _P, _P, _P, _S, _P],
        "moe_router_bwd": [_P, _P, _P, _P, _P, _P, _P, _S, _P],
        "moe_load_stats": [_P, _I, _P, _P, _P],
        "moe_layer_fwd": [_P, _P, _P, _P, _P, _P, _P, _P, _S, _P, _S, _P],
        "moe_layer_bwd": [_P, _P, _P, _P, _S, _P, _P, _P, _P, _P, _P, _P, _P, _P, _S, _P],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.restype = _I
        fn.argtypes = args
    _lib = lib
    return lib


def status_string(status: int) -> str:
    try:
        return load().moe_status_string(int(status)).decode()
    except Exception:  # noqa: BLE001 - only used to format an error
        return "unknown"


def _ptr(t):
    """Device address of a tensor argument.  The kernels read every buffer as a dense
    row-major array in device memory, so a host tensor (whose address a kernel cannot
    read) or a strided view is refused here, before anything is launched."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("moe: tensor arguments must live in device memory")
    if not t.is_contiguous():
        raise ValueError("moe: tensor arguments must be contiguous (dense row-major)")
    return t.data_ptr()


def _arg(t, dtype, numel, name):
    """_ptr after checking a tensor argument's element type and that it holds at least
    the `numel` elements the call reads or writes: the library sees only the address,
    so a buffer of the wrong type or too short would be misread or overrun."""
    if t is None or isinstance(t, int):
        return _ptr(t)
    if t.dtype != dtype:
        raise ValueError(f"moe: {name} must be {dtype}, got {t.dtype}")
    if t.numel() < numel:
        raise ValueError(f"moe: {name} holds {t.numel()} elements, the call needs {numel}")
    return _ptr(t)


def _dims(desc):
    """(T, d, d_ff, E, k, R, act dtype, dW dtype, weight slices) of a descriptor."""
    act = act_dtype(desc)
    dw = torch.float32 if desc.flags & MOE_FLAG_DW_FP32 else act
    nw = desc.E + (1 if desc.flags & MOE_FLAG_SHARED_EXPERT else 0)
    return desc.T, desc.d, desc.d_ff, desc.E, desc.k, rows_of(desc), act, dw, nw


def _stream(stream=None):
    if stream is None:
        if torch.cuda.is_available():
            return torch.cuda.current_stream().cuda_stream
        return None
    return int(stream) if isinstance(stream, int) else stream.cuda_stream


def _check(st: int, what: str):
    if st != MOE_OK:
        raise MoEError(st, what)


def make_desc(T, d, d_ff, E, k, dtype="bf16", flags=0, capacity=0) -> moe_desc:
    return moe_desc(T, d, d_ff, E, k, DTYPES[dtype] if isinstance(dtype, str) else dtype, flags,
                    capacity)


def rows_of(desc: moe_desc) -> int:
    """Routed rows R: T*k, or E*capacity in the capacity-padded layout (0 without tokens)."""
    if desc.T == 0:
        return 0
    return desc.E * desc.capacity if desc.capacity > 0 else desc.T * desc.k


def act_dtype(desc: moe_desc) -> torch.dtype:
    return torch.float32 if desc.dtype == MOE_FP32 else torch.bfloat16


# ------------------------------------------------------------------------------ sizes
def moe_check_desc(desc) -> int:
    return load().moe_check_desc(ctypes.byref(desc))


def moe_workspace_size(desc) -> int:
    n = _S(0)
    _check(load().moe_workspace_size(ctypes.byref(desc), ctypes.byref(n)), "moe_workspace_size")
    return n.value


def moe_saved_layout_get(desc) -> moe_saved_layout:
    out = moe_saved_layout()
    _check(load().moe_saved_layout_get(ctypes.byref(desc), ctypes.byref(out)),
           "moe_saved_layout_get")
    return out


def moe_workspace_init(ws, stream=None):
    _check(load().moe_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "moe_workspace_init")


def moe_read_device_status(ws, stream=None) -> int:
    bits = _I(0)
    st = load().moe_read_device_status(_ptr(ws), _stream(stream), ctypes.byref(bits))
    if st not in (MOE_OK, MOE_EDEVICE):
        _check(st, "moe_read_device_status")
    return bits.value


def alloc_workspace(desc, device="cuda") -> torch.Tensor:
    """Caller-owned workspace (torch allocation) with its status word cleared."""
    ws = torch.empty(moe_workspace_size(desc), dtype=torch.uint8, device=device)
    moe_workspace_init(ws)
    return ws


def _nbytes(t):
    return t.numel() * t.element_size()


# ------------------------------------------------------------------------------ stages
def moe_router_logits(desc, x, Wr, logits, stream=None):
    T, d, f, E, k, R, act, dw, nw = _dims(desc)
    _check(load().moe_router_logits(ctypes.byref(desc), _arg(x, act, T * d, "x"),
                                    _arg(Wr, act, d * E, "Wr"),
                                    _arg(logits, torch.float32, T * E, "logits"),
                                    _stream(stream)), "moe_router_logits")


def moe_route(desc, logits, topk_idx, gates, counts, offsets, slot, row_token, row_gate, ws,
              stream=None):
    T, d, f, E, k, R, act, dw, nw = _dims(desc)
    i32, f32 = torch.int32, torch.float32
    _check(load().moe_route(ctypes.byref(desc), _arg(logits, f32, T * E, "logits"),
                            _arg(topk_idx, i32, T * k, "topk_idx"), _arg(gates, f32, T * k, "gates"),
                            _arg(counts, i32, E, "counts"), _arg(offsets, i32, E + 1, "offsets"),
                            _arg(slot, i32, T * k, "slot"), _arg(row_token, i32, R, "row_token"),
                            _arg(row_gate, f32, R, "row_gate"), _ptr(ws),
                            _nbytes(ws), _stream(stream)), "moe_route")


def moe_route_noalloc(desc, logits, topk_idx, gates, counts, offsets, slot, row_token, row_gate,
                      stream=None):
    """moe_route for callers that cannot provide a workspace: the scratch lives in a
    fixed static device array inside the library (see include/moe.h)."""
    T, d, f, E, k, R, act, dw, nw = _dims(desc)
    i32, f32 = torch.int32, torch.float32
    _check(load().moe_route_noalloc(ctypes.byref(desc), _arg(logits, f32, T * E, "logits"),
                                    _arg(topk_idx, i32, T * k, "topk_idx"),
                                    _arg(gates, f32, T * k, "gates"), _arg(counts, i32, E, "counts"),
                                    _arg(offsets, i32, E + 1, "offsets"),
                                    _arg(slot, i32, T * k, "slot"),
                                    _arg(row_token, i32, R, "row_token"),
                                    _arg(row_gate, f32, R, "row_gate"), _stream(stream)),
           "moe_route_noalloc")


def moe_mx_scale_bytes(rows, cols, num_segments) -> int:
    n = _S(0)
    _check(load().moe_mx_scale_bytes(rows, cols, num_segments, ctypes.byref(n)),
           "moe_mx_scale_bytes")
    return n.value


def moe_mx_quantize(x, seg_offsets, colwise, codes, scales, ws, stream=None):
    """MXFP8 quantisation of bf16 x [rows, cols] in row segments (see include/moe.h)."""
    rows, cols = x.shape
    nseg = seg_offsets.numel() - 1
    nsf = moe_mx_scale_bytes(rows, cols, nseg)
    _check(load().moe_mx_quantize(_arg(x, torch.bfloat16, rows * cols, "x"), rows, cols,
                                  _arg(seg_offsets, torch.int32, nseg + 1, "seg_offsets"), nseg,
                                  1 if colwise else 0, _arg(codes, torch.uint8, rows * cols, "codes"),
                                  _arg(scales, torch.uint8, nsf, "scales"), _ptr(ws), _nbytes(ws),
                                  _stream(stream)),
           "moe_mx_quantize")


def moe_dispatch(desc, x, slot, x_perm, ws, x_perm_sf=None, stream=None):
    T, d, f, E, k, R, act, dw, nw = _dims(desc)
    _check(load().moe_dispatch(ctypes.byref(desc), _arg(x, act, T * d, "x"),
                               _arg(slot, torch.int32, T * k, "slot"),
                               _arg(x_perm, act, R * d, "x_perm"), _ptr(x_perm_sf), _ptr(ws),
                               _nbytes(ws), _stream(stream)),
           "moe_dispatch")


def moe_grouped_gemm_fwd(desc, x_perm, W13, W2, offsets, H13, a, y_perm, ws, x_perm_sf=None,
                         stream=None):
    T, d, f, E, k, R, act, dw, nw = _dims(desc)
    _check(load().moe_grouped_gemm_fwd(ctypes.byref(desc), _arg(x_perm, act, R * d, "x_perm"),
                                       _ptr(x_perm_sf), _arg(W13, act, E * 2 * f * d, "W13"),
                                       _arg(W2, act, E * d * f, "W2"),
                                       _arg(offsets, torch.int32, E + 1, "offsets"),
                                       _arg(H13, act, R * 2 * f, "H13"), _arg(a, act, R * f, "a"),
                                       _arg(y_perm, act, R * d, "y_perm"), _ptr(ws), _nbytes(ws),
                                       _stream(stream)),
           "moe_grouped_gemm_fwd")


def moe_combine(desc, y_perm, gates, slot, y, ws, stream=None):
    T, d, f, E, k, R, act, dw, nw = _dims(desc)
    _check(load().moe_combine(ctypes.byref(desc), _arg(y_perm, act, R * d, "y_perm"),
                              _arg(gates, torch.float32, T * k, "gates"),
                              _arg(slot, torch.int32, T * k, "slot"), _arg(y, act, T * d, "y"),
                              _ptr(ws), _nbytes(ws), _stream(stream)), "moe_combine")


def moe_combine_bwd(desc, dy, y_perm, gates, topk_idx, slot, dy_perm, d_logits, ws, stream=None):
    T, d, f, E, k, R, act, dw, nw = _dims(desc)
    i32, f32 = torch.int32, torch.float32
    _check(load().moe_combine_bwd(ctypes.byref(desc), _arg(dy, act, T * d, "dy"),
                                  _arg(y_perm, act, R * d, "y_perm"),
                                  _arg(gates, f32, T * k, "gates"),
                                  _arg(topk_idx, i32, T * k, "topk_idx"),
                                  _arg(slot, i32, T * k, "slot"),
                                  _arg(dy_perm, act, R * d, "dy_perm"),
                                  _arg(d_logits, f32, T * E, "d_logits"), _ptr(ws), _nbytes(ws),
                                  _stream(stream)), "moe_combine_bwd")


def moe_grouped_gemm_bwd(desc, dy_perm, x_perm, H13, a, W13, W2, offsets, dH13, dx_perm, dW13,
                         dW2, ws, stream=None):
    T, d, f, E, k, R, act, dw, nw = _dims(desc)
    _check(load().moe_grouped_gemm_bwd(ctypes.byref(desc), _arg(dy_perm, act, R * d, "dy_perm"),
                                       _arg(x_perm, act, R * d, "x_perm"),
                                       _arg(H13, act, R * 2 * f, "H13"), _arg(a, act, R * f, "a"),
                                       _arg(W13, act, E * 2 * f * d, "W13"),
                                       _arg(W2, act, E * d * f, "W2"),
                                       _arg(offsets, torch.int32, E + 1, "offsets"),
                                       _arg(dH13, act, R * 2 * f, "dH13"),
                                       _arg(dx_perm, act, R * d, "dx_perm"),
                                       _arg(dW13, dw, E * 2 * f * d, "dW13"),
                                       _arg(dW2, dw, E * d * f, "dW2"), _ptr(ws), _nbytes(ws),
                                       _stream(stream)), "moe_grouped_gemm_bwd")


def moe_dispatch_bwd(desc, dx_perm, slot, dx, ws, stream=None):
    T, d, f, E, k, R, act, dw, nw = _dims(desc)
    _check(load().moe_dispatch_bwd(ctypes.byref(desc), _arg(dx_perm, act, R * d, "dx_perm"),
                                   _arg(slot, torch.int32, T * k, "slot"),
                                   _arg(dx, act, T * d, "dx"), _ptr(ws), _nbytes(ws),
                                   _stream(stream)), "moe_dispatch_bwd")


def moe_router_bwd(desc, x, Wr, d_logits, dx, dWr, ws, stream=None):
    T, d, f, E, k, R, act, dw, nw = _dims(desc)
    _check(load().moe_router_bwd(ctypes.byref(desc), _arg(x, act, T * d, "x"),
                                 _arg(Wr, act, d * E, "Wr"),
                                 _arg(d_logits, torch.float32, T * E, "d_logits"),
                                 _arg(dx, act, T * d, "dx"), _arg(dWr, act, d * E, "dWr"), _ptr(ws),
                                 _nbytes(ws), _stream(stream)),
           "moe_router_bwd")


LOAD_STATS_BYTES = ctypes.sizeof(moe_load_stats_t)


def moe_load_stats(counts, out, status=None, stream=None):
    """counts: int32 [E] device tensor; out: a device tensor of at least LOAD_STATS_BYTES
    bytes (16-byte aligned) that receives a moe_load_stats_t; status: optional int32
    device word for MOE_DEV_BAD_OFFSETS."""
    if out.numel() * out.element_size() < LOAD_STATS_BYTES:
        raise MoEError(MOE_EWORKSPACE, "moe_load_stats")
    _check(load().moe_load_stats(_arg(counts, torch.int32, 0, "counts"), int(counts.numel()),
                                 _ptr(out), _arg(status, torch.int32, 1, "status"),
                                 _stream(stream)), "moe_load_stats")


def decode_load_stats(out) -> dict:
    """The moe_load_stats_t in `out` (copied to the host) as a dict."""
    raw = bytes(out.detach().cpu().view(torch.uint8)[:LOAD_STATS_BYTES].numpy().tobytes())
    st = moe_load_stats_t.from_buffer_copy(raw)
    return {name: getattr(st, name) for name, _ in moe_load_stats_t._fields_}


def moe_layer_fwd(desc, x, logits, Wr, W13, W2, y, saved, ws, stream=None):
    T, d, f, E, k, R, act, dw, nw = _dims(desc)
    _check(load().moe_layer_fwd(ctypes.byref(desc), _arg(x, act, T * d, "x"),
                                _arg(logits, torch.float32, T * E, "logits"),
                                _arg(Wr, act, d * E, "Wr"), _arg(W13, act, nw * 2 * f * d, "W13"),
                                _arg(W2, act, nw * d * f, "W2"), _arg(y, act, T * d, "y"),
                                _ptr(saved), _nbytes(saved), _ptr(ws), _nbytes(ws),
                                _stream(stream)), "moe_layer_fwd")


def moe_layer_bwd(desc, dy, x, saved, W13, W2, Wr, dx, d_logits, dW13, dW2, dWr, ws, stream=None):
    T, d, f, E, k, R, act, dw, nw = _dims(desc)
    _check(load().moe_layer_bwd(ctypes.byref(desc), _arg(dy, act, T * d, "dy"),
                                _arg(x, act, T * d, "x"), _ptr(saved), _nbytes(saved),
                                _arg(W13, act, nw * 2 * f * d, "W13"),
                                _arg(W2, act, nw * d * f, "W2"), _arg(Wr, act, d * E, "Wr"),
                                _arg(dx, act, T * d, "dx"),
                                _arg(d_logits, torch.float32, T * E, "d_logits"),
                                _arg(dW13, dw, nw * 2 * f * d, "dW13"),
                                _arg(dW2, dw, nw * d * f, "dW2"), _arg(dWr, act, d * E, "dWr"),
                                _ptr(ws), _nbytes(ws), _stream(stream)), "moe_layer_bwd")


# ------------------------------------------------------------------------------ views
def saved_views(desc, saved: torch.Tensor) -> dict:
    """Typed views of the tensors moe_layer_fwd keeps in ``saved``."""
    L = moe_saved_layout_get(desc)
    T, k, E, d, f = desc.T, desc.k, desc.E, desc.d, desc.d_ff
    R = rows_of(desc)
    act = act_dtype(desc)

    def view(off, n, dt, shape):
        es = torch.empty((), dtype=dt).element_size()
        return saved[off:off + n * es].view(dt).view(*shape)

    out = dict(topk_idx=view(L.topk_idx, T * k, torch.int32, (T, k)),
               gates=view(L.gates, T * k, torch.float32, (T, k)),
               counts=view(L.counts, E, torch.int32, (E,)),
               offsets=view(L.offsets, E + 1, torch.int32, (E + 1,)),
               slot=view(L.slot, T * k, torch.int32, (T, k)),
               row_token=view(L.row_token, R, torch.int32, (R,)),
               row_gate=view(L.row_gate, R, torch.float32, (R,)))
    if not desc.flags & MOE_FLAG_RECOMPUTE:     # else the backward recomputes them
        out.update(x_perm=view(L.x_perm, R * d, act, (R, d)),
                   H13=view(L.H13, R * 2 * f, act, (R, 2 * f)),
                   a=view(L.a, R * f, act, (R, f)),
                   y_perm=view(L.y_perm, R * d, act, (R, d)))
        if desc.flags & MOE_FLAG_SHARED_EXPERT:
            out.update(H13_shared=view(L.H13_shared, T * 2 * f, act, (T, 2 * f)),
                       a_shared=view(L.a_shared, T * f, act, (T, f)))
    if desc.flags & MOE_FLAG_ROUTER:
        out["logits"] = view(L.logits, T * E, torch.float32, (T, E))
    return out


class Layer:
    """Convenience holder of one descriptor with its torch-allocated saved buffer and
    workspace; ``fwd``/``bwd`` call moe_layer_fwd / moe_layer_bwd."""

    def __init__(self, desc, device="cuda"):
        self.desc = desc
        self.device = device
        self.saved = torch.empty(moe_saved_layout_get(desc).total, dtype=torch.uint8, device=device)
        self.ws = alloc_workspace(desc, device)

    def fwd(self, x, W13, W2, logits=None, Wr=None, y=None, stream=None):
        if y is None:
            y = torch.empty(self.desc.T, self.desc.d, dtype=act_dtype(self.desc), device=self.device)
        moe_layer_fwd(self.desc, x, logits, Wr, W13, W2, y, self.saved, self.ws, stream)
        return y

    def bwd(self, dy, W13, W2, x=None, Wr=None, out=None, stream=None):
        d = self.desc
        act = act_dtype(d)
        dw_dt = torch.float32 if d.flags & MOE_FLAG_DW_FP32 else act
        nw = d.E + (1 if d.flags & MOE_FLAG_SHARED_EXPERT else 0)   # weight slices
        if out is None:
            out = dict(dx=torch.empty(d.T, d.d, dtype=act, device=self.device),
                       d_logits=torch.empty(d.T, d.E, dtype=torch.float32, device=self.device),
                       dW13=torch.empty(nw, 2 * d.d_ff, d.d, dtype=dw_dt, device=self.device),
                       dW2=torch.empty(nw, d.d, d.d_ff, dtype=dw_dt, device=self.device),
                       dWr=(torch.empty(d.d, d.E, dtype=act, device=self.device)
                            if d.flags & MOE_FLAG_ROUTER else None))
        moe_layer_bwd(d, dy, x, self.saved, W13, W2, Wr, out["dx"], out["d_logits"], out["dW13"],
                      out["dW2"], out.get("dWr"), self.ws, stream)
        return out

    def views(self) -> dict:
        return saved_views(self.desc, self.saved)
