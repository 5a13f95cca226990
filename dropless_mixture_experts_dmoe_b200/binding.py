"""Thin ctypes binding of libdmoe.so (declared in include/dmoe.h).

Argument marshalling only: every step of the layer runs in the library's CUDA kernels.
PyTorch is used for device memory and streams.  There is no fallback: if the library is
missing or the device is not a B200 the calls raise.

The functions carry the C names (``dmoe_sparse_map``, ``dmoe_forward``, ``dmoe_backward`` and
the step entry points) and take torch tensors where the C call takes device pointers.
"""
from __future__ import annotations

import ctypes
import os

import torch

from .build import LIB

BLOCKING = 128
MAX_EXPERTS = 1024
MAX_TOP_K = 32

WS_MAP, WS_FORWARD, WS_BACKWARD, WS_FORWARD_TRAIN, WS_ROUTER_BACKWARD = 0, 1, 2, 3, 4
DGLU_TILE_COLS = 128

STATUS_NONFINITE_LOGITS = 0x1
STATUS_EXPERT_OUT_OF_RANGE = 0x2
STATUS_DUPLICATE_EXPERT = 0x4
STATUS_TIMEOUT = 0x8

_P = ctypes.c_void_p
_SZ = ctypes.c_size_t
_I = ctypes.c_int


ROUTE_RENORMALIZE = 0x1
ROUTE_TOKEN_ROUNDING = 0x2
SAVE_X_ONLY = 0x4
FUSED_COMBINE = 0x8
SCALE_COLS = 128  # block floating point of Y_pad / dX_pad: one scale per row and 128 columns


def scale_stride(h: int) -> int:
    """Row stride of the scale arrays: ceil(h/128) scales padded to a multiple of 4."""
    return (h + 511) // 512 * 4


class dmoe_dims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("hidden", ctypes.c_int32), ("ffn", ctypes.c_int32),
                ("num_experts", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("flags", ctypes.c_int32)]

    def __repr__(self):
        return (f"dmoe_dims(T={self.T}, hidden={self.hidden}, ffn={self.ffn}, "
                f"num_experts={self.num_experts}, top_k={self.top_k}, "
                f"flags={self.flags})")


MAP_FIELDS = ("top_experts", "weights", "tokens_per_expert", "bins", "padded_bins", "indices",
              "bin_ids", "dest_row", "block_expert", "num_blocks", "status", "entry_offsets")


class dmoe_map(ctypes.Structure):
    _fields_ = [(n, _P) for n in MAP_FIELDS]


class DMoEError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {error_string(code)} ({code})")
        self.code = code


_lib = None


def load():
    """Load the in-tree libdmoe.so (build it first with ``build.build()``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB):
        raise ImportError(f"libdmoe.so not built: {LIB} is missing "
                          "(run python -m dropless_mixture_experts_dmoe_b200.build)")
    lib = ctypes.CDLL(LIB)
    D = ctypes.POINTER(dmoe_dims)
    M = ctypes.POINTER(dmoe_map)
    lib.dmoe_padded_rows_max.argtypes = [D]
    lib.dmoe_padded_rows_max.restype = _SZ
    lib.dmoe_entries_max.argtypes = [D]
    lib.dmoe_entries_max.restype = _SZ
    lib.dmoe_workspace_bytes.argtypes = [D, _I]
    lib.dmoe_workspace_bytes.restype = _SZ
    lib.dmoe_saved_bytes.argtypes = [D, ctypes.POINTER(_SZ)]
    lib.dmoe_saved_bytes.restype = _SZ
    lib.dmoe_sparse_map.argtypes = [D, _P, M, _P, _SZ, _P]
    lib.dmoe_forward.argtypes = [D, _P, _P, _P, _P, M, _P, _P, _P, _SZ, _P]
    lib.dmoe_backward.argtypes = [D, _P, _P, _P, _P, M, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]
    lib.dmoe_padded_gather.argtypes = [D, _P, M, _P, _P]
    lib.dmoe_expert_glu.argtypes = [D, _P, _P, _P, M, _P, _P, _P, _P]
    lib.dmoe_expert_glu_gather.argtypes = [D, _P, _P, _P, M, _P, _P, _P, _P]
    lib.dmoe_expert_down.argtypes = [D, _P, _P, M, _P, _P, _P]
    lib.dmoe_padded_scatter.argtypes = [D, _P, _P, M, _P, _P, _P]
    lib.dmoe_expert_down_combine.argtypes = [D, _P, _P, M, _P, _P, _P]
    lib.dmoe_bwd_dglu.argtypes = [D, _P, _P, _P, _P, M, _P, _P, _P, _P, _P]
    lib.dmoe_bwd_scatter.argtypes = [D, _P, _P, _P, M, _P, _P, _P]
    lib.dmoe_router_forward.argtypes = [D, _P, _P, _P, _P, _P]
    lib.dmoe_router_dlogits.argtypes = [D, _P, M, _P, _P, _P]
    lib.dmoe_router_backward.argtypes = [D, _P, _P, _P, M, _P, _P, _P, _P, _SZ, _P]
    lib.dmoe_bwd_dx.argtypes = [D, _P, _P, _P, _P, M, _P, _P, _P]
    lib.dmoe_bwd_wgrad.argtypes = [D, _P, _P, _P, _P, _P, M, _P, _P, _P, _P]
    lib.dmoe_sparse_map_noalloc.argtypes = [D, _P, M, _P]
    for fn in ("dmoe_sparse_map", "dmoe_sparse_map_noalloc", "dmoe_forward", "dmoe_backward",
               "dmoe_padded_gather",
               "dmoe_expert_glu", "dmoe_expert_glu_gather", "dmoe_expert_down", "dmoe_padded_scatter",
               "dmoe_expert_down_combine",
               "dmoe_bwd_dglu", "dmoe_bwd_dx", "dmoe_bwd_wgrad", "dmoe_bwd_scatter",
               "dmoe_router_forward", "dmoe_router_dlogits", "dmoe_router_backward"):
        getattr(lib, fn).restype = _I
    lib.dmoe_error_string.argtypes = [_I]
    lib.dmoe_error_string.restype = ctypes.c_char_p
    lib.dmoe_status_string.argtypes = [ctypes.c_int32]
    lib.dmoe_status_string.restype = ctypes.c_char_p
    lib.dmoe_version.argtypes = []
    lib.dmoe_version.restype = ctypes.c_char_p
    lib.dmoe_debug_inject_stall.argtypes = [_I]
    lib.dmoe_debug_inject_stall.restype = _I
    _lib = lib
    return lib


def error_string(code: int) -> str:
    return load().dmoe_error_string(code).decode()


def status_string(status: int) -> str:
    return load().dmoe_status_string(int(status)).decode()


def version() -> str:
    return load().dmoe_version().decode()


def dmoe_debug_inject_stall(enable: bool = True) -> None:
    """Test-only: the next grouped-GEMM launch stalls on purpose and reports
    STATUS_TIMEOUT (see include/dmoe.h)."""
    _check(load().dmoe_debug_inject_stall(1 if enable else 0), "dmoe_debug_inject_stall")


def make_dims(T: int, hidden: int, ffn: int, num_experts: int, top_k: int,
              flags: int = 0) -> dmoe_dims:
    """flags: an OR of ROUTE_RENORMALIZE (weights = softmax over the k chosen logits) and
    SAVE_X_ONLY (the forward saves X_pad only; the backward recomputes A and Bm)."""
    return dmoe_dims(T, hidden, ffn, num_experts, top_k, flags)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, what: str):
    if rc != 0:
        raise DMoEError(rc, what)


# ---- sizes ------------------------------------------------------------------------------------

def dmoe_padded_rows_max(dims: dmoe_dims) -> int:
    return int(load().dmoe_padded_rows_max(ctypes.byref(dims)))


def dmoe_entries_max(dims: dmoe_dims) -> int:
    return int(load().dmoe_entries_max(ctypes.byref(dims)))


def dmoe_workspace_bytes(dims: dmoe_dims, kind: int) -> int:
    return int(load().dmoe_workspace_bytes(ctypes.byref(dims), kind))


def dmoe_saved_bytes(dims: dmoe_dims):
    offs = (_SZ * 3)()
    total = int(load().dmoe_saved_bytes(ctypes.byref(dims), offs))
    return total, [int(o) for o in offs]


# ---- the sparse map -----------------------------------------------------------------------------

class SparseMap:
    """Device tensors of the sparse map (torch allocations) and their C view."""

    def __init__(self, dims: dmoe_dims, device="cuda"):
        T, E, k = dims.T, dims.num_experts, dims.top_k
        P = dmoe_padded_rows_max(dims)
        if P == 0:
            raise DMoEError(-2, "SparseMap")
        i32 = dict(dtype=torch.int32, device=device)
        self.dims = dims
        rounding = bool(dims.flags & ROUTE_TOKEN_ROUNDING)
        N = dmoe_entries_max(dims)
        if rounding:  # experts and weights of the token-major entry list
            self.top_experts = torch.empty(N, **i32)
            self.weights = torch.empty(N, dtype=torch.float32, device=device)
        else:
            self.top_experts = torch.empty((T, k), **i32)
            self.weights = torch.empty((T, k), dtype=torch.float32, device=device)
        self.tokens_per_expert = torch.empty(E, **i32)
        self.bins = torch.empty(E, **i32)
        self.padded_bins = torch.empty(E, **i32)
        self.indices = torch.empty(N, **i32)
        self.bin_ids = torch.empty(N, **i32)
        self.dest_row = torch.empty(N, **i32)
        self.block_expert = torch.empty(max(P // BLOCKING, 1), **i32)
        self.num_blocks = torch.empty(1, **i32)
        self.status = torch.zeros(1, **i32)
        # token rounding: a token-major entry list (see include/dmoe.h)
        self.entry_offsets = torch.empty(T + 1, **i32) if rounding else None
        self._c = dmoe_map(*[0 if getattr(self, n) is None else getattr(self, n).data_ptr()
                             for n in MAP_FIELDS])

    @property
    def c(self) -> dmoe_map:
        return self._c

    def as_dict(self) -> dict:
        return {n: getattr(self, n) for n in MAP_FIELDS if getattr(self, n) is not None}


def dmoe_sparse_map(dims: dmoe_dims, logits, smap: SparseMap, ws, stream=None):
    """Routing + sparse map.  logits: [T,E] bf16 CUDA tensor or None (top_experts given)."""
    ws_bytes = ws.numel() * ws.element_size()
    rc = load().dmoe_sparse_map(ctypes.byref(dims), _ptr(logits), ctypes.byref(smap.c), _ptr(ws),
                                ws_bytes, _stream(stream))
    _check(rc, "dmoe_sparse_map")


def dmoe_forward(dims: dmoe_dims, x, w1, w3, w2, smap: SparseMap, y, saved=None, ws=None,
                 stream=None):
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    rc = load().dmoe_forward(ctypes.byref(dims), _ptr(x), _ptr(w1), _ptr(w3), _ptr(w2),
                             ctypes.byref(smap.c), _ptr(y), _ptr(saved), _ptr(ws), ws_bytes,
                             _stream(stream))
    _check(rc, "dmoe_forward")


def dmoe_backward(dims: dmoe_dims, dy, w1, w3, w2, smap: SparseMap, saved, dx, dw1, dw3, dw2,
                  dweights, ws, stream=None):
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    rc = load().dmoe_backward(ctypes.byref(dims), _ptr(dy), _ptr(w1), _ptr(w3), _ptr(w2),
                              ctypes.byref(smap.c), _ptr(saved), _ptr(dx), _ptr(dw1), _ptr(dw3),
                              _ptr(dw2), _ptr(dweights), _ptr(ws), ws_bytes, _stream(stream))
    _check(rc, "dmoe_backward")


def dmoe_padded_gather(dims, x, smap: SparseMap, x_pad, stream=None):
    _check(load().dmoe_padded_gather(ctypes.byref(dims), _ptr(x), ctypes.byref(smap.c), _ptr(x_pad),
                                     _stream(stream)), "dmoe_padded_gather")


def dmoe_expert_glu(dims, x_pad, w1, w3, smap: SparseMap, h_out, a_out=None, b_out=None,
                    stream=None):
    _check(load().dmoe_expert_glu(ctypes.byref(dims), _ptr(x_pad), _ptr(w1), _ptr(w3),
                                  ctypes.byref(smap.c), _ptr(h_out), _ptr(a_out), _ptr(b_out),
                                  _stream(stream)), "dmoe_expert_glu")


def dmoe_expert_glu_gather(dims, x, w1, w3, smap: SparseMap, h_out, a_out=None, b_out=None,
                           stream=None):
    _check(load().dmoe_expert_glu_gather(ctypes.byref(dims), _ptr(x), _ptr(w1), _ptr(w3),
                                         ctypes.byref(smap.c), _ptr(h_out), _ptr(a_out),
                                         _ptr(b_out), _stream(stream)), "dmoe_expert_glu_gather")


def dmoe_expert_down(dims, h_in, w2, smap: SparseMap, y_pad, y_scale, stream=None):
    """y_pad [P_max,h] fp16 and y_scale [P_max, scale_stride(h)] fp32: block floating point."""
    _check(load().dmoe_expert_down(ctypes.byref(dims), _ptr(h_in), _ptr(w2), ctypes.byref(smap.c),
                                   _ptr(y_pad), _ptr(y_scale), _stream(stream)), "dmoe_expert_down")


def dmoe_expert_down_combine(dims, h_in, w2, smap: SparseMap, y, y_acc, stream=None):
    """y = the weighted combine of the down GEMM, fused (y_acc: T*h fp32 workspace)."""
    _check(load().dmoe_expert_down_combine(ctypes.byref(dims), _ptr(h_in), _ptr(w2),
                                           ctypes.byref(smap.c), _ptr(y), _ptr(y_acc),
                                           _stream(stream)), "dmoe_expert_down_combine")


def dmoe_padded_scatter(dims, y_pad, y_scale, smap: SparseMap, weights, y, stream=None):
    """y_scale None: y_pad is bf16; else block floating point (fp16 y_pad and its scales)."""
    _check(load().dmoe_padded_scatter(ctypes.byref(dims), _ptr(y_pad), _ptr(y_scale),
                                      ctypes.byref(smap.c), _ptr(weights), _ptr(y),
                                      _stream(stream)), "dmoe_padded_scatter")


def dmoe_bwd_dglu(dims, dy_pad, w2, a_saved, bm_saved, smap: SparseMap, da, dbm, hw, dw_part,
                  stream=None):
    _check(load().dmoe_bwd_dglu(ctypes.byref(dims), _ptr(dy_pad), _ptr(w2), _ptr(a_saved),
                                _ptr(bm_saved), ctypes.byref(smap.c), _ptr(da), _ptr(dbm),
                                _ptr(hw), _ptr(dw_part), _stream(stream)), "dmoe_bwd_dglu")


def dmoe_bwd_scatter(dims, dx_pad, dx_scale, dw_part, smap: SparseMap, dx, dweights,
                     stream=None):
    _check(load().dmoe_bwd_scatter(ctypes.byref(dims), _ptr(dx_pad), _ptr(dx_scale),
                                   _ptr(dw_part), ctypes.byref(smap.c), _ptr(dx), _ptr(dweights),
                                   _stream(stream)), "dmoe_bwd_scatter")


def dmoe_bwd_dx(dims, da, dbm, w1, w3, smap: SparseMap, dx_pad, dx_scale, stream=None):
    """dx_pad [P_max,h] fp16 and dx_scale [P_max, scale_stride(h)] fp32: block floating point."""
    _check(load().dmoe_bwd_dx(ctypes.byref(dims), _ptr(da), _ptr(dbm), _ptr(w1), _ptr(w3),
                              ctypes.byref(smap.c), _ptr(dx_pad), _ptr(dx_scale),
                              _stream(stream)), "dmoe_bwd_dx")


def dmoe_bwd_wgrad(dims, x_pad, hw, dy_pad, da, dbm, smap: SparseMap, dw1, dw3, dw2,
                   stream=None):
    _check(load().dmoe_bwd_wgrad(ctypes.byref(dims), _ptr(x_pad), _ptr(hw), _ptr(dy_pad),
                                 _ptr(da), _ptr(dbm), ctypes.byref(smap.c), _ptr(dw1), _ptr(dw3),
                                 _ptr(dw2), _stream(stream)), "dmoe_bwd_wgrad")


def dmoe_router_forward(dims, x, w_router, logits, status, stream=None):
    """logits [T,E] bf16 = x W_r^T (the linear router; E % 8 == 0)."""
    _check(load().dmoe_router_forward(ctypes.byref(dims), _ptr(x), _ptr(w_router), _ptr(logits),
                                      _ptr(status), _stream(stream)), "dmoe_router_forward")


def dmoe_router_dlogits(dims, logits, smap: SparseMap, dweights, dlogits, stream=None):
    _check(load().dmoe_router_dlogits(ctypes.byref(dims), _ptr(logits), ctypes.byref(smap.c),
                                      _ptr(dweights), _ptr(dlogits), _stream(stream)),
           "dmoe_router_dlogits")


def dmoe_router_backward(dims, x, w_router, logits, smap: SparseMap, dweights, dx, dw_router, ws,
                         stream=None):
    """dx += dlogits W_r (in place), dw_router = dlogits^T x (fp32)."""
    ws_bytes = ws.numel() * ws.element_size()
    _check(load().dmoe_router_backward(ctypes.byref(dims), _ptr(x), _ptr(w_router), _ptr(logits),
                                       ctypes.byref(smap.c), _ptr(dweights), _ptr(dx),
                                       _ptr(dw_router), _ptr(ws), ws_bytes, _stream(stream)),
           "dmoe_router_backward")


def dmoe_sparse_map_noalloc(dims: dmoe_dims, logits, smap: SparseMap, stream=None):
    """Allocation-free routing + sparse map (static scratch inside the library; see
    include/dmoe.h).  For callers that cannot allocate a workspace."""
    _check(load().dmoe_sparse_map_noalloc(ctypes.byref(dims), _ptr(logits),
                                          ctypes.byref(smap.c), _stream(stream)),
           "dmoe_sparse_map_noalloc")


# ---- buffers (allocation only) ----------------------------------------------------------------

class Buffers:
    """Caller-side device allocations for one layer shape: map, workspaces, saved activations.

    train=True: ``saved`` (X_pad, A, Bm for the backward), the training forward workspace
    ``ws_fwd`` (H, Y_pad and its scales), the backward workspace, and separate step buffers
    ``bstep`` (dy_pad, da, dbm, hw, dw_part, dx_pad, dx_scale) for driving the backward step
    entry points one by one.  train=False: the inference workspace of ``dmoe_forward`` plus
    separate X_pad / H / Y_pad / Y_pad-scale tensors (``step``) for the forward step entry
    points.  ``view(name)`` gives [P_max, cols] views: x_pad, a, bm (bf16) of the saved buffer,
    and h (bf16), y_pad (fp16) and y_scale (fp32) of the forward workspace (valid until the
    workspace is reused)."""

    def __init__(self, dims: dmoe_dims, train: bool = False, device="cuda"):
        self.dims = dims
        self.P = dmoe_padded_rows_max(dims)
        self.map = SparseMap(dims, device)
        u8 = dict(dtype=torch.uint8, device=device)
        self.ws_map = torch.empty(max(dmoe_workspace_bytes(dims, WS_MAP), 16), **u8)
        self.train = train
        P, h, f = self.P, dims.hidden, dims.ffn
        nsc = scale_stride(h)
        bf = dict(dtype=torch.bfloat16, device=device)
        f32 = dict(dtype=torch.float32, device=device)
        self.saved = self.ws_bwd = None
        self.step = {}
        if train:
            total, offs = dmoe_saved_bytes(dims)
            self.saved = torch.empty(total, **u8)
            self.offsets = dict(x_pad=offs[0], a=offs[1], bm=offs[2])
            if dims.flags & SAVE_X_ONLY:  # A and Bm are not saved
                del self.offsets["a"], self.offsets["bm"]
            self.ws_fwd = torch.empty(dmoe_workspace_bytes(dims, WS_FORWARD_TRAIN), **u8)
            self.ws_bwd = torch.empty(max(dmoe_workspace_bytes(dims, WS_BACKWARD), 16), **u8)
            nt = (f + DGLU_TILE_COLS - 1) // DGLU_TILE_COLS
            self.bstep = dict(dy_pad=torch.empty((P, h), **bf), da=torch.empty((P, f), **bf),
                              dbm=torch.empty((P, f), **bf), hw=torch.empty((P, f), **bf),
                              dw_part=torch.empty((P, nt), **f32),
                              dx_pad=torch.empty((P, h), dtype=torch.float16, device=device),
                              dx_scale=torch.empty((P, nsc), **f32))
        else:
            self.ws_fwd = torch.empty(dmoe_workspace_bytes(dims, WS_FORWARD), **u8)
            self.step = dict(x_pad=torch.empty((P, h), **bf), h=torch.empty((P, f), **bf),
                             y_pad=torch.empty((P, h), dtype=torch.float16, device=device),
                             y_scale=torch.empty((P, nsc), **f32),
                             y_acc=torch.empty((dims.T, h), **f32))

    def view(self, name: str) -> torch.Tensor:
        """[P, cols] view of a saved activation (x_pad, a, bm) or, after a training forward,
        of its workspace (h, y_pad, y_scale)."""
        if not self.train:
            return self.step[name]
        P, h, f = self.P, self.dims.hidden, self.dims.ffn
        if name in self.offsets:
            cols = h if name == "x_pad" else f
            off = self.offsets[name]
            return self.saved[off:off + P * cols * 2].view(torch.bfloat16).view(P, cols)
        # forward workspace layout: H [P,f] bf16 | Y_pad [P,h] fp16 | scales [P, scale_stride(h)]
        # fp32, each start aligned to 256 bytes
        up = lambda v: (v + 255) // 256 * 256
        nsc = scale_stride(h)
        o_y = up(P * f * 2)
        o_s = up(o_y + P * h * 2)
        if name == "h":
            return self.ws_fwd[:P * f * 2].view(torch.bfloat16).view(P, f)
        if name == "y_acc" and self.dims.flags & FUSED_COMBINE:  # [T,h] fp32 after H
            T = self.dims.T
            return self.ws_fwd[o_y:o_y + T * h * 4].view(torch.float32).view(T, h)
        if name == "y_pad":
            return self.ws_fwd[o_y:o_y + P * h * 2].view(torch.float16).view(P, h)
        if name == "y_scale":
            return self.ws_fwd[o_s:o_s + P * nsc * 4].view(torch.float32).view(P, nsc)
        raise KeyError(f"{name} is not saved with these flags")
