"""The dMoE layer as a ``torch.autograd.Function`` over the three layer calls of the C ABI.

Forward: ``dmoe_sparse_map`` (routing from the logits) and ``dmoe_forward``, which keeps X_pad
and the two GEMM1 pre-activations for the backward.  Backward: ``dmoe_backward`` (dx, dW1, dW3,
dW2 and the gradient of every routing weight) and, when the logits need a gradient,
``dmoe_router_dlogits`` (through the softmax that produced the weights).  Every step runs in
libdmoe.so; this module only allocates the buffers and orders the calls on the current stream.

Inputs: x [T, hidden] and logits [T, E] bf16, W1 and W3 [E, ffn, hidden] and W2
[E, hidden, ffn] bf16, all contiguous CUDA tensors.  The weight gradients are computed in fp32
and handed to autograd, which stores them in the weights' dtype.  A logit gradient needs
E % 8 == 0.  Device-side conditions (non-finite logits, a bounded wait that gave up) are left
in ``last_status()``'s word, which a caller may read after synchronising.
"""
from __future__ import annotations

import torch

from . import binding as B

_last_map = None


def last_status() -> int:
    """Status word of the most recent forward's sparse map (synchronises the device)."""
    return 0 if _last_map is None else int(_last_map.status.item())


def _check_inputs(x, logits, w1, w3, w2):
    for name, t in (("x", x), ("logits", logits), ("w1", w1), ("w3", w3), ("w2", w2)):
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
    T, h = x.shape
    E, f, h1 = w1.shape
    if logits.shape != (T, E) or h1 != h or w3.shape != w1.shape or w2.shape != (E, h, f):
        raise ValueError("shapes: x [T,h], logits [T,E], w1/w3 [E,f,h], w2 [E,h,f]")
    return T, h, f, E


class DMoEFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, logits, w1, w3, w2, top_k: int, flags: int = 0):
        global _last_map
        T, h, f, E = _check_inputs(x, logits, w1, w3, w2)
        dims = B.make_dims(T, h, f, E, top_k, flags=flags)
        dev = x.device
        u8 = dict(dtype=torch.uint8, device=dev)
        smap = B.SparseMap(dims, dev)
        ws_map = torch.empty(max(B.dmoe_workspace_bytes(dims, B.WS_MAP), 16), **u8)
        saved_bytes, _ = B.dmoe_saved_bytes(dims)
        saved = torch.empty(saved_bytes, **u8)
        ws_fwd = torch.empty(B.dmoe_workspace_bytes(dims, B.WS_FORWARD_TRAIN), **u8)
        y = torch.empty_like(x)
        B.dmoe_sparse_map(dims, logits, smap, ws_map)
        B.dmoe_forward(dims, x, w1, w3, w2, smap, y, saved=saved, ws=ws_fwd)
        ctx.save_for_backward(logits, w1, w3, w2)
        ctx.dims, ctx.smap, ctx.saved_act = dims, smap, saved
        _last_map = smap
        return y

    @staticmethod
    def backward(ctx, dy):
        logits, w1, w3, w2 = ctx.saved_tensors
        dims, smap = ctx.dims, ctx.smap
        dy = dy.to(torch.bfloat16).contiguous()
        dev = dy.device
        f32 = dict(dtype=torch.float32, device=dev)
        dx = torch.empty_like(dy)
        dw1 = torch.empty(w1.shape, **f32)
        dw3 = torch.empty(w3.shape, **f32)
        dw2 = torch.empty(w2.shape, **f32)
        rounded = bool(dims.flags & B.ROUTE_TOKEN_ROUNDING)  # one weight per listed entry
        dweights = torch.empty(B.dmoe_entries_max(dims) if rounded else (dims.T, dims.top_k), **f32)
        ws_bwd = torch.empty(max(B.dmoe_workspace_bytes(dims, B.WS_BACKWARD), 16),
                             dtype=torch.uint8, device=dev)
        B.dmoe_backward(dims, dy, w1, w3, w2, smap, ctx.saved_act, dx, dw1, dw3, dw2, dweights,
                        ws_bwd)
        dlogits = None
        if ctx.needs_input_grad[1]:
            if rounded:
                raise NotImplementedError("the logit gradient of the token-rounded routing is "
                                          "not provided")
            dlogits = torch.empty_like(logits)
            B.dmoe_router_dlogits(dims, logits, smap, dweights, dlogits)
        return dx, dlogits, dw1, dw3, dw2, None, None


def dmoe(x, logits, w1, w3, w2, top_k: int, flags: int = 0):
    """y = dMoE(x) with the experts chosen by the top-k of softmax(logits); differentiable in
    x, logits, W1, W3 and W2."""
    return DMoEFunction.apply(x, logits, w1, w3, w2, top_k, flags)
