"""Parity of the linear router: the logits GEMM, the gradient through the softmax routing
weights (dlogits), dx += dlogits W_r and the split-K router weight gradient, against the
oracle.  The routing decision is taken on the same bf16 logits on both sides."""
import numpy as np
import pytest
import torch

import bf16_model
import oracle
from dropless_mixture_experts_dmoe_b200 import binding as B
from dropless_mixture_experts_dmoe_b200.workloads import custom, make_inputs

from helpers import assert_close, dims_of, sample_tokens, to_np


def assert_increment_close(got_total, base, ref_inc, what):
    """The router adds its dx increment to the experts' dx in fp32 and rounds the total once
    to bf16, so the increment read back as total - base carries that rounding: up to half a
    bf16 ulp of the total, which can be far above the increment's own size.  Each element must
    be within that plus 5e-2 of the increment's RMS, and the relative L2 error within 1e-2."""
    inc = got_total - base
    rms = float(np.sqrt(np.mean(ref_inc * ref_inc)))
    bound = 2.0 ** -8 * np.abs(got_total) + 5e-2 * rms
    assert (np.abs(inc - ref_inc) <= bound).all(), what
    rel = float(np.linalg.norm(inc - ref_inc) / np.linalg.norm(ref_inc))
    assert rel <= 1e-2, f"{what}: relative L2 {rel:.3e}"

pytestmark = pytest.mark.gpu

SMALL = [
    custom(256, 128, 128, 8, 2),      # E = 8: narrower than one 64-column box
    custom(300, 384, 128, 64, 8),     # ragged T (not a multiple of 128), ragged 256-column tile
    custom(1000, 256, 256, 32, 4),
    custom(129, 128, 128, 1024, 8),   # the largest E: four 256-column tiles, a 1-row tail
]


def _forward_backward(w, flags=0):
    """Router forward, map, expert forward + backward, router backward, all on the GPU."""
    inp = make_inputs(w, with_dy=True, with_router=True)
    dims = B.make_dims(w.T, w.hidden, w.ffn, w.E, w.top_k, flags=flags)
    dev = {k: v.cuda() for k, v in inp.items()}
    bufs = B.Buffers(dims, train=True)
    bf = dict(dtype=torch.bfloat16, device="cuda")
    f32 = dict(dtype=torch.float32, device="cuda")
    logits = torch.empty((w.T, w.E), **bf)
    rstatus = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.dmoe_router_forward(dims, dev["x"], dev["w_router"], logits, rstatus)
    B.dmoe_sparse_map(dims, logits, bufs.map, bufs.ws_map)
    y = torch.empty((w.T, w.hidden), **bf)
    B.dmoe_forward(dims, dev["x"], dev["w1"], dev["w3"], dev["w2"], bufs.map, y,
                   saved=bufs.saved, ws=bufs.ws_fwd)
    g = dict(dx=torch.empty((w.T, w.hidden), **bf), dw1=torch.empty((w.E, w.ffn, w.hidden), **f32),
             dw3=torch.empty((w.E, w.ffn, w.hidden), **f32),
             dw2=torch.empty((w.E, w.hidden, w.ffn), **f32), dw=torch.empty((w.T, w.top_k), **f32))
    B.dmoe_backward(dims, dev["dy"], dev["w1"], dev["w3"], dev["w2"], bufs.map, bufs.saved,
                    g["dx"], g["dw1"], g["dw3"], g["dw2"], g["dw"], bufs.ws_bwd)
    dx_experts = g["dx"].clone()
    dwr = torch.full((w.E, w.hidden), float("nan"), **f32)
    ws = torch.empty(B.dmoe_workspace_bytes(dims, B.WS_ROUTER_BACKWARD), dtype=torch.uint8,
                     device="cuda")
    B.dmoe_router_backward(dims, dev["x"], dev["w_router"], logits, bufs.map, g["dw"], g["dx"],
                           dwr, ws)
    torch.cuda.synchronize()
    assert int(rstatus.item()) == 0 and int(bufs.map.status.item()) == 0
    return inp, dims, dev, bufs, logits, g, dx_experts, dwr, ws


THIN = [  # thin routers (E <= 32): logits GEMMs whose 256-column tile is mostly padding
    custom(4096, 4096, 128, 8, 2),    # the Mixtral-shaped router (its ffn plays no part; sampled rows)
    custom(1000, 128, 128, 16, 4),
    custom(333, 640, 128, 24, 4),     # E not a power of two, a ragged last row tile
    custom(77, 8192, 128, 32, 8),     # long K (128 steps of 64), one partial row tile
    custom(3, 384, 128, 8, 2),        # three tokens: a tile of almost only zero-filled rows
]


@pytest.mark.parametrize("w", SMALL + THIN + [custom(4096, 2048, 512, 256, 8)],
                         ids=lambda w: w.describe())
def test_router_logits_parity(w):
    inp = make_inputs(w, with_router=True)
    dims = dims_of(w)
    logits = torch.full((w.T, w.E), float("nan"), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.dmoe_router_forward(dims, inp["x"].cuda(), inp["w_router"].cuda(), logits, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    toks = None if w.T <= 1024 else sample_tokens(np.zeros((w.T, 1), np.int32), 1, 256, seed=3)
    ref = oracle.router_logits(inp["x"].float().numpy(), inp["w_router"].float().numpy(),
                               tokens=toks, threads=oracle.max_threads())
    got = to_np(logits) if toks is None else to_np(logits)[toks]
    rms = float(np.sqrt(np.mean(ref * ref)))
    # one bf16 rounding of an fp32-accumulated dot product
    assert (np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-4 * rms).all()


@pytest.mark.parametrize("renorm", [False, True], ids=["softmax", "renormalised"])
@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.describe())
def test_router_backward_full_chain_parity(w, renorm):
    """x -> router -> map -> experts -> loss, backward into x, W_r (and the experts); both
    routing variants."""
    flags = B.ROUTE_RENORMALIZE if renorm else 0
    inp, dims, dev, bufs, logits, g, dx_experts, dwr, _ = _forward_backward(w, flags)
    o = {k: v.float().numpy() for k, v in inp.items()}
    lg = logits.float().cpu().numpy()  # the routed scores (bf16, widened exactly)
    top, wts = oracle.route(lg, w.top_k, renorm=renorm)
    assert (bufs.map.top_experts.cpu().numpy() == top).all()
    ref = oracle.backward(o["x"], o["dy"], o["w1"], o["w3"], o["w2"], top, wts)
    r = oracle.router_backward(o["x"], o["w_router"], lg, top, ref["dw"],
                               threads=oracle.max_threads(), renorm=renorm)
    tol = bf16_model.bounds(bf16_model.backward_model(inp, top, wts), ref)["dx"]
    assert_close(to_np(g["dx"]), ref["dx"] + r["dx_r"], f"dx {w.describe()}",
                 max_abs_rms=max(tol, 5e-2))
    # the modelled pipeline: the layer's routing-weight gradients as the bf16 model gives them,
    # through the router's softmax gradient, rounded to bf16, times x
    mdw = bf16_model.backward_model(inp, top, wts)["dw"]
    rm = oracle.router_backward(o["x"], o["w_router"], lg, top, mdw, want_dx=False,
                                want_dwr=False, renorm=renorm)
    dwr_tol = bf16_model.bounds({"dWr": bf16_model.router_wgrad_model(rm["dlogits"], inp["x"])},
                                {"dWr": r["dWr"]})["dWr"]
    assert_close(to_np(dwr), r["dWr"], f"dW_r {w.describe()}", max_abs_rms=dwr_tol)


@pytest.mark.parametrize("renorm", [False, True], ids=["softmax", "renormalised"])
@pytest.mark.parametrize("w", SMALL[1:3], ids=lambda w: w.describe())
def test_router_steps_against_oracle_on_gpu_inputs(w, renorm):
    """Each router backward step on the GPU's own inputs: dlogits from the GPU's dweights, the
    dx increment, and dW_r, each against the oracle given exactly those inputs."""
    flags = B.ROUTE_RENORMALIZE if renorm else 0
    inp, dims, dev, bufs, logits, g, dx_experts, dwr, ws = _forward_backward(w, flags)
    lg = logits.float().cpu().numpy()
    top = bufs.map.top_experts.cpu().numpy()
    dw_gpu = g["dw"].double().cpu().numpy()
    r = oracle.router_backward(inp["x"].float().numpy(), inp["w_router"].float().numpy(), lg, top,
                               dw_gpu, renorm=renorm)
    dl = torch.empty((w.T, w.E), dtype=torch.bfloat16, device="cuda")
    B.dmoe_router_dlogits(dims, logits, bufs.map, g["dw"], dl)
    torch.cuda.synchronize()
    got = to_np(dl)
    ref = r["dlogits"]
    # fp32 softmax, then one bf16 rounding
    assert (np.abs(got - ref) <= 2.0 ** -7 * np.abs(ref) + 1e-4 * np.abs(ref).max()).all()
    # the dx increment: its rounding adds at most one bf16 ulp of the sum
    assert_increment_close(to_np(g["dx"]), to_np(dx_experts), r["dx_r"], "dx_r")
    assert_close(to_np(dwr), r["dWr"], "dW_r")


def test_router_backward_deterministic_and_full_size_sampled():
    """A 4096-token, E = 256 case (many K splits of dW_r): two runs give the same bits, and
    sampled tokens of dx_r and sampled dW_r elements match the oracle."""
    w = custom(4096, 2048, 512, 256, 8)
    inp, dims, dev, bufs, logits, g, dx_experts, dwr, ws = _forward_backward(w)
    dx2 = dx_experts.clone()
    dwr2 = torch.empty_like(dwr)
    B.dmoe_router_backward(dims, dev["x"], dev["w_router"], logits, bufs.map, g["dw"], dx2, dwr2, ws)
    torch.cuda.synchronize()
    assert torch.equal(dx2.view(torch.int16), g["dx"].view(torch.int16))
    assert torch.equal(dwr2.view(torch.int32), dwr.view(torch.int32))
    lg = logits.float().cpu().numpy()
    top = bufs.map.top_experts.cpu().numpy()
    toks = sample_tokens(top, w.E, 64, seed=11)
    rng = np.random.default_rng(13)
    el = np.stack([rng.integers(0, w.E, 200), rng.integers(0, w.hidden, 200)], 1)
    r = oracle.router_backward(inp["x"].float().numpy(), inp["w_router"].float().numpy(), lg, top,
                               g["dw"].double().cpu().numpy(), tokens=toks, elems=el,
                               threads=oracle.max_threads())
    assert_increment_close(to_np(g["dx"])[toks], to_np(dx_experts)[toks], r["dx_r"], "dx_r sampled")
    assert_close(to_np(dwr)[el[:, 0], el[:, 1]], r["dWr"], "dW_r sampled")
