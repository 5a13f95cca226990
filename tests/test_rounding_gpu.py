"""Tile-aware token rounding (the SonicMoE abstract's routing variant, DMOE_ROUTE_TOKEN_ROUNDING)
against the oracle: the rounded routing as a token-major entry list bit for bit, its padded
map (no padding rows: every count is a multiple of 128), and the layer's forward and backward
over it."""
import numpy as np
import pytest
import torch

import oracle
from dropless_mixture_experts_dmoe_b200 import binding as B
from dropless_mixture_experts_dmoe_b200.workloads import WORKLOADS, custom, make_inputs

import bf16_model
from helpers import MAX_ABS_RMS, WEIGHT_RTOL, assert_close, to_np

pytestmark = pytest.mark.gpu

RT = B.ROUTE_TOKEN_ROUNDING


def _dims(w):
    return B.make_dims(w.T, w.hidden, w.ffn, w.E, w.top_k, flags=RT)


def _oracle_rounded(logits, k, E):
    top, _ = oracle.route(logits, k)
    tr, wr = oracle.round_tokens(logits, top)
    offsets, experts, weights = oracle.compact_entries(tr, wr)
    return tr, wr, offsets, experts, weights


def _check_map(bufs, logits, w):
    """Every array of the GPU's rounded map against the oracle; returns the oracle routing."""
    m = bufs.map
    tr, wr, offsets, experts, weights = _oracle_rounded(logits, w.top_k, w.E)
    n = int(offsets[-1])
    assert int(m.status.item()) == 0
    np.testing.assert_array_equal(m.entry_offsets.cpu().numpy(), offsets)
    te = m.top_experts.cpu().numpy()
    np.testing.assert_array_equal(te[:n], experts)
    assert (te[n:] == -1).all()
    np.testing.assert_allclose(m.weights.cpu().numpy()[:n], weights, rtol=WEIGHT_RTOL, atol=0)
    assert (m.weights.cpu().numpy()[n:] == 0).all()
    ref = oracle.sparse_map(experts.reshape(-1, 1), w.E)
    for key in ("tokens_per_expert", "bins", "padded_bins"):
        np.testing.assert_array_equal(getattr(m, key).cpu().numpy(), ref[key], err_msg=key)
    for key in ("indices", "bin_ids", "dest_row"):
        np.testing.assert_array_equal(getattr(m, key).cpu().numpy()[:n], ref[key], err_msg=key)
    assert (m.dest_row.cpu().numpy()[n:] == -1).all()
    assert int(m.num_blocks.item()) == ref["num_blocks"]
    be = m.block_expert.cpu().numpy()
    nref = len(ref["block_expert"])
    np.testing.assert_array_equal(be[:nref], ref["block_expert"][:len(be)])
    assert (be[nref:] == -1).all()
    # the point of the rounding: no padding rows
    assert (ref["tokens_per_expert"] % 128 == 0).all()
    assert ref["num_blocks"] * 128 == n
    return tr, wr, offsets


CASES = [
    custom(3000, 128, 128, 16, 2, number=31),
    custom(1000, 128, 128, 8, 3, number=32),
    custom(700, 128, 128, 64, 8, number=33),   # many experts below 64 entries: dropped to 0
    custom(256, 128, 128, 4, 1, number=34),
    custom(20000, 128, 128, 256, 8, number=35, zipf_bias=True),  # skewed: heavy and light
    WORKLOADS[4],                               # the high-granularity workload's routing
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.describe())
def test_rounded_map_parity(w):
    dims = _dims(w)
    inp = make_inputs(w, with_dy=False)
    bufs = B.Buffers(dims, train=False)
    B.dmoe_sparse_map(dims, inp["logits"].cuda(), bufs.map, bufs.ws_map)
    torch.cuda.synchronize()
    _check_map(bufs, inp["logits"].float().numpy(), w)


def test_rounded_map_ties():
    """Few distinct logit values (+0 and -0 among them): the rank ties are broken by the token
    index exactly as in the oracle."""
    T, E, k = 3000, 16, 2
    g = torch.Generator().manual_seed(9)
    vals = torch.tensor([-1.0, -0.0, 0.0, 0.5, 2.0])
    logits = vals[torch.randint(0, 5, (T, E), generator=g)].to(torch.bfloat16)
    w = custom(T, 128, 128, E, k)
    dims = _dims(w)
    bufs = B.Buffers(dims, train=False)
    B.dmoe_sparse_map(dims, logits.cuda(), bufs.map, bufs.ws_map)
    torch.cuda.synchronize()
    _check_map(bufs, logits.float().numpy(), w)


@pytest.mark.parametrize("w", [custom(3000, 256, 256, 16, 2, number=41),
                               custom(700, 384, 128, 32, 4, number=42)],
                         ids=lambda w: w.describe())
def test_rounded_layer_forward_backward(w):
    """Forward and backward over the rounded routing against the oracle run on the same
    rounded routing (absent positions skipped); dweights per listed entry."""
    dims = _dims(w)
    inp = make_inputs(w, with_dy=True)
    bufs = B.Buffers(dims, train=True)
    dev = {k: v.cuda() for k, v in inp.items()}
    B.dmoe_sparse_map(dims, dev["logits"], bufs.map, bufs.ws_map)
    y = torch.empty((w.T, w.hidden), dtype=torch.bfloat16, device="cuda")
    B.dmoe_forward(dims, dev["x"], dev["w1"], dev["w3"], dev["w2"], bufs.map, y, saved=bufs.saved,
                   ws=bufs.ws_fwd)
    E, f, h, T = w.E, w.ffn, w.hidden, w.T
    f32 = dict(dtype=torch.float32, device="cuda")
    dx = torch.empty_like(y)
    dw1 = torch.empty((E, f, h), **f32)
    dw3 = torch.empty_like(dw1)
    dw2 = torch.empty((E, h, f), **f32)
    dwt = torch.empty(B.dmoe_entries_max(dims), **f32)
    B.dmoe_backward(dims, dev["dy"], dev["w1"], dev["w3"], dev["w2"], bufs.map, bufs.saved, dx,
                    dw1, dw3, dw2, dwt, bufs.ws_bwd)
    torch.cuda.synchronize()
    o = {k: v.float().numpy() for k, v in inp.items()}
    tr, wr, offsets = _check_map(bufs, o["logits"], w)
    # stress shapes (few rows per expert): the bf16 rounding model of the pipeline sizes the
    # max-abs bound where it exceeds 5e-2 / 1.25 (tests/bf16_model.py)
    yref = oracle.forward(o["x"], o["w1"], o["w3"], o["w2"], tr, wr, threads=8)
    ytol = bf16_model.bounds({"y": bf16_model.forward_model(inp, tr, wr)}, {"y": yref})["y"]
    assert_close(to_np(y), yref, f"y {w.describe()}", max_abs_rms=ytol)
    g = oracle.backward(o["x"], o["dy"], o["w1"], o["w3"], o["w2"], tr, wr)
    tol = bf16_model.bounds(bf16_model.backward_model(inp, tr, wr), g)
    for got, name in ((dx, "dx"), (dw1, "dW1"), (dw3, "dW3"), (dw2, "dW2")):
        assert_close(to_np(got), g[name], f"{name} {w.describe()}", max_abs_rms=tol[name])
    n = int(offsets[-1])
    assert_close(to_np(dwt)[:n], g["dw"][tr >= 0], f"dw {w.describe()}", max_abs_rms=tol["dw"])


def test_rounded_forward_high_granularity():
    """The high-granularity workload (T = 16384, E = 128, top-8) with the rounded routing: every
    token's output against the oracle, and no padding rows left in the padded layout."""
    w = WORKLOADS[4]
    dims = _dims(w)
    inp = make_inputs(w, with_dy=False)
    bufs = B.Buffers(dims, train=False)
    dev = {k: v.cuda() for k, v in inp.items()}
    B.dmoe_sparse_map(dims, dev["logits"], bufs.map, bufs.ws_map)
    y = torch.empty((w.T, w.hidden), dtype=torch.bfloat16, device="cuda")
    B.dmoe_forward(dims, dev["x"], dev["w1"], dev["w3"], dev["w2"], bufs.map, y, ws=bufs.ws_fwd)
    torch.cuda.synchronize()
    o = {k: v.float().numpy() for k, v in inp.items()}
    tr, wr, offsets = _check_map(bufs, o["logits"], w)
    yref = oracle.forward(o["x"], o["w1"], o["w3"], o["w2"], tr, wr, threads=oracle.max_threads())
    assert_close(to_np(y), yref, "y high-granularity rounded")
