"""The forward variant whose down GEMM does the weighted combine in its epilogue
(DMOE_FUSED_COMBINE: fp32 vector reductions into a token accumulator, no Y_pad) against the
oracle, its reproducibility for top_k <= 2, and its agreement with the default path."""
import numpy as np
import pytest
import torch

import bf16_model
import oracle
from dropless_mixture_experts_dmoe_b200 import binding as B
from dropless_mixture_experts_dmoe_b200.workloads import WORKLOADS, custom, make_inputs

from helpers import MAX_ABS_RMS, assert_close, compare_map, to_np, tokens_covering_blocks

pytestmark = pytest.mark.gpu


def _forward(w, inp, flags, train=False):
    dims = B.make_dims(w.T, w.hidden, w.ffn, w.E, w.top_k, flags=flags)
    bufs = B.Buffers(dims, train=train)
    dev = {k: v.cuda() for k, v in inp.items()}
    B.dmoe_sparse_map(dims, dev["logits"], bufs.map, bufs.ws_map)
    y = torch.empty((w.T, w.hidden), dtype=torch.bfloat16, device="cuda")
    B.dmoe_forward(dims, dev["x"], dev["w1"], dev["w3"], dev["w2"], bufs.map, y,
                   saved=bufs.saved if train else None, ws=bufs.ws_fwd)
    torch.cuda.synchronize()
    return bufs, y


SHAPES = [WORKLOADS[1], custom(512, 384, 384, 8, 2), custom(300, 256, 256, 16, 4),
          custom(1000, 128, 512, 5, 3), custom(200, 640, 128, 64, 8)]


@pytest.mark.parametrize("train", [False, True], ids=["inference", "training"])
@pytest.mark.parametrize("w", SHAPES, ids=lambda w: w.describe())
def test_fused_combine_parity(w, train):
    inp = make_inputs(w)
    bufs, y = _forward(w, inp, B.FUSED_COMBINE, train)
    assert int(bufs.map.status.item()) == 0
    o = {k: v.float().numpy() for k, v in inp.items()}
    top, wts = oracle.route(o["logits"], w.top_k)
    ref = oracle.forward(o["x"], o["w1"], o["w3"], o["w2"], top, wts, threads=8)
    tol = tol0 = MAX_ABS_RMS
    if not w.number:  # stress shape: the rounding model's bound, for the fused path (fp32
        # rows summed) and for the default one (rows in block floating point)
        tol = bf16_model.bounds({"y": bf16_model.forward_model(inp, top, wts, fused=True)},
                                {"y": ref})["y"]
        tol0 = bf16_model.bounds({"y": bf16_model.forward_model(inp, top, wts)}, {"y": ref})["y"]
    assert_close(to_np(y), ref, f"y fused {w.describe()}", max_abs_rms=tol)
    _, y0 = _forward(w, inp, 0, train)  # the default path, within the larger of the bounds
    assert_close(to_np(y), to_np(y0), f"y fused vs default {w.describe()}",
                 max_abs_rms=max(tol, tol0))


@pytest.mark.parametrize("w", [SHAPES[1], WORKLOADS[1]], ids=lambda w: w.describe())
def test_fused_combine_reproducible_top2(w):
    """top_k = 2: each output element is 0 + a + b in some order, and a + b = b + a, so two
    runs give the same bits."""
    inp = make_inputs(w)
    _, y1 = _forward(w, inp, B.FUSED_COMBINE)
    _, y2 = _forward(w, inp, B.FUSED_COMBINE)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_fused_combine_mixtral_shaped_full_size():
    """The Mixtral-shaped workload (top-2, hidden 4096): the tokens holding the first and last
    row of every 128-row block against the oracle."""
    w = WORKLOADS[2]
    inp = make_inputs(w, with_dy=False)
    bufs, y = _forward(w, inp, B.FUSED_COMBINE)
    assert int(bufs.map.status.item()) == 0
    lg = inp["logits"].float().numpy()
    top, wts = oracle.route(lg, w.top_k)
    m = oracle.sparse_map(top, w.E)
    toks = tokens_covering_blocks(m, w.top_k, w.T, 256, seed=2)
    o = {k: inp[k].float().numpy() for k in ("x", "w1", "w3", "w2")}
    ref = oracle.forward(o["x"], o["w1"], o["w3"], o["w2"], top, wts, tokens=toks,
                         threads=oracle.max_threads())
    assert_close(to_np(y)[toks], ref, f"y fused mixtral-shaped ({len(toks)} tokens)")
    assert torch.isfinite(y.float()).all()
