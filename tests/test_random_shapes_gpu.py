"""Seeded sweep of random small shapes through the whole layer (forward and backward) and
of map-only shapes up to the maximum sizes, against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from dropless_mixture_experts_dmoe_b200 import binding as B
from dropless_mixture_experts_dmoe_b200.workloads import custom, make_inputs, make_tensor

import bf16_model
from helpers import assert_close, compare_map, dims_of, gpu_backward, gpu_map, oracle_inputs, to_np

pytestmark = pytest.mark.gpu


def _random_shapes(n, seed):
    rng = np.random.default_rng(seed)
    out = [custom(1, 128, 128, 1, 1), custom(3, 256, 128, 4, 4), custom(129, 128, 256, 1, 1)]
    while len(out) < n:
        E = int(rng.choice([1, 2, 3, 7, 16, 33]))
        k = int(rng.integers(1, min(E, 8) + 1))
        T = int(rng.integers(1, 700))
        h = int(rng.choice([128, 256, 384, 640]))
        f = int(rng.choice([128, 256, 512]))
        out.append(custom(T, h, f, E, k, number=0))
    return out


@pytest.mark.parametrize("w", _random_shapes(10, seed=2024), ids=lambda w: w.describe())
def test_random_shape_forward_backward(w):
    inp = make_inputs(w, with_dy=True)
    dims = dims_of(w)
    bufs, dev, y, g = gpu_backward(dims, inp)
    assert int(bufs.map.status.item()) == 0
    o = oracle_inputs(inp)
    top, wts = oracle.route(o["logits"], w.top_k)
    assert (bufs.map.top_experts.cpu().numpy() == top).all()
    yref = oracle.forward(o["x"], o["w1"], o["w3"], o["w2"], top, wts, threads=8)
    ytol = bf16_model.bounds({"y": bf16_model.forward_model(inp, top, wts)}, {"y": yref})["y"]
    assert_close(to_np(y), yref, f"y {w.describe()}", max_abs_rms=ytol)
    ref = oracle.backward(o["x"], o["dy"], o["w1"], o["w3"], o["w2"], top, wts)
    tol = bf16_model.bounds(bf16_model.backward_model(inp, top, wts), ref)
    for gk, rk in (("dx", "dx"), ("dw1", "dW1"), ("dw3", "dW3"), ("dw2", "dW2"), ("dw", "dw")):
        assert_close(to_np(g[gk]), ref[rk], f"{rk} {w.describe()}", max_abs_rms=tol[rk])


@pytest.mark.parametrize("T,E,k", [(262144, 256, 8), (65536, 1024, 8), (200000, 8, 2)])
def test_map_parity_maximum_sizes(T, E, k):
    w = custom(T, 128, 128, E, k, number=7)
    logits = make_tensor(w, "logits")
    dims = B.make_dims(T, 128, 128, E, k)
    _, g = gpu_map(dims, logits)
    top, wts = oracle.route(logits.float().numpy(), k)
    compare_map(g, oracle.sparse_map(top, E), top_expected=top)
    np.testing.assert_allclose(g["weights"], wts, rtol=2e-6, atol=0)
