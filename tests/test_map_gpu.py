"""Sparse-map parity: routing and every map array bit-exact against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from dropless_mixture_experts_dmoe_b200 import binding as B
from dropless_mixture_experts_dmoe_b200.workloads import WORKLOADS, make_inputs, make_tensor

from helpers import WEIGHT_RTOL, compare_map, gpu_map

pytestmark = pytest.mark.gpu


def _logits_only(w):
    return make_tensor(w, "logits")


@pytest.mark.parametrize("num", [1, 2, 3, 4, 5])
def test_map_parity_workloads(num):
    w = WORKLOADS[num]
    logits = _logits_only(w)
    dims = B.make_dims(w.T, w.hidden, w.ffn, w.E, w.top_k)
    _, g = gpu_map(dims, logits)
    top, wts = oracle.route(logits.float().numpy(), w.top_k)
    o = oracle.sparse_map(top, w.E)
    compare_map(g, o, top_expected=top)
    np.testing.assert_allclose(g["weights"], wts, rtol=WEIGHT_RTOL, atol=0)
    assert g["status"] == 0


def test_map_parity_real_inputs_tiny():
    w = WORKLOADS[1]
    inp = make_inputs(w)
    dims = B.make_dims(w.T, w.hidden, w.ffn, w.E, w.top_k)
    _, g = gpu_map(dims, inp["logits"])
    top, wts = oracle.route(inp["logits"].float().numpy(), w.top_k)
    compare_map(g, oracle.sparse_map(top, w.E), top_expected=top)


@pytest.mark.parametrize("T,E,k,kind", [
    (300, 8, 2, "all_equal"),      # every row ties: experts 0..k-1
    (257, 16, 4, "few_values"),    # many ties, +0 / -0 mixed
    (130, 8, 8, "continuous"),     # k = E
    (1000, 1, 1, "continuous"),    # E = 1
    (999, 64, 1, "continuous"),    # k = 1
    (2000, 1024, 8, "continuous"),  # maximum E
    (4097, 32, 32, "few_values"),  # maximum k
    (1, 8, 2, "continuous"),       # single token
    (8192, 64, 8, "continuous"),   # the issue's failing shape with 4096-long sequences
    # logits layouts of the routing kernel: two experts per word for even E (word c of lane l
    # = experts 64c + 2l, 64c + 2l + 1), lane l = experts l, l + 32, ... for odd E; rounds
    # unrolled for top-2 and top-8
    (7, 7, 3, "few_values"),        # 1 per lane, a partial tile
    (1000, 33, 4, "continuous"),    # 2 per lane, odd E
    (1000, 100, 8, "few_values"),   # 4 per lane, paired, ties
    (1500, 250, 8, "continuous"),   # 8 per lane, paired, a partial last word group
    (1500, 251, 8, "continuous"),   # 8 per lane, odd E
    (300, 256, 32, "few_values"),   # 8 per lane, 32 picks drain whole lanes (refilled rounds)
    (600, 384, 8, "few_values"),    # 16 per lane, paired
    (700, 1000, 8, "continuous"),   # 32 per lane, paired
    (700, 999, 8, "continuous"),    # 32 per lane, odd E
    (40000, 16, 4, "continuous"),   # 625 tiles: the scan re-reads past its register cache
    (500, 64, 8, "tiny_values"),    # bf16 subnormals of both signs next to +0 / -0
    (2048, 256, 8, "skewed"),       # the skewed workload's bias on the low expert indices
    # two logits per word, word c of lane l = experts 64c + 2l, 64c + 2l + 1
    (2048, 256, 8, "lane_heavy"),   # lane 0's experts win: the rounds run again with refills
    (1000, 200, 8, "continuous"),   # a partial last word group (lanes 0-3 of the fourth)
    (1000, 66, 4, "few_values"),    # one lane of the second group, ties
    (777, 512, 2, "lane_heavy"),    # 16 per lane, top-2
])
def test_map_parity_edge_cases(T, E, k, kind):
    g = torch.Generator().manual_seed(T * 7 + E)
    if kind == "all_equal":
        logits = torch.full((T, E), 0.5)
    elif kind == "few_values":
        vals = torch.tensor([-1.0, -0.0, 0.0, 0.5, 0.5, 2.0])
        logits = vals[torch.randint(0, len(vals), (T, E), generator=g)]
    elif kind == "tiny_values":
        vals = torch.tensor([-2e-39, -1e-39, -0.0, 0.0, 1e-39, 2e-39, 3e-39, 1e-38])
        logits = vals[torch.randint(0, len(vals), (T, E), generator=g)]
    elif kind == "skewed":
        logits = torch.randn((T, E), generator=g) - 1.5 * torch.log(torch.arange(E) + 1.0)
    elif kind == "lane_heavy":  # experts 64c, 64c + 1 (the first lane's) far above the rest
        logits = torch.randn((T, E), generator=g) - 8.0
        logits[:, (torch.arange(E) % 64) < 2] += 16.0
    else:
        logits = torch.randn((T, E), generator=g)
    logits = logits.to(torch.bfloat16)
    dims = B.make_dims(T, 128, 128, E, k)
    _, gm = gpu_map(dims, logits)
    top, wts = oracle.route(logits.float().numpy(), k)
    compare_map(gm, oracle.sparse_map(top, E), top_expected=top)
    np.testing.assert_allclose(gm["weights"], wts, rtol=WEIGHT_RTOL, atol=0)


@pytest.mark.parametrize("T,E,k", [(4096, 64, 8), (1000, 8, 2), (300, 16, 16), (777, 1024, 1),
                                   (2000, 256, 32)])
def test_map_renormalised_weights(T, E, k):
    """Routing variant DMOE_ROUTE_RENORMALIZE: the same choice, weights = softmax over the k
    chosen logits (summing to 1), against the oracle's renormalised mode."""
    g = torch.Generator().manual_seed(T + 31 * E + k)
    logits = torch.randn((T, E), generator=g).to(torch.bfloat16)
    dims = B.make_dims(T, 128, 128, E, k, flags=B.ROUTE_RENORMALIZE)
    _, gm = gpu_map(dims, logits)
    top, wts = oracle.route(logits.float().numpy(), k, renorm=True)
    compare_map(gm, oracle.sparse_map(top, E), top_expected=top)
    np.testing.assert_allclose(gm["weights"], wts, rtol=WEIGHT_RTOL, atol=0)
    np.testing.assert_allclose(gm["weights"].sum(1), 1.0, rtol=0, atol=k * 2e-7)
    assert gm["status"] == 0


def test_map_skew_and_empty_experts_given_top():
    """Caller-given top_experts: one expert takes every token, most experts are empty."""
    T, E, k = 5000, 256, 8
    top = np.zeros((T, k), np.int32)
    top[:, 1:] = (np.arange(T)[:, None] * 7 + np.arange(1, k)[None, :]) % 5 + 1
    dims = B.make_dims(T, 128, 128, E, k)
    _, g = gpu_map(dims, top_experts=top)
    compare_map(g, oracle.sparse_map(top, E), top_expected=top)
    assert g["status"] & B.STATUS_DUPLICATE_EXPERT  # slots 1..7 repeat experts within a token


def test_map_given_top_out_of_range_is_dropped():
    T, E, k = 100, 8, 2
    top = np.tile(np.array([[1, 2]], np.int32), (T, 1))
    top[5, 1] = 8
    top[17, 0] = -3
    dims = B.make_dims(T, 128, 128, E, k)
    _, g = gpu_map(dims, top_experts=top)
    assert g["status"] & B.STATUS_EXPERT_OUT_OF_RANGE
    assert g["dest_row"][5 * k + 1] == -1 and g["dest_row"][17 * k] == -1
    valid = top.ravel()[(top.ravel() >= 0) & (top.ravel() < E)]
    assert g["tokens_per_expert"].sum() == valid.size


def test_map_nonfinite_logits_flagged():
    logits = torch.randn(64, 8)
    logits[3, 2] = float("nan")
    dims = B.make_dims(64, 128, 128, 8, 2)
    _, g = gpu_map(dims, logits.to(torch.bfloat16))
    assert g["status"] & B.STATUS_NONFINITE_LOGITS


@pytest.mark.parametrize("E,k", [(256, 8), (64, 4), (250, 8), (255, 8), (33, 2)])
def test_map_nonfinite_logits_ranked(E, k):
    """NaN ranks below every value (-inf included), +-inf at its place; the choice and the map
    stay bit-exact and the call is flagged."""
    T = 700
    g = torch.Generator().manual_seed(E + k)
    logits = torch.randn((T, E), generator=g)
    r = torch.rand((T, E), generator=g)
    logits[r < 0.01] = float("nan")
    logits[(r >= 0.01) & (r < 0.015)] = float("inf")
    logits[(r >= 0.015) & (r < 0.02)] = float("-inf")
    logits[5, :] = float("nan")             # a row of NaN only
    logits[6, : E // 2] = float("-inf")     # half of a row at -inf
    logits = logits.to(torch.bfloat16)
    dims = B.make_dims(T, 128, 128, E, k)
    _, gm = gpu_map(dims, logits)
    top, _ = oracle.route(logits.float().numpy(), k)
    compare_map(gm, oracle.sparse_map(top, E), top_expected=top)
    assert gm["status"] & B.STATUS_NONFINITE_LOGITS


def test_map_status_is_the_calls_own():
    """The map call's status word holds its own bits: a flag left by an earlier call, or
    garbage put there by the caller, does not survive a clean call."""
    dims = B.make_dims(64, 128, 128, 8, 2)
    bad = torch.randn(64, 8)
    bad[3, 2] = float("nan")
    bufs, g = gpu_map(dims, bad.to(torch.bfloat16))
    assert g["status"] == B.STATUS_NONFINITE_LOGITS
    _, g = gpu_map(dims, torch.randn(64, 8).to(torch.bfloat16), bufs=bufs)
    assert g["status"] == 0
    bufs.map.status.fill_(0x1234)
    _, g = gpu_map(dims, torch.randn(64, 8).to(torch.bfloat16), bufs=bufs)
    assert g["status"] == 0


def test_map_deterministic_repeat():
    w = WORKLOADS[5]
    logits = _logits_only(w)
    dims = B.make_dims(w.T, w.hidden, w.ffn, w.E, w.top_k)
    bufs, g1 = gpu_map(dims, logits)
    _, g2 = gpu_map(dims, logits, bufs=bufs)
    for key in ("top_experts", "weights", "indices", "dest_row", "block_expert"):
        assert (g1[key] == g2[key]).all()
