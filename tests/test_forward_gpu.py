"""Forward parity of the whole layer (map + gather + tcgen05 GEMMs + combine) against the
oracle, plus checks of the GEMM intermediates against float64 PyTorch on the same bf16
operands."""
import numpy as np
import pytest
import torch

import oracle
from dropless_mixture_experts_dmoe_b200 import binding as B
from dropless_mixture_experts_dmoe_b200.workloads import WORKLOADS, custom, make_inputs

import bf16_model
from helpers import (MAX_ABS_RMS, assert_close, compare_map, dims_of, gpu_forward, oracle_inputs,
                     to_np, tokens_covering_blocks)

pytestmark = pytest.mark.gpu

SMALL = [
    WORKLOADS[1],                     # tiny: 8 experts, top-2, one column tile each
    custom(512, 384, 384, 8, 2),      # 3 GLU column tiles; down GEMM 256 + ragged 128 columns
    custom(300, 256, 256, 16, 4),     # ragged row blocks, top-4
    custom(1000, 128, 512, 5, 3),     # top-3, K = 128
    custom(200, 640, 128, 64, 8),     # many experts, many empty or single-row blocks
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.describe())
def test_forward_full_parity_small(w):
    inp = make_inputs(w)
    dims = dims_of(w)
    bufs, dev, y = gpu_forward(dims, inp)
    o = oracle_inputs(inp)
    top, wts = oracle.route(o["logits"], w.top_k)
    m = oracle.sparse_map(top, w.E)
    g = {k: to_np(v) for k, v in bufs.map.as_dict().items()}
    g["num_blocks"] = int(g["num_blocks"][0])
    compare_map(g, m, top_expected=top)
    assert int(g["status"][0]) == 0
    ref = oracle.forward(o["x"], o["w1"], o["w3"], o["w2"], top, wts, threads=8)
    tol = MAX_ABS_RMS
    if not w.number:  # stress shape: the modelled bf16 error decides (tests/bf16_model.py)
        tol = bf16_model.bounds({"y": bf16_model.forward_model(inp, top, wts)}, {"y": ref})["y"]
    assert_close(to_np(y), ref, f"y {w.describe()}", max_abs_rms=tol)


@pytest.mark.parametrize("w", SMALL[:3], ids=lambda w: w.describe())
def test_gemm_intermediates(w):
    """H and Y_pad block by block against float64 matmuls of the same bf16 operands."""
    inp = make_inputs(w)
    dims = dims_of(w)
    bufs, dev, y = gpu_forward(dims, inp)
    nb = int(bufs.map.num_blocks.item())
    be = bufs.map.block_expert.cpu().numpy()
    xp = bufs.view("x_pad")[: nb * 128].double().cpu()
    A = bufs.view("a")[: nb * 128].double().cpu()
    Bm = bufs.view("bm")[: nb * 128].double().cpu()
    H = bufs.view("h")[: nb * 128].double().cpu()
    # Y_pad is block floating point: fp16 values times one power-of-two scale per 128 columns,
    # each row weighted by its routing weight (0 for a padding row)
    ys = bufs.view("y_scale")[: nb * 128].double().cpu().abs().repeat_interleave(128, dim=1)
    Yp = bufs.view("y_pad")[: nb * 128].double().cpu() * ys[:, : w.hidden]
    wrow = torch.zeros(nb * 128, dtype=torch.float64)
    wrow[bufs.map.dest_row.cpu().long()] = bufs.map.weights.cpu().double().reshape(-1)
    W1 = inp["w1"].double()
    W3 = inp["w3"].double()
    W2 = inp["w2"].double()
    for b in range(nb):
        e = int(be[b])
        rows = slice(b * 128, (b + 1) * 128)
        a_ref = xp[rows] @ W1[e].T
        b_ref = xp[rows] @ W3[e].T
        h_ref = torch.nn.functional.silu(a_ref) * b_ref
        assert torch.allclose(A[rows], a_ref, rtol=1e-2, atol=1e-2), b
        assert torch.allclose(Bm[rows], b_ref, rtol=1e-2, atol=1e-2), b
        assert torch.allclose(H[rows], h_ref, rtol=2e-2, atol=2e-3), b
        y_ref = wrow[rows, None] * (H[rows] @ W2[e].T)
        assert torch.allclose(Yp[rows], y_ref, rtol=1e-2, atol=1e-4), b


@pytest.mark.parametrize("num", [2, 3, 4, 5])
def test_forward_parity_full_size(num):
    """The full-size workloads as the bench runs them.  The fine-grained and high-granularity
    workloads compare every token of y with the oracle; the Mixtral-shaped and skewed ones the
    tokens whose entries hold the first and the last real row of every 128-row block (so both
    halves of every pair of blocks, every expert's ragged last block and every column tile
    are checked), plus random tokens."""
    w = WORKLOADS[num]
    inp = make_inputs(w, with_dy=False)
    dims = dims_of(w)
    bufs, dev, y = gpu_forward(dims, inp, train=False)
    assert int(bufs.map.status.item()) == 0
    del dev
    lg = inp["logits"].float().numpy()
    top, wts = oracle.route(lg, w.top_k)
    g = {k: to_np(v) for k, v in bufs.map.as_dict().items()}
    g["num_blocks"] = int(g["num_blocks"][0])
    m = oracle.sparse_map(top, w.E)
    compare_map(g, m, top_expected=top)
    if num in (3, 4):
        toks = None
    else:
        toks = tokens_covering_blocks(m, w.top_k, w.T, 256, seed=num, last_rows=(num == 2))
        covered = np.unique(m["dest_row"].reshape(w.T, w.top_k)[toks] // 128)
        assert len(covered) == m["num_blocks"]  # every block holds a sampled row
    o = {k: inp[k].float().numpy() for k in ("x", "w1", "w3", "w2")}
    ref = oracle.forward(o["x"], o["w1"], o["w3"], o["w2"], top, wts, tokens=toks,
                         threads=oracle.max_threads())
    got = to_np(y) if toks is None else to_np(y)[toks]
    assert_close(got, ref, f"y workload {num} ({len(ref)} tokens)")
    # properties at every token: finite output, no NaN from padding rows
    assert torch.isfinite(y.float()).all()


@pytest.mark.parametrize("w", SMALL + [WORKLOADS[3]], ids=lambda w: w.describe())
def test_gathered_glu_matches_padded_glu(w):
    """The GLU GEMM that gathers its rows from x must equal, bit for bit, gather + GLU on the
    materialised X_pad (padding rows, odd last blocks and all)."""
    inp = make_inputs(w)
    dims = dims_of(w)
    bufs, dev, y = gpu_forward(dims, inp, train=True)
    P = bufs.P
    h2 = torch.full((P, w.ffn), float("nan"), dtype=torch.bfloat16, device="cuda")
    a2 = torch.full_like(h2, float("nan"))
    b2 = torch.full_like(h2, float("nan"))
    B.dmoe_expert_glu_gather(dims, dev["x"], dev["w1"], dev["w3"], bufs.map, h2, a2, b2)
    torch.cuda.synchronize()
    rows = int(bufs.map.num_blocks.item()) * 128
    for name, got in (("h", h2), ("a", a2), ("bm", b2)):
        ref = bufs.view(name)[:rows]
        assert torch.equal(got[:rows].view(torch.int16), ref.view(torch.int16)), name


def test_forward_deterministic():
    w = SMALL[1]
    inp = make_inputs(w)
    dims = dims_of(w)
    _, _, y1 = gpu_forward(dims, inp)
    _, _, y2 = gpu_forward(dims, inp)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_forward_inference_equals_training_mode():
    w = SMALL[2]
    inp = make_inputs(w)
    dims = dims_of(w)
    _, _, y1 = gpu_forward(dims, inp, train=True)
    _, _, y2 = gpu_forward(dims, inp, train=False)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
