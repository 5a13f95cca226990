"""padded_gather / padded_scatter data-movement parity (bit-exact where the maths is exact)."""
import numpy as np
import pytest
import torch

import oracle
from dropless_mixture_experts_dmoe_b200 import binding as B
from dropless_mixture_experts_dmoe_b200.workloads import WORKLOADS, custom, make_tensor

from helpers import compare_map, gpu_map, to_np

pytestmark = pytest.mark.gpu

SHAPES = [
    WORKLOADS[1],
    WORKLOADS[3],
    custom(1000, 384, 128, 5, 3),    # h/8 = 48 vectors per row: a ragged vector chunk
    custom(777, 4096, 128, 16, 2),   # wide rows (two 256-vector chunks)
    custom(64, 128, 128, 300, 8),    # most experts empty
]


def _setup(w):
    dims = B.make_dims(w.T, w.hidden, w.ffn, w.E, w.top_k)
    logits = make_tensor(w, "logits")
    bufs, g = gpu_map(dims, logits)
    top, _ = oracle.route(logits.float().numpy(), w.top_k)
    compare_map(g, oracle.sparse_map(top, w.E), top_expected=top)
    x = make_tensor(w, "x").cuda()
    return dims, bufs, g, x


@pytest.mark.parametrize("w", SHAPES, ids=lambda w: w.describe())
def test_gather_bit_exact_and_zero_padding(w):
    dims, bufs, g, x = _setup(w)
    xp = bufs.view("x_pad")
    xp.view(torch.int16).fill_(0x7F81)  # sentinel (a NaN pattern) to see untouched rows
    B.dmoe_padded_gather(dims, x, bufs.map, xp)
    torch.cuda.synchronize()
    P = g["num_blocks"] * 128
    xp16 = xp.view(torch.int16).cpu().numpy()
    x16 = x.view(torch.int16).cpu().numpy()
    t_of_j = np.arange(w.T * w.top_k) // w.top_k
    np.testing.assert_array_equal(xp16[g["dest_row"]], x16[t_of_j])
    real = np.zeros(P, bool)
    real[g["dest_row"]] = True
    assert (xp16[:P][~real] == 0).all(), "padding rows must be zero"
    assert (xp16[P:] == 0x7F81).all(), "rows past the padded size must be untouched"


@pytest.mark.parametrize("w", SHAPES, ids=lambda w: w.describe())
def test_scatter_of_gather_is_k_times_x(w):
    dims, bufs, g, x = _setup(w)
    xp = bufs.view("x_pad")
    B.dmoe_padded_gather(dims, x, bufs.map, xp)
    y = torch.empty_like(x)
    B.dmoe_padded_scatter(dims, xp, None, bufs.map, None, y)  # w = 1, bf16 rows
    torch.cuda.synchronize()
    ref = (x.float() * w.top_k).to(torch.bfloat16)  # k*x is exact in fp32
    assert torch.equal(y.view(torch.int16), ref.view(torch.int16))


@pytest.mark.parametrize("w", SHAPES[:3], ids=lambda w: w.describe())
def test_weighted_scatter(w):
    dims, bufs, g, x = _setup(w)
    yp = torch.randn((bufs.P, w.hidden), device="cuda").to(torch.bfloat16)
    y = torch.empty_like(x)
    B.dmoe_padded_scatter(dims, yp, None, bufs.map, bufs.map.weights, y)
    torch.cuda.synchronize()
    ypn = to_np(yp).astype(np.float64)
    wts = g["weights"].astype(np.float64)
    rows = g["dest_row"].reshape(w.T, w.top_k)
    ref = np.einsum("ts,tsh->th", wts, ypn[rows])
    got = to_np(y).astype(np.float64)
    # one bf16 rounding of an fp32 sum: within 2^-8 relative, plus fp32 summation slack
    assert (np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5).all()


def _add_round_f32(a: torch.Tensor, p: torch.Tensor) -> torch.Tensor:
    """fp32 a + p rounded once to fp32 (round to nearest even), p a float64 tensor holding an
    exact product: the double sum plus its exact remainder (two-sum), then a correction where
    the double sum sits exactly halfway between two floats."""
    a = a.double()
    s = a + p
    bb = s - a
    err = (a - (s - bb)) + (p - bb)  # s + err == a + p exactly (finite values)
    r = s.float()
    inf = torch.tensor(float("inf"))
    lo = torch.where(r.double() <= s, r, torch.nextafter(r, -inf))
    hi = torch.nextafter(lo, inf)
    fix = (s == (lo.double() + hi.double()) / 2) & torch.isfinite(err) & (err != 0)
    return torch.where(fix & (err > 0), hi, torch.where(fix & (err < 0), lo, r))


@pytest.mark.parametrize("weighted", [False, True], ids=["unweighted", "weighted"])
@pytest.mark.parametrize("kind", ["normal", "wide", "nonfinite"])
@pytest.mark.parametrize("w", SHAPES[:3], ids=lambda w: w.describe())
def test_weighted_scatter_block_floating_point(w, kind, weighted):
    """Rows in block floating point (fp16 values, one power-of-two scale per row and 128
    columns, the format of the down and dX GEMMs' output): y_t = bf16(sum_s fma(w_s * |scale|,
    value)), bit for bit against the same fp32 sum in slot order.  Unweighted rows with a scale
    that fp16 holds take the kernel's mixed-precision path, the others its converting path.
    "wide" adds zeros, fp16 subnormals and scales from 2^-30 to 2^24 (both paths); "nonfinite"
    marks some groups with scale -1 and puts an inf or a NaN in them."""
    dims, bufs, g, x = _setup(w)
    P, h = bufs.P, w.hidden
    nsc = B.scale_stride(h)  # ceil(h/128) scales per row, padded to a multiple of 4
    gen = torch.Generator(device="cpu").manual_seed(5)
    vals = (torch.randn((P, h), generator=gen) * 4096).to(torch.float16)
    expo = torch.randint(-20, 5, (P, nsc), generator=gen).float()
    if kind == "wide":
        tiny = (torch.randn((P, h), generator=gen) * 2.0 ** -18).to(torch.float16)  # subnormal
        pick = torch.randint(0, 4, (P, h), generator=gen)
        vals = torch.where(pick == 0, tiny, vals)
        vals = torch.where(pick == 1, torch.zeros_like(vals), vals)
        expo = torch.randint(-30, 25, (P, nsc), generator=gen).float()
    scale = torch.pow(2.0, expo)
    if kind == "nonfinite":
        grp = torch.rand((P, nsc), generator=gen) < 0.05
        grp[:, (h + 127) // 128:] = False
        scale = torch.where(grp, torch.full_like(scale, -1.0), scale)
        cols = grp.repeat_interleave(128, dim=1)[:, :h]
        hit = cols & (torch.rand((P, h), generator=gen) < 0.02)
        special = torch.where(torch.rand((P, h), generator=gen) < 0.5,
                              torch.full_like(vals, float("inf")),
                              torch.full_like(vals, float("nan")))
        vals = torch.where(hit, special, vals)
    y = torch.empty_like(x)
    B.dmoe_padded_scatter(dims, vals.cuda(), scale.cuda(), bufs.map,
                          bufs.map.weights if weighted else None, y)
    torch.cuda.synchronize()
    full = vals.double() * scale.abs().double().repeat_interleave(128, dim=1)[:, :h]  # exact
    wts = torch.from_numpy(g["weights"]).float() if weighted else torch.ones(w.T, w.top_k)
    rows = torch.from_numpy(g["dest_row"].reshape(w.T, w.top_k)).long()
    acc = torch.zeros((w.T, h), dtype=torch.float32)
    for s in range(w.top_k):  # w * |scale| * value (exact in double), one rounding: an fma
        acc = _add_round_f32(acc, wts[:, s:s + 1].double() * full[rows[:, s]])
    ref = acc.to(torch.bfloat16)
    got = y.cpu()
    nan_ref, nan_got = torch.isnan(ref), torch.isnan(got)
    assert torch.equal(nan_ref, nan_got)
    if kind == "nonfinite":
        assert nan_ref.any() and torch.isinf(ref).any()
    assert torch.equal(torch.where(nan_got, 0, got.view(torch.int16)),
                       torch.where(nan_ref, 0, ref.view(torch.int16)))
