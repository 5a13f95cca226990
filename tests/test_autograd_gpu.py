"""The autograd wrapper: its output and every gradient equal the direct C-ABI calls bit for bit
(the weight gradients as stored in the weights' bf16), and its logit gradient matches the
oracle's gradient through the routing softmax."""
import numpy as np
import pytest
import torch

import oracle
from dropless_mixture_experts_dmoe_b200 import autograd as A
from dropless_mixture_experts_dmoe_b200 import binding as B
from dropless_mixture_experts_dmoe_b200.workloads import custom, make_inputs

from helpers import assert_close, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("renorm", [False, True], ids=["softmax", "renormalised"])
@pytest.mark.parametrize("w", [custom(300, 256, 256, 16, 4), custom(1000, 384, 128, 8, 2)],
                         ids=lambda w: w.describe())
def test_autograd_matches_direct_calls(w, renorm):
    flags = B.ROUTE_RENORMALIZE if renorm else 0
    inp = make_inputs(w, with_dy=True)
    dev = {k: v.cuda() for k, v in inp.items()}
    leaves = {k: dev[k].clone().requires_grad_(True) for k in ("x", "logits", "w1", "w3", "w2")}
    y = A.dmoe(leaves["x"], leaves["logits"], leaves["w1"], leaves["w3"], leaves["w2"], w.top_k,
               flags)
    (y.float() * dev["dy"].float()).sum().backward()
    torch.cuda.synchronize()
    assert A.last_status() == 0

    # the same steps through the C ABI
    dims = B.make_dims(w.T, w.hidden, w.ffn, w.E, w.top_k, flags=flags)
    bufs = B.Buffers(dims, train=True)
    bf, f32 = dict(dtype=torch.bfloat16, device="cuda"), dict(dtype=torch.float32, device="cuda")
    y_ref = torch.empty((w.T, w.hidden), **bf)
    B.dmoe_sparse_map(dims, dev["logits"], bufs.map, bufs.ws_map)
    B.dmoe_forward(dims, dev["x"], dev["w1"], dev["w3"], dev["w2"], bufs.map, y_ref,
                   saved=bufs.saved, ws=bufs.ws_fwd)
    g = dict(dx=torch.empty_like(y_ref), dw1=torch.empty((w.E, w.ffn, w.hidden), **f32),
             dw3=torch.empty((w.E, w.ffn, w.hidden), **f32),
             dw2=torch.empty((w.E, w.hidden, w.ffn), **f32), dw=torch.empty((w.T, w.top_k), **f32))
    B.dmoe_backward(dims, dev["dy"], dev["w1"], dev["w3"], dev["w2"], bufs.map, bufs.saved,
                    g["dx"], g["dw1"], g["dw3"], g["dw2"], g["dw"], bufs.ws_bwd)
    dl = torch.empty_like(dev["logits"])
    B.dmoe_router_dlogits(dims, dev["logits"], bufs.map, g["dw"], dl)
    torch.cuda.synchronize()

    def same(a, b):
        return torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert same(y, y_ref)
    assert same(leaves["x"].grad, g["dx"])
    assert same(leaves["logits"].grad, dl)
    for name, key in (("w1", "dw1"), ("w3", "dw3"), ("w2", "dw2")):
        assert leaves[name].grad.dtype == torch.bfloat16
        assert same(leaves[name].grad, g[key].to(torch.bfloat16)), name

    # the logit gradient against the oracle, given the GPU's routing-weight gradients
    lg = inp["logits"].float().numpy()
    top, _ = oracle.route(lg, w.top_k, renorm=renorm)
    wr = np.zeros((w.E, w.hidden), np.float32)  # only dlogits is asked for
    r = oracle.router_backward(inp["x"].float().numpy(), wr, lg, top,
                               g["dw"].double().cpu().numpy(), want_dx=False, want_dwr=False,
                               renorm=renorm)
    # dlogits: fp32 arithmetic rounded once to bf16 per element
    got, ref = to_np(leaves["logits"].grad), r["dlogits"]
    assert (np.abs(got - ref) <= 2.0 ** -7 * np.abs(ref) + 1e-4 * np.abs(ref).max()).all()
    assert_close(got, ref, "dlogits")


def test_autograd_rejects_bad_inputs():
    x = torch.zeros(4, 128, dtype=torch.float32, device="cuda")
    with pytest.raises(ValueError):
        A.dmoe(x, x, x, x, x, 1)
