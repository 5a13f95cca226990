"""The layer's calls inside a CUDA graph: map, forward and backward captured once and
replayed give the eager results bit for bit, and a replay after new inputs are written into
the captured buffers follows the new inputs (nothing is baked into the graph but pointers)."""
import pytest
import torch

from dropless_mixture_experts_dmoe_b200 import binding as B
from dropless_mixture_experts_dmoe_b200.workloads import custom, make_inputs

from helpers import dims_of

pytestmark = pytest.mark.gpu


def _alloc(w, dims):
    bufs = B.Buffers(dims, train=True)
    bf = dict(dtype=torch.bfloat16, device="cuda")
    f32 = dict(dtype=torch.float32, device="cuda")
    out = dict(y=torch.empty((w.T, w.hidden), **bf), dx=torch.empty((w.T, w.hidden), **bf),
               dw1=torch.empty((w.E, w.ffn, w.hidden), **f32),
               dw3=torch.empty((w.E, w.ffn, w.hidden), **f32),
               dw2=torch.empty((w.E, w.hidden, w.ffn), **f32), dw=torch.empty((w.T, w.top_k), **f32))
    return bufs, out


def _step(dims, dev, bufs, out):
    """One training step of the layer on the current stream (eager or being captured)."""
    B.dmoe_sparse_map(dims, dev["logits"], bufs.map, bufs.ws_map)
    B.dmoe_forward(dims, dev["x"], dev["w1"], dev["w3"], dev["w2"], bufs.map, out["y"],
                   saved=bufs.saved, ws=bufs.ws_fwd)
    B.dmoe_backward(dims, dev["dy"], dev["w1"], dev["w3"], dev["w2"], bufs.map, bufs.saved,
                    out["dx"], out["dw1"], out["dw3"], out["dw2"], out["dw"], bufs.ws_bwd)


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


@pytest.mark.parametrize("w", [custom(1000, 256, 384, 16, 4), custom(512, 512, 256, 8, 2)],
                         ids=lambda w: w.describe())
def test_layer_step_replays_from_a_cuda_graph(w):
    dims = dims_of(w)
    inp = make_inputs(w, with_dy=True)
    dev = {k: v.cuda() for k, v in inp.items()}
    # eager reference (also the first call of every launcher, outside any capture)
    bufs_e, ref = _alloc(w, dims)
    _step(dims, dev, bufs_e, ref)
    torch.cuda.synchronize()

    bufs, out = _alloc(w, dims)
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        _step(dims, dev, bufs, out)  # warm the capture stream
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    with torch.cuda.graph(graph):
        _step(dims, dev, bufs, out)
    for v in out.values():  # poison, then the replay must rewrite every output
        v.fill_(float("nan"))
    graph.replay()
    torch.cuda.synchronize()
    assert int(bufs.map.status.item()) == 0
    for k in ref:
        assert torch.equal(_bits(out[k]), _bits(ref[k])), k

    # new inputs written into the captured buffers: the replay follows them
    inp2 = make_inputs(w, seed=w.seed + 77, with_dy=True)
    for k in ("x", "logits", "dy"):
        dev[k].copy_(inp2[k])
    _step(dims, dev, bufs_e, ref)  # eager on the new inputs
    graph.replay()
    torch.cuda.synchronize()
    for k in ref:
        assert torch.equal(_bits(out[k]), _bits(ref[k])), k
    del graph
