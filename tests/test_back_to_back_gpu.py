"""Steps issued back to back on one stream, with no synchronisation between them, give the same
bits as steps run in isolation.  Each kernel may be scheduled before the previous one has
finished (programmatic dependent launch); this checks that no kernel reads or writes global
memory before the earlier ones are complete: the next step's map rewrites the routing
weights, rows and block table that the previous step's copies and GEMMs read, and its
forward overwrites the padded buffers the previous backward still reads."""
import pytest
import torch

from dropless_mixture_experts_dmoe_b200 import binding as B
from dropless_mixture_experts_dmoe_b200.workloads import custom, make_inputs

from helpers import dims_of

pytestmark = pytest.mark.gpu


def _outputs(w):
    bf = dict(dtype=torch.bfloat16, device="cuda")
    f32 = dict(dtype=torch.float32, device="cuda")
    return dict(y=torch.empty((w.T, w.hidden), **bf), dx=torch.empty((w.T, w.hidden), **bf),
                dw1=torch.empty((w.E, w.ffn, w.hidden), **f32),
                dw3=torch.empty((w.E, w.ffn, w.hidden), **f32),
                dw2=torch.empty((w.E, w.hidden, w.ffn), **f32),
                dw=torch.empty((w.T, w.top_k), **f32))


def _step(dims, dev, bufs, out):
    B.dmoe_sparse_map(dims, dev["logits"], bufs.map, bufs.ws_map)
    B.dmoe_forward(dims, dev["x"], dev["w1"], dev["w3"], dev["w2"], bufs.map, out["y"],
                   saved=bufs.saved, ws=bufs.ws_fwd)
    B.dmoe_backward(dims, dev["dy"], dev["w1"], dev["w3"], dev["w2"], bufs.map, bufs.saved,
                    out["dx"], out["dw1"], out["dw3"], out["dw2"], out["dw"], bufs.ws_bwd)


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


@pytest.mark.parametrize("w", [custom(2048, 256, 256, 64, 8), custom(700, 384, 128, 8, 2)],
                         ids=lambda w: w.describe())
def test_back_to_back_steps_equal_isolated_steps(w):
    dims = dims_of(w)
    # two input sets that route differently; the weights are shared
    sets = []
    for s in range(2):
        inp = make_inputs(w, seed=w.seed + 31 * s, with_dy=True)
        sets.append({k: v.cuda() for k, v in inp.items()})
    for k in ("w1", "w3", "w2"):
        sets[1][k] = sets[0][k]
    bufs = B.Buffers(dims, train=True)
    # isolated: each input set alone, synchronised
    ref = []
    for s in range(2):
        out = _outputs(w)
        _step(dims, sets[s], bufs, out)
        torch.cuda.synchronize()
        ref.append(out)
    # back to back: A B A B A B on the same buffers, one stream, no synchronisation
    outs = [_outputs(w) for _ in range(6)]
    for i, out in enumerate(outs):
        _step(dims, sets[i % 2], bufs, out)
    torch.cuda.synchronize()
    assert int(bufs.map.status.item()) == 0
    for i, out in enumerate(outs):
        for name, v in out.items():
            assert torch.equal(_bits(v), _bits(ref[i % 2][name])), (i, name)
