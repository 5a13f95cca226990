"""Failure detection on the GPU without a fault: a bounded in-kernel wait is made to run out
on purpose (the pair leaders of one GEMM launch withhold their first operand stage); the
kernel must report DMOE_STATUS_TIMEOUT through the status word, return, and leave the
context usable for a clean run that still matches the oracle."""
import time

import pytest
import torch

import oracle
from dropless_mixture_experts_dmoe_b200 import binding as B
from dropless_mixture_experts_dmoe_b200.workloads import WORKLOADS, custom, make_inputs

from helpers import assert_close, dims_of, gpu_forward, oracle_inputs, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("w", [WORKLOADS[1], custom(600, 256, 384, 8, 2)],
                         ids=lambda w: w.describe())
def test_injected_stall_reports_timeout_and_context_survives(w):
    inp = make_inputs(w)
    dims = dims_of(w)
    bufs = B.Buffers(dims, train=False)
    dev = {k: v.cuda() for k, v in inp.items()}
    y = torch.empty((w.T, w.hidden), dtype=torch.bfloat16, device="cuda")
    B.dmoe_sparse_map(dims, dev["logits"], bufs.map, bufs.ws_map)
    torch.cuda.synchronize()
    assert int(bufs.map.status.item()) == 0
    B.dmoe_debug_inject_stall(True)  # consumed by the GLU GEMM launch of this forward
    t0 = time.time()
    B.dmoe_forward(dims, dev["x"], dev["w1"], dev["w3"], dev["w2"], bufs.map, y, ws=bufs.ws_fwd)
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    status = int(bufs.map.status.item())
    assert status & B.STATUS_TIMEOUT, B.status_string(status)
    assert elapsed < 10.0  # the waits gave up after their short budget
    # the context is still usable and a clean run is correct
    bufs2, dev2, y2 = gpu_forward(dims, inp, train=False)
    assert int(bufs2.map.status.item()) == 0
    o = oracle_inputs(inp)
    top, wts = oracle.route(o["logits"], w.top_k)
    ref = oracle.forward(o["x"], o["w1"], o["w3"], o["w2"], top, wts, threads=8)
    assert_close(to_np(y2), ref, f"y after an injected stall {w.describe()}")
