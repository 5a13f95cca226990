"""The allocation-free map entry point against the regular one.

dmoe_sparse_map_noalloc serves callers that cannot allocate a device workspace (a plugin
whose host application owns all device memory, or a loop that must not call cudaMalloc);
it keeps its scratch in a static device array inside the library.  Here it must give the
same map as dmoe_sparse_map (which takes a caller workspace) on two calls in a row with
different inputs, so stale scratch from the first call cannot leak into the second.  This
file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from dropless_mixture_experts_dmoe_b200 import binding as B
from dropless_mixture_experts_dmoe_b200 import build as build_mod
from dropless_mixture_experts_dmoe_b200.workloads import WORKLOADS, make_tensor

pytestmark = pytest.mark.gpu

FIELDS = ("top_experts", "weights", "tokens_per_expert", "bins", "padded_bins", "indices",
          "bin_ids", "dest_row", "block_expert", "num_blocks", "status")


def _snapshot(smap):
    torch.cuda.synchronize()
    return {n: getattr(smap, n).cpu().clone() for n in FIELDS}


def _regular(dims, logits):
    smap = B.SparseMap(dims)
    ws = torch.empty(B.dmoe_workspace_bytes(dims, B.WS_MAP), dtype=torch.uint8, device="cuda")
    B.dmoe_sparse_map(dims, logits, smap, ws)
    return _snapshot(smap)


def test_noalloc_map_matches_regular_two_calls():
    build_mod.build()
    B.load()
    cases = [WORKLOADS[5], WORKLOADS[3]]  # large then smaller: the second call sees stale scratch
    smap_cache = {}
    for w in cases:
        dims = B.make_dims(w.T, w.hidden, w.ffn, w.E, w.top_k)
        logits = make_tensor(w, "logits").cuda()
        ref = _regular(dims, logits)
        smap = smap_cache.setdefault(w.name, B.SparseMap(dims))
        for name in FIELDS:
            getattr(smap, name).fill_(-7)
        B.dmoe_sparse_map_noalloc(dims, logits, smap)
        got = _snapshot(smap)
        # same kernels and arithmetic as the regular entry point: every integer array and
        # the fp32 routing weights must be identical (tolerance 0)
        for name in FIELDS:
            assert torch.equal(got[name], ref[name]), name
        assert int(got["status"][0]) == 0


def test_noalloc_map_given_top_experts_and_limit():
    build_mod.build()
    lib = B.load()
    w = WORKLOADS[4]
    dims = B.make_dims(w.T, w.hidden, w.ffn, w.E, w.top_k)
    logits = make_tensor(w, "logits").cuda()
    ref = _regular(dims, logits)
    smap = B.SparseMap(dims)
    smap.top_experts.copy_(ref["top_experts"].cuda())
    B.dmoe_sparse_map_noalloc(dims, None, smap)  # top_experts given, weights untouched
    got = _snapshot(smap)
    for name in ("tokens_per_expert", "bins", "padded_bins", "indices", "bin_ids", "dest_row",
                 "block_expert", "num_blocks"):
        assert torch.equal(got[name], ref[name]), name
    # beyond the static capacity: rejected on the host before any launch
    big = B.make_dims(262144, 128, 128, 1024, 8)
    rc = lib.dmoe_sparse_map_noalloc(ctypes.byref(big), None, ctypes.byref(smap.c), None)
    assert rc == -4  # DMOE_ERR_WORKSPACE
    assert np.ceil(262144 / 64) * 1024 * 4 > (1 << 20)
