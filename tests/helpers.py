"""Shared test helpers: run the CUDA path through the C ABI, run the oracle, compare.

The CUDA side goes through ``dropless_mixture_experts_dmoe_b200.binding`` only; the oracle
side through ``oracle`` only.  Inputs for both come from ``workloads`` (seeded, bf16)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from dropless_mixture_experts_dmoe_b200 import binding as B
from dropless_mixture_experts_dmoe_b200.workloads import Workload

# Float tolerance of the layer's outputs and gradients against the fp32-input oracle
# (relative L2 error and max-abs error relative to the reference RMS).
REL_L2 = 1e-2
MAX_ABS_RMS = 5e-2
# fp32 routing weights (fp32 expf/sum on the GPU, double in the oracle).
WEIGHT_RTOL = 2e-6


def metrics(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    diff = got - ref
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))
    mx = float(np.max(np.abs(diff))) if ref.size else 0.0
    return rel, mx, rms


# Every comparison made through assert_close, (what, rel L2, max-abs / RMS, bound): written to
# the JSON file named by DMOE_PARITY_LOG at the end of the session (tests/conftest.py).
RECORD: list = []


def assert_close(got, ref, what="", max_abs_rms=MAX_ABS_RMS):
    """Relative L2 <= REL_L2 and max-abs <= max_abs_rms * RMS(ref).  The five named workloads
    use MAX_ABS_RMS; stress shapes pass the bound that tests/bf16_model.py derives."""
    rel, mx, rms = metrics(got, ref)
    RECORD.append((what, rel, mx / rms if rms else 0.0, max_abs_rms))
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    assert rel <= REL_L2, f"{what}: relative L2 {rel:.3e} > {REL_L2}"
    assert mx <= max_abs_rms * rms, f"{what}: max abs {mx:.3e} > {max_abs_rms} * RMS {rms:.3e}"
    return rel, mx, rms


def dims_of(w: Workload):
    return B.make_dims(w.T, w.hidden, w.ffn, w.E, w.top_k)


def to_np(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.detach().cpu().numpy()


def gpu_map(dims, logits=None, top_experts=None, bufs=None):
    """Run dmoe_sparse_map; returns (Buffers, dict of numpy arrays)."""
    if bufs is None:
        bufs = B.Buffers(dims, train=True)
    if top_experts is not None:
        bufs.map.top_experts.copy_(torch.as_tensor(top_experts, dtype=torch.int32))
    lg = None if logits is None else logits.cuda()
    B.dmoe_sparse_map(dims, lg, bufs.map, bufs.ws_map)
    torch.cuda.synchronize()
    out = {k: to_np(v) for k, v in bufs.map.as_dict().items()}
    out["num_blocks"] = int(out["num_blocks"][0])
    out["status"] = int(out["status"][0])
    return bufs, out


def compare_map(g: dict, o: dict, top_expected=None):
    """Bit-exact comparison of every integer map array."""
    if top_expected is not None:
        np.testing.assert_array_equal(g["top_experts"], top_expected)
    for k in ("tokens_per_expert", "bins", "padded_bins", "indices", "bin_ids", "dest_row"):
        np.testing.assert_array_equal(g[k], o[k], err_msg=k)
    assert g["num_blocks"] == o["num_blocks"]
    np.testing.assert_array_equal(g["block_expert"], o["block_expert"], err_msg="block_expert")


def oracle_inputs(inp: dict) -> dict:
    """fp32 numpy copies (exact widening of the bf16 inputs) for the oracle."""
    return {k: v.float().numpy() for k, v in inp.items()}


def gpu_forward(dims, inp: dict, train=True):
    """Full layer forward through the C ABI: map (from logits) + dmoe_forward."""
    bufs = B.Buffers(dims, train=train)
    dev = {k: v.cuda() for k, v in inp.items()}
    B.dmoe_sparse_map(dims, dev["logits"], bufs.map, bufs.ws_map)
    y = torch.empty((dims.T, dims.hidden), dtype=torch.bfloat16, device="cuda")
    B.dmoe_forward(dims, dev["x"], dev["w1"], dev["w3"], dev["w2"], bufs.map, y,
                   saved=bufs.saved, ws=bufs.ws_fwd)
    torch.cuda.synchronize()
    return bufs, dev, y


def sample_tokens(top: np.ndarray, E: int, n: int, seed: int = 0) -> np.ndarray:
    """A token sample that touches as many experts as possible plus random tokens,
    including the last token (ragged tail)."""
    rng = np.random.default_rng(seed)
    T = top.shape[0]
    picks = {T - 1, 0}
    seen = set()
    for t in rng.permutation(T):
        if len(picks) >= n:
            break
        if not set(top[t].tolist()) <= seen:
            picks.add(int(t))
            seen |= set(top[t].tolist())
    while len(picks) < min(n, T):
        picks.add(int(rng.integers(T)))
    return np.array(sorted(picks), np.int32)


def tokens_covering_blocks(m: dict, k: int, T: int, n_min: int, seed: int = 0,
                           last_rows: bool = True) -> np.ndarray:
    """Tokens whose entries land in every 128-row block of the map: for each block the token
    of its first real row and (last_rows) of its last real row -- so both halves of every
    pair of blocks, each expert's ragged last block and every column tile of the GEMMs are
    sampled -- plus token 0, token T-1 and random tokens up to n_min."""
    dest = np.asarray(m["dest_row"]).astype(np.int64)
    j = np.nonzero(dest >= 0)[0]
    order = j[np.argsort(dest[j], kind="stable")]
    blk = dest[order] // 128
    _, first = np.unique(blk, return_index=True)
    picks = set((order[first] // k).tolist())
    if last_rows:
        _, last = np.unique(blk[::-1], return_index=True)
        picks |= set((order[len(order) - 1 - last] // k).tolist())
    picks |= {0, T - 1}
    rng = np.random.default_rng(seed)
    while len(picks) < min(n_min, T):
        picks.add(int(rng.integers(T)))
    return np.array(sorted(picks), np.int32)


def gpu_backward(dims, inp: dict):
    """Map + training forward + dmoe_backward through the C ABI.

    Returns (bufs, dev, y, grads) with grads = dict(dx, dw1, dw3, dw2, dw) on the device."""
    bufs, dev, y = gpu_forward(dims, inp, train=True)
    dev["dy"] = inp["dy"].cuda()
    E, f, h, T, k = dims.num_experts, dims.ffn, dims.hidden, dims.T, dims.top_k
    bf = dict(dtype=torch.bfloat16, device="cuda")
    f32 = dict(dtype=torch.float32, device="cuda")
    g = dict(dx=torch.empty((T, h), **bf), dw1=torch.empty((E, f, h), **f32),
             dw3=torch.empty((E, f, h), **f32), dw2=torch.empty((E, h, f), **f32),
             dw=torch.empty((T, k), **f32))
    for v in g.values():  # poison: every output element must be written
        v.fill_(float("nan"))
    B.dmoe_backward(dims, dev["dy"], dev["w1"], dev["w3"], dev["w2"], bufs.map, bufs.saved,
                    g["dx"], g["dw1"], g["dw3"], g["dw2"], g["dw"], bufs.ws_bwd)
    torch.cuda.synchronize()
    return bufs, dev, y, g
