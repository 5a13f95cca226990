"""CPU oracle for the dropless-MoE (dMoE) expert layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import this package.  The product path never does, and this package
imports nothing from the product package: the two share no code.

The arithmetic lives in ``dmoe_oracle.c`` (plain C, double accumulation, built with gcc and
no fast-math); this module only marshals numpy arrays into it with ctypes.  Every routine
cites the passage of the pages it follows, in the C source:

* ``route``           -- top-k of softmax over the E logits (Fast-LLM issue #56 "[feat]
                         Support sparse copy for a large number of experts", error log:
                         ``(scores, top_experts)``; MegaBlocks walkthrough "02 · dropless MoE
                         与 block-sparse 重构" §4.5 ``router(x)``).
* ``sparse_map``      -- histogram, cumsum, round_up to 128, stable sort, the padded-row index
                         math, the block->expert table (walkthrough §2, §4.1-§4.3).
* ``round_tokens``    -- tile-aware token rounding of a routing (SonicMoE abstract).
* ``forward``         -- per-token loop y_t = sum_s w_ts W2_e(silu(W1_e x_t) * W3_e x_t)
                         (walkthrough §4.5 schematic, gated SiLU per the issue's config).
* ``backward``, ``backward_tokens``, ``wgrad_elements``, ``wgrad_expert`` -- chain rule per
                         (token, slot);
                         role swap and routing-weight gradient of walkthrough §4.2, activation
                         recompute of §4.4.
* ``router_logits``, ``router_backward`` -- the linear router whose output is the issue's
                         ``(scores, top_experts)`` (walkthrough §4.5 ``router(x)``), and the
                         chain rule through the softmax routing weights into the logits, the
                         router input and the router weight.

Pins (tests/test_oracle_pins.py) tie every routine to something other than itself: brute
force, closed forms, library special cases, the walkthrough's block diagram (§3), invariants
(§2, §5) and central finite differences.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dmoe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

BLOCKING = 128


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP on, no fast-math, no FP contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-std=c11", "-o", _LIB_PATH + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_route.argtypes = [I, I, I, I, P, P, P]
        lib.oracle_sparse_map.argtypes = [I, I, I, P, P, P, P, P, P, P, P, I, P]
        lib.oracle_forward.argtypes = [I, I, I, I, I, P, P, P, P, P, P, I, P, P, P, I]
        lib.oracle_backward.argtypes = [I, I, I, I, I, P, P, P, P, P, P, P, P, P, P, P, P]
        lib.oracle_backward_tokens.argtypes = [I, I, I, I, I, P, P, P, P, P, P, P, I, P, P, P, I]
        lib.oracle_wgrad_elements.argtypes = [I, I, I, I, I, P, P, P, P, P, P, P, I, P, P, I]
        lib.oracle_wgrad_expert.argtypes = [I, I, I, I, I, P, P, P, P, P, P, P, I, P, P, P, I]
        lib.oracle_round_tokens.argtypes = [I, I, I, I, P, P, I, P, P]
        lib.oracle_router_logits.argtypes = [I, I, I, P, P, I, P, P, I]
        lib.oracle_router_backward.argtypes = [I, I, I, I, I, P, P, P, P, P, P, I, P, P, I, P, P, I]
        for fn in (lib.oracle_route, lib.oracle_sparse_map, lib.oracle_forward, lib.oracle_backward,
                   lib.oracle_backward_tokens, lib.oracle_wgrad_elements, lib.oracle_wgrad_expert,
                   lib.oracle_round_tokens,
                   lib.oracle_max_threads,
                   lib.oracle_router_logits, lib.oracle_router_backward):
            fn.restype = ctypes.c_int
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _f32(a) -> np.ndarray:
    """fp32 C-contiguous view/copy (bf16 inputs are widened exactly by the caller)."""
    return np.ascontiguousarray(a, dtype=np.float32)


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.int32)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def padded_rows_max(T: int, E: int, k: int) -> int:
    """Static bound on the padded row count: floor((T*k + 127*E)/128)*128."""
    return ((T * k + (BLOCKING - 1) * E) // BLOCKING) * BLOCKING


def route(logits, k: int, renorm: bool = False):
    """logits [T,E] -> (top_experts [T,k] int32, weights [T,k] float64); renorm: weights are
    the softmax over the k chosen logits (they sum to 1)."""
    lg = _f32(logits)
    T, E = lg.shape
    top = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    rc = _load().oracle_route(T, E, k, int(bool(renorm)), _p(lg), _p(top), _p(w))
    if rc != 0:
        raise ValueError(f"oracle_route failed ({rc})")
    return top, w


def round_tokens(logits, top_experts, block: int = BLOCKING, kmax: int | None = None):
    """Tile-aware token rounding of a top-k routing (dmoe_oracle.c, oracle_round_tokens).
    Returns (top [T, kmax] int32 with -1 in unused positions, weights [T, kmax] float64)."""
    lg, top = _f32(logits), _i32(top_experts)
    T, E = lg.shape
    k = top.shape[1]
    kmax = E if kmax is None else kmax
    out_top = np.empty((T, kmax), np.int32)
    out_w = np.empty((T, kmax), np.float64)
    rc = _load().oracle_round_tokens(T, E, k, int(block), _p(lg), _p(top), kmax, _p(out_top),
                                     _p(out_w))
    if rc < 0:
        raise ValueError(f"oracle_round_tokens failed ({rc})")
    return out_top[:, :max(rc, 1)].copy(), out_w[:, :max(rc, 1)].copy()


def compact_entries(top, weights):
    """Token-major entry list of a routing with absent (-1) positions: (offsets [T+1],
    experts [N'], weights [N']), each token's entries in position order."""
    top = np.asarray(top)
    keep = top >= 0
    offsets = np.concatenate([[0], np.cumsum(keep.sum(1))]).astype(np.int32)
    return offsets, top[keep].astype(np.int32), np.asarray(weights)[keep]


def sparse_map(top_experts, E: int, nblk_cap: int | None = None) -> dict:
    """top_experts [T,k] -> dict of the sparse-map arrays (see dmoe_oracle.c)."""
    top = _i32(top_experts)
    T, k = top.shape
    N = T * k
    if nblk_cap is None:
        nblk_cap = padded_rows_max(T, E, k) // BLOCKING
    out = dict(
        tokens_per_expert=np.empty(E, np.int32), bins=np.empty(E, np.int32),
        padded_bins=np.empty(E, np.int32), indices=np.empty(N, np.int32),
        bin_ids=np.empty(N, np.int32), dest_row=np.empty(N, np.int32),
        block_expert=np.empty(max(nblk_cap, 1), np.int32), num_blocks=np.empty(1, np.int32))
    rc = _load().oracle_sparse_map(
        T, E, k, _p(top), _p(out["tokens_per_expert"]), _p(out["bins"]), _p(out["padded_bins"]),
        _p(out["indices"]), _p(out["bin_ids"]), _p(out["dest_row"]), _p(out["block_expert"]),
        nblk_cap, _p(out["num_blocks"]))
    if rc != 0:
        raise ValueError(f"oracle_sparse_map failed ({rc})")
    out["block_expert"] = out["block_expert"][:nblk_cap]
    out["num_blocks"] = int(out["num_blocks"][0])
    return out


def forward(x, W1, W3, W2, top_experts, weights, tokens=None, want_yts=False, threads=1):
    """Per-token forward.  x [T,h]; W1, W3 [E,f,h]; W2 [E,h,f]; top/weights [T,k].

    Returns y [n,h] float64 for the listed tokens (all when ``tokens`` is None) and, if
    ``want_yts``, the per-slot expert outputs [n,k,h]."""
    x, W1, W3, W2 = _f32(x), _f32(W1), _f32(W3), _f32(W2)
    top, w = _i32(top_experts), _f64(weights)
    T, h = x.shape
    E, f, _ = W1.shape
    k = top.shape[1]
    toks = None if tokens is None else _i32(tokens)
    n = T if toks is None else toks.shape[0]
    y = np.empty((n, h), np.float64)
    yts = np.empty((n, k, h), np.float64) if want_yts else None
    rc = _load().oracle_forward(T, h, f, E, k, _p(x), _p(W1), _p(W3), _p(W2), _p(top), _p(w), n,
                                None if toks is None else _p(toks), _p(y),
                                None if yts is None else _p(yts), int(threads))
    if rc != 0:
        raise RuntimeError(f"oracle_forward failed ({rc})")
    return (y, yts) if want_yts else y


def backward(x, dy, W1, W3, W2, top_experts, weights):
    """Full backward (small shapes).  Returns dict dx, dW1, dW3, dW2, dw (float64)."""
    x, dy, W1, W3, W2 = _f32(x), _f32(dy), _f32(W1), _f32(W3), _f32(W2)
    top, w = _i32(top_experts), _f64(weights)
    T, h = x.shape
    E, f, _ = W1.shape
    k = top.shape[1]
    out = dict(dx=np.empty((T, h)), dW1=np.empty((E, f, h)), dW3=np.empty((E, f, h)),
               dW2=np.empty((E, h, f)), dw=np.empty((T, k)))
    rc = _load().oracle_backward(T, h, f, E, k, _p(x), _p(dy), _p(W1), _p(W3), _p(W2), _p(top),
                                 _p(w), _p(out["dx"]), _p(out["dW1"]), _p(out["dW3"]),
                                 _p(out["dW2"]), _p(out["dw"]))
    if rc != 0:
        raise RuntimeError(f"oracle_backward failed ({rc})")
    return out


def backward_tokens(x, dy, W1, W3, W2, top_experts, weights, tokens, threads=1):
    """dx [n,h] and dw [n,k] (float64) for the listed tokens."""
    x, dy, W1, W3, W2 = _f32(x), _f32(dy), _f32(W1), _f32(W3), _f32(W2)
    top, w, toks = _i32(top_experts), _f64(weights), _i32(tokens)
    T, h = x.shape
    E, f, _ = W1.shape
    k = top.shape[1]
    n = toks.shape[0]
    dx = np.empty((n, h))
    dw = np.empty((n, k))
    rc = _load().oracle_backward_tokens(T, h, f, E, k, _p(x), _p(dy), _p(W1), _p(W3), _p(W2),
                                        _p(top), _p(w), n, _p(toks), _p(dx), _p(dw), int(threads))
    if rc != 0:
        raise RuntimeError(f"oracle_backward_tokens failed ({rc})")
    return dx, dw


def wgrad_elements(x, dy, W1, W3, W2, top_experts, weights, queries, threads=1):
    """queries [n,4] rows (which in {1,2,3}, e, r, c) -> float64 [n] weight-gradient elements."""
    x, dy, W1, W3, W2 = _f32(x), _f32(dy), _f32(W1), _f32(W3), _f32(W2)
    top, w, q = _i32(top_experts), _f64(weights), _i32(queries)
    T, h = x.shape
    E, f, _ = W1.shape
    k = top.shape[1]
    out = np.empty(q.shape[0])
    rc = _load().oracle_wgrad_elements(T, h, f, E, k, _p(x), _p(dy), _p(W1), _p(W3), _p(W2),
                                       _p(top), _p(w), q.shape[0], _p(q), _p(out), int(threads))
    if rc != 0:
        raise RuntimeError(f"oracle_wgrad_elements failed ({rc})")
    return out


def wgrad_expert(x, dy, W1, W3, W2, top_experts, weights, e: int, threads=1):
    """Whole weight-gradient slabs of expert ``e``: (dW1_e [f,h], dW3_e [f,h], dW2_e [h,f]),
    float64, each element summed over the expert's entries in entry order."""
    x, dy, W1, W3, W2 = _f32(x), _f32(dy), _f32(W1), _f32(W3), _f32(W2)
    top, w = _i32(top_experts), _f64(weights)
    T, h = x.shape
    E, f, _ = W1.shape
    k = top.shape[1]
    d1, d3, d2 = np.empty((f, h)), np.empty((f, h)), np.empty((h, f))
    rc = _load().oracle_wgrad_expert(T, h, f, E, k, _p(x), _p(dy), _p(W1), _p(W3), _p(W2),
                                     _p(top), _p(w), int(e), _p(d1), _p(d3), _p(d2), int(threads))
    if rc != 0:
        raise RuntimeError(f"oracle_wgrad_expert failed ({rc})")
    return d1, d3, d2


def router_logits(x, Wr, tokens=None, threads=1):
    """logits [n,E] float64 = x[tokens] Wr^T (all tokens when ``tokens`` is None)."""
    x, Wr = _f32(x), _f32(Wr)
    T, h = x.shape
    E = Wr.shape[0]
    toks = None if tokens is None else _i32(tokens)
    n = T if toks is None else toks.shape[0]
    out = np.empty((n, E), np.float64)
    rc = _load().oracle_router_logits(T, h, E, _p(x), _p(Wr), n,
                                      None if toks is None else _p(toks), _p(out), int(threads))
    if rc != 0:
        raise ValueError(f"oracle_router_logits failed ({rc})")
    return out


def router_backward(x, Wr, logits, top_experts, dweights, tokens=None, elems=None,
                    want_dx=True, want_dwr=True, threads=1, renorm=False):
    """Gradient through the routing weights.  Returns dict dlogits [T,E], dx_r ([n,h] for
    ``tokens`` or [T,h]) and dWr ([len(elems)] for ``elems`` = [(e, c), ...] or [E,h]),
    all float64."""
    x, Wr, lg = _f32(x), _f32(Wr), _f32(logits)
    top, dw = _i32(top_experts), _f64(dweights)
    T, h = x.shape
    E = Wr.shape[0]
    k = top.shape[1]
    dl = np.empty((T, E), np.float64)
    toks = None if tokens is None else _i32(tokens)
    n_tok = T if toks is None else toks.shape[0]
    dx = np.empty((n_tok, h), np.float64) if want_dx else None
    el = None if elems is None else _i32(np.asarray(elems).reshape(-1, 2))
    n_el = E * h if el is None else el.shape[0]
    dwr = np.empty(n_el, np.float64) if want_dwr else None
    rc = _load().oracle_router_backward(
        T, h, E, k, int(bool(renorm)), _p(x), _p(Wr), _p(lg), _p(top), _p(dw), _p(dl), n_tok,
        None if toks is None else _p(toks), None if dx is None else _p(dx),
        n_el, None if el is None else _p(el), None if dwr is None else _p(dwr), int(threads))
    if rc != 0:
        raise ValueError(f"oracle_router_backward failed ({rc})")
    out = dict(dlogits=dl)
    if dx is not None:
        out["dx_r"] = dx
    if dwr is not None:
        out["dWr"] = dwr if el is not None else dwr.reshape(E, h)
    return out

