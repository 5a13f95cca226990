"""Pins for the CPU oracle: each routine checked against something other than itself.

Routing  -- brute force over all k-subsets; all-equal logits; k = E; +0/-0 and NaN order;
            softmax weights against torch's float64 softmax (library special case).
Map      -- the block diagram of the MegaBlocks walkthrough (section 3, golden fixture);
            invariants of sections 2 and 5 (padding <= 127, one expert per 128-row block,
            sum of counts = T*k); numpy's stable argsort (library) for the sorted order; the
            padded-row index math of section 4.2 restated element by element.
Forward  -- closed form with permutation/selection weights (catches transposed operands and
            wrong indices); zero inputs; exact scaling; E = 1, k = 1 against torch float64
            (textbook gated MLP); invariance under relabelling experts.
Backward -- central finite differences of the oracle's own forward (in double) for x, W1,
            W3, W2 and the routing weights; dw = <dy, y_ts>; linearity in dy; the sampled
            routines against the full backward; whole per-expert weight-gradient slabs
            against torch float64 autograd of the layer's composition.
Router   -- logits: one-hot tokens read a column of the router weight (closed form), numpy's
            float64 matmul (library); gradient through the routing weights: central finite
            differences of sum dw * softmax(x Wr^T)[picks] in the logits, x and Wr; torch
            float64 autograd of the same composition; shift invariance (each token's logit
            gradient sums to zero); k = E with equal dw gives zero; sampled = full.
Token rounding (variant flag) -- every count a multiple of the tile and the nearest one (ties
            up), the dropped / added entries against sorted() of the rank key, slot order kept,
            weights against torch's float64 softmax, block 1 = identity; absent positions (-1)
            contribute nothing in the forward and backward.
Renormalised routing (variant flag) -- weights sum to 1, their ratios are exp(l_i - l_j),
            k = 1 gives 1 and k = E gives the plain softmax; torch float64 softmax over the
            chosen logits; its logit gradient by finite differences and autograd, zero outside
            the chosen experts.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------------------
# routing
# ----------------------------------------------------------------------------------------

def _beats(a, ia, b, ib):
    """Total order used for selection: larger value first, NaN lowest, then lower index."""
    if math.isnan(a) and math.isnan(b):
        return ia < ib
    if math.isnan(a):
        return False
    if math.isnan(b):
        return True
    if a != b:
        return a > b
    return ia < ib


def test_route_brute_force_subsets(oracle_mod):
    rng = np.random.default_rng(7)
    vals = np.array([-1.5, -0.0, 0.0, 0.25, 0.25, 1.0, 2.0, -np.inf], dtype=np.float32)
    for E in (1, 2, 3, 5, 8):
        for k in range(1, E + 1):
            logits = rng.choice(vals, size=(64, E)).astype(np.float32)
            top, _ = oracle_mod.route(logits, k)
            for t in range(64):
                l = [float(v) for v in logits[t]]
                dominant = []
                for S in itertools.combinations(range(E), k):
                    rest = [e for e in range(E) if e not in S]
                    if all(_beats(l[a], a, l[b], b) for a in S for b in rest):
                        dominant.append(set(S))
                assert len(dominant) == 1
                assert set(top[t].tolist()) == dominant[0]
                for s in range(k - 1):  # slot order follows the same total order
                    a, b = top[t, s], top[t, s + 1]
                    assert _beats(l[a], a, l[b], b)


def test_route_all_equal_logits(oracle_mod):
    for E, k in ((8, 2), (64, 8), (256, 8), (4, 4)):
        logits = np.full((5, E), 0.375, np.float32)
        top, w = oracle_mod.route(logits, k)
        assert (top == np.arange(k)[None, :]).all()
        assert (w.astype(np.float32) == np.float32(1.0 / E)).all()


def test_route_k_equals_E_descending(oracle_mod):
    rng = np.random.default_rng(3)
    logits = rng.standard_normal((32, 6)).astype(np.float32)
    top, _ = oracle_mod.route(logits, 6)
    # library special case: a stable descending argsort (no ties in continuous draws)
    ref = np.argsort(-logits, axis=1, kind="stable")
    assert (top == ref).all()


def test_route_signed_zero_and_nan(oracle_mod):
    top, _ = oracle_mod.route(np.array([[-0.0, 0.0, -1.0]], np.float32), 1)
    assert top[0, 0] == 0  # -0 == +0: the lower index wins
    top, _ = oracle_mod.route(np.array([[0.0, -0.0, -1.0]], np.float32), 2)
    assert top[0].tolist() == [0, 1]
    top, _ = oracle_mod.route(np.array([[np.nan, -np.inf, -3.0]], np.float32), 3)
    assert top[0].tolist() == [2, 1, 0]  # NaN ranks below -inf


def test_route_weights_match_library_softmax(oracle_mod):
    rng = np.random.default_rng(11)
    for E, k in ((8, 2), (64, 8), (256, 8)):
        logits = torch.randn(128, E, generator=torch.Generator().manual_seed(E)).to(torch.bfloat16).float()
        top, w = oracle_mod.route(logits.numpy(), k)
        sm = torch.softmax(logits.double(), dim=1).numpy()
        ref = np.take_along_axis(sm, top.astype(np.int64), axis=1)
        np.testing.assert_allclose(w, ref, rtol=1e-13, atol=0)
        assert (w.sum(1) <= 1 + 1e-12).all()  # no renormalisation over the chosen k


# ----------------------------------------------------------------------------------------
# sparse map
# ----------------------------------------------------------------------------------------

def test_map_block_diagram_golden(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "block_diagram.json")))
    E = g["E"]
    top = np.concatenate([np.full(c, e, np.int32) for e, c in enumerate(g["counts"])])
    np.random.default_rng(0).shuffle(top)
    m = oracle_mod.sparse_map(top[:, None], E)
    assert m["tokens_per_expert"].tolist() == g["counts"]
    assert m["bins"].tolist() == g["expected_bins"]
    assert m["padded_bins"].tolist() == g["expected_padded_bins"]
    assert np.diff([0] + m["padded_bins"].tolist()).tolist() == g["expected_padded_tokens_per_expert"]
    assert m["num_blocks"] == g["expected_num_blocks"]
    nb = m["num_blocks"]
    assert m["block_expert"][:nb].tolist() == g["expected_block_expert"]
    assert (m["block_expert"][nb:] == -1).all()
    cb = g["ffn"] // 128
    cols = [[int(e) * cb + c for c in range(cb)] for e in m["block_expert"][:nb]]
    assert cols == g["expected_column_blocks"]


def _check_map_invariants(top, E, m):
    T, k = top.shape
    N = T * k
    c = m["tokens_per_expert"].astype(np.int64)
    assert c.sum() == N
    assert (c == np.bincount(top.ravel(), minlength=E)).all()
    padded = np.diff(np.concatenate([[0], m["padded_bins"].astype(np.int64)]))
    assert (padded % 128 == 0).all()
    assert ((padded - c >= 0) & (padded - c <= 127)).all()
    assert (m["bins"] == np.cumsum(c)).all()
    # stable sort: numpy's stable argsort is the library special case
    assert (m["indices"] == np.argsort(top.ravel(), kind="stable")).all()
    assert (m["bin_ids"] == top.ravel()[m["indices"]]).all()
    assert (np.diff(m["bin_ids"]) >= 0).all()
    # the index math of section 4.2, element by element
    bins_ex = np.concatenate([[0], m["bins"][:-1]])
    pb_ex = np.concatenate([[0], m["padded_bins"][:-1]])
    i = np.arange(N)
    e = m["bin_ids"]
    dest = np.empty(N, np.int64)
    dest[m["indices"]] = (i - bins_ex[e]) + pb_ex[e]
    assert (m["dest_row"] == dest).all()
    P = int(m["padded_bins"][-1])
    assert len(set(m["dest_row"].tolist())) == N and m["dest_row"].min() >= 0 and m["dest_row"].max() < P
    # every 128-row block belongs to exactly one expert (section 2)
    nb = m["num_blocks"]
    assert nb * 128 == P
    owner = np.full(P, -1)
    owner[m["dest_row"]] = top.ravel()
    for b in range(nb):
        rows = owner[b * 128:(b + 1) * 128]
        real = rows[rows >= 0]
        assert len(real) > 0 and (real == m["block_expert"][b]).all()
    assert (m["block_expert"][nb:] == -1).all()


@pytest.mark.parametrize("T,E,k,seed", [(256, 8, 2, 0), (1000, 64, 8, 1), (37, 300, 3, 2),
                                         (300, 1, 1, 3), (129, 5, 5, 4), (5000, 256, 8, 5)])
def test_map_invariants_random(oracle_mod, T, E, k, seed):
    rng = np.random.default_rng(seed)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    top, _ = oracle_mod.route(logits, k)
    m = oracle_mod.sparse_map(top, E)
    _check_map_invariants(top, E, m)


def test_map_skewed_and_empty_experts(oracle_mod):
    T, E, k = 700, 16, 2
    top = np.zeros((T, k), np.int32)
    top[:, 1] = 1 + (np.arange(T) % 3)  # experts 4..15 are empty, expert 0 holds every token
    m = oracle_mod.sparse_map(top, E)
    _check_map_invariants(top, E, m)
    assert (m["tokens_per_expert"][4:] == 0).all()


def test_map_rejects_bad_expert(oracle_mod):
    with pytest.raises(ValueError):
        oracle_mod.sparse_map(np.array([[0], [3]], np.int32), 3)


# ----------------------------------------------------------------------------------------
# forward
# ----------------------------------------------------------------------------------------

def _silu(z):
    return z / (1.0 + np.exp(-z))


def test_forward_closed_form_selection_weights(oracle_mod):
    """Weights that select one input element per output: the FFN is then an elementwise
    closed form, and any transposed operand or wrong index changes it."""
    rng = np.random.default_rng(5)
    T, h, f, E, k = 16, 128, 256, 3, 2
    x = rng.standard_normal((T, h)).astype(np.float32)
    W1 = np.zeros((E, f, h), np.float32)
    W3 = np.zeros((E, f, h), np.float32)
    W2 = np.zeros((E, h, f), np.float32)
    p1 = rng.integers(0, h, (E, f))
    p3 = rng.integers(0, h, (E, f))
    p2 = rng.integers(0, f, (E, h))
    al, be, ga = [np.float32(v) for v in (0.75, -1.25, 0.5)]
    for e in range(E):
        W1[e, np.arange(f), p1[e]] = al * (e + 1)
        W3[e, np.arange(f), p3[e]] = be
        W2[e, np.arange(h), p2[e]] = ga * (e + 2)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    top, w = oracle_mod.route(logits, k)
    y = oracle_mod.forward(x, W1, W3, W2, top, w)
    ref = np.zeros((T, h))
    for t in range(T):
        for s in range(k):
            e = top[t, s]
            xt = x[t].astype(np.float64)
            hh = _silu(float(al) * (e + 1) * xt[p1[e]]) * (float(be) * xt[p3[e]])
            ref[t] += w[t, s] * float(ga) * (e + 2) * hh[p2[e]]
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-14)


def _rand_layer(rng, T, h, f, E, k, scale=0.05):
    x = rng.standard_normal((T, h)).astype(np.float32)
    W1 = (scale * rng.standard_normal((E, f, h))).astype(np.float32)
    W3 = (scale * rng.standard_normal((E, f, h))).astype(np.float32)
    W2 = (scale * rng.standard_normal((E, h, f))).astype(np.float32)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    return x, W1, W3, W2, logits


def test_forward_zero_and_scaling(oracle_mod):
    rng = np.random.default_rng(9)
    x, W1, W3, W2, logits = _rand_layer(rng, 12, 128, 128, 4, 2)
    top, w = oracle_mod.route(logits, 2)
    assert (oracle_mod.forward(np.zeros_like(x), W1, W3, W2, top, w) == 0).all()
    assert (oracle_mod.forward(x, W1, W3, np.zeros_like(W2), top, w) == 0).all()
    assert (oracle_mod.forward(x, W1, np.zeros_like(W3), W2, top, w) == 0).all()
    y = oracle_mod.forward(x, W1, W3, W2, top, w)
    y2 = oracle_mod.forward(x, W1, W3, 2 * W2, top, w)
    assert (y2 == 2 * y).all()  # scaling W2 by 2 is exact in binary floating point


def test_forward_single_expert_is_textbook_gated_mlp(oracle_mod):
    rng = np.random.default_rng(13)
    x, W1, W3, W2, logits = _rand_layer(rng, 20, 128, 256, 1, 1)
    top, w = oracle_mod.route(logits, 1)
    assert (top == 0).all() and (w == 1.0).all()
    y = oracle_mod.forward(x, W1, W3, W2, top, w)
    X = torch.from_numpy(x).double()
    ref = (torch.nn.functional.silu(X @ torch.from_numpy(W1[0]).double().T)
           * (X @ torch.from_numpy(W3[0]).double().T)) @ torch.from_numpy(W2[0]).double().T
    np.testing.assert_allclose(y, ref.numpy(), rtol=1e-10, atol=1e-12)


def test_forward_expert_relabelling_invariance(oracle_mod):
    rng = np.random.default_rng(17)
    x, W1, W3, W2, logits = _rand_layer(rng, 24, 128, 128, 6, 3)
    top, w = oracle_mod.route(logits, 3)
    y = oracle_mod.forward(x, W1, W3, W2, top, w)
    perm = rng.permutation(6)  # new expert id of old expert e is perm[e]
    inv = np.argsort(perm)
    top2, w2 = oracle_mod.route(logits[:, inv], 3)
    assert (top2 == perm[top]).all()
    y2 = oracle_mod.forward(x, W1[inv], W3[inv], W2[inv], top2, w2)
    np.testing.assert_allclose(y2, y, rtol=1e-12, atol=1e-13)


def test_forward_token_subset_matches_full(oracle_mod):
    rng = np.random.default_rng(19)
    x, W1, W3, W2, logits = _rand_layer(rng, 30, 128, 128, 4, 2)
    top, w = oracle_mod.route(logits, 2)
    y, yts = oracle_mod.forward(x, W1, W3, W2, top, w, want_yts=True, threads=2)
    toks = np.array([29, 0, 7], np.int32)
    ys = oracle_mod.forward(x, W1, W3, W2, top, w, tokens=toks)
    assert (ys == y[toks]).all()
    np.testing.assert_allclose((w[:, :, None] * yts).sum(1), y, rtol=1e-12, atol=1e-14)


# ----------------------------------------------------------------------------------------
# backward
# ----------------------------------------------------------------------------------------

def _loss(oracle_mod, x, W1, W3, W2, top, w, dy):
    return float((oracle_mod.forward(x, W1, W3, W2, top, w) * dy).sum())


def _fd_check(oracle_mod, name, args, grad, idxs, top, w, dy, step):
    x, W1, W3, W2 = args
    for ix in idxs:
        plus = [a.copy() for a in args]
        minus = [a.copy() for a in args]
        i = ["x", "W1", "W3", "W2"].index(name)
        plus[i][ix] += np.float32(step)
        minus[i][ix] -= np.float32(step)
        delta = float(plus[i][ix]) - float(minus[i][ix])
        fd = (_loss(oracle_mod, *plus, top, w, dy) - _loss(oracle_mod, *minus, top, w, dy)) / delta
        assert abs(fd - grad[ix]) <= 2e-6 + 2e-5 * abs(grad[ix]), (name, ix, fd, grad[ix])


def test_backward_finite_differences(oracle_mod):
    rng = np.random.default_rng(23)
    T, h, f, E, k = 8, 128, 128, 4, 2
    x, W1, W3, W2, logits = _rand_layer(rng, T, h, f, E, k, scale=0.1)
    dy = rng.standard_normal((T, h)).astype(np.float32)
    top, w = oracle_mod.route(logits, k)
    g = oracle_mod.backward(x, dy, W1, W3, W2, top, w)
    args = (x, W1, W3, W2)
    pick = lambda shape, n: [tuple(rng.integers(0, s) for s in shape) for _ in range(n)]
    used = sorted(set(top.ravel().tolist()))
    for name, grad, shape in (("x", g["dx"], x.shape), ("W1", g["dW1"], W1.shape),
                              ("W3", g["dW3"], W3.shape), ("W2", g["dW2"], W2.shape)):
        idxs = pick(shape, 12)
        if name != "x":  # make sure most probes land on experts that receive tokens
            idxs = [(used[i % len(used)],) + ix[1:] for i, ix in enumerate(idxs)]
        _fd_check(oracle_mod, name, args, grad, idxs, top, w, dy, step=2.0 ** -7)
    # routing-weight gradient: perturb w directly
    for (t, s) in [(0, 0), (3, 1), (7, 0)]:
        wp, wm = w.copy(), w.copy()
        wp[t, s] += 1e-3
        wm[t, s] -= 1e-3
        fd = (_loss(oracle_mod, *args, top, wp, dy) - _loss(oracle_mod, *args, top, wm, dy)) / 2e-3
        assert abs(fd - g["dw"][t, s]) <= 1e-8 + 1e-8 * abs(fd)
    # unrouted experts get exactly zero gradient
    for e in range(E):
        if e not in used:
            assert (g["dW1"][e] == 0).all() and (g["dW2"][e] == 0).all()


def test_backward_dw_identity_and_linearity(oracle_mod):
    rng = np.random.default_rng(29)
    T, h, f, E, k = 10, 128, 128, 4, 2
    x, W1, W3, W2, logits = _rand_layer(rng, T, h, f, E, k)
    top, w = oracle_mod.route(logits, k)
    dy = rng.standard_normal((T, h)).astype(np.float32)
    g = oracle_mod.backward(x, dy, W1, W3, W2, top, w)
    _, yts = oracle_mod.forward(x, W1, W3, W2, top, w, want_yts=True)
    np.testing.assert_allclose(g["dw"], np.einsum("th,tsh->ts", dy.astype(np.float64), yts),
                               rtol=1e-12, atol=1e-13)
    g2 = oracle_mod.backward(x, 2 * dy, W1, W3, W2, top, w)
    assert (g2["dx"] == 2 * g["dx"]).all() and (g2["dW1"] == 2 * g["dW1"]).all()


def test_backward_sampled_routines_match_full(oracle_mod):
    rng = np.random.default_rng(31)
    T, h, f, E, k = 12, 128, 256, 4, 2
    x, W1, W3, W2, logits = _rand_layer(rng, T, h, f, E, k)
    top, w = oracle_mod.route(logits, k)
    dy = rng.standard_normal((T, h)).astype(np.float32)
    g = oracle_mod.backward(x, dy, W1, W3, W2, top, w)
    toks = np.array([11, 2, 5], np.int32)
    dx, dw = oracle_mod.backward_tokens(x, dy, W1, W3, W2, top, w, toks, threads=2)
    np.testing.assert_allclose(dx, g["dx"][toks], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dw, g["dw"][toks], rtol=1e-12, atol=1e-14)
    q = []
    for e in range(E):
        q += [(1, e, rng.integers(f), rng.integers(h)), (3, e, rng.integers(f), rng.integers(h)),
              (2, e, rng.integers(h), rng.integers(f))]
    q = np.array(q, np.int32)
    vals = oracle_mod.wgrad_elements(x, dy, W1, W3, W2, top, w, q, threads=2)
    full = {1: g["dW1"], 3: g["dW3"], 2: g["dW2"]}
    ref = np.array([full[a][b, c, d] for a, b, c, d in q])
    np.testing.assert_allclose(vals, ref, rtol=1e-11, atol=1e-14)


def test_wgrad_expert_slabs_against_autograd(oracle_mod):
    """Whole per-expert weight-gradient slabs against torch float64 autograd of the layer's
    composition y = sum_s w_ts W2_e(silu(W1_e x_t) * W3_e x_t), loss = <dy, y>; and the
    same bits as the full backward's slabs (one ordered sum per element)."""
    rng = np.random.default_rng(37)
    T, h, f, E, k = 40, 24, 16, 5, 3
    x, W1, W3, W2, logits = _rand_layer(rng, T, h, f, E, k, scale=0.2)
    dy = rng.standard_normal((T, h)).astype(np.float32)
    top, w = oracle_mod.route(logits, k)
    tw = [torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (W1, W3, W2)]
    tx, tdy = torch.tensor(x, dtype=torch.float64), torch.tensor(dy, dtype=torch.float64)
    idx = torch.tensor(top, dtype=torch.long)
    a = torch.einsum("tkfh,th->tkf", tw[0][idx], tx)
    b = torch.einsum("tkfh,th->tkf", tw[1][idx], tx)
    yts = torch.einsum("tkhf,tkf->tkh", tw[2][idx], torch.nn.functional.silu(a) * b)
    y = (torch.tensor(w) [:, :, None] * yts).sum(1)
    (y * tdy).sum().backward()
    full = oracle_mod.backward(x, dy, W1, W3, W2, top, w)
    counts = np.bincount(top.ravel(), minlength=E)
    for e in range(E):
        d1, d3, d2 = oracle_mod.wgrad_expert(x, dy, W1, W3, W2, top, w, e, threads=3)
        for got, ref, n in ((d1, tw[0].grad[e], "dW1"), (d3, tw[1].grad[e], "dW3"),
                            (d2, tw[2].grad[e], "dW2")):
            np.testing.assert_allclose(got, ref.numpy(), rtol=1e-10, atol=1e-12, err_msg=(n, e))
        assert (d1 == full["dW1"][e]).all() and (d3 == full["dW3"][e]).all()
        assert (d2 == full["dW2"][e]).all()
        if counts[e] == 0:
            assert not d1.any() and not d3.any() and not d2.any()


# ----------------------------------------------------------------------------------------
# tile-aware token rounding
# ----------------------------------------------------------------------------------------

def _rank_key(lg, t, e):
    """Rank of token t for expert e, larger first: (logit, -token)."""
    return (float(lg[t, e]), -int(t))


def _check_rounding(oracle_mod, lg, k, B):
    T, E = lg.shape
    top, w = oracle_mod.route(lg, k)
    tr, wr = oracle_mod.round_tokens(lg, top, block=B)
    c = np.bincount(top.ravel(), minlength=E)
    c2 = np.bincount(tr[tr >= 0], minlength=E)
    for e in range(E):
        r = c[e] % B
        routed = set(np.nonzero((top == e).any(1))[0].tolist())
        now = set(np.nonzero((tr == e).any(1))[0].tolist())
        if r == 0:
            assert now == routed, e
            continue
        up = 2 * r >= B and T - c[e] >= B - r
        if up:  # the B - r best-ranked tokens not routed to e are added, nothing dropped
            assert c2[e] == c[e] + (B - r) and routed <= now
            cand = sorted(set(range(T)) - routed, key=lambda t: _rank_key(lg, t, e), reverse=True)
            assert now - routed == set(cand[:B - r]), e
        else:  # e's r worst-ranked entries are dropped, nothing added
            assert c2[e] == c[e] - r and now <= routed
            ranked = sorted(routed, key=lambda t: _rank_key(lg, t, e))
            assert routed - now == set(ranked[:r]), e
        assert c2[e] % B == 0
        assert abs(int(c2[e]) - int(c[e])) <= B // 2
    # each token: its surviving slots in slot order, then added experts in increasing order
    p = torch.softmax(torch.tensor(lg, dtype=torch.float64), dim=1).numpy()
    for t in range(T):
        row = [e for e in tr[t] if e >= 0]
        kept = [e for e in top[t] if e in row]
        assert row[:len(kept)] == kept
        assert row[len(kept):] == sorted(set(row) - set(top[t].tolist()))
        assert len(set(row)) == len(row)
        np.testing.assert_allclose(wr[t, :len(row)], p[t, row], rtol=1e-12)
        assert (tr[t, len(row):] == -1).all() and (wr[t, len(row):] == 0).all()
    return top, tr, wr


@pytest.mark.parametrize("T,E,k,B,seed", [(3000, 16, 2, 128, 0), (700, 8, 3, 128, 1),
                                          (40, 5, 2, 4, 2), (9, 3, 1, 2, 3), (500, 64, 8, 16, 4),
                                          (200, 4, 2, 128, 5)])
def test_token_rounding_definition(oracle_mod, T, E, k, B, seed):
    """Every count becomes the nearest multiple of the tile (ties upward; downward when too
    few tokens are left to add), the dropped entries are the worst-ranked ones and the added
    tokens the best-ranked unrouted ones (checked against sorted() of the rank key), the
    slot order is kept, and every weight is the float64 softmax at its expert."""
    rng = np.random.default_rng(seed)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    if seed == 2:  # ties: few distinct values, +0 and -0 among them
        lg = np.array([-1.0, -0.0, 0.0, 0.5, 2.0], np.float32)[rng.integers(0, 5, (T, E))]
    _check_rounding(oracle_mod, lg, k, B)


def test_token_rounding_identity_and_skew(oracle_mod):
    """Block 1 leaves the routing unchanged; a skewed routing (the skewed workload's bias)
    rounds every expert, including ones with fewer than 64 entries, which drop to zero."""
    rng = np.random.default_rng(7)
    lg = rng.standard_normal((300, 8)).astype(np.float32)
    top, w = oracle_mod.route(lg, 2)
    tr, wr = oracle_mod.round_tokens(lg, top, block=1)
    assert (tr == top).all() and np.allclose(wr, w, rtol=1e-15)
    lg = (rng.standard_normal((2000, 32)) - 1.5 * np.log(np.arange(32) + 1.0)).astype(np.float32)
    top, tr, wr = _check_rounding(oracle_mod, lg, 4, 128)
    c2 = np.bincount(tr[tr >= 0], minlength=32)
    assert (c2 % 128 == 0).all() and (c2 == 0).any()


def test_absent_entries_contribute_nothing(oracle_mod):
    """Forward and backward skip positions whose expert is -1 (the rounded routing's unused
    positions): the same as a valid expert with weight 0 in the forward and in dx, with the
    position's own routing-weight gradient 0."""
    rng = np.random.default_rng(41)
    T, h, f, E, k = 6, 128, 128, 4, 3
    x, W1, W3, W2, logits = _rand_layer(rng, T, h, f, E, k)
    top, w = oracle_mod.route(logits, k)
    dy = rng.standard_normal((T, h)).astype(np.float32)
    top_a, w_a = top.copy(), w.copy()
    top_a[[1, 4], [2, 0]] = -1
    w_z = w.copy()
    w_z[[1, 4], [2, 0]] = 0.0
    ya = oracle_mod.forward(x, W1, W3, W2, top_a, w_a)
    yz = oracle_mod.forward(x, W1, W3, W2, top, w_z)
    np.testing.assert_array_equal(ya, yz)
    ga = oracle_mod.backward(x, dy, W1, W3, W2, top_a, w_a)
    gz = oracle_mod.backward(x, dy, W1, W3, W2, top, w_z)
    np.testing.assert_allclose(ga["dx"], gz["dx"], rtol=1e-13, atol=1e-15)
    assert ga["dw"][1, 2] == 0 and ga["dw"][4, 0] == 0
    assert ga["dw"][0, 0] == gz["dw"][0, 0]


# ----------------------------------------------------------------------------------------
# router GEMM and the gradient through the routing weights
# ----------------------------------------------------------------------------------------

def _router_loss(lg64, top, dw):
    """sum_t sum_s dw_ts * softmax(l_t)[top_ts], in float64 (picks held fixed)."""
    z = lg64 - lg64.max(1, keepdims=True)
    p = np.exp(z)
    p /= p.sum(1, keepdims=True)
    return float((dw * np.take_along_axis(p, top.astype(np.int64), 1)).sum())


def test_router_logits_closed_form_and_library_matmul(oracle_mod):
    rng = np.random.default_rng(61)
    T, h, E = 7, 48, 5
    Wr = rng.standard_normal((E, h)).astype(np.float32)
    x = np.zeros((T, h), np.float32)
    cols = rng.integers(0, h, T)
    x[np.arange(T), cols] = 1.0
    lg = oracle_mod.router_logits(x, Wr)
    assert (lg == Wr[:, cols].T.astype(np.float64)).all()  # a one-hot token reads a column
    x = rng.standard_normal((T, h)).astype(np.float32)
    lg = oracle_mod.router_logits(x, Wr)
    np.testing.assert_allclose(lg, x.astype(np.float64) @ Wr.astype(np.float64).T,
                               rtol=1e-13, atol=1e-12)
    assert (oracle_mod.router_logits(x, Wr, tokens=np.array([6, 0, 3])) == lg[[6, 0, 3]]).all()


def _router_case(oracle_mod, seed, T=6, h=32, E=7, k=3):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, h)).astype(np.float32)
    Wr = (0.3 * rng.standard_normal((E, h))).astype(np.float32)
    lg = (x.astype(np.float64) @ Wr.astype(np.float64).T).astype(np.float32)
    top, _ = oracle_mod.route(lg, k)
    dw = rng.standard_normal((T, k))
    return x, Wr, lg, top, dw


def test_router_backward_finite_differences(oracle_mod):
    x, Wr, lg, top, dw = _router_case(oracle_mod, 67)
    g = oracle_mod.router_backward(x, Wr, lg, top, dw)
    T, E = lg.shape
    l64 = lg.astype(np.float64)
    eps = 1e-6
    for t in range(T):  # every logit: the picks stay fixed under a perturbation this small
        for i in range(E):
            lp, lm = l64.copy(), l64.copy()
            lp[t, i] += eps
            lm[t, i] -= eps
            fd = (_router_loss(lp, top, dw) - _router_loss(lm, top, dw)) / (2 * eps)
            assert abs(fd - g["dlogits"][t, i]) <= 1e-8 + 1e-6 * abs(fd), (t, i)
    # through logits = x Wr^T: perturb x and Wr (the oracle's dlogits is taken at the
    # fp32-rounded logits, hence the looser relative bound)
    rng = np.random.default_rng(71)
    x64, W64 = x.astype(np.float64), Wr.astype(np.float64)
    for _ in range(12):
        t, c = int(rng.integers(T)), int(rng.integers(x.shape[1]))
        xp, xm = x64.copy(), x64.copy()
        xp[t, c] += eps
        xm[t, c] -= eps
        fd = (_router_loss(xp @ W64.T, top, dw) - _router_loss(xm @ W64.T, top, dw)) / (2 * eps)
        assert abs(fd - g["dx_r"][t, c]) <= 1e-7 + 1e-5 * abs(fd), ("x", t, c)
        e = int(rng.integers(E))
        wp, wm = W64.copy(), W64.copy()
        wp[e, c] += eps
        wm[e, c] -= eps
        fd = (_router_loss(x64 @ wp.T, top, dw) - _router_loss(x64 @ wm.T, top, dw)) / (2 * eps)
        assert abs(fd - g["dWr"][e, c]) <= 1e-7 + 1e-5 * abs(fd), ("Wr", e, c)


def test_router_backward_autograd_and_invariants(oracle_mod):
    x, Wr, lg, top, dw = _router_case(oracle_mod, 73, T=9, h=40, E=8, k=4)
    g = oracle_mod.router_backward(x, Wr, lg, top, dw)
    l = torch.tensor(lg, dtype=torch.float64, requires_grad=True)
    p = torch.softmax(l, dim=1)
    (torch.tensor(dw) * p.gather(1, torch.from_numpy(top).long())).sum().backward()
    np.testing.assert_allclose(g["dlogits"], l.grad.numpy(), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(g["dx_r"], l.grad.numpy() @ Wr.astype(np.float64), rtol=1e-12,
                               atol=1e-14)
    np.testing.assert_allclose(g["dWr"], l.grad.numpy().T @ x.astype(np.float64), rtol=1e-12,
                               atol=1e-14)
    # softmax is shift-invariant: each token's logit gradient sums to zero
    assert np.abs(g["dlogits"].sum(1)).max() <= 1e-14
    # all experts picked with the same dw: the weights sum to 1, so no gradient reaches the logits
    T, E = lg.shape
    topE, _ = oracle_mod.route(lg, E)
    z = oracle_mod.router_backward(x, Wr, lg, topE, np.full((T, E), 0.7))
    assert np.abs(z["dlogits"]).max() <= 1e-15
    # sampled routines equal the full ones
    toks = np.array([8, 2, 5])
    el = np.array([[0, 3], [7, 39], [4, 0]])
    s = oracle_mod.router_backward(x, Wr, lg, top, dw, tokens=toks, elems=el)
    assert (s["dx_r"] == g["dx_r"][toks]).all()
    assert (s["dWr"] == g["dWr"][el[:, 0], el[:, 1]]).all()


# ----------------------------------------------------------------------------------------
# renormalised routing (the weights are the softmax over the k chosen logits)
# ----------------------------------------------------------------------------------------

def test_route_renorm_closed_forms(oracle_mod):
    rng = np.random.default_rng(83)
    T, E = 40, 12
    lg = rng.standard_normal((T, E)).astype(np.float32)
    for k in (1, 3, E):
        top, w = oracle_mod.route(lg, k, renorm=True)
        top0, w0 = oracle_mod.route(lg, k)
        assert (top == top0).all()  # the choice does not depend on the weights
        np.testing.assert_allclose(w.sum(1), 1.0, rtol=0, atol=1e-15)
        sel = np.take_along_axis(lg.astype(np.float64), top.astype(np.int64), 1)
        np.testing.assert_allclose(w[:, :1] / w, np.exp(sel[:, :1] - sel), rtol=1e-13)
        if k == 1:
            assert (w == 1.0).all()
        if k == E:
            np.testing.assert_allclose(w, w0, rtol=1e-14, atol=1e-16)
        ref = torch.softmax(torch.from_numpy(sel), dim=1).numpy()  # library softmax
        np.testing.assert_allclose(w, ref, rtol=1e-13, atol=1e-16)


def test_router_backward_renorm_finite_differences_and_autograd(oracle_mod):
    rng = np.random.default_rng(89)
    T, h, E, k = 5, 24, 9, 3
    x = rng.standard_normal((T, h)).astype(np.float32)
    Wr = (0.3 * rng.standard_normal((E, h))).astype(np.float32)
    lg = (x.astype(np.float64) @ Wr.astype(np.float64).T).astype(np.float32)
    top, _ = oracle_mod.route(lg, k, renorm=True)
    dw = rng.standard_normal((T, k))
    g = oracle_mod.router_backward(x, Wr, lg, top, dw, renorm=True)

    def loss(l64):
        sel = np.take_along_axis(l64, top.astype(np.int64), 1)
        z = np.exp(sel - sel.max(1, keepdims=True))
        return float((dw * z / z.sum(1, keepdims=True)).sum())

    l64 = lg.astype(np.float64)
    eps = 1e-6
    for t in range(T):
        for i in range(E):
            lp, lm = l64.copy(), l64.copy()
            lp[t, i] += eps
            lm[t, i] -= eps
            fd = (loss(lp) - loss(lm)) / (2 * eps)
            assert abs(fd - g["dlogits"][t, i]) <= 1e-8 + 1e-6 * abs(fd), (t, i)
    chosen = np.zeros((T, E), bool)
    np.put_along_axis(chosen, top.astype(np.int64), True, 1)
    assert (g["dlogits"][~chosen] == 0).all()
    assert np.abs(g["dlogits"].sum(1)).max() <= 1e-14
    l = torch.tensor(lg, dtype=torch.float64, requires_grad=True)
    sel = l.gather(1, torch.from_numpy(top).long())
    (torch.tensor(dw) * torch.softmax(sel, dim=1)).sum().backward()
    np.testing.assert_allclose(g["dlogits"], l.grad.numpy(), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(g["dx_r"], l.grad.numpy() @ Wr.astype(np.float64), rtol=1e-12,
                               atol=1e-14)



# ---- property sweeps (hypothesis) ----------------------------------------------------------


@settings(max_examples=60, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(T=st.integers(1, 300), E=st.integers(1, 64), data=st.data())
def test_map_invariants_property(oracle_mod, T, E, data):
    """Every map invariant on random routings: k distinct experts per token, any T and E."""
    k = data.draw(st.integers(1, min(E, 8)), label="k")
    rng = np.random.default_rng(data.draw(st.integers(0, 2 ** 31 - 1), label="seed"))
    top = np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)
    _check_map_invariants(top, E, oracle_mod.sparse_map(top, E))


@settings(max_examples=60, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(E=st.integers(1, 7), data=st.data())
def test_route_brute_force_property(oracle_mod, E, data):
    """The chosen k-subset is the unique one that beats every other expert under (value
    descending, index ascending), on logits drawn from a small set full of ties and signed
    zeros; slots follow the same order."""
    k = data.draw(st.integers(1, E), label="k")
    vals = np.array([-2.0, -0.0, 0.0, 0.5, 0.5, 3.0, -np.inf], dtype=np.float32)
    rng = np.random.default_rng(data.draw(st.integers(0, 2 ** 31 - 1), label="seed"))
    logits = rng.choice(vals, size=(16, E)).astype(np.float32)
    top, _ = oracle_mod.route(logits, k)
    for t in range(16):
        l = [float(v) for v in logits[t]]
        winners = [set(S) for S in itertools.combinations(range(E), k)
                   if all(_beats(l[a], a, l[b], b) for a in S for b in range(E) if b not in S)]
        assert len(winners) == 1 and set(top[t].tolist()) == winners[0]
        for s in range(k - 1):
            assert _beats(l[top[t, s]], top[t, s], l[top[t, s + 1]], top[t, s + 1])
