"""The routing kernel's selection scheme, modelled on the host and checked by brute force.

The CUDA routing kernel does not sort a token's E logits.  Each of the 32 lanes of a warp
holds its share of the integer keys (order-preserving image of the bf16 logit in the high 16
bits, 0xFFFF - expert in the low 16, so larger key = larger logit, equal logits -> lower
expert) and keeps only its three largest; k rounds of a warp-wide maximum over the lanes'
best candidates give the picks in rank order.  Afterwards one check decides whether those are
the top-k of all keys: if a lane has used up its candidates and holds more than three keys at
or above the last pick, the rounds run again with refills (a lane that runs dry takes its
keys below the last pick).  This module restates that scheme in Python (the kernel's lane
layouts: for even E two experts per word, word c of lane l = experts 64c + 2l and
64c + 2l + 1; for odd E lane l holds experts l, l + 32, ...) and checks, on
tie-heavy and lane-heavy inputs, that it returns exactly the top-k that a full sort gives.  It
models the scheme, not the CUDA code; the GPU tests compare the kernel with the oracle.
No GPU, no product code."""
import numpy as np
import pytest
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

LANES = 32
C = 3  # candidates per lane


def _order_image(bits16: int) -> int:
    """Order-preserving image of a bf16 bit pattern (-0 taken as +0; not for NaN)."""
    if bits16 == 0x8000:
        bits16 = 0
    return (~bits16) & 0xFFFF if bits16 & 0x8000 else bits16 | 0x8000


def _keys_per_lane(values: np.ndarray):
    """Keys of one token, dealt to lanes as the kernel does."""
    E = len(values)
    kpl = 1
    while 32 * kpl < E:
        kpl *= 2
    bits = torch.from_numpy(values.astype(np.float32)).to(torch.bfloat16).view(torch.int16)
    bits = bits.numpy().astype(np.int64) & 0xFFFF
    packed = kpl >= 2 and E % 2 == 0  # else lane l holds experts l, l + 32, ...
    lanes = [[] for _ in range(LANES)]
    for lane in range(LANES):
        for i in range(kpl):
            e = 64 * (i >> 1) + 2 * lane + (i & 1) if packed else lane + 32 * i
            if e < E:
                lanes[lane].append((_order_image(int(bits[e])) << 16) | (0xFFFF - e))
    return lanes


def _rounds(lanes, k, refill):
    cand = [sorted(keys, reverse=True)[:C] for keys in lanes]
    picks = []
    for s in range(k):
        wb = max((c[0] for c in cand if c), default=0)
        picks.append(wb)
        for lane, c in enumerate(cand):
            if c and c[0] == wb:
                c.pop(0)
                if refill and not c and s + 1 < k:  # dry: refill from the keys below wb
                    cand[lane] = sorted((x for x in lanes[lane] if x < wb), reverse=True)[:C]
    dry = [not c for c in cand]
    return picks, dry


def kernel_scheme_topk(values: np.ndarray, k: int):
    """Expert ids in rank order, as the routing kernel's scheme finds them."""
    lanes = _keys_per_lane(values)
    picks, dry = _rounds(lanes, k, refill=False)
    last = picks[-1]
    if any(d and sum(x >= last for x in keys) > C for d, keys in zip(dry, lanes)):
        picks, _ = _rounds(lanes, k, refill=True)
    return [0xFFFF - (p & 0xFFFF) for p in picks]


def sorted_topk(values: np.ndarray, k: int):
    """The definition: largest bf16 value first, equal values by the lower expert index."""
    v = torch.from_numpy(values.astype(np.float32)).to(torch.bfloat16).double().numpy()
    return sorted(range(len(v)), key=lambda e: (-v[e], e))[:k]


def _check(values, k):
    assert kernel_scheme_topk(values, k) == sorted_topk(values, k)


@pytest.mark.parametrize("E,k", [(64, 8), (128, 8), (256, 8), (256, 32), (200, 8), (66, 4),
                                 (512, 2), (8, 8), (33, 4)])
def test_selection_scheme_random(E, k):
    rng = np.random.default_rng(E * 100 + k)
    for _ in range(40):
        _check(rng.standard_normal(E), k)


@pytest.mark.parametrize("E,k", [(256, 8), (256, 32), (128, 16)])
def test_selection_scheme_one_lane_holds_the_top(E, k):
    """Lane 0's experts (64c, 64c + 1) far above the rest: it holds up to eight of the top-k,
    so the check after the rounds must send the token through the refilling rounds."""
    rng = np.random.default_rng(E + k)
    for _ in range(20):
        v = rng.standard_normal(E) - 8.0
        v[(np.arange(E) % 64) < 2] += 16.0
        _check(v, k)


@pytest.mark.parametrize("E,k", [(256, 8), (64, 8), (100, 8)])
def test_selection_scheme_ties_and_signed_zeros(E, k):
    rng = np.random.default_rng(7 * E + k)
    vals = np.array([-1.0, -0.0, 0.0, 0.5, 0.5, 2.0])
    for _ in range(30):
        _check(vals[rng.integers(0, len(vals), E)], k)
    _check(np.full(E, 0.25), k)  # every logit equal: experts 0 .. k-1


def test_selection_scheme_skewed_bias():
    rng = np.random.default_rng(5)
    bias = -1.5 * np.log(np.arange(256) + 1.0)
    for _ in range(40):
        _check(rng.standard_normal(256) + bias, 8)


@settings(max_examples=150, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(st.integers(2, 96), st.data())
def test_selection_scheme_hypothesis(E, data):
    k = data.draw(st.integers(1, min(E, 32)))
    pool = data.draw(st.lists(st.sampled_from([-3.0, -1.0, -0.0, 0.0, 0.5, 1.0, 4.0]),
                              min_size=2, max_size=4))
    idx = data.draw(st.lists(st.integers(0, len(pool) - 1), min_size=E, max_size=E))
    _check(np.array([pool[i] for i in idx]), k)
