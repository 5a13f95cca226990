"""C-ABI checks that need no GPU: the library builds/loads, exports every symbol the header
declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

from dropless_mixture_experts_dmoe_b200 import binding as B
from dropless_mixture_experts_dmoe_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.load()


def _declared_symbols():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"DMOE_API\s+[\w\s\*]+?\b(dmoe_\w+)\s*\(", txt)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = _declared_symbols()
    assert len(names) >= 13
    for n in names:
        assert hasattr(lib, n), n
    assert B.version().startswith("dmoe-b200")


def test_sizes():
    d = B.make_dims(4096, 4096, 14336, 8, 2)
    P = B.dmoe_padded_rows_max(d)
    assert P == ((4096 * 2 + 127 * 8) // 128) * 128
    assert B.dmoe_workspace_bytes(d, B.WS_MAP) >= 4 * 64 * 8
    assert B.dmoe_workspace_bytes(d, B.WS_FORWARD) >= P * (2 * 4096 + 14336) * 2
    # a training forward keeps X_pad in the saved buffer: its workspace holds H and Y_pad only
    assert P * (4096 + 14336) * 2 <= B.dmoe_workspace_bytes(d, B.WS_FORWARD_TRAIN) < \
        B.dmoe_workspace_bytes(d, B.WS_FORWARD)
    # backward: dY_pad (reused for dX_pad), dA, dBm, Hw and the routing-weight partials
    assert B.dmoe_workspace_bytes(d, B.WS_BACKWARD) >= P * (4096 + 3 * 14336) * 2 + P * 56 * 4
    total, offs = B.dmoe_saved_bytes(d)
    assert len(offs) == 3  # X_pad, A, Bm: neither H nor Y_pad outlives the forward
    assert offs == sorted(offs) and offs[0] == 0 and all(o % 256 == 0 for o in offs)
    assert offs[1] >= P * 4096 * 2 and offs[2] >= offs[1] + P * 14336 * 2
    assert total >= offs[2] + P * 14336 * 2
    assert B.dmoe_workspace_bytes(d, 5) == 0  # unknown workspace kind


@pytest.mark.parametrize("dims,code", [
    ((256, 128, 100, 8, 2), -2),    # ffn % 128 != 0 (the walkthrough's topology guard)
    ((256, 96, 128, 8, 2), -2),     # hidden % 128 != 0
    ((256, 128, 128, 8, 9), -2),    # top_k > E
    ((256, 128, 128, 64, 33), -2),  # top_k > 32
    ((0, 128, 128, 8, 2), -2),      # T < 1
    ((256, 128, 128, 1025, 2), -3),  # E > 1024
    ((256, 128, 128, 0, 1), -3),
    ((2 ** 28, 128, 128, 32, 16), -8),  # T*k overflows int32
])
def test_bad_dims_rejected_before_launch(lib, dims, code):
    d = B.make_dims(*dims)
    assert B.dmoe_padded_rows_max(d) == 0
    m = B.dmoe_map()
    rc = lib.dmoe_sparse_map(ctypes.byref(d), None, ctypes.byref(m), None, 0, None)
    assert rc == code
    rc = lib.dmoe_forward(ctypes.byref(d), None, None, None, None, ctypes.byref(m), None, None, None,
                          0, None)
    assert rc == code
    assert B.error_string(code) != "unknown error"


def test_unknown_flag_rejected(lib):
    m = B.dmoe_map()
    for bad in (0x10, 0x40, B.ROUTE_TOKEN_ROUNDING | B.ROUTE_RENORMALIZE,
                B.ROUTE_TOKEN_ROUNDING | B.FUSED_COMBINE):
        d = B.make_dims(256, 128, 128, 8, 2, flags=bad)
        assert B.dmoe_padded_rows_max(d) == 0
        assert lib.dmoe_sparse_map(ctypes.byref(d), None, ctypes.byref(m), None, 0, None) == -2
    for fl in (B.ROUTE_RENORMALIZE, B.SAVE_X_ONLY, B.ROUTE_RENORMALIZE | B.SAVE_X_ONLY,
               B.ROUTE_TOKEN_ROUNDING, B.ROUTE_TOKEN_ROUNDING | B.SAVE_X_ONLY, B.FUSED_COMBINE,
               B.FUSED_COMBINE | B.ROUTE_RENORMALIZE | B.SAVE_X_ONLY):
        d = B.make_dims(256, 128, 128, 8, 2, flags=fl)
        assert B.dmoe_padded_rows_max(d) > 0  # the defined flags are accepted


def test_token_rounding_sizes(lib):
    """DMOE_ROUTE_TOKEN_ROUNDING: up to 64 added entries per expert (T*k + 64E), the padded
    bound from that, and T above 2^20 rejected; the router calls reject the flag."""
    d = B.make_dims(4096, 128, 128, 64, 8, flags=B.ROUTE_TOKEN_ROUNDING)
    assert B.dmoe_entries_max(d) == 4096 * 8 + 64 * 64
    assert B.dmoe_padded_rows_max(d) == (4096 * 8 + 64 * 64 + 127 * 64) // 128 * 128
    assert B.dmoe_entries_max(B.make_dims(4096, 128, 128, 64, 8)) == 4096 * 8
    assert B.dmoe_entries_max(B.make_dims((1 << 20) + 1, 128, 128, 8, 1,
                                          flags=B.ROUTE_TOKEN_ROUNDING)) == 0
    m = B.dmoe_map()
    assert lib.dmoe_router_dlogits(ctypes.byref(d), None, ctypes.byref(m), None, None, None) == -2


def test_save_x_only_sizes(lib):
    """DMOE_SAVE_X_ONLY: the saved activations shrink to X_pad (2h bytes per padded row, from
    2h + 4f) and the backward workspace grows by the recomputed A and Bm (4f per row)."""
    T, h, f, E, k = 32768, 2048, 512, 256, 8
    d0 = B.make_dims(T, h, f, E, k)
    d1 = B.make_dims(T, h, f, E, k, flags=B.SAVE_X_ONLY)
    P = B.dmoe_padded_rows_max(d0)
    s0, off0 = B.dmoe_saved_bytes(d0)
    s1, off1 = B.dmoe_saved_bytes(d1)
    assert s0 >= P * (2 * h + 4 * f) and s1 == P * 2 * h and off1 == [0, 0, 0]
    assert off0[1] >= P * 2 * h and off0[2] >= off0[1] + P * 2 * f
    assert abs((1 - s1 / s0) - 4 * f / (2 * h + 4 * f)) < 1e-3  # a third at this shape
    w0 = B.dmoe_workspace_bytes(d0, B.WS_BACKWARD)
    w1 = B.dmoe_workspace_bytes(d1, B.WS_BACKWARD)
    assert P * 4 * f <= w1 - w0 <= P * 4 * f + 512
    assert B.dmoe_workspace_bytes(d1, B.WS_FORWARD_TRAIN) == B.dmoe_workspace_bytes(d0, B.WS_FORWARD_TRAIN)


def test_router_needs_E_multiple_of_8(lib):
    """The router's [T, E] rows must be multiples of 16 bytes: E % 8 != 0 is a shape error,
    reported before any launch (and before the null-pointer checks)."""
    m = B.dmoe_map()
    for E, code in ((12, -2), (8, -1), (1025, -3)):
        d = B.make_dims(256, 128, 128, E, 2)
        assert lib.dmoe_router_forward(ctypes.byref(d), None, None, None, None, None) == code
        assert lib.dmoe_router_dlogits(ctypes.byref(d), None, ctypes.byref(m), None, None, None) == code
        assert lib.dmoe_router_backward(ctypes.byref(d), None, None, None, ctypes.byref(m), None,
                                        None, None, None, 0, None) == code
    d = B.make_dims(4096, 2048, 512, 256, 8)
    # dlogits [T, E] bf16 plus 16 split slabs of round_up(E, 128) x h fp32 partials
    assert B.dmoe_workspace_bytes(d, B.WS_ROUTER_BACKWARD) >= 4096 * 256 * 2 + 16 * 256 * 2048 * 4


def test_null_and_workspace_checks(lib):
    d = B.make_dims(256, 128, 128, 8, 2)
    m = B.dmoe_map()
    assert lib.dmoe_sparse_map(ctypes.byref(d), None, ctypes.byref(m), None, 0, None) == -1
    fake = 1 << 20  # host-side checks only: nothing is launched when a check fails
    m = B.dmoe_map(*([fake] * len(B.MAP_FIELDS)))
    assert lib.dmoe_sparse_map(ctypes.byref(d), fake, ctypes.byref(m), fake, 16, None) == -4
    assert lib.dmoe_sparse_map(ctypes.byref(d), fake + 2, ctypes.byref(m), fake, 1 << 20, None) == -5


def test_status_strings(lib):
    assert B.status_string(0) == "ok"
    s = B.status_string(B.STATUS_TIMEOUT | B.STATUS_NONFINITE_LOGITS)
    assert "timeout" in s and "nonfinite" in s


@pytest.mark.parametrize("T,E", [(1, 1), (4096, 8), (32768, 256), (32769, 256), (262144, 256),
                                 (65536, 1024)])
def test_map_workspace_formula(T, E):
    """The map workspace is what include/dmoe.h states: per-tile histograms ceil(T/64)*E, one
    ticket counter, one status word per tile and the scan's per-segment totals
    ceil(T/32768)*E, int32 each (rounded up to the 256-byte alignment)."""
    d = B.make_dims(T, 128, 128, E, 1)
    tiles = -(-T // 64)
    segs = -(-tiles // 512)
    need = 4 * (tiles * E + 1 + tiles + segs * E)
    assert need <= B.dmoe_workspace_bytes(d, B.WS_MAP) < need + 256


def test_noalloc_capacity_limits(lib):
    """dmoe_sparse_map_noalloc's static scratch holds exactly the documented sizes: the largest
    T that fits passes the capacity check (and is then refused for its unaligned logits pointer,
    still before any device call); 64 more tokens are refused with DMOE_ERR_WORKSPACE."""
    fake = 1 << 20  # host-side checks only: every case below is refused before a launch
    m = B.dmoe_map(*([fake] * len(B.MAP_FIELDS)))
    for E, t_max in ((256, 65152), (1024, 16256)):
        fits = B.make_dims(t_max, 128, 128, E, 1)
        over = B.make_dims(t_max + 64, 128, 128, E, 1)
        assert lib.dmoe_sparse_map_noalloc(ctypes.byref(over), fake, ctypes.byref(m), None) == -4
        assert lib.dmoe_sparse_map_noalloc(ctypes.byref(fits), fake + 2, ctypes.byref(m),
                                           None) == -5


def test_autograd_wrapper_validates_inputs_on_the_host():
    """dmoe() rejects non-CUDA, non-bf16 or mis-shaped inputs before calling the library."""
    import torch

    from dropless_mixture_experts_dmoe_b200 import autograd as A

    x = torch.zeros(4, 128, dtype=torch.bfloat16)  # a CPU tensor
    w = torch.zeros(2, 128, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        A.dmoe(x, torch.zeros(4, 2, dtype=torch.bfloat16), w, w, w, 1)
    with pytest.raises(ValueError):
        A.dmoe(x.float(), x, w, w, w, 1)
