"""dMoE expert layer for NVIDIA B200 (sm_100a): routing, sparse map, padded gather, grouped
tcgen05 gated-SiLU expert GEMMs, weighted combine and backward, behind the C ABI of
``libdmoe.so`` (include/dmoe.h).  ``binding`` is the thin ctypes layer over it."""
from . import autograd, binding  # noqa: F401
from .autograd import DMoEFunction, dmoe  # noqa: F401
from .binding import (Buffers, DMoEError, SparseMap, dmoe_backward, dmoe_bwd_dglu,  # noqa: F401
                      dmoe_bwd_dx, dmoe_bwd_scatter, dmoe_bwd_wgrad, dmoe_expert_down,
                      dmoe_expert_glu, dmoe_expert_glu_gather, dmoe_forward, dmoe_padded_gather, dmoe_padded_rows_max,
                      dmoe_padded_scatter, dmoe_router_backward, dmoe_router_dlogits,
                      dmoe_router_forward, dmoe_saved_bytes, dmoe_sparse_map,
                      dmoe_sparse_map_noalloc, dmoe_workspace_bytes, make_dims)

__version__ = "0.1"
