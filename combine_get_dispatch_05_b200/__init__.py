"""B200 (sm_100a) MoE token dispatch / combine: a C-ABI CUDA library plus a thin
Python binding.

* ``ep_*`` functions: the C entry points of ``include/ep_b200.h``, one to one,
  taking torch tensors for device memory (argument marshalling only).
* :class:`Buffer`: the DeepEP-style call shapes (dispatch / combine /
  low_latency_dispatch / low_latency_combine) on top of them.
* :class:`EpGroup`: dispatch / combine across the ranks of a process group (one
  GPU each), through NCCL all-to-all or straight through peer memory.

Importing this package loads ``libep_b200.so``; if it is missing the import
fails (there is no fallback implementation).
"""
from ._lib import (  # noqa: F401
    EP_DEV_CAPACITY, EP_DEV_INDEX_RANGE, EP_DEV_TIMEOUT, EP_ERR_CUDA, EP_ERR_INVALID_ARG,
    EP_ERR_SHAPE, EP_ERR_WORKSPACE, EP_OK, EP_QUANT_FP8_E4M3_1X128, EP_QUANT_FP8_E4M3_1X128_POW2,
    EP_QUANT_NONE, EP_QUANT_SCALES_MN_MAJOR, EpError, scales_ld,
    Layout, LowLatencyHandle, LIB_PATH, ep_combine, ep_combine_backward, ep_debug_wait_probe,
    ep_combine_dedup, ep_dispatch, ep_dispatch_backward, ep_dispatch_dedup,
    ep_get_dispatch_layout, ep_lb_prefetch_weights, ep_lb_reduce_grads, ep_low_latency_combine,
    ep_low_latency_dispatch, ep_read_status, ep_workspace_bytes, ep_workspace_init, lib,
    status_string, EP_IPC_HANDLE_BYTES, PeerTables, device_bytes, ep_ipc_alloc, ep_ipc_close,
    ep_ipc_free, ep_ipc_open, ep_peer_combine, ep_peer_dispatch, ep_peer_plan,
    ep_get_dispatch_layout_dedup, ep_peer_combine_dedup, ep_peer_dispatch_dedup,
    ep_peer_low_latency_combine, ep_peer_low_latency_dispatch,
)
from .buffer import Buffer  # noqa: F401
from .ep_group import EpContext, EpGroup  # noqa: F401

__version__ = "0.1.0"
