"""B200-native MoE expert-parallel dispatch / combine.

The public calls (``ep_get_dispatch_layout``, ``ep_dispatch``, ``ep_combine``)
are thin ctypes bindings over the C-ABI library ``libep.so`` built from
``csrc/``; every step of the path runs in its sm_100a kernels.  They are loaded
on first use, so importing the input generators (``workloads``) does not need
the CUDA library.
"""

_API = ("ep_get_dispatch_layout", "ep_dispatch", "ep_combine", "ep_group_limited_gating", "EPHandle",
        "DispatchBuffers", "alloc_dispatch_buffers", "EPError", "recv_capacity_bound",
        "workspace_bytes", "library_path")


def __getattr__(name):
    if name in _API:
        from . import ep
        return getattr(ep, name)
    raise AttributeError(name)


__all__ = list(_API)
