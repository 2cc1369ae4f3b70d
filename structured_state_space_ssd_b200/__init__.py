"""B200-native (sm_100a) SSD layer forward: ``Y = SSD(A, B, C)(X)``.

The work runs in ``libssd.so`` (hand-written CUDA kernels behind a C ABI,
declared in ``include/ssd.h``); :mod:`.ssd` is the thin ctypes binding that
marshals torch tensors into it.  Importing this package loads nothing: the
library is opened on the first call, and a missing or unloadable library is
an error, never a fallback.
"""
from .inputs import HEADLINE, WORKLOADS, Workload, make_inputs, make_output_grads, workload_inputs  # noqa: F401

__all__ = ["HEADLINE", "WORKLOADS", "Workload", "make_inputs", "make_output_grads", "workload_inputs",
           "ssd_fwd", "ssd_fwd_workspace_bytes", "ssd_status_string", "SSDError"]


def __getattr__(name):
    if name in ("ssd_fwd", "ssd_fwd_workspace_bytes", "ssd_status_string", "SSDError"):
        from . import ssd
        return getattr(ssd, name)
    raise AttributeError(name)
