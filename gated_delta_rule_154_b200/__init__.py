"""Gated delta-rule recurrence on NVIDIA B200 (sm_100a).

The CUDA library ``libgdr.so`` (built from ``csrc/``) holds every kernel; the
Python side only marshals torch tensors into its C ABI.  Importing this
package does not load the library; the first call does, and it raises if the
library is missing.
"""

__all__ = ["forward_chunked", "decode_step", "workspace_size", "Desc"]


def __getattr__(name):
    if name in __all__:
        from . import api
        return getattr(api, name)
    raise AttributeError(name)
