"""ctypes view of libgdr.so's C ABI (declared in include/gdr.h).

Argument marshalling only.  Loading fails loudly if the library is missing:
there is no other implementation behind these names.
"""

from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdr.so")

# gdr_status
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT, ERR_RANGE = range(7)
# gdr_dtype
F32, BF16 = 0, 1
# gdr_gate
GATE_ONE, GATE_SCALAR, GATE_VECTOR, GATE_FG2 = 0, 1, 2, 3

EXPORTS = ("gdr_workspace_size", "gdr_forward_chunked", "gdr_decode_step",
           "gdr_last_device_error", "gdr_status_string", "gdr_version", "gdr_test_skip_signal",
           "gdr_decode_step_paged", "gdr_forward_varlen", "gdr_backward_workspace_size",
           "gdr_backward_chunked", "gdr_backward_varlen", "gdr_backward_varlen_workspace_size",
           "gdr_backward_chunked_noalloc", "gdr_segment_maps_workspace_size",
           "gdr_segment_maps", "gdr_segment_scan", "gdr_segmented_workspace_size",
           "gdr_forward_segmented")

# bytes of the library-owned scratch of gdr_backward_chunked_noalloc
NOALLOC_SCRATCH_BYTES = 64 << 20


class GdrDesc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int),
                ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("chunk", ctypes.c_int),
                ("in_dtype", ctypes.c_int), ("decay", ctypes.c_int),
                ("erase", ctypes.c_int), ("write", ctypes.c_int)]


class GdrError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s: %s" % (what, status_string(status)))


_lib = None


def load(path: str = LIB_PATH):
    """Load libgdr.so once and declare its signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError("libgdr.so not found at %s; build it with "
                           "`python -m gated_delta_rule_154_b200.build`" % path)
    lib = ctypes.CDLL(path)
    vp, sz, i = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    dp = ctypes.POINTER(GdrDesc)
    lib.gdr_workspace_size.restype = sz
    lib.gdr_workspace_size.argtypes = [dp]
    lib.gdr_forward_chunked.restype = i
    lib.gdr_forward_chunked.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.gdr_decode_step.restype = i
    lib.gdr_decode_step.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.gdr_last_device_error.restype = i
    lib.gdr_last_device_error.argtypes = [vp]
    lib.gdr_status_string.restype = ctypes.c_char_p
    lib.gdr_status_string.argtypes = [i]
    lib.gdr_version.restype = i
    lib.gdr_version.argtypes = []
    lib.gdr_forward_varlen.restype = i
    lib.gdr_forward_varlen.argtypes = [dp, vp, i, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.gdr_decode_step_paged.restype = i
    lib.gdr_decode_step_paged.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, i, vp, vp]
    lib.gdr_backward_workspace_size.restype = sz
    lib.gdr_backward_workspace_size.argtypes = [dp]
    lib.gdr_backward_chunked.restype = i
    lib.gdr_backward_chunked.argtypes = [dp] + [vp] * 17 + [sz, vp]
    lib.gdr_backward_varlen_workspace_size.restype = sz
    lib.gdr_backward_varlen_workspace_size.argtypes = [dp, i]
    lib.gdr_backward_varlen.restype = i
    lib.gdr_backward_varlen.argtypes = [dp, vp, i] + [vp] * 17 + [sz, vp]
    lib.gdr_backward_chunked_noalloc.restype = i
    lib.gdr_backward_chunked_noalloc.argtypes = [dp] + [vp] * 16 + [vp]
    lib.gdr_segment_maps_workspace_size.restype = sz
    lib.gdr_segment_maps_workspace_size.argtypes = [dp]
    lib.gdr_segment_maps.restype = i
    lib.gdr_segment_maps.argtypes = [dp] + [vp] * 9 + [sz, vp]
    ll = ctypes.c_longlong
    lib.gdr_segment_scan.restype = i
    lib.gdr_segment_scan.argtypes = [i, i, i, i, i, ll, ll, vp, vp, vp, vp, vp, vp]
    lib.gdr_segmented_workspace_size.restype = sz
    lib.gdr_segmented_workspace_size.argtypes = [dp, i]
    lib.gdr_forward_segmented.restype = i
    lib.gdr_forward_segmented.argtypes = [dp, i] + [vp] * 10 + [sz, vp]
    lib.gdr_test_skip_signal.restype = None
    lib.gdr_test_skip_signal.argtypes = [i]
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().gdr_status_string(int(status)).decode()


def workspace_size(desc: GdrDesc) -> int:
    return int(load().gdr_workspace_size(ctypes.byref(desc)))


def forward_chunked(desc: GdrDesc, q, k, v, a, b, w, s0, o, s_final, workspace, ws_bytes,
                    stream) -> int:
    """Raw call: every pointer an int (0 = NULL).  Returns the gdr_status."""
    return int(load().gdr_forward_chunked(ctypes.byref(desc), q, k, v, a, b, w, s0, o,
                                          s_final, workspace, ws_bytes, stream))


def decode_step(desc: GdrDesc, q, k, v, a, b, w, state, o, stream) -> int:
    """Raw call: every pointer an int (0 = NULL).  Returns the gdr_status."""
    return int(load().gdr_decode_step(ctypes.byref(desc), q, k, v, a, b, w, state, o, stream))


def forward_varlen(desc: GdrDesc, cu_seqlens, n_seqs, q, k, v, a, b, w, s0, o, s_final,
                   workspace, ws_bytes, stream) -> int:
    """Raw call: every pointer an int (0 = NULL).  Returns the gdr_status."""
    return int(load().gdr_forward_varlen(ctypes.byref(desc), cu_seqlens, int(n_seqs), q, k, v,
                                         a, b, w, s0, o, s_final, workspace, ws_bytes, stream))


def decode_step_paged(desc: GdrDesc, q, k, v, a, b, w, pool, slot, n_slots, o, stream) -> int:
    """Raw call: every pointer an int (0 = NULL).  Returns the gdr_status."""
    return int(load().gdr_decode_step_paged(ctypes.byref(desc), q, k, v, a, b, w, pool, slot,
                                            int(n_slots), o, stream))


def backward_workspace_size(desc: GdrDesc) -> int:
    return int(load().gdr_backward_workspace_size(ctypes.byref(desc)))


def backward_chunked(desc: GdrDesc, q, k, v, a, b, w, s0, d_o, ds_final, dq, dk, dv, da, db,
                     dw, ds0, workspace, ws_bytes, stream) -> int:
    """Raw call: every pointer an int (0 = NULL).  Returns the gdr_status."""
    return int(load().gdr_backward_chunked(ctypes.byref(desc), q, k, v, a, b, w, s0, d_o,
                                           ds_final, dq, dk, dv, da, db, dw, ds0, workspace,
                                           ws_bytes, stream))


def backward_chunked_noalloc(desc: GdrDesc, q, k, v, a, b, w, s0, d_o, ds_final, dq, dk, dv,
                             da, db, dw, ds0, stream) -> int:
    """Raw call: every pointer an int (0 = NULL).  Returns the gdr_status."""
    return int(load().gdr_backward_chunked_noalloc(ctypes.byref(desc), q, k, v, a, b, w, s0,
                                                   d_o, ds_final, dq, dk, dv, da, db, dw, ds0,
                                                   stream))


def backward_varlen_workspace_size(desc: GdrDesc, n_seqs: int) -> int:
    return int(load().gdr_backward_varlen_workspace_size(ctypes.byref(desc), int(n_seqs)))


def backward_varlen(desc: GdrDesc, cu_seqlens, n_seqs, q, k, v, a, b, w, s0, d_o, ds_final,
                    dq, dk, dv, da, db, dw, ds0, workspace, ws_bytes, stream) -> int:
    """Raw call: every pointer an int (0 = NULL).  Returns the gdr_status."""
    return int(load().gdr_backward_varlen(ctypes.byref(desc), cu_seqlens, int(n_seqs), q, k, v,
                                          a, b, w, s0, d_o, ds_final, dq, dk, dv, da, db, dw,
                                          ds0, workspace, ws_bytes, stream))


def segment_maps_workspace_size(desc: GdrDesc) -> int:
    return int(load().gdr_segment_maps_workspace_size(ctypes.byref(desc)))


def segment_maps(desc: GdrDesc, q, k, v, a, b, w, m_out, n_out, workspace, ws_bytes,
                 stream) -> int:
    """Raw call: every pointer an int (0 = NULL).  Returns the gdr_status."""
    return int(load().gdr_segment_maps(ctypes.byref(desc), q, k, v, a, b, w, m_out, n_out,
                                       workspace, ws_bytes, stream))


def segment_scan(n_segments, B, H, dk, dv, seg_stride, batch_stride, m, n, s0, s_start,
                 s_final, stream) -> int:
    """Raw call: every pointer an int (0 = NULL).  Returns the gdr_status."""
    return int(load().gdr_segment_scan(int(n_segments), int(B), int(H), int(dk), int(dv),
                                       int(seg_stride), int(batch_stride), m, n, s0, s_start,
                                       s_final, stream))


def segmented_workspace_size(desc: GdrDesc, n_segments: int) -> int:
    return int(load().gdr_segmented_workspace_size(ctypes.byref(desc), int(n_segments)))


def forward_segmented(desc: GdrDesc, n_segments, q, k, v, a, b, w, s0, o, s_final, workspace,
                      ws_bytes, stream) -> int:
    """Raw call: every pointer an int (0 = NULL).  Returns the gdr_status."""
    return int(load().gdr_forward_segmented(ctypes.byref(desc), int(n_segments), q, k, v, a, b,
                                            w, s0, o, s_final, workspace, ws_bytes, stream))


def last_device_error(stream) -> int:
    return int(load().gdr_last_device_error(stream))
