"""float64 CPU oracle of the gated delta-rule recurrence.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The CUDA library never
imports, links or loads anything from here, and this package imports nothing
from the CUDA side.

The arithmetic lives in ``gdr_oracle.c`` (plain loops, double precision), built
into ``liboracle.so`` with gcc and OpenMP by :func:`build`.  This module only
marshals numpy arrays into it.

Recurrence (per (batch, head), S in R^{dk x dv}), from the FG^2-GDN page
(gist.science 2604.19021), section 2 "Methodology", update rule, with the
decoupled erase/write gates of the Gated DeltaNet-2 page (needhelp.icu), gates
table::

    S'  = Diag(a_t) S_{t-1}
    S_t = S' - (b_t * k_t)(k_t^T S') + k_t (w_t * v_t)^T
    o_t = S_t^T q_t
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdr_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

GATE_ONE, GATE_SCALAR, GATE_VECTOR = 0, 1, 2

_default = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile a C oracle source into a shared library (gcc -O2 -fopenmp)."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    tmp = out + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared",
           "-fno-fast-math", "-ffp-contract=off", src, "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


class Oracle:
    """ctypes view of one compiled oracle library."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        f32p = ctypes.POINTER(ctypes.c_float)
        f64p = ctypes.POINTER(ctypes.c_double)
        i = ctypes.c_int
        lib.oracle_forward.restype = i
        lib.oracle_forward.argtypes = [i, i, i, i, i, i, i, i,
                                       f32p, f32p, f32p, f32p, f32p, f32p,
                                       f64p, f64p, f64p, i]
        lib.oracle_decode_step.restype = i
        lib.oracle_decode_step.argtypes = [i, i, i, i, i, i, i,
                                           f32p, f32p, f32p, f32p, f32p, f32p,
                                           f64p, f64p, i]
        lib.oracle_backward.restype = i
        lib.oracle_backward.argtypes = [i, i, i, i, i, i, i, i,
                                        f32p, f32p, f32p, f32p, f32p, f32p,
                                        f64p, f64p, f64p,
                                        f64p, f64p, f64p, f64p, f64p, f64p, f64p, i]
        lib.oracle_max_threads.restype = i
        lib.oracle_max_threads.argtypes = []
        self.lib = lib
        self.path = path

    def max_threads(self) -> int:
        return int(self.lib.oracle_max_threads())

    def forward(self, q, k, v, a=None, b=None, w=None, s0=None, *, want_o=True,
                nthreads: int = 0):
        return _forward(self.lib, q, k, v, a, b, w, s0, want_o, nthreads)

    def decode_step(self, q, k, v, a, b, w, state, *, nthreads: int = 0):
        return _decode_step(self.lib, q, k, v, a, b, w, state, nthreads)

    def backward(self, q, k, v, a, b, w, s0, do, dsT=None, *, nthreads: int = 0):
        return _backward(self.lib, q, k, v, a, b, w, s0, do, dsT, nthreads)


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def max_threads() -> int:
    """OpenMP threads the oracle runs with by default."""
    return default().max_threads()


def _f32(x):
    if x is None:
        return None, None
    arr = np.ascontiguousarray(x, dtype=np.float32)
    return arr, arr.ctypes.data_as(ctypes.POINTER(ctypes.c_float))


def _f64(x):
    if x is None:
        return None, None
    arr = np.ascontiguousarray(x, dtype=np.float64)
    return arr, arr.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _kind(g, full_shape_k, scalar_shape):
    if g is None:
        return GATE_ONE
    g = np.asarray(g)
    if g.shape == tuple(scalar_shape):
        return GATE_SCALAR
    if g.shape == tuple(full_shape_k):
        return GATE_VECTOR
    raise ValueError("gate shape %s matches neither %s nor %s"
                     % (g.shape, scalar_shape, full_shape_k))


def _forward(lib, q, k, v, a, b, w, s0, want_o, nthreads):
    q = np.asarray(q)
    B, T, H, dk = q.shape
    dv = np.asarray(v).shape[-1]
    ak = _kind(a, (B, T, H, dk), (B, T, H))
    bk = _kind(b, (B, T, H, dk), (B, T, H))
    wk = _kind(w, (B, T, H, dv), (B, T, H))
    keep = []
    ptrs = []
    for x in (q, k, v, a, b, w):
        arr, p = _f32(x)
        keep.append(arr)
        ptrs.append(p)
    s0a, s0p = _f64(s0)
    o = np.empty((B, T, H, dv), np.float64) if want_o else None
    sT = np.empty((B, H, dk, dv), np.float64)
    op = o.ctypes.data_as(ctypes.POINTER(ctypes.c_double)) if want_o else None
    rc = lib.oracle_forward(B, T, H, dk, dv, ak, bk, wk, *ptrs, s0p, op,
                            sT.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                            int(nthreads))
    if rc != 0:
        raise RuntimeError("oracle_forward failed (%d)" % rc)
    del keep, s0a
    return o, sT


def _backward(lib, q, k, v, a, b, w, s0, do, dsT, nthreads):
    q = np.asarray(q)
    B, T, H, dk = q.shape
    dv = np.asarray(v).shape[-1]
    ak = _kind(a, (B, T, H, dk), (B, T, H))
    bk = _kind(b, (B, T, H, dk), (B, T, H))
    wk = _kind(w, (B, T, H, dv), (B, T, H))
    keep = []
    ptrs = []
    for x in (q, k, v, a, b, w):
        arr, p = _f32(x)
        keep.append(arr)
        ptrs.append(p)
    for x in (s0, do, dsT):
        arr, p = _f64(x)
        keep.append(arr)
        ptrs.append(p)
    f64 = lambda shape: np.zeros(shape, np.float64)
    gate_shape = lambda kind, d: None if kind == GATE_ONE else (
        (B, T, H) if kind == GATE_SCALAR else (B, T, H, d))
    out = {"dq": f64((B, T, H, dk)), "dk": f64((B, T, H, dk)), "dv": f64((B, T, H, dv)),
           "da": None, "db": None, "dw": None, "ds0": f64((B, H, dk, dv))}
    for name, kind, d in (("da", ak, dk), ("db", bk, dk), ("dw", wk, dv)):
        shp = gate_shape(kind, d)
        out[name] = f64(shp) if shp is not None else None
    optr = [None if out[n] is None else out[n].ctypes.data_as(ctypes.POINTER(ctypes.c_double))
            for n in ("dq", "dk", "dv", "da", "db", "dw", "ds0")]
    rc = lib.oracle_backward(B, T, H, dk, dv, ak, bk, wk, *ptrs, *optr, int(nthreads))
    if rc != 0:
        raise RuntimeError("oracle_backward failed (%d)" % rc)
    del keep
    return out


def _decode_step(lib, q, k, v, a, b, w, state, nthreads):
    q = np.asarray(q)
    B, H, dk = q.shape
    dv = np.asarray(v).shape[-1]
    ak = _kind(a, (B, H, dk), (B, H))
    bk = _kind(b, (B, H, dk), (B, H))
    wk = _kind(w, (B, H, dv), (B, H))
    keep = []
    ptrs = []
    for x in (q, k, v, a, b, w):
        arr, p = _f32(x)
        keep.append(arr)
        ptrs.append(p)
    st = np.array(state, dtype=np.float64, copy=True, order="C")
    o = np.empty((B, H, dv), np.float64)
    rc = lib.oracle_decode_step(
        B, H, dk, dv, ak, bk, wk, *ptrs,
        st.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
        o.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), int(nthreads))
    if rc != 0:
        raise RuntimeError("oracle_decode_step failed (%d)" % rc)
    del keep
    return o, st


def forward(q, k, v, a=None, b=None, w=None, s0=None, *, want_o=True,
            nthreads: int = 0):
    """Run the recurrence over all T steps.

    q, k: [B, T, H, dk]; v: [B, T, H, dv]; a, b: [B, T, H, dk] or [B, T, H]
    or None (gate == 1); w: [B, T, H, dv] or [B, T, H] or None;
    s0: [B, H, dk, dv] or None (zeros).  Values are taken as float32 (exact for
    bf16 and fp32 inputs) and the arithmetic runs in float64.

    Returns (o [B, T, H, dv] float64 or None, sT [B, H, dk, dv] float64).
    """
    return default().forward(q, k, v, a, b, w, s0, want_o=want_o, nthreads=nthreads)


def decode_step(q, k, v, a, b, w, state, *, nthreads: int = 0):
    """One decode step, returning (o [B, H, dv], new_state [B, H, dk, dv]).

    q, k: [B, H, dk]; v: [B, H, dv]; a, b: [B, H, dk] or [B, H] or None;
    w: [B, H, dv] or [B, H] or None; state: [B, H, dk, dv] (not modified).
    """
    return default().decode_step(q, k, v, a, b, w, state, nthreads=nthreads)


def backward(q, k, v, a=None, b=None, w=None, s0=None, do=None, dsT=None, *,
             nthreads: int = 0):
    """Gradients of  L = sum_t <o_t, do_t> + <S_T, dsT>  with respect to every
    input of :func:`forward` (reverse-mode differentiation of the recurrence,
    step by step; see ``oracle_backward`` in gdr_oracle.c).

    do: [B, T, H, dv]; dsT: [B, H, dk, dv] or None (zero).  Returns a dict of
    float64 arrays: dq, dk [B, T, H, dk]; dv [B, T, H, dv]; da, db, dw in the
    shape of a, b, w (None where the gate is None); ds0 [B, H, dk, dv].
    """
    return default().backward(q, k, v, a, b, w, s0, do, dsT, nthreads=nthreads)
