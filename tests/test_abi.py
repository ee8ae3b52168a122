"""The C ABI without a GPU: the library loads, exports every entry point that
include/gdr.h declares, and rejects bad arguments on the host before any CUDA
call (no compute call is made here)."""

import ctypes
import os
import re

import pytest

from gated_delta_rule_154_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "gdr.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdr_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_documented_calls():
    names = _declared_functions()
    for n in ("gdr_forward_chunked", "gdr_decode_step", "gdr_workspace_size",
              "gdr_status_string", "gdr_last_device_error"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name
    assert set(_lib.EXPORTS) <= set(_declared_functions())


def test_status_strings(lib):
    assert _lib.status_string(_lib.OK) == "GDR_OK"
    assert _lib.status_string(_lib.ERR_RANGE) == "GDR_ERR_RANGE"
    assert _lib.status_string(99) == "GDR_UNKNOWN_STATUS"
    assert lib.gdr_version() >= 0x000100


def _desc(**kw):
    base = dict(B=2, T=128, H=4, dk=128, dv=128, chunk=64, in_dtype=_lib.BF16,
                decay=_lib.GATE_VECTOR, erase=_lib.GATE_VECTOR, write=_lib.GATE_VECTOR)
    base.update(kw)
    return _lib.GdrDesc(**base)


def test_workspace_is_host_only_and_zero(lib):
    assert _lib.workspace_size(_desc()) == 0
    assert lib.gdr_workspace_size(None) == 0


P = 1 << 20  # a 16-byte-aligned fake address: never dereferenced, checks fail first


@pytest.mark.parametrize("field,value", [
    ("B", 0), ("H", 0), ("T", -1), ("dk", 96), ("dv", 32), ("chunk", 48),
    ("in_dtype", 7), ("decay", 3), ("erase", -1), ("write", 5)])
def test_bad_descriptor_rejected(lib, field, value):
    d = _desc(**{field: value})
    st = _lib.forward_chunked(d, P, P, P, P, P, P, 0, P, 0, 0, 0, 0)
    assert st == _lib.ERR_INVALID_ARG
    d.T = 1
    setattr(d, field, value)
    if field != "T":
        st = _lib.decode_step(d, P, P, P, P, P, P, P, P, 0)
        assert st == _lib.ERR_INVALID_ARG


@pytest.mark.parametrize("which", range(7))
def test_null_or_misaligned_pointer_rejected(lib, which):
    ptrs = [P] * 7  # q k v a b w o
    for bad in (0, P + 8):
        p = list(ptrs)
        p[which] = bad
        q, k, v, a, b, w, o = p
        assert _lib.forward_chunked(_desc(), q, k, v, a, b, w, 0, o, 0, 0, 0, 0) == _lib.ERR_INVALID_ARG
        assert _lib.decode_step(_desc(T=1), q, k, v, a, b, w, P, o, 0) == _lib.ERR_INVALID_ARG


def test_misaligned_state_rejected(lib):
    assert _lib.forward_chunked(_desc(), P, P, P, P, P, P, P + 4, P, 0, 0, 0, 0) == _lib.ERR_INVALID_ARG
    assert _lib.forward_chunked(_desc(), P, P, P, P, P, P, 0, P, P + 4, 0, 0, 0) == _lib.ERR_INVALID_ARG
    assert _lib.decode_step(_desc(T=1), P, P, P, P, P, P, 0, P, 0) == _lib.ERR_INVALID_ARG


def test_decode_needs_t_equal_one(lib):
    assert _lib.decode_step(_desc(T=2), P, P, P, P, P, P, P, P, 0) == _lib.ERR_INVALID_ARG


def test_gate_one_needs_no_pointer_and_empty_is_a_no_op(lib):
    # T = 0 with no final state: nothing to do, no CUDA call, GDR_OK.
    d = _desc(T=0, decay=_lib.GATE_ONE, erase=_lib.GATE_ONE, write=_lib.GATE_ONE)
    assert _lib.forward_chunked(d, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0) == _lib.OK


def test_null_descriptor(lib):
    assert lib.gdr_forward_chunked(None, *([None] * 9), None, 0, None) == _lib.ERR_INVALID_ARG
    assert lib.gdr_decode_step(None, *([None] * 9)) == _lib.ERR_INVALID_ARG


def test_fg2_gate_kind_accepted_for_erase_and_write_only(lib):
    # accepted (T = 0 and no final state: validated, nothing launched)
    d = _desc(T=0, erase=_lib.GATE_FG2, write=_lib.GATE_FG2)
    assert _lib.forward_chunked(d, P, P, P, P, P, P, 0, P, 0, 0, 0, 0) == _lib.OK
    # FG2 is no decay form, and its learning-rate pointers are required
    assert _lib.forward_chunked(_desc(decay=_lib.GATE_FG2), P, P, P, P, P, P, 0, P, 0, 0, 0,
                                0) == _lib.ERR_INVALID_ARG
    d = _desc(erase=_lib.GATE_FG2, write=_lib.GATE_FG2)
    assert _lib.forward_chunked(d, P, P, P, P, 0, P, 0, P, 0, 0, 0, 0) == _lib.ERR_INVALID_ARG
    assert _lib.forward_chunked(d, P, P, P, P, P, 0, 0, P, 0, 0, 0, 0) == _lib.ERR_INVALID_ARG
    for bad in (4, 99):
        assert _lib.forward_chunked(_desc(erase=bad), P, P, P, P, P, P, 0, P, 0, 0, 0,
                                    0) == _lib.ERR_INVALID_ARG


def test_paged_decode_argument_checks(lib):
    d = _desc(T=1)
    ok = dict(q=P, k=P, v=P, a=P, b=P, w=P, pool=P, slot=P, n=4, o=P)

    def call(**kw):
        x = dict(ok)
        x.update(kw)
        return _lib.decode_step_paged(d, x["q"], x["k"], x["v"], x["a"], x["b"], x["w"],
                                      x["pool"], x["slot"], x["n"], x["o"], 0)
    assert call(slot=0) == _lib.ERR_INVALID_ARG        # slot array required
    assert call(slot=P + 2) == _lib.ERR_INVALID_ARG    # int32 alignment
    assert call(pool=0) == _lib.ERR_INVALID_ARG
    assert call(pool=P + 4) == _lib.ERR_INVALID_ARG
    assert call(n=0) == _lib.ERR_INVALID_ARG
    d.T = 2
    assert call() == _lib.ERR_INVALID_ARG


def test_varlen_argument_checks(lib):
    cu = P
    d = _desc(B=1)
    assert _lib.forward_varlen(d, 0, 2, P, P, P, P, P, P, 0, P, 0, 0, 0, 0) == _lib.ERR_INVALID_ARG
    assert _lib.forward_varlen(d, P + 2, 2, P, P, P, P, P, P, 0, P, 0, 0, 0, 0) == _lib.ERR_INVALID_ARG
    assert _lib.forward_varlen(d, cu, 0, P, P, P, P, P, P, 0, P, 0, 0, 0, 0) == _lib.ERR_INVALID_ARG
    assert _lib.forward_varlen(_desc(B=2), cu, 2, P, P, P, P, P, P, 0, P, 0, 0, 0,
                               0) == _lib.ERR_INVALID_ARG
    assert _lib.forward_varlen(d, cu, 2, 0, P, P, P, P, P, 0, P, 0, 0, 0, 0) == _lib.ERR_INVALID_ARG
    # nothing to do: no tokens and no final state
    d0 = _desc(B=1, T=0)
    assert _lib.forward_varlen(d0, cu, 2, P, P, P, P, P, P, 0, P, 0, 0, 0, 0) == _lib.OK


def _bwd(d, **kw):
    """gdr_backward_chunked with every pointer a valid fake address unless given."""
    names = ("q", "k", "v", "a", "b", "w", "s0", "d_o", "ds_final", "dq", "dk", "dv", "da",
             "db", "dw", "ds0", "ws")
    p = {n: P for n in names}
    p["s0"] = p["ds_final"] = p["ds0"] = 0
    p.update(kw)
    ws_bytes = kw.pop("ws_bytes", None)
    if ws_bytes is None:
        ws_bytes = _lib.backward_workspace_size(d)
    return _lib.backward_chunked(d, *(p[n] for n in names), ws_bytes, 0)


def test_backward_workspace_size(lib):
    d = _desc(B=2, T=100, H=4, dk=128, dv=64)
    # chunk-start states on a 32-token grid plus one running state gradient
    assert _lib.backward_workspace_size(d) == 2 * 4 * 128 * 64 * 4 * (4 + 1)
    assert _lib.backward_workspace_size(_desc(T=0)) == 2 * 4 * 128 * 128 * 4
    # bf16, d = 128: bf16 states at 64-token chunk starts and S_T, E, five
    # bf16 intermediates, two rows per chunk and head
    tc = _desc(B=2, T=100, H=4)
    assert _lib.backward_workspace_size(tc) == 2 * 4 * (2 * 33792 + 65536) + 2 * 100 * 4 * 1536
    # packed sequences keep the 32-token layout
    assert _lib.backward_varlen_workspace_size(_desc(B=1, T=100, H=4), 3) == \
        4 * 128 * 128 * 4 * (4 + 2 * 3)
    assert _lib.backward_workspace_size(_desc(dk=96)) == 0
    assert lib.gdr_backward_workspace_size(None) == 0


def test_backward_argument_checks(lib):
    d = _desc()
    assert _bwd(_desc(dk=96)) == _lib.ERR_INVALID_ARG
    for name in ("q", "k", "v", "a", "b", "w", "d_o", "dq", "dk", "dv", "da", "db", "dw"):
        assert _bwd(d, **{name: 0}) == _lib.ERR_INVALID_ARG, name
        assert _bwd(d, **{name: P + 8}) == _lib.ERR_INVALID_ARG, name
    for name in ("s0", "ds_final", "ds0"):
        assert _bwd(d, **{name: P + 4}) == _lib.ERR_INVALID_ARG, name
    assert _bwd(d, ws=0) == _lib.ERR_WORKSPACE
    assert _bwd(d, ws_bytes=_lib.backward_workspace_size(d) - 1) == _lib.ERR_WORKSPACE
    assert _bwd(d, ws=P + 8) == _lib.ERR_INVALID_ARG
    # FG^2-GDN learning rates are accepted (no tokens, no dS0: validated, nothing launched)
    fg2 = _desc(T=0, erase=_lib.GATE_FG2, write=_lib.GATE_FG2)
    assert _bwd(fg2) == _lib.OK
    # absent gates need neither the gate nor its gradient
    one = _desc(T=0, decay=_lib.GATE_ONE, erase=_lib.GATE_ONE, write=_lib.GATE_ONE)
    assert _bwd(one, a=0, b=0, w=0, da=0, db=0, dw=0) == _lib.OK  # nothing to write


def test_backward_varlen_workspace_and_checks(lib):
    d = _desc(B=1, T=100, H=4, dk=128, dv=64)
    mat = 128 * 64 * 4
    # at most ceil(T / 32) + n_seqs chunk-start states per head, then n_seqs running dS
    assert _lib.backward_varlen_workspace_size(d, 3) == 4 * mat * (4 + 3 + 3)
    assert _lib.backward_varlen_workspace_size(d, 0) == 0
    assert _lib.backward_varlen_workspace_size(_desc(dk=96), 2) == 0
    need = _lib.backward_varlen_workspace_size(d, 3)
    args = lambda **kw: dict(dict(q=P, k=P, v=P, a=P, b=P, w=P, s0=0, d_o=P, ds_final=0, dq=P,
                                  dk=P, dv=P, da=P, db=P, dw=P, ds0=0, ws=P, ws_bytes=need), **kw)
    def call(desc, cu, n, **kw):
        x = args(**kw)
        return _lib.backward_varlen(desc, cu, n, x["q"], x["k"], x["v"], x["a"], x["b"], x["w"],
                                    x["s0"], x["d_o"], x["ds_final"], x["dq"], x["dk"], x["dv"],
                                    x["da"], x["db"], x["dw"], x["ds0"], x["ws"], x["ws_bytes"], 0)
    assert call(d, 0, 3) == _lib.ERR_INVALID_ARG            # no cu_seqlens
    assert call(d, P + 2, 3) == _lib.ERR_INVALID_ARG        # misaligned cu_seqlens
    assert call(d, P, 0) == _lib.ERR_INVALID_ARG            # no sequence
    assert call(_desc(B=2), P, 3) == _lib.ERR_INVALID_ARG   # packed sequences need B = 1
    assert call(d, P, 3, ws_bytes=need - 1) == _lib.ERR_WORKSPACE
    assert call(d, P, 3, dq=0) == _lib.ERR_INVALID_ARG
    # no tokens and no dS0: validated, nothing launched
    assert call(_desc(B=1, T=0), P, 2, ws_bytes=_lib.backward_varlen_workspace_size(
        _desc(B=1, T=0), 2)) == _lib.OK


@pytest.mark.parametrize("dtype,T", [("bf16", 40000), ("f32", 32 * 1024)])
def test_noalloc_refuses_a_problem_larger_than_its_scratch_before_any_cuda_call(lib, dtype, T):
    """The no-allocation backward refuses a problem whose workspace exceeds its
    64 MiB scratch with GDR_ERR_WORKSPACE, on the host, before any CUDA call
    (so also here, without a GPU): bf16 at d = 128 takes the tensor-core path
    (about 2 KiB per token-head), float32 the mma.sync one (64 KiB per 32
    tokens and head)."""
    desc = _lib.GdrDesc(B=1, T=T, H=1, dk=128, dv=128, chunk=64,
                        in_dtype=_lib.BF16 if dtype == "bf16" else _lib.F32,
                        decay=_lib.GATE_VECTOR, erase=_lib.GATE_VECTOR, write=_lib.GATE_VECTOR)
    assert _lib.backward_workspace_size(desc) > _lib.NOALLOC_SCRATCH_BYTES
    p = 1 << 20   # never dereferenced
    assert _lib.backward_chunked_noalloc(desc, *([p] * 16), 0) == _lib.ERR_WORKSPACE
