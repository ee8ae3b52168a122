"""GPU parity of the chunked prefill against the float64 oracle, through the
library's C ABI (via the thin torch binding), plus the properties the
recurrence fixes at any size: chunk-size invariance, resume, head
permutation, in-place state, empty input, and agreement with the decode
kernel run token by token.

Tolerances (max |x - ref| / max |ref| per tensor): 1e-4 for float32 inputs,
2e-2 for bf16 inputs (state float32 in both)."""

import numpy as np
import pytest
import torch

from gated_delta_rule_154_b200 import _lib, api
from gated_delta_rule_154_b200 import workload as W
from gpu_helpers import (TOL, gpu_prefill, inputs_to_dev, oracle_prefill, rel_err, report,
                         to_dev, to_host)

pytestmark = pytest.mark.gpu


def _check_full(wl, inp, chunk=None):
    o, s = gpu_prefill(wl, inp, chunk)
    o_ref, s_ref = oracle_prefill(wl, inp)
    eo, es = rel_err(to_host(o), o_ref), rel_err(to_host(s), s_ref)
    assert eo <= TOL[wl.dtype] and es <= TOL[wl.dtype], (wl.name, chunk, eo, es)
    return eo, es


def test_gdn_fp32_full_workload():
    """Gated DeltaNet, scalar gates, float32: B=1 H=2 T=256 d=64 chunk 64."""
    wl = W.WORKLOADS["gdn_fp32"]
    _check_full(wl, W.make_prefill(wl))


@pytest.mark.parametrize("name", ["gdn_fp32", "kda_bf16", "gdn2_bf16", "long_bf16"])
@pytest.mark.parametrize("T", [64, 200, 333])
def test_small_shapes_every_gate_kind(name, T):
    """Reduced B/H/T of each prefill workload, with ragged tails."""
    wl = W.WORKLOADS[name].replace(B=2, H=3, T=T)
    _check_full(wl, W.make_prefill(wl, seed=T))


@pytest.mark.parametrize("chunk", [16, 32, 64])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 64), (64, 128), (128, 128)])
def test_chunk_sizes_and_head_dims_fp32(chunk, dk, dv):
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=1, H=2, T=150, dk=dk, dv=dv, dtype="f32", chunk=chunk)
    _check_full(wl, W.make_prefill(wl, seed=chunk + dk + dv))


@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_chunk_sizes_bf16(chunk):
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=1, H=2, T=300, chunk=chunk)
    _check_full(wl, W.make_prefill(wl, seed=7))


def test_gate_one_everywhere():
    """a = b = w = 1 given as GATE_ONE (no gate tensors): plain DeltaNet."""
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=1, H=2, T=130, dtype="f32")
    inp = W.make_prefill(wl, seed=3)
    d = inputs_to_dev(inp, wl)
    o, s = api.forward_chunked(d["q"], d["k"], d["v"], None, None, None, d["s0"], chunk=64)
    ones_k = np.ones_like(inp["a"])
    ref = dict(inp, a=ones_k, b=ones_k, w=np.ones_like(inp["w"]))
    o_ref, s_ref = oracle_prefill(wl, ref)
    assert rel_err(to_host(o), o_ref) <= 1e-4 and rel_err(to_host(s), s_ref) <= 1e-4


def test_chunk_size_invariance_fp32():
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=2, H=2, T=256, dtype="f32")
    inp = W.make_prefill(wl, seed=11)
    o16, s16 = gpu_prefill(wl, inp, 16)
    o64, s64 = gpu_prefill(wl, inp, 64)
    assert rel_err(to_host(o16), to_host(o64)) <= 1e-4
    assert rel_err(to_host(s16), to_host(s64)) <= 1e-4


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_resume_split_sequence(dtype):
    """forward(T1) then forward(T2, s0 = S_T1) equals forward(T1 + T2)."""
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=2, H=2, T=320, dtype=dtype)
    inp = W.make_prefill(wl, seed=5)
    d = inputs_to_dev(inp, wl)
    o, s = api.forward_chunked(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"], d["s0"])
    c = 192
    part = lambda x, sl: x[:, sl].contiguous()
    o1, s1 = api.forward_chunked(*(part(d[k], slice(0, c)) for k in "qkvabw"), d["s0"])
    o2, s2 = api.forward_chunked(*(part(d[k], slice(c, None)) for k in "qkvabw"), s1)
    tol = TOL[dtype]
    assert rel_err(to_host(torch.cat([o1, o2], 1)), to_host(o)) <= tol
    assert rel_err(to_host(s2), to_host(s)) <= tol


def test_head_permutation():
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=1, H=4, T=100)
    inp = W.make_prefill(wl, seed=9)
    d = inputs_to_dev(inp, wl)
    perm = torch.tensor([2, 0, 3, 1], device="cuda")
    o, s = api.forward_chunked(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"], d["s0"])
    p = lambda x: x.index_select(2, perm).contiguous()
    op, sp = api.forward_chunked(*(p(d[k]) for k in "qkvabw"), d["s0"].index_select(1, perm).contiguous())
    assert torch.equal(op, o.index_select(2, perm))
    assert torch.equal(sp, s.index_select(1, perm))


def test_in_place_final_state_and_no_final_state():
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=1, H=2, T=130)
    inp = W.make_prefill(wl, seed=2)
    d = inputs_to_dev(inp, wl)
    o, s = api.forward_chunked(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"], d["s0"])
    st = d["s0"].clone()
    o2, s2 = api.forward_chunked(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"], st, s_final=st)
    assert s2.data_ptr() == st.data_ptr()
    assert torch.equal(o2, o) and torch.equal(st, s)
    o3, s3 = api.forward_chunked(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"], d["s0"],
                                 return_final=False)
    assert s3 is None and torch.equal(o3, o)


def test_empty_sequence_returns_initial_state():
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=2, H=2, T=0)
    inp = W.make_prefill(wl.replace(T=1), seed=1)
    s0 = to_dev(inp["s0"], "f32")
    e = lambda d: torch.empty((2, 0, 2, d), dtype=torch.bfloat16, device="cuda")
    o, s = api.forward_chunked(e(128), e(128), e(128), e(128), e(128), e(128), s0)
    torch.cuda.synchronize()
    assert o.shape == (2, 0, 2, 128) and torch.equal(s, s0)
    o, s = api.forward_chunked(e(128), e(128), e(128), e(128), e(128), e(128), None)
    assert torch.count_nonzero(s) == 0


def test_matches_decode_kernel_token_by_token():
    """The chunked kernel and the decode kernel run step by step agree."""
    wl = W.WORKLOADS["kda_bf16"].replace(B=2, H=2, T=70, dtype="f32")
    inp = W.make_prefill(wl, seed=4)
    d = inputs_to_dev(inp, wl)
    o, s = api.forward_chunked(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"], None)
    state = torch.zeros_like(s)
    outs = []
    for t in range(wl.T):
        g = lambda x: x[:, t].contiguous()
        outs.append(api.decode_step(g(d["q"]), g(d["k"]), g(d["v"]), g(d["a"]), g(d["b"]),
                                    g(d["w"]), state))
    torch.cuda.synchronize()
    assert rel_err(to_host(torch.stack(outs, 1)), to_host(o)) <= 1e-4
    assert rel_err(to_host(state), to_host(s)) <= 1e-4


def test_no_device_error_recorded():
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=1, H=2, T=64)
    gpu_prefill(wl, W.make_prefill(wl))
    assert api.last_device_error() == 0


def test_bounded_wait_runs_out_and_reports_timeout():
    """A completion signal that nothing sets (test hook): the kernel's bounded
    wait gives up, everything in flight is drained, the launch ends with
    GDR_ERR_TIMEOUT, and the context stays usable: the next launch is exact
    and records no error."""
    import time
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=1, H=2, T=200)
    inp = W.make_prefill(wl, seed=5)
    assert api.last_device_error() == 0
    api.test_skip_signal(True)
    t = time.perf_counter()
    gpu_prefill(wl, inp)
    assert api.last_device_error() == _lib.ERR_TIMEOUT
    assert time.perf_counter() - t < 60.0
    _check_full(wl, inp)            # the hook was consumed by one launch
    assert api.last_device_error() == 0


# ------------------------------------------------------ full-size workloads

@pytest.mark.parametrize("name,split", [("kda_bf16", True), ("gdn2_bf16", True),
                                        ("long_bf16", True), ("long_bf16", False)])
def test_full_size_every_head(name, split):
    """Full workload on the GPU in the bench's launch configuration, compared
    element by element with the oracle on every (b, h): all outputs o and
    every final state.  The long-context workload (32 heads) runs both ways:
    split into segments by the library (its default with a workspace) and on
    the one-pass kernel.  The per-tensor error, its margin to the tolerance
    and the element-wise error (floor 1e-6) are printed."""
    wl = W.WORKLOADS[name]
    inp = W.make_prefill(wl, seed=0, threads=16)
    o, s = gpu_prefill(wl, inp, split=split)
    name = name + ("" if split else " one launch")
    o_h, s_h = to_host(o), to_host(s)
    del o, s
    o_ref, s_ref = oracle_prefill(wl, inp)
    tol = TOL[wl.dtype]
    msg = [report("%s o" % name, o_h, o_ref, tol), report("%s S_T" % name, s_h, s_ref, tol)]
    assert np.isfinite(o_h).all() and np.isfinite(s_h).all()
    assert rel_err(o_h, o_ref) <= tol and rel_err(s_h, s_ref) <= tol, msg
    # and per head: no single (b, h) may exceed the tolerance on its own scale
    worst = 0.0
    for b in range(wl.B):
        for h in range(wl.H):
            worst = max(worst, rel_err(o_h[b, :, h], o_ref[b, :, h]),
                        rel_err(s_h[b, h], s_ref[b, h]))
    print("%s worst single head: %.3e" % (name, worst), flush=True)
    assert worst <= tol, (name, worst)


@pytest.mark.parametrize("name", ["kda_bf16", "gdn2_bf16"])
def test_tensor_core_kernel_matches_decode_kernel_token_by_token(name):
    """The chunked form on the tcgen05 kernel (bf16, chunk 64) against the
    sequential form run token by token by the decode kernel, same bf16 inputs:
    the two forms must agree within the bf16 tolerance (o per token and the
    final state), with a random initial state and a ragged tail."""
    wl = W.WORKLOADS[name].replace(B=2, H=3, T=203, random_s0=True)
    inp = W.make_prefill(wl, seed=31)
    d = inputs_to_dev(inp, wl)
    o, s = api.forward_chunked(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"], d["s0"],
                               chunk=64)
    state = d["s0"].clone()
    outs = []
    for t in range(wl.T):
        g = lambda x: x[:, t].contiguous()
        outs.append(api.decode_step(g(d["q"]), g(d["k"]), g(d["v"]), g(d["a"]), g(d["b"]),
                                    g(d["w"]), state))
    torch.cuda.synchronize()
    assert api.last_device_error() == 0
    seq_o = to_host(torch.stack(outs, 1))
    msg = [report("%s chunked vs sequential o" % name, to_host(o), seq_o, TOL["bf16"]),
           report("%s chunked vs sequential S_T" % name, to_host(s), to_host(state),
                  TOL["bf16"])]
    assert rel_err(to_host(o), seq_o) <= TOL["bf16"], msg
    assert rel_err(to_host(s), to_host(state)) <= TOL["bf16"], msg


@pytest.mark.parametrize("a_val", [0.25, 0.2])
def test_strong_decay_inside_the_range_matches_oracle(a_val):
    """One key channel decays by a_val at every token of whole chunks: the
    decay over the chunk (0.25^64 = 2^-128) is below float32's normal range,
    but every factor the kernel forms (a product over at most half a chunk)
    is representable, so the result must match the oracle with no error
    reported."""
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=1, H=2, T=192)
    inp = W.make_prefill(wl, seed=3)
    a = inp["a"].copy()
    a[0, :128, 1, 5] = W.f32_to_bf16_bits(np.full(128, a_val, np.float32))
    a[0, 64:, 0, 77] = W.f32_to_bf16_bits(np.full(128, a_val, np.float32))
    inp = dict(inp, a=a)
    o, s = gpu_prefill(wl, inp, 64)
    assert api.last_device_error() == 0
    o_ref, s_ref = oracle_prefill(wl, inp)
    msg = [report("a=%g o" % a_val, to_host(o), o_ref, TOL["bf16"]),
           report("a=%g S_T" % a_val, to_host(s), s_ref, TOL["bf16"])]
    assert np.isfinite(to_host(o)).all() and np.isfinite(to_host(s)).all()
    assert rel_err(to_host(o), o_ref) <= TOL["bf16"], msg
    assert rel_err(to_host(s), s_ref) <= TOL["bf16"], msg


def test_zero_decay_on_a_chunks_first_token():
    """a = 0 at the first token of a chunk resets that channel's state there;
    no divisor holds that token's decay, so the kernel computes it exactly."""
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=1, H=2, T=192)
    inp = W.make_prefill(wl, seed=8)
    a = inp["a"].copy()
    a[0, 64, :, :9] = W.f32_to_bf16_bits(np.zeros((2, 9), np.float32))
    inp = dict(inp, a=a)
    o, s = gpu_prefill(wl, inp, 64)
    assert api.last_device_error() == 0
    o_ref, s_ref = oracle_prefill(wl, inp)
    assert rel_err(to_host(o), o_ref) <= TOL["bf16"]
    assert rel_err(to_host(s), s_ref) <= TOL["bf16"]


@pytest.mark.parametrize("name", ["kda_bf16", "gdn2_bf16"])
def test_full_size_repeatable_bit_for_bit(name):
    """The kernels fix every reduction order, so repeated launches on the same
    inputs must agree bit for bit; a shared-memory or tensor-memory race
    between a chunk's steps shows up here as a difference (or a non-finite
    value) somewhere in the full output, not only in sampled heads."""
    wl = W.WORKLOADS[name]
    inp = W.make_prefill(wl, seed=1)
    d = inputs_to_dev(inp, wl)
    runs = []
    for _ in range(4):
        o, s = api.forward_chunked(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"], d["s0"],
                                   chunk=wl.chunk)
        torch.cuda.synchronize()
        runs.append((o.clone(), s.clone()))
    o0, s0 = runs[0]
    assert torch.isfinite(o0.float()).all() and torch.isfinite(s0).all()
    for o, s in runs[1:]:
        assert torch.equal(o, o0) and torch.equal(s, s0)


# ------------------------------------------- tensor-core kernel specific checks

@pytest.mark.parametrize("name", ["kda_bf16", "gdn2_bf16"])
def test_tensor_core_kernel_matches_float32_kernel(name):
    """bf16 inputs, chunk 64 runs on the tcgen05 kernel; chunk 32 on the
    float32 CUDA-core kernel.  Same inputs, same recurrence."""
    wl = W.WORKLOADS[name].replace(B=2, H=4, T=517)
    inp = W.make_prefill(wl, seed=17)
    o64, s64 = gpu_prefill(wl, inp, 64)
    o32, s32 = gpu_prefill(wl, inp, 32)
    assert rel_err(to_host(o64), to_host(o32)) <= TOL["bf16"]
    assert rel_err(to_host(s64), to_host(s32)) <= TOL["bf16"]


def test_tensor_core_scalar_decay_and_gate_one():
    """Scalar decay, no erase gate (b = 1), scalar write gate, bf16."""
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=1, H=3, T=190, decay="scalar", erase="scalar",
                                          write="scalar")
    inp = W.make_prefill(wl, seed=23)
    d = inputs_to_dev(inp, wl)
    o, s = api.forward_chunked(d["q"], d["k"], d["v"], d["a"], None, d["w"], d["s0"], chunk=64)
    torch.cuda.synchronize()
    ref = dict(inp, b=np.full_like(inp["b"], W.f32_to_bf16_bits(np.float32(1.0))))
    o_ref, s_ref = oracle_prefill(wl, ref)
    assert rel_err(to_host(o), o_ref) <= TOL["bf16"]
    assert rel_err(to_host(s), s_ref) <= TOL["bf16"]
    assert api.last_device_error() == 0


def test_decay_beyond_tensor_core_range_is_reported():
    """A decay strong enough that exp(decay over half a chunk) leaves float
    range is flagged as GDR_ERR_RANGE on the tensor-core kernel, and the
    error word is cleared once read."""
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=1, H=2, T=64)
    inp = W.make_prefill(wl, seed=1)
    a = inp["a"].copy()
    a[0, :, 1, 5] = W.f32_to_bf16_bits(np.full(64, 0.01, np.float32))  # log(0.01)*32 < -80
    inp = dict(inp, a=a)
    gpu_prefill(wl, inp, 64)
    assert api.last_device_error() == 6   # GDR_ERR_RANGE
    assert api.last_device_error() == 0
    # the float32 kernel (chunk 32) has no such limit and matches the oracle
    o, s = gpu_prefill(wl, inp, 32)
    o_ref, s_ref = oracle_prefill(wl, inp)
    assert rel_err(to_host(o), o_ref) <= TOL["bf16"] and rel_err(to_host(s), s_ref) <= TOL["bf16"]
