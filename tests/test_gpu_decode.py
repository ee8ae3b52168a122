"""GPU parity of the single-token decode step against the float64 oracle.

Full decode workload (batch 256, H = 32, d = 128, bf16 inputs, float32 state
~ N(0, 0.1)) checked on every head for 100 consecutive steps; a 64-head slice
is carried through 1000 consecutive steps with fresh inputs each step.
Tolerance 2e-2 for bf16 inputs, 1e-4 for float32 (max |x - ref| / max |ref|)."""

import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_154_b200 import api
from gated_delta_rule_154_b200 import workload as W
from gpu_helpers import TOL, rel_err, report, to_dev, to_host

pytestmark = pytest.mark.gpu


def _step_dev(inp, wl):
    d = {k: to_dev(inp[k], wl.dtype) for k in ("q", "k", "v", "a", "b", "w")}
    if d["w"] is None:
        d["w"] = d["b"]
    return d


def _step_f32(inp, wl):
    f = {k: W.as_f32(inp[k], wl.dtype) for k in ("q", "k", "v", "a", "b", "w")}
    if f["w"] is None:
        f["w"] = f["b"]
    return f


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64), (64, 128)])
@pytest.mark.parametrize("gates", ["vector", "scalar"])
def test_decode_small(dtype, dk, dv, gates):
    shared = "shared" if gates == "scalar" else "vector"
    wl = W.WORKLOADS["decode_bf16"].replace(B=3, H=5, dk=dk, dv=dv, dtype=dtype,
                                            decay=gates, erase=gates, write=shared)
    state_np = W.make_decode_state(wl)
    state = to_dev(state_np, "f32")
    ref_state = state_np.astype(np.float64)
    for step in (1, 2, 3):
        inp = W.make_decode_step(wl, step)
        d, f = _step_dev(inp, wl), _step_f32(inp, wl)
        o = api.decode_step(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"], state)
        o_ref, ref_state = oracle.decode_step(f["q"], f["k"], f["v"], f["a"], f["b"], f["w"],
                                              ref_state)
        torch.cuda.synchronize()
        assert rel_err(to_host(o), o_ref) <= TOL[dtype]
        assert rel_err(to_host(state), ref_state) <= TOL[dtype]


def test_decode_full_batch_hundred_steps():
    """The whole decode batch (256 x 32 heads) through 100 consecutive steps
    with fresh inputs each step, every head compared with the oracle at every
    step (o) and the carried state at steps 1, 10, 50 and 100."""
    wl = W.WORKLOADS["decode_bf16"]
    state_np = W.make_decode_state(wl, threads=16)
    state = to_dev(state_np, "f32")
    ref_state = state_np.astype(np.float64)
    worst_o = 0.0
    for step in range(1, 101):
        inp = W.make_decode_step(wl, step, threads=16)
        d, f = _step_dev(inp, wl), _step_f32(inp, wl)
        o = api.decode_step(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"], state)
        o_ref, ref_state = oracle.decode_step(f["q"], f["k"], f["v"], f["a"], f["b"], f["w"],
                                              ref_state)
        torch.cuda.synchronize()
        eo = rel_err(to_host(o), o_ref)
        worst_o = max(worst_o, eo)
        assert eo <= TOL["bf16"], (step, eo)
        if step in (1, 10, 50, 100):
            msg = report("decode step %d state" % step, to_host(state), ref_state, TOL["bf16"])
            assert rel_err(to_host(state), ref_state) <= TOL["bf16"], msg
    report("decode step 100 o", to_host(o), o_ref, TOL["bf16"])
    print("decode worst o over 100 steps: %.3e" % worst_o, flush=True)


def test_decode_thousand_steps_head_slice():
    """64 heads (the decode workload's H = 32 on 2 batch rows) through 1000
    steps: the float32 state must not drift from the float64 one."""
    wl = W.WORKLOADS["decode_bf16"].replace(B=2)
    state_np = W.make_decode_state(wl)
    state = to_dev(state_np, "f32")
    ref_state = state_np.astype(np.float64)
    worst = 0.0
    for step in range(1, wl.steps + 1):
        inp = W.make_decode_step(wl, step, threads=1)
        d, f = _step_dev(inp, wl), _step_f32(inp, wl)
        o = api.decode_step(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"], state)
        o_ref, ref_state = oracle.decode_step(f["q"], f["k"], f["v"], f["a"], f["b"], f["w"],
                                              ref_state, nthreads=1)
        if step % 100 == 0 or step < 4:
            torch.cuda.synchronize()
            worst = max(worst, rel_err(to_host(o), o_ref))
            assert worst <= TOL["bf16"], (step, worst)
    torch.cuda.synchronize()
    assert rel_err(to_host(state), ref_state) <= TOL["bf16"]


def test_prefill_then_decode_continuity():
    """Prefill of T tokens followed by one decode step equals prefill of T + 1."""
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=2, H=3, T=129, dtype="f32")
    inp = W.make_prefill(wl, seed=21)
    d = {k: to_dev(inp[k], "f32") for k in ("q", "k", "v", "a", "b", "w", "s0")}
    o_all, s_all = api.forward_chunked(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"], d["s0"])
    T = wl.T - 1
    head = lambda x: x[:, :T].contiguous()
    _, s_T = api.forward_chunked(*(head(d[k]) for k in "qkvabw"), d["s0"])
    last = lambda x: x[:, T].contiguous()
    o_last = api.decode_step(*(last(d[k]) for k in "qkvabw"), s_T)
    torch.cuda.synchronize()
    assert rel_err(to_host(o_last), to_host(o_all[:, T])) <= 1e-4
    assert rel_err(to_host(s_T), to_host(s_all)) <= 1e-4
