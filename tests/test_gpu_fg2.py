"""FG^2-GDN and FG^2-GDN+ through the same kernels (gate kind FG2): the
learning rates beta^k (and beta^v) enter through their square roots inside
the kernels.  The oracle runs the spec rule on the mapped inputs
k~ = sqrt(beta^k) k, b = 1, w = sqrt(beta^v) (FG^2-GDN page, section 2
"Methodology": FG2-GDN update rule; the oracle pin pin_fg2gdn_symmetric ties
this mapping to the symmetric form (I - k~k~^T) Diag(a) S + k~ v~^T).
Tolerances as elsewhere: 1e-4 float32, 2e-2 bf16 (max |x - ref| / max |ref|)."""

import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_154_b200 import api
from gated_delta_rule_154_b200 import workload as W
from gpu_helpers import TOL, oracle_prefill, rel_err, to_dev, to_host

pytestmark = pytest.mark.gpu


def _mapped(inp, wl, plus):
    """Inputs of the spec rule that FG^2-GDN(+) stands for (float64 maths,
    handed to the oracle as float32 images)."""
    f = {k: W.as_f32(inp[k], wl.dtype).astype(np.float64) for k in ("k", "b", "w")}
    beta_k = f["b"]
    beta_v = f["w"] if plus else f["b"]
    out = dict(inp)
    for k in ("q", "v", "a"):
        out[k] = W.as_f32(inp[k], wl.dtype)
    out["k"] = (np.sqrt(beta_k) * f["k"]).astype(np.float32)
    out["b"] = np.ones_like(beta_k, dtype=np.float32)
    out["w"] = np.sqrt(beta_v).astype(np.float32)
    return out


@pytest.mark.parametrize("plus", [False, True])
@pytest.mark.parametrize("dtype,d,chunk,T", [("bf16", 128, 64, 200), ("bf16", 128, 64, 64),
                                             ("f32", 64, 64, 150), ("f32", 128, 32, 97)])
def test_fg2_prefill(dtype, d, chunk, T, plus):
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=2, H=3, T=T, dk=d, dv=d, dtype=dtype, chunk=chunk)
    inp = W.make_prefill(wl, seed=T + d)
    dev = {k: to_dev(inp[k], dtype) for k in ("q", "k", "v", "a", "b", "w")}
    s0 = to_dev(inp["s0"], "f32") if inp.get("s0") is not None else None
    o, s = api.forward_fg2(dev["q"], dev["k"], dev["v"], dev["a"], dev["b"],
                           dev["w"] if plus else None, s0, chunk=chunk)
    torch.cuda.synchronize()
    assert api.last_device_error() == 0
    m = _mapped(inp, wl, plus)
    mwl = wl.replace(dtype="f32")  # the mapped inputs are float32 images already
    o_ref, s_ref = oracle_prefill(mwl, m)
    assert rel_err(to_host(o), o_ref) <= TOL[dtype]
    assert rel_err(to_host(s), s_ref) <= TOL[dtype]


@pytest.mark.parametrize("plus", [False, True])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_fg2_decode(dtype, plus):
    wl = W.WORKLOADS["decode_bf16"].replace(B=3, H=5, dtype=dtype)
    state_np = W.make_decode_state(wl)
    state = to_dev(state_np, "f32")
    ref_state = state_np.astype(np.float64)
    for step in (1, 2, 3):
        inp = W.make_decode_step(wl, step)
        d = {k: to_dev(inp[k], dtype) for k in ("q", "k", "v", "a", "b", "w")}
        o = api.decode_step_fg2(d["q"], d["k"], d["v"], d["a"], d["b"],
                                d["w"] if plus else None, state)
        f = _mapped(inp, wl, plus)
        o_ref, ref_state = oracle.decode_step(f["q"], f["k"], f["v"], f["a"], f["b"], f["w"],
                                              ref_state)
        torch.cuda.synchronize()
        assert rel_err(to_host(o), o_ref) <= TOL[dtype]
        assert rel_err(to_host(state), ref_state) <= TOL[dtype]


def test_fg2_prefill_then_decode_continues_the_state():
    """FG^2-GDN prefill of T tokens, then one decode step, equals the prefill
    of T + 1 tokens (bf16, tensor-core prefill path)."""
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=1, H=2, T=129)
    inp = W.make_prefill(wl, seed=11)
    dev = {k: to_dev(inp[k], "bf16") for k in ("q", "k", "v", "a", "b", "w")}
    s0 = to_dev(inp["s0"], "f32")
    o_all, s_all = api.forward_fg2(dev["q"], dev["k"], dev["v"], dev["a"], dev["b"], None, s0)
    cut = lambda t: t[:, :128].contiguous()
    last = lambda t: t[:, 128].contiguous()
    _, s_head = api.forward_fg2(*(cut(dev[k]) for k in ("q", "k", "v", "a", "b")), None, s0)
    o_last = api.decode_step_fg2(*(last(dev[k]) for k in ("q", "k", "v", "a", "b")), None,
                                 s_head)
    torch.cuda.synchronize()
    assert rel_err(to_host(o_last), to_host(o_all[:, 128])) <= TOL["bf16"]
    assert rel_err(to_host(s_head), to_host(s_all)) <= TOL["bf16"]
