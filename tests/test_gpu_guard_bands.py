"""Guard bands around every buffer the kernels write: each output (o, the
final state, the decode state updated in place) is a view into the middle of
a larger allocation whose two ends hold a fixed bit pattern; after the launch
the ends must be bit-for-bit unchanged (no write outside the tensor), and the
outputs must still match the float64 oracle.  Ragged token counts put the
last chunk's partial TMA box and the masked tail rows right at the edge."""

import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_154_b200 import api
from gated_delta_rule_154_b200 import workload as W
from gpu_helpers import TOL, inputs_to_dev, oracle_prefill, rel_err, to_dev, to_host

pytestmark = pytest.mark.gpu

GUARD = 4096  # elements on each side; keeps the inner view 16-byte aligned
PATTERN = {torch.float32: (torch.int32, 0x7FBADBAD), torch.bfloat16: (torch.int16, 0x7FBD)}


def _guarded(shape, dtype):
    n = int(np.prod(shape))
    buf = torch.empty(n + 2 * GUARD, dtype=dtype, device="cuda")
    ity, pat = PATTERN[dtype]
    buf.view(ity).fill_(pat)
    return buf, buf[GUARD:GUARD + n].view(shape)


def _guards_intact(buf):
    ity, pat = PATTERN[buf.dtype]
    bits = buf.view(ity)
    return bool((bits[:GUARD] == pat).all()) and bool((bits[-GUARD:] == pat).all())


@pytest.mark.parametrize("name,T", [("gdn2_bf16", 200), ("kda_bf16", 129), ("gdn_fp32", 77),
                                    ("gdn2_bf16", 64)])
def test_prefill_writes_stay_inside_o_and_final_state(name, T):
    wl = W.WORKLOADS[name].replace(B=2, H=3, T=T)
    inp = W.make_prefill(wl, seed=T)
    d = inputs_to_dev(inp, wl)
    dt = d["q"].dtype
    obuf, o = _guarded((wl.B, wl.T, wl.H, wl.dv), dt)
    sbuf, s = _guarded((wl.B, wl.H, wl.dk, wl.dv), torch.float32)
    api.forward_chunked(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"], d["s0"],
                        chunk=wl.chunk, out=o, s_final=s)
    torch.cuda.synchronize()
    assert _guards_intact(obuf) and _guards_intact(sbuf)
    o_ref, s_ref = oracle_prefill(wl, inp)
    assert rel_err(to_host(o), o_ref) <= TOL[wl.dtype]
    assert rel_err(to_host(s), s_ref) <= TOL[wl.dtype]
    assert api.last_device_error() == 0


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_writes_stay_inside_state_and_o(dtype):
    wl = W.WORKLOADS["decode_bf16"].replace(B=3, H=5, dtype=dtype)
    state_np = W.make_decode_state(wl)
    sbuf, state = _guarded((wl.B, wl.H, wl.dk, wl.dv), torch.float32)
    state.copy_(to_dev(state_np, "f32"))
    inp = W.make_decode_step(wl, 1)
    d = {k: to_dev(inp[k], wl.dtype) for k in ("q", "k", "v", "a", "b", "w")}
    if d["w"] is None:
        d["w"] = d["b"]
    obuf, o = _guarded((wl.B, wl.H, wl.dv), d["q"].dtype)
    api.decode_step(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"], state, out=o)
    torch.cuda.synchronize()
    assert _guards_intact(sbuf) and _guards_intact(obuf)
    f = {k: W.as_f32(inp[k], wl.dtype) for k in ("q", "k", "v", "a", "b", "w")}
    if f["w"] is None:
        f["w"] = f["b"]
    o_ref, s_ref = oracle.decode_step(f["q"], f["k"], f["v"], f["a"], f["b"], f["w"],
                                      state_np.astype(np.float64))
    assert rel_err(to_host(o), o_ref) <= TOL[dtype]
    assert rel_err(to_host(state), s_ref) <= TOL[dtype]
