"""The backward pass for callers that cannot allocate device memory.

Some callers have no way to call cudaMalloc: a plugin inside a host runtime
that owns all device memory and gives the library no allocator, or
latency-critical code that must not allocate because allocation may
synchronise the device.  gdr_backward_chunked_noalloc serves them: it takes no
workspace and runs the same backward with the library's own file-scope
scratch.  This test calls it through the C ABI (ctypes, raw pointers) and
checks that its gradients equal those of gdr_backward_chunked with a
caller-owned workspace, on two calls in a row (the scratch keeps the first
call's contents when the second starts), and that a problem larger than the
scratch is refused.

The file is named so that pytest collects it after every other test file."""

import ctypes

import numpy as np
import pytest
import torch

from gated_delta_rule_154_b200 import _lib, api
from gated_delta_rule_154_b200 import workload as W
from gpu_helpers import TOL, inputs_to_dev, rel_err, to_dev, to_host

pytestmark = pytest.mark.gpu

GRADS = ("dq", "dk", "dv", "da", "db", "dw", "ds0")


def _ptr(t):
    return 0 if t is None else int(t.data_ptr())


def _run(wl, seed, noalloc):
    inp = W.make_prefill(wl, seed=seed)
    up = W.make_upstream(wl, seed=seed)
    d = inputs_to_dev(inp, wl)
    d_o = to_dev(up["do"], wl.dtype)
    dsT = to_dev(up["dsT"], "f32")
    desc = api.desc_for(d["q"], d["v"], d["a"], d["b"], d["w"], 32)
    g = {"dq": torch.empty_like(d["q"]), "dk": torch.empty_like(d["k"]),
         "dv": torch.empty_like(d["v"]), "da": torch.empty_like(d["a"]),
         "db": torch.empty_like(d["b"]), "dw": torch.empty_like(d["w"]),
         "ds0": torch.empty_like(d["s0"])}
    # garbage in the outputs: every element must be written by the call
    for t in g.values():
        t.fill_(float("nan"))
    ins = [_ptr(d[x]) for x in ("q", "k", "v", "a", "b", "w", "s0")] + [_ptr(d_o), _ptr(dsT)]
    outs = [_ptr(g[n]) for n in GRADS]
    stream = torch.cuda.current_stream().cuda_stream
    if noalloc:
        st = _lib.backward_chunked_noalloc(desc, *ins, *outs, stream)
    else:
        need = _lib.backward_workspace_size(desc)
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        st = _lib.backward_chunked(desc, *ins, *outs, _ptr(ws), need, stream)
    assert st == _lib.OK, _lib.status_string(st)
    torch.cuda.synchronize()
    assert api.last_device_error() == 0
    return {n: to_host(t) for n, t in g.items()}


@pytest.mark.parametrize("name", ["gdn2_bf16", "kda_bf16"])
def test_noalloc_matches_workspace_entry_point_on_two_calls(name):
    wl = W.WORKLOADS[name].replace(B=1, H=2, T=200, random_s0=True)
    desc = _lib.GdrDesc(B=wl.B, T=wl.T, H=wl.H, dk=wl.dk, dv=wl.dv, chunk=32,
                        in_dtype=_lib.BF16, decay=_lib.GATE_VECTOR, erase=_lib.GATE_VECTOR,
                        write=_lib.GATE_VECTOR)
    assert _lib.backward_workspace_size(desc) <= _lib.NOALLOC_SCRATCH_BYTES
    for seed in (5, 6):   # two calls in a row on the shared scratch
        ref = _run(wl, seed, noalloc=False)
        got = _run(wl, seed, noalloc=True)
        for n in GRADS:
            assert np.isfinite(got[n]).all(), (n, seed)
            assert rel_err(got[n], ref[n]) <= TOL["bf16"], (n, seed, rel_err(got[n], ref[n]))


def test_noalloc_refuses_a_problem_larger_than_its_scratch():
    """bf16, dk = dv = 128 needs about 2 KiB per token and head (chunk-start
    states, E, the bf16 intermediates): 32k tokens of one head do not fit
    and are refused with GDR_ERR_WORKSPACE before anything is launched."""
    desc = _lib.GdrDesc(B=1, T=32 * 1024, H=1, dk=128, dv=128, chunk=32, in_dtype=_lib.BF16,
                        decay=_lib.GATE_VECTOR, erase=_lib.GATE_VECTOR, write=_lib.GATE_VECTOR)
    assert _lib.backward_workspace_size(desc) > _lib.NOALLOC_SCRATCH_BYTES
    p = 1 << 20   # never dereferenced: the size check comes first
    st = _lib.backward_chunked_noalloc(desc, *([p] * 16), 0)
    assert st == _lib.ERR_WORKSPACE
