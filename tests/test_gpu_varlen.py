"""Packed sequences of different lengths in one launch (gdr_forward_varlen):
each sequence must equal its own separate prefill (and the float64 oracle),
tokens after the last sequence stay untouched, and a sequence range outside
the tensor is skipped and reported as GDR_ERR_INVALID_ARG.  Lengths mix
empty, single-token, partial-chunk and multi-chunk sequences, so the last
chunk of one sequence sits next to the first tokens of the following one.
Tolerances: 1e-4 float32, 2e-2 bf16 (max |x - ref| / max |ref|)."""

import numpy as np
import pytest
import torch

from gated_delta_rule_154_b200 import _lib, api
from gated_delta_rule_154_b200 import workload as W
from gpu_helpers import TOL, oracle_prefill, rel_err, to_dev, to_host

pytestmark = pytest.mark.gpu

LENS = [200, 64, 1, 130, 0, 77, 63]
PAD = 64  # tokens after the last sequence, never part of one


def _packed(name, dtype, d, chunk, seed):
    total = sum(LENS) + PAD
    wl = W.WORKLOADS[name].replace(B=1, H=3, T=total, dk=d, dv=d, dtype=dtype, chunk=chunk)
    inp = W.make_prefill(wl, seed=seed)
    cu = np.concatenate([[0], np.cumsum(LENS)]).astype(np.int32)
    rng = np.random.default_rng(seed)
    s0 = rng.normal(0.0, 0.1, size=(len(LENS), wl.H, d, d)).astype(np.float32)
    return wl, inp, cu, s0


def _slice(inp, wl, t0, t1):
    sub = {}
    for key in ("q", "k", "v", "a", "b", "w"):
        x = inp.get(key)
        sub[key] = None if x is None else np.ascontiguousarray(x[:, t0:t1])
    return sub


@pytest.mark.parametrize("name,dtype,d,chunk,fg2", [
    ("gdn2_bf16", "bf16", 128, 64, False),    # tensor-core kernel, vector gates
    ("kda_bf16", "bf16", 128, 64, False),     # tensor-core kernel, scalar beta
    ("gdn2_bf16", "bf16", 128, 64, True),     # tensor-core kernel, FG^2-GDN+
    ("gdn_fp32", "f32", 64, 32, False),       # float32 kernel
])
def test_packed_sequences_match_separate_runs(name, dtype, d, chunk, fg2):
    wl, inp, cu, s0 = _packed(name, dtype, d, chunk, seed=sum(LENS) + d)
    dev = {k: to_dev(inp[k], dtype) for k in ("q", "k", "v", "a", "b", "w")}
    if dev["w"] is None:
        dev["w"] = dev["b"]
    ity, pat = (torch.int16, 0x7FBD) if dtype == "bf16" else (torch.int32, 0x7FBADBAD)
    o = torch.empty((1, wl.T, wl.H, d), dtype=dev["q"].dtype, device="cuda")
    o.view(ity).fill_(pat)
    s0_d = torch.from_numpy(s0).cuda()
    o, sT = api.forward_varlen(dev["q"], dev["k"], dev["v"], dev["a"], dev["b"], dev["w"],
                               torch.from_numpy(cu).cuda(), s0_d, chunk=chunk, out=o, fg2=fg2)
    torch.cuda.synchronize()
    assert api.last_device_error() == 0
    # the padding tokens were not written
    assert bool((o[:, int(cu[-1]):].view(ity) == pat).all())
    for n, L in enumerate(LENS):
        t0, t1 = int(cu[n]), int(cu[n + 1])
        if L == 0:
            assert torch.equal(sT[n], s0_d[n])
            continue
        # fresh (16-byte aligned) copies: a slice of a scalar gate is not aligned
        sub = {k: None if x is None else x[:, t0:t1].clone() for k, x in dev.items()}
        o1, s1 = api.forward_chunked(sub["q"], sub["k"], sub["v"], sub["a"], sub["b"], sub["w"],
                                     s0_d[n:n + 1].contiguous(), chunk=chunk, fg2=fg2)
        torch.cuda.synchronize()
        assert rel_err(to_host(o[:, t0:t1]), to_host(o1)) <= TOL[dtype] / 4
        assert rel_err(to_host(sT[n:n + 1]), to_host(s1)) <= TOL[dtype] / 4
        if not fg2 and n in (0, 2, 3):   # and the oracle on a few sequences
            swl = wl.replace(T=L)
            ref_in = _slice(inp, wl, t0, t1)
            ref_in["s0"] = s0[n:n + 1]
            o_ref, s_ref = oracle_prefill(swl, ref_in)
            assert rel_err(to_host(o[:, t0:t1]), o_ref) <= TOL[dtype]
            assert rel_err(to_host(sT[n:n + 1]), s_ref) <= TOL[dtype]


def test_out_of_range_sequence_is_skipped_and_reported():
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=1, H=2, T=192)
    inp = W.make_prefill(wl, seed=4)
    dev = {k: to_dev(inp[k], "bf16") for k in ("q", "k", "v", "a", "b", "w")}
    cu = torch.tensor([0, 100, 500], dtype=torch.int32, device="cuda")  # second ends past T
    o, sT = api.forward_varlen(dev["q"], dev["k"], dev["v"], dev["a"], dev["b"], dev["w"], cu)
    assert api.last_device_error() == _lib.ERR_INVALID_ARG
    o1, s1 = api.forward_chunked(*(x[:, :100].clone() for x in
                                   (dev["q"], dev["k"], dev["v"], dev["a"], dev["b"], dev["w"])))
    torch.cuda.synchronize()
    assert rel_err(to_host(o[:, :100]), to_host(o1)) <= TOL["bf16"] / 4
    assert rel_err(to_host(sT[:1]), to_host(s1)) <= TOL["bf16"] / 4
    assert api.last_device_error() == 0
