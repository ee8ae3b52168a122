"""GPU parity of the sequence-parallel prefill against the float64 oracle.

forward_segmented splits every sequence into P segments that run side by
side on one GPU: their affine maps (M, N), a scan for the start states, and a
second pass.  The multi-GPU form runs the same two library calls around an
all-gather; here its ranks are emulated one after another in one process
(no kernel waits on another), so the maps, the scan on the gathered maps and
the per-rank second pass are exercised exactly as ranks would call them.
Tolerance 2e-2 for bf16 inputs (max |x - ref| / max |ref| per tensor)."""

import numpy as np
import pytest
import torch

from gated_delta_rule_154_b200 import api
from gated_delta_rule_154_b200 import workload as W
from gpu_helpers import TOL, inputs_to_dev, oracle_prefill, rel_err, report, to_host

import oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("P", [2, 3, 5])
@pytest.mark.parametrize("name", ["gdn2_bf16", "kda_bf16"])
def test_segmented_matches_oracle(name, P):
    wl = W.WORKLOADS[name].replace(B=2, H=3, T=333, random_s0=True)
    inp = W.make_prefill(wl, seed=40 + P)
    d = inputs_to_dev(inp, wl)
    o, s = api.forward_segmented(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"], d["s0"],
                                 n_segments=P)
    torch.cuda.synchronize()
    assert api.last_device_error() == 0
    o_ref, s_ref = oracle_prefill(wl, inp)
    msg = [report("%s P=%d o" % (name, P), to_host(o), o_ref, TOL["bf16"]),
           report("%s P=%d S_T" % (name, P), to_host(s), s_ref, TOL["bf16"])]
    assert rel_err(to_host(o), o_ref) <= TOL["bf16"], msg
    assert rel_err(to_host(s), s_ref) <= TOL["bf16"], msg


def test_segment_maps_match_oracle():
    """M from S = I with the writes off, N from S = 0, against the oracle run
    the same way."""
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=1, H=2, T=100, random_s0=False)
    inp = W.make_prefill(wl, seed=3)
    d = inputs_to_dev(inp, wl)
    m, n = api.segment_maps(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"])
    torch.cuda.synchronize()
    f = lambda key: W.as_f32(inp[key], wl.dtype)
    eye = np.broadcast_to(np.eye(128), (1, 2, 128, 128)).copy()
    _, m_ref = oracle.forward(f("q"), f("k"), np.zeros_like(f("v")), f("a"), f("b"),
                              np.zeros_like(f("w")), eye, want_o=False)
    _, n_ref = oracle.forward(f("q"), f("k"), f("v"), f("a"), f("b"), f("w"), None, want_o=False)
    assert rel_err(to_host(m), m_ref) <= TOL["bf16"]
    assert rel_err(to_host(n), n_ref) <= TOL["bf16"]


def test_emulated_ranks_match_oracle():
    """P ranks each holding one segment: maps per rank, the scan over the
    gathered maps (segment-major, as an all-gather leaves them), then each
    rank's segment from its start state."""
    P = 4
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=2, H=2, T=4 * 96, random_s0=True)
    inp = W.make_prefill(wl, seed=9)
    d = inputs_to_dev(inp, wl)
    L = wl.T // P
    seg = lambda x, r: x[:, r * L:(r + 1) * L].contiguous()
    maps = [api.segment_maps(*(seg(d[k], r) for k in "qkvabw")) for r in range(P)]
    s_start, s_final = api.segment_scan(torch.stack([m for m, _ in maps]),
                                        torch.stack([n for _, n in maps]), d["s0"])
    outs = [api.forward_chunked(*(seg(d[k], r) for k in "qkvabw"), s_start[r].contiguous(),
                                return_final=False)[0] for r in range(P)]
    torch.cuda.synchronize()
    o_ref, s_ref = oracle_prefill(wl, inp)
    assert rel_err(to_host(torch.cat(outs, 1)), o_ref) <= TOL["bf16"]
    assert rel_err(to_host(s_final), s_ref) <= TOL["bf16"]


def test_segmented_long_workload_every_head():
    """The long-context workload's shape (H = 32, d = 128) at T = 16384, four
    segments, against the oracle on every head."""
    wl = W.WORKLOADS["long_bf16"].replace(T=16384)
    inp = W.make_prefill(wl, seed=0, threads=16)
    d = inputs_to_dev(inp, wl)
    o, s = api.forward_segmented(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"], None,
                                 n_segments=4)
    torch.cuda.synchronize()
    assert api.last_device_error() == 0
    o_ref, s_ref = oracle_prefill(wl, inp)
    msg = [report("long T=16384 P=4 o", to_host(o), o_ref, TOL["bf16"]),
           report("long T=16384 P=4 S_T", to_host(s), s_ref, TOL["bf16"])]
    assert rel_err(to_host(o), o_ref) <= TOL["bf16"], msg
    assert rel_err(to_host(s), s_ref) <= TOL["bf16"], msg
