"""Decode over a state pool (many sequences, paged state): batch entry b
updates pool[slot[b]] in place.  Checked against the float64 oracle on the
gathered states; slots not named stay bit-for-bit unchanged; an out-of-range
slot is skipped and reported as GDR_ERR_INVALID_ARG, the other entries still
exact.  Tolerances: 1e-4 float32, 2e-2 bf16 (max |x - ref| / max |ref|)."""

import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_154_b200 import _lib, api
from gated_delta_rule_154_b200 import workload as W
from gpu_helpers import TOL, rel_err, to_dev, to_host

pytestmark = pytest.mark.gpu


def _step_inputs(wl, step, fg2=False):
    inp = W.make_decode_step(wl, step)
    d = {k: to_dev(inp[k], wl.dtype) for k in ("q", "k", "v", "a", "b", "w")}
    f = {k: W.as_f32(inp[k], wl.dtype) for k in ("q", "k", "v", "a", "b", "w")}
    if d["w"] is None:
        d["w"], f["w"] = d["b"], f["b"]
    return d, f


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_paged_decode_matches_oracle_and_leaves_other_slots(dtype):
    wl = W.WORKLOADS["decode_bf16"].replace(B=4, H=3, dtype=dtype)
    n_slots = 10
    rng = np.random.default_rng(3)
    pool_np = rng.normal(0.0, 0.1, size=(n_slots, wl.H, wl.dk, wl.dv)).astype(np.float32)
    pool = torch.from_numpy(pool_np).cuda()
    slots = np.array([7, 2, 9, 0], dtype=np.int32)
    slot = torch.from_numpy(slots).cuda()
    ref = pool_np.astype(np.float64)
    for step in (1, 2):
        d, f = _step_inputs(wl, step)
        o = api.decode_step_paged(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"], pool, slot)
        o_ref, new = oracle.decode_step(f["q"], f["k"], f["v"], f["a"], f["b"], f["w"],
                                        ref[slots])
        ref[slots] = new
        torch.cuda.synchronize()
        assert api.last_device_error() == 0
        assert rel_err(to_host(o), o_ref) <= TOL[dtype]
        assert rel_err(to_host(pool[slots.tolist()]), ref[slots]) <= TOL[dtype]
    untouched = [s for s in range(n_slots) if s not in slots]
    assert torch.equal(pool[untouched].cpu(), torch.from_numpy(pool_np[untouched]))


def test_paged_decode_out_of_range_slot_is_skipped_and_reported():
    wl = W.WORKLOADS["decode_bf16"].replace(B=3, H=2)
    n_slots = 4
    pool_np = np.random.default_rng(5).normal(0.0, 0.1, size=(n_slots, wl.H, wl.dk, wl.dv)
                                              ).astype(np.float32)
    pool = torch.from_numpy(pool_np).cuda()
    slots = np.array([1, 11, 3], dtype=np.int32)     # entry 1 is out of range
    d, f = _step_inputs(wl, 1)
    o = api.decode_step_paged(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"], pool,
                              torch.from_numpy(slots).cuda())
    assert api.last_device_error() == _lib.ERR_INVALID_ARG
    keep = [0, 2]
    sel = lambda x: x[keep]
    o_ref, new = oracle.decode_step(*(sel(f[k]) for k in ("q", "k", "v", "a", "b", "w")),
                                    pool_np[slots[keep]].astype(np.float64))
    assert rel_err(to_host(o[keep]), o_ref) <= TOL["bf16"]
    assert rel_err(to_host(pool[slots[keep].tolist()]), new) <= TOL["bf16"]
    # slots 0 and 2 were never named: unchanged
    assert torch.equal(pool[[0, 2]].cpu(), torch.from_numpy(pool_np[[0, 2]]))
    assert api.last_device_error() == 0
