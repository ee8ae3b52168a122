"""Shared helpers of the GPU parity tests: move seeded inputs to the device,
run the CUDA path through the library's API, run the oracle on the same
values, and measure the error the way the tolerances are stated
(max |x - ref| / max |ref|, per tensor)."""

from __future__ import annotations

import numpy as np
import torch

import oracle
from gated_delta_rule_154_b200 import api
from gated_delta_rule_154_b200 import workload as W

TOL = {"f32": 1e-4, "bf16": 2e-2}


def rel_err(x, ref) -> float:
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    den = float(np.max(np.abs(ref))) if ref.size else 0.0
    if den == 0.0:
        return float(np.max(np.abs(x))) if x.size else 0.0
    return float(np.max(np.abs(x - ref)) / den)


def elem_err(x, ref, floor: float = 1e-6) -> float:
    """Largest element-wise relative error |x - ref| / max(|ref|, floor); logged
    next to rel_err, which is the metric the tolerances apply to."""
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    if not ref.size:
        return 0.0
    return float(np.max(np.abs(x - ref) / np.maximum(np.abs(ref), floor)))


def report(tag: str, x, ref, tol: float) -> str:
    """One line with the per-tensor error, its margin to the tolerance and the
    element-wise error (floor 1e-6); printed so that runs with -s log it."""
    e = rel_err(x, ref)
    line = "%s: max|x-ref|/max|ref| = %.3e (tolerance %.0e, margin x%.1f); " \
           "element-wise max (floor 1e-6) = %.3e" % (tag, e, tol, tol / max(e, 1e-30),
                                                      elem_err(x, ref))
    print(line, flush=True)
    return line


def to_dev(x, dtype: str, device="cuda"):
    if x is None:
        return None
    if dtype == "bf16" and x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)


def to_host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def inputs_to_dev(inp, wl):
    d = {k: to_dev(inp[k], wl.dtype) for k in ("q", "k", "v", "a", "b", "w")}
    if d["w"] is None:           # shared beta: the write gate is the erase tensor
        d["w"] = d["b"]
    d["s0"] = None if inp.get("s0") is None else to_dev(inp["s0"], "f32")
    return d


def gpu_prefill(wl, inp, chunk=None, s0=None, **kw):
    d = inputs_to_dev(inp, wl)
    if s0 is not None:
        d["s0"] = s0
    o, s = api.forward_chunked(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"], d["s0"],
                               chunk=chunk or wl.chunk, **kw)
    torch.cuda.synchronize()
    return o, s


def oracle_prefill(wl, inp, heads=None, nthreads=0):
    """float64 oracle on the exact float32 images of the inputs.  With
    ``heads`` only those (b, h) are run; results come back stacked
    [n_heads, T, dv] and [n_heads, dk, dv]."""
    f = lambda key: W.as_f32(inp[key], wl.dtype)
    q, k, v, a, b = f("q"), f("k"), f("v"), f("a"), f("b")
    w = f("w") if inp.get("w") is not None else b
    s0 = inp.get("s0")
    if heads is None:
        return oracle.forward(q, k, v, a, b, w, s0, nthreads=nthreads)
    sel = lambda x, bi, hi: None if x is None else x[bi:bi + 1, :, hi:hi + 1]
    bs = np.array([bh[0] for bh in heads])
    hs = np.array([bh[1] for bh in heads])
    # stack the sampled heads along H of one batch row so the oracle runs them in parallel
    cat = lambda x: None if x is None else np.concatenate([sel(x, bi, hi) for bi, hi in heads], axis=2)
    s0s = None if s0 is None else s0[bs, hs][None]
    o, s = oracle.forward(cat(q), cat(k), cat(v), cat(a), cat(b), cat(w), s0s, nthreads=nthreads)
    return np.moveaxis(o[0], 1, 0), s[0]
