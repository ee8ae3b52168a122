"""GPU parity of the backward pass (gdr_backward_chunked) against the float64
oracle's reverse-mode gradients (oracle.backward, itself pinned by finite
differences of the forward), through the C ABI.  Loss
L = sum_t <o_t, do_t> + <S_T, dsT> with seeded upstream gradients
(workload.make_upstream).  The pages train the recurrence in its chunked WY
form (FG^2-GDN page, gist.science 2604.19021, section 2 "Methodology").

Tolerances as for the forward (max |x - ref| / max |ref| per gradient
tensor): 1e-4 for float32 inputs, 2e-2 for bf16 inputs (gradients are
returned in the input dtype; dS0 in float32)."""

import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_154_b200 import _lib, api
from gated_delta_rule_154_b200 import workload as W
from gpu_helpers import TOL, inputs_to_dev, rel_err, to_dev, to_host

pytestmark = pytest.mark.gpu

GRADS = ("dq", "dk", "dv", "da", "db", "dw", "ds0")


def _gpu(wl, inp, up, with_dsT=True, s0=True):
    d = inputs_to_dev(inp, wl)
    do = to_dev(up["do"], wl.dtype)
    dsT = to_dev(up["dsT"], "f32") if with_dsT else None
    g = api.backward(d["q"], d["k"], d["v"], d["a"], d["b"], d["w"], d["s0"] if s0 else None,
                     do, dsT)
    torch.cuda.synchronize()
    return g


def _oracle(wl, inp, up, with_dsT=True, s0=True, heads=None):
    f = lambda key: W.as_f32(inp[key], wl.dtype)
    q, k, v, a, b = f("q"), f("k"), f("v"), f("a"), f("b")
    w = f("w") if inp.get("w") is not None else b
    do = W.as_f32(up["do"], wl.dtype)
    s0v = inp.get("s0") if s0 else None
    dsT = up["dsT"] if with_dsT else None
    if heads is None:
        return oracle.backward(q, k, v, a, b, w, s0v, do, dsT)
    # sampled heads stacked along H of one batch row
    cat = lambda x: None if x is None else np.concatenate(
        [x[bi:bi + 1, :, hi:hi + 1] for bi, hi in heads], axis=2)
    st = lambda x: None if x is None else np.stack([x[bi, hi] for bi, hi in heads])[None]
    return oracle.backward(cat(q), cat(k), cat(v), cat(a), cat(b), cat(w), st(s0v), cat(do),
                           st(dsT))


def _compare(g, ref, tol, where=""):
    errs = {}
    for name in GRADS:
        if ref[name] is None:
            assert g[name] is None, name
            continue
        errs[name] = rel_err(to_host(g[name]), ref[name])
    bad = {k: e for k, e in errs.items() if not e <= tol}
    assert not bad, (where, errs)
    return errs


@pytest.mark.parametrize("name", ["gdn_fp32", "kda_bf16", "gdn2_bf16", "long_bf16"])
@pytest.mark.parametrize("T", [1, 32, 97, 200])
def test_small_shapes_every_gate_kind(name, T):
    """Reduced B/H/T of each prefill workload (scalar gates, shared beta,
    decoupled vector gates, zero s0), ragged chunk tails included."""
    wl = W.WORKLOADS[name].replace(B=2, H=2, T=T)
    inp = W.make_prefill(wl, seed=T)
    up = W.make_upstream(wl, seed=T)
    g = _gpu(wl, inp, up)
    assert api.last_device_error() == 0
    _compare(g, _oracle(wl, inp, up), TOL[wl.dtype], (name, T))


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 64), (64, 128), (128, 128)])
def test_head_dims_fp32(dk, dv):
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=1, H=2, T=70, dk=dk, dv=dv, dtype="f32")
    inp = W.make_prefill(wl, seed=dk + dv)
    up = W.make_upstream(wl, seed=dk + dv)
    _compare(_gpu(wl, inp, up), _oracle(wl, inp, up), TOL["f32"], (dk, dv))


def test_scalar_gates_bf16():
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=1, H=3, T=100, decay="scalar", erase="scalar",
                                          write="scalar")
    inp = W.make_prefill(wl, seed=5)
    up = W.make_upstream(wl, seed=5)
    _compare(_gpu(wl, inp, up), _oracle(wl, inp, up), TOL["bf16"])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_gate_one_everywhere(dtype):
    """No gate tensors (a = b = w = 1): plain DeltaNet; no gate gradients
    (bf16: the tensor-core path, 75 tokens = one full chunk and a tail)."""
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=1, H=2, T=75, dtype=dtype)
    inp = W.make_prefill(wl, seed=3)
    up = W.make_upstream(wl, seed=3)
    d = inputs_to_dev(inp, wl)
    g = api.backward(d["q"], d["k"], d["v"], None, None, None, d["s0"], to_dev(up["do"], dtype),
                     to_dev(up["dsT"], "f32"))
    torch.cuda.synchronize()
    assert api.last_device_error() == 0
    f = lambda key: W.as_f32(inp[key], dtype)
    ref = oracle.backward(f("q"), f("k"), f("v"), None, None, None, inp["s0"],
                          W.as_f32(up["do"], dtype), up["dsT"])
    _compare(g, ref, TOL[dtype])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_without_state_gradient_or_initial_state(dtype):
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=2, H=1, T=90, dtype=dtype)
    inp = W.make_prefill(wl, seed=9)
    up = W.make_upstream(wl, seed=9)
    g = _gpu(wl, inp, up, with_dsT=False, s0=False)
    assert api.last_device_error() == 0
    _compare(g, _oracle(wl, inp, up, with_dsT=False, s0=False), TOL[dtype])


def test_zero_length_passes_the_state_gradient_through():
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=1, H=2, T=0, dtype="f32")
    inp = W.make_prefill(wl.replace(T=1), seed=2)
    up = W.make_upstream(wl.replace(T=1), seed=2)
    z = lambda d: torch.zeros((1, 0, 2, d), dtype=torch.float32, device="cuda")
    dsT = to_dev(up["dsT"], "f32")
    g = api.backward(z(128), z(128), z(128), z(128), z(128), z(128), None, z(128), dsT)
    torch.cuda.synchronize()
    assert torch.equal(g["ds0"], dsT)


def test_decay_beyond_range_is_reported():
    """Every channel's decay must multiply to at least about exp(-80) over a
    32-token chunk (the tensor-core path: over tokens 1-31 and 32-63 of each
    64-token chunk); a stronger one is flagged as GDR_ERR_RANGE."""
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=1, H=2, T=64)
    inp = W.make_prefill(wl, seed=1)
    a = inp["a"].copy()
    a[0, :, 1, 5] = W.f32_to_bf16_bits(np.full(64, 0.01, np.float32))  # log(0.01)*32 < -80
    _gpu(wl, dict(inp, a=a), W.make_upstream(wl, seed=1))
    assert api.last_device_error() == 6   # GDR_ERR_RANGE
    assert api.last_device_error() == 0


def test_repeatable_bit_for_bit():
    """Every reduction order is fixed: repeated calls agree bit for bit."""
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=2, H=4, T=333)
    inp = W.make_prefill(wl, seed=4)
    up = W.make_upstream(wl, seed=4)
    g0 = _gpu(wl, inp, up)
    for _ in range(2):
        g = _gpu(wl, inp, up)
        for name in GRADS:
            assert torch.equal(g[name], g0[name]), name


def test_full_size_sampled_heads():
    """The bench-sized workload (B=8, T=8192, H=16, d=128, bf16) on the GPU;
    the oracle recomputes the gradients of one whole head of every batch row
    (eight heads, spread over the head index)."""
    wl = W.WORKLOADS["gdn2_bf16"]
    heads = [(bi, (5 * bi + 3) % wl.H) for bi in range(wl.B)]
    inp = W.make_prefill(wl, seed=0)
    up = W.make_upstream(wl, seed=0)
    g = _gpu(wl, inp, up)
    assert api.last_device_error() == 0
    ref = _oracle(wl, inp, up, heads=heads)
    for i, (bi, hi) in enumerate(heads):
        for name in GRADS:
            x = g[name][bi, hi] if name == "ds0" else g[name][bi, :, hi]
            r = ref[name][0, i] if name == "ds0" else ref[name][0, :, i]
            e = rel_err(to_host(x), r)
            assert e <= TOL["bf16"], (bi, hi, name, e)


@pytest.mark.parametrize("plus", [False, True])
@pytest.mark.parametrize("dtype,d,T", [("bf16", 128, 97), ("f32", 64, 70)])
def test_fg2_learning_rates(dtype, d, T, plus):
    """FG^2-GDN (one beta for key and value) and FG^2-GDN+ (beta^k, beta^v):
    the oracle runs the mapped rule (key sqrt(beta^k) k, erase gate 1, write
    gate sqrt(beta^v); FG^2-GDN page, section 2) and its gradients are
    carried back through the square roots by the chain rule."""
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=2, H=2, T=T, dk=d, dv=d, dtype=dtype)
    inp = W.make_prefill(wl, seed=T + d)
    up = W.make_upstream(wl, seed=T + d)
    dev = {x: to_dev(inp[x], dtype) for x in ("q", "k", "v", "a", "b", "w")}
    beta_v_dev = dev["w"] if plus else dev["b"]
    g = api.backward(dev["q"], dev["k"], dev["v"], dev["a"], dev["b"], beta_v_dev,
                     to_dev(inp["s0"], "f32"), to_dev(up["do"], dtype), to_dev(up["dsT"], "f32"),
                     fg2=True)
    torch.cuda.synchronize()
    assert api.last_device_error() == 0
    f = lambda key: W.as_f32(inp[key], dtype).astype(np.float64)
    kk, beta_k = f("k"), f("b")
    beta_v = f("w") if plus else beta_k
    sk, sv = np.sqrt(beta_k), np.sqrt(beta_v)
    m = oracle.backward(W.as_f32(inp["q"], dtype), (sk * kk).astype(np.float32),
                        W.as_f32(inp["v"], dtype), W.as_f32(inp["a"], dtype),
                        np.ones(beta_k.shape, np.float32), sv.astype(np.float32), inp["s0"],
                        W.as_f32(up["do"], dtype), up["dsT"])
    ref = {"dq": m["dq"], "dk": sk * m["dk"], "dv": m["dv"], "da": m["da"],
           "db": m["dk"] * kk / (2 * sk), "dw": m["dw"] / (2 * sv), "ds0": m["ds0"]}
    _compare(g, ref, TOL[dtype], (dtype, d, T, plus))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_packed_sequences(dtype):
    """Sequences of different lengths (0 to 100 tokens) packed in one row:
    each sequence's gradients equal the oracle's for that sequence alone, and
    the tokens after the last sequence are never written."""
    lens = [0, 5, 32, 33, 100, 1, 64]
    H = 2
    T = sum(lens) + 5
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=1, H=H, T=T, dtype=dtype)
    inp = W.make_prefill(wl, seed=21)
    up = W.make_upstream(wl, seed=21)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    N = len(lens)
    rng = np.random.default_rng(5)
    s0 = (0.1 * rng.standard_normal((N, H, 128, 128))).astype(np.float32)
    dsT = (0.1 * rng.standard_normal((N, H, 128, 128))).astype(np.float32)
    dev = {x: to_dev(inp[x], dtype) for x in ("q", "k", "v", "a", "b", "w")}
    src = {"dq": "q", "dk": "k", "dv": "v", "da": "a", "db": "b", "dw": "w"}
    out = {n: torch.full_like(dev[x], 7.0) for n, x in src.items()}
    g = api.backward(dev["q"], dev["k"], dev["v"], dev["a"], dev["b"], dev["w"],
                     to_dev(s0, "f32"), to_dev(up["do"], dtype), to_dev(dsT, "f32"),
                     cu_seqlens=torch.from_numpy(cu).cuda(), out=out)
    torch.cuda.synchronize()
    assert api.last_device_error() == 0
    f = lambda key: W.as_f32(inp[key], dtype)
    do = W.as_f32(up["do"], dtype)
    for n, (t0, t1) in enumerate(zip(cu[:-1], cu[1:])):
        sl = lambda x: x[:, t0:t1]
        ref = oracle.backward(sl(f("q")), sl(f("k")), sl(f("v")), sl(f("a")), sl(f("b")),
                              sl(f("w")), s0[n:n + 1].astype(np.float64), sl(do),
                              dsT[n:n + 1].astype(np.float64))
        for name in src:
            e = rel_err(to_host(g[name][:, t0:t1]), ref[name])
            assert e <= TOL[dtype], (n, name, e)
        assert rel_err(to_host(g["ds0"][n:n + 1]), ref["ds0"]) <= TOL[dtype], n
    for name in src:
        assert torch.all(g[name][:, cu[-1]:] == 7.0), name


def test_unordered_packed_sequences_are_reported():
    """A decreasing offset makes the sequences after it unordered: they are
    skipped and reported (GDR_ERR_INVALID_ARG); the ordered ones before it are
    computed."""
    H = 1
    wl = W.WORKLOADS["gdn2_bf16"].replace(B=1, H=H, T=96, dtype="f32")
    inp = W.make_prefill(wl, seed=2)
    up = W.make_upstream(wl, seed=2)
    cu = np.array([0, 40, 20, 96], np.int32)
    dev = {x: to_dev(inp[x], "f32") for x in ("q", "k", "v", "a", "b", "w")}
    out = {"dq": torch.full_like(dev["q"], 7.0)}
    g = api.backward(dev["q"], dev["k"], dev["v"], dev["a"], dev["b"], dev["w"], None,
                     to_dev(up["do"], "f32"), None, cu_seqlens=torch.from_numpy(cu).cuda(),
                     out=out)
    torch.cuda.synchronize()
    assert api.last_device_error() == _lib.ERR_INVALID_ARG
    f = lambda key: W.as_f32(inp[key], "f32")
    sl = lambda x: x[:, 0:40]
    ref = oracle.backward(sl(f("q")), sl(f("k")), sl(f("v")), sl(f("a")), sl(f("b")), sl(f("w")),
                          None, sl(up["do"]), None)
    assert rel_err(to_host(g["dq"][:, 0:40]), ref["dq"]) <= TOL["f32"]
    assert torch.all(g["dq"][:, 40:] == 7.0)
