"""Pins of the oracle's backward pass (``oracle.backward``).

The backward is the reverse-mode derivative of the recurrence of the
FG^2-GDN page (gist.science 2604.19021), section 2 "Methodology", FG2-GDN
update rule, with the decoupled erase/write gates of the Gated DeltaNet-2
page (needhelp.icu), gates table; the pages use the chunked form for training
(FG^2-GDN page, section 2: WY representation kept for chunked training).

Pinned against something other than itself: five-point central differences
of the forward oracle (pinned on its own in test_oracle_pins.py) for every
input element, on small cases with vector, scalar and absent gates.  The
inputs are multiples of 2^-12 below 2 in magnitude, so every perturbed value
x +- h, x +- 2h (h = 2^-8) is exact in float32; the stencil's truncation
error is O(h^4) of the fifth derivative, far below the 1e-9 bound.
``test_backward_mutants_are_caught`` plants plausible mistakes in a copy of
the backward and checks that the pin fails for each.
"""

import os
import shutil
import tempfile

import numpy as np
import pytest

import oracle

H_STEP = 2.0 ** -8
TOL = 1e-9


def _quant(x):
    return (np.round(np.asarray(x, np.float64) * 4096.0) / 4096.0).astype(np.float32)


def _case(seed, B, T, H, dk, dv, gates):
    rng = np.random.default_rng(seed)
    q = _quant(rng.uniform(-1, 1, (B, T, H, dk)))
    k = _quant(rng.uniform(-1, 1, (B, T, H, dk)) / np.sqrt(dk))
    v = _quant(rng.uniform(-1, 1, (B, T, H, dv)))
    if gates == "vector":
        a = _quant(rng.uniform(0.5, 0.99, (B, T, H, dk)))
        b = _quant(rng.uniform(0.05, 0.95, (B, T, H, dk)))
        w = _quant(rng.uniform(0.05, 0.95, (B, T, H, dv)))
    elif gates == "scalar":
        a = _quant(rng.uniform(0.5, 0.99, (B, T, H)))
        b = _quant(rng.uniform(0.05, 0.95, (B, T, H)))
        w = _quant(rng.uniform(0.05, 0.95, (B, T, H)))
    else:
        a = b = w = None
    s0 = rng.uniform(-1, 1, (B, H, dk, dv))
    do = rng.uniform(-1, 1, (B, T, H, dv))
    dsT = rng.uniform(-1, 1, (B, H, dk, dv))
    return dict(q=q, k=k, v=v, a=a, b=b, w=w, s0=s0), do, dsT


def _loss(orc, x, do, dsT):
    o, s = orc.forward(x["q"], x["k"], x["v"], x["a"], x["b"], x["w"], x["s0"])
    return float(np.sum(o * do) + np.sum(s * dsT))


def _fd_grad(orc, x, name, do, dsT):
    """Five-point central difference of the loss for every element of x[name]."""
    base = x[name]
    g = np.zeros(base.shape, np.float64)
    for idx in np.ndindex(base.shape):
        vals = []
        for m in (-2, -1, 1, 2):
            y = dict(x)
            arr = base.copy()
            arr[idx] = arr[idx] + m * H_STEP
            y[name] = arr
            vals.append(_loss(orc, y, do, dsT))
        g[idx] = (vals[0] - 8 * vals[1] + 8 * vals[2] - vals[3]) / (12 * H_STEP)
    return g


def _rel(x, ref):
    return float(np.max(np.abs(x - ref)) / max(np.max(np.abs(ref)), 1e-300))


def pin_finite_differences(orc, gates, seed=0, shape=(1, 5, 2, 3, 2)):
    x, do, dsT = _case(seed, *shape, gates)
    g = orc.backward(x["q"], x["k"], x["v"], x["a"], x["b"], x["w"], x["s0"], do, dsT)
    err = 0.0
    for name, gname in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("a", "da"), ("b", "db"),
                        ("w", "dw"), ("s0", "ds0")):
        if x[name] is None:
            assert g[gname] is None
            continue
        err = max(err, _rel(g[gname], _fd_grad(orc, x, name, do, dsT)))
    return err


@pytest.mark.parametrize("gates", ["vector", "scalar", "none"])
def test_backward_matches_finite_differences(gates):
    assert pin_finite_differences(oracle.default(), gates) <= TOL


def test_backward_without_state_gradient_and_initial_state():
    """dsT = None is a zero upstream state gradient, s0 = None a zero state."""
    orc = oracle.default()
    x, do, _ = _case(3, 1, 4, 1, 3, 2, "vector")
    x["s0"] = None
    g = orc.backward(x["q"], x["k"], x["v"], x["a"], x["b"], x["w"], None, do, None)
    g0 = orc.backward(x["q"], x["k"], x["v"], x["a"], x["b"], x["w"],
                      np.zeros((1, 1, 3, 2)), do, np.zeros((1, 1, 3, 2)))
    for key in ("dq", "dk", "dv", "da", "db", "dw", "ds0"):
        assert np.array_equal(g[key], g0[key])


def test_backward_zero_length():
    """T = 0: the only gradient is dS0 = dS_T."""
    orc = oracle.default()
    z = lambda d: np.zeros((1, 0, 2, d), np.float32)
    dsT = np.random.default_rng(1).standard_normal((1, 2, 3, 4))
    g = orc.backward(z(3), z(3), z(4), None, None, None, None,
                     np.zeros((1, 0, 2, 4)), dsT)
    assert g["dq"].shape == (1, 0, 2, 3) and np.array_equal(g["ds0"], dsT)


# ----------------------------------------------------------- mutation check

MUTANTS = {
    "erase_reads_state_not_key_term": ("G[(size_t)i * dv + j] += ki * de[j];", "(void)0;"),
    "erase_sign": ("dp[i] = -s1;", "dp[i] = s1;"),
    "decay_grad_from_new_state": ("s += G[(size_t)i * dv + j] * Sprev[(size_t)i * dv + j];",
                                  "s += G[(size_t)i * dv + j] * Scur[(size_t)i * dv + j];"),
    "state_grad_not_decayed": ("for (int j = 0; j < dv; ++j) G[(size_t)i * dv + j] *= ag[i];",
                               "for (int j = 0; j < dv; ++j) G[(size_t)i * dv + j] *= 1.0;"),
    "query_grad_from_old_state": ("acc += Scur[(size_t)i * dv + j] * dot[j];",
                                  "acc += Sprev[(size_t)i * dv + j] * dot[j];"),
    "key_read_term_dropped": ("gk[i] += s;", "(void)s;"),
    "write_gate_grad_uses_gate": ("gg[j] = (double)v[vbase + j] * du[j];",
                                  "gg[j] = gate_at(w, w_kind, tok, vbase, j) * du[j];"),
}


@pytest.fixture(scope="module")
def mutant_dir():
    d = tempfile.mkdtemp(prefix="gdr_oracle_bwd_mutants_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_backward_mutants_are_caught(name, mutant_dir):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "gdr_oracle.c")).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, "mutation anchor not found: %s" % name
    path = os.path.join(mutant_dir, name + ".c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib = oracle.build(force=True, src=path, out=os.path.join(mutant_dir, name + ".so"))
    orc = oracle.Oracle(lib)
    errs = [pin_finite_differences(orc, g, shape=(1, 4, 1, 3, 2)) for g in ("vector", "scalar")]
    assert max(errs) > 1e-4, "mutant %s passed the pin: %s" % (name, errs)
