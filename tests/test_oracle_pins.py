"""Pins of the float64 oracle against facts fixed by the pages and by algebra.

Each pin computes its expected value WITHOUT the oracle's rank-1 loop: from a
hand-worked example, from explicit transition-matrix products, from closed
forms of special cases (pure decay, gated linear attention, the textbook delta
rule, the symmetric FG^2-GDN form), or from invariants of the recurrence
(projection property, linearity in the initial state, resume, head
permutation).  ``test_mutants_are_caught`` plants plausible mistakes in a copy
of the oracle's C source and checks that some pin fails for each one.

Recurrence: FG^2-GDN page (gist.science 2604.19021), section 2 "Methodology",
FG2-GDN update rule; decoupled erase/write gates: Gated DeltaNet-2 page
(needhelp.icu), gates table; scalar versus per-channel decay: FG^2-GDN page,
section 1 "Problem statement".
"""

import json
import os
import shutil
import subprocess
import tempfile

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
TOL = 1e-12


def _rel(x, ref):
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.max(np.abs(x - ref)) / max(np.max(np.abs(ref)), 1e-300))


def _rand_inputs(rng, B, T, H, dk, dv, gates="vector", s0=True):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    if gates == "vector":
        a = rng.uniform(0.5, 1.0, (B, T, H, dk))
        b = rng.uniform(0.0, 1.0, (B, T, H, dk))
        w = rng.uniform(0.0, 1.0, (B, T, H, dv))
    else:
        a = rng.uniform(0.5, 1.0, (B, T, H))
        b = rng.uniform(0.0, 1.0, (B, T, H))
        w = rng.uniform(0.0, 1.0, (B, T, H))
    S0 = rng.standard_normal((B, H, dk, dv)) if s0 else None
    f = lambda x: None if x is None else x.astype(np.float32)
    return [f(x) for x in (q, k, v, a, b, w)] + [None if S0 is None else S0]


# ------------------------------------------------------------------ the pins

def pin_hand_example(orc):
    g = json.load(open(os.path.join(HERE, "golden", "hand_two_steps.json")))
    sh = lambda key: np.array(g[key], np.float32)[None, :, None, :]   # [1,T,1,d]
    s0 = np.array(g["s0"], np.float64)[None, None]
    o, sT = orc.forward(sh("q"), sh("k"), sh("v"), sh("a"), sh("b"), sh("w"), s0)
    return max(_rel(o[0, :, 0, :], g["o"]), _rel(sT[0, 0], g["sT"]))


def pin_brute_force(orc, seed=1):
    """S_T = (A_T...A_1) S0 + sum_s (A_T...A_{s+1}) k_s u_s^T with explicit
    transition matrices A_t = (I - (b_t*k_t) k_t^T) Diag(a_t), u_s = w_s*v_s."""
    rng = np.random.default_rng(seed)
    B, T, H, dk, dv = 1, 4, 2, 3, 2
    q, k, v, a, b, w, S0 = _rand_inputs(rng, B, T, H, dk, dv)
    o, sT = orc.forward(q, k, v, a, b, w, S0)
    err = 0.0
    for h in range(H):
        f64 = lambda x: x[0, :, h].astype(np.float64)
        qh, kh, vh, ah, bh, wh = map(f64, (q, k, v, a, b, w))
        A = [(np.eye(dk) - np.outer(bh[t] * kh[t], kh[t])) @ np.diag(ah[t]) for t in range(T)]
        C = [np.outer(kh[t], wh[t] * vh[t]) for t in range(T)]

        def prod(lo, hi):  # A_{hi-1} ... A_lo
            P = np.eye(dk)
            for r in range(lo, hi):
                P = A[r] @ P
            return P

        for t in range(T):
            St = prod(0, t + 1) @ S0[0, h] + sum(prod(s + 1, t + 1) @ C[s] for s in range(t + 1))
            err = max(err, _rel(o[0, t, h], St.T @ qh[t]))
            if t == T - 1:
                err = max(err, _rel(sT[0, h], St))
    return err


def pin_delta_invariant(orc, seed=2):
    """a = 1, b = w = 1, |k_t| = 1: the state maps k_t exactly to v_t."""
    rng = np.random.default_rng(seed)
    B, T, H, d = 2, 6, 2, 8
    _, _, v, _, _, _, S0 = _rand_inputs(rng, B, T, H, d, d)
    # keys with exactly unit norm in float32: +-1/2 on four random channels
    k = np.zeros((B, T, H, d), np.float32)
    for idx in np.ndindex(B, T, H):
        pos = rng.choice(d, 4, replace=False)
        k[idx][pos] = rng.choice([-0.5, 0.5], 4)
    err = 0.0
    for gates in ("none", "ones"):
        if gates == "none":
            a = b = w = None
        else:
            a = np.ones((B, T, H, d), np.float32)
            b = np.ones((B, T, H, d), np.float32)
            w = np.ones((B, T, H, d), np.float32)
        o, _ = orc.forward(k, k, v, a, b, w, S0)   # query = key
        err = max(err, _rel(o, v))
    return err


def pin_gla_closed_form(orc, seed=3):
    """b = 0: gated linear attention,
    o_t = (gamma_t*q_t)^T S0 + sum_{s<=t} sum_i q_ti (gamma_ti/gamma_si) k_si (w_s*v_s)."""
    rng = np.random.default_rng(seed)
    B, T, H, dk, dv = 1, 7, 2, 4, 3
    q, k, v, a, _, w, S0 = _rand_inputs(rng, B, T, H, dk, dv)
    b = np.zeros((B, T, H, dk), np.float32)
    o, sT = orc.forward(q, k, v, a, b, w, S0)
    err = 0.0
    for h in range(H):
        qh, kh, vh, ah, wh = (x[0, :, h].astype(np.float64) for x in (q, k, v, a, w))
        gam = np.cumprod(ah, axis=0)
        for t in range(T):
            ref = (gam[t] * qh[t]) @ S0[0, h]
            for s in range(t + 1):
                ref = ref + np.sum(qh[t] * gam[t] / gam[s] * kh[s]) * (wh[s] * vh[s])
            err = max(err, _rel(o[0, t, h], ref))
        Sref = np.diag(gam[-1]) @ S0[0, h] + sum(
            np.outer(gam[-1] / gam[s] * kh[s], wh[s] * vh[s]) for s in range(T))
        err = max(err, _rel(sT[0, h], Sref))
    return err


def pin_pure_decay(orc, seed=4):
    """k = 0: S_t = Diag(gamma_t) S0, o_t = S_t^T q_t."""
    rng = np.random.default_rng(seed)
    B, T, H, dk, dv = 1, 5, 3, 4, 6
    q, k, v, a, b, w, S0 = _rand_inputs(rng, B, T, H, dk, dv)
    k = np.zeros_like(k)
    o, sT = orc.forward(q, k, v, a, b, w, S0)
    err = 0.0
    for h in range(H):
        gam = np.cumprod(a[0, :, h].astype(np.float64), axis=0)
        for t in range(T):
            St = np.diag(gam[t]) @ S0[0, h]
            err = max(err, _rel(o[0, t, h], St.T @ q[0, t, h].astype(np.float64)))
        err = max(err, _rel(sT[0, h], np.diag(gam[-1]) @ S0[0, h]))
    return err


def pin_textbook_delta_rule(orc, seed=5):
    """a = 1, b = w = beta (scalar): S_t = S_{t-1} + beta_t k_t (v_t - S_{t-1}^T k_t)^T."""
    rng = np.random.default_rng(seed)
    B, T, H, dk, dv = 1, 6, 2, 5, 3
    q, k, v, _, beta, _, S0 = _rand_inputs(rng, B, T, H, dk, dv, gates="scalar")
    o, sT = orc.forward(q, k, v, None, beta, beta, S0)
    err = 0.0
    for h in range(H):
        S = S0[0, h].copy()
        for t in range(T):
            kt = k[0, t, h].astype(np.float64)
            S = S + beta[0, t, h] * np.outer(kt, v[0, t, h].astype(np.float64) - S.T @ kt)
            err = max(err, _rel(o[0, t, h], S.T @ q[0, t, h].astype(np.float64)))
        err = max(err, _rel(sT[0, h], S))
    return err


def pin_fg2gdn_symmetric(orc, seed=6):
    """FG^2-GDN: S_t = (I - kk kk^T) Diag(alpha_t) S + kk vv^T, kk = sqrt(beta)*k,
    vv = sqrt(beta)*v, equals the general rule fed key sqrt(beta)*k, b = 1,
    w = sqrt(beta)."""
    rng = np.random.default_rng(seed)
    B, T, H, d = 1, 5, 2, 4
    q, k, v, alpha, beta, _, S0 = _rand_inputs(rng, B, T, H, d, d)
    kt = (np.sqrt(beta.astype(np.float64)) * k).astype(np.float32)
    wt = np.sqrt(beta.astype(np.float64)).astype(np.float32)
    o, sT = orc.forward(q, kt, v, alpha, None, wt, S0)
    err = 0.0
    for h in range(H):
        S = S0[0, h].copy()
        for t in range(T):
            kk = kt[0, t, h].astype(np.float64)
            vv = wt[0, t, h].astype(np.float64) * v[0, t, h]
            S = (np.eye(d) - np.outer(kk, kk)) @ np.diag(alpha[0, t, h].astype(np.float64)) @ S \
                + np.outer(kk, vv)
            err = max(err, _rel(o[0, t, h], S.T @ q[0, t, h].astype(np.float64)))
        err = max(err, _rel(sT[0, h], S))
    return err


def pin_linear_in_s0(orc, seed=7):
    """S_T(S0 + D) - S_T(S0) equals the run from D with every write removed."""
    rng = np.random.default_rng(seed)
    B, T, H, dk, dv = 2, 6, 2, 4, 5
    q, k, v, a, b, w, S0 = _rand_inputs(rng, B, T, H, dk, dv)
    D = rng.standard_normal(S0.shape)
    o1, s1 = orc.forward(q, k, v, a, b, w, S0)
    o2, s2 = orc.forward(q, k, v, a, b, w, S0 + D)
    o3, s3 = orc.forward(q, k, np.zeros_like(v), a, b, w, D)
    return max(_rel(s2 - s1, s3), _rel(o2 - o1, o3))


def pin_resume(orc, seed=8):
    """forward(T1) then forward(T2, s0 = S_T1) equals forward(T1 + T2)."""
    rng = np.random.default_rng(seed)
    B, T, H, dk, dv = 2, 9, 2, 4, 3
    q, k, v, a, b, w, S0 = _rand_inputs(rng, B, T, H, dk, dv)
    o, s = orc.forward(q, k, v, a, b, w, S0)
    c = 4
    cut = lambda x, sl: x[:, sl]
    oa, sa = orc.forward(*(cut(x, slice(0, c)) for x in (q, k, v, a, b, w)), S0)
    ob, sb = orc.forward(*(cut(x, slice(c, T)) for x in (q, k, v, a, b, w)), sa)
    return max(_rel(np.concatenate([oa, ob], axis=1), o), _rel(sb, s))


def pin_head_permutation(orc, seed=9):
    rng = np.random.default_rng(seed)
    B, T, H, dk, dv = 1, 5, 4, 3, 3
    q, k, v, a, b, w, S0 = _rand_inputs(rng, B, T, H, dk, dv)
    perm = np.array([2, 0, 3, 1])
    o, s = orc.forward(q, k, v, a, b, w, S0)
    p = lambda x: x[:, :, perm]
    op, sp = orc.forward(*(p(x) for x in (q, k, v, a, b, w)), S0[:, perm])
    return max(_rel(op, o[:, :, perm]), _rel(sp, s[:, perm]))


def pin_scalar_broadcast(orc, seed=10):
    rng = np.random.default_rng(seed)
    B, T, H, dk, dv = 1, 5, 2, 4, 3
    q, k, v, a, b, w, S0 = _rand_inputs(rng, B, T, H, dk, dv, gates="scalar")
    o, s = orc.forward(q, k, v, a, b, w, S0)
    bc = lambda x, d: np.ascontiguousarray(np.broadcast_to(x[..., None], x.shape + (d,)))
    o2, s2 = orc.forward(q, k, v, bc(a, dk), bc(b, dk), bc(w, dv), S0)
    return max(_rel(o2, o), _rel(s2, s))


def pin_decode_is_one_step(orc, seed=11):
    rng = np.random.default_rng(seed)
    B, T, H, dk, dv = 2, 1, 3, 4, 5
    q, k, v, a, b, w, S0 = _rand_inputs(rng, B, T, H, dk, dv)
    o, s = orc.forward(q, k, v, a, b, w, S0)
    sq = lambda x: x[:, 0]
    od, sd = orc.decode_step(*(sq(x) for x in (q, k, v, a, b, w)), S0)
    return max(_rel(od, o[:, 0]), _rel(sd, s))


PINS = [pin_hand_example, pin_brute_force, pin_delta_invariant, pin_gla_closed_form,
        pin_pure_decay, pin_textbook_delta_rule, pin_fg2gdn_symmetric, pin_linear_in_s0,
        pin_resume, pin_head_permutation, pin_scalar_broadcast, pin_decode_is_one_step]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    assert pin(oracle.default()) <= TOL


def test_zero_length_and_empty_batch():
    orc = oracle.default()
    S0 = np.random.default_rng(0).standard_normal((1, 2, 3, 4))
    z = lambda d: np.zeros((1, 0, 2, d), np.float32)
    o, s = orc.forward(z(3), z(3), z(4), None, None, None, S0)
    assert o.shape == (1, 0, 2, 4) and np.array_equal(s, S0)
    o, s = orc.forward(np.zeros((0, 3, 2, 3), np.float32), np.zeros((0, 3, 2, 3), np.float32),
                       np.zeros((0, 3, 2, 4), np.float32))
    assert o.shape == (0, 3, 2, 4) and s.shape == (0, 2, 3, 4)


# ----------------------------------------------------------- mutation check

MUTANTS = {
    "no_decay": ("S[(size_t)i * dv + j] *= ag[i];", "S[(size_t)i * dv + j] *= 1.0;"),
    "erase_sign": ("+= -bk[i] * e[j] + ki * wv[j];", "+= bk[i] * e[j] + ki * wv[j];"),
    "erase_gate_dropped": ("bk[i] = gate_at(b, b_kind, tok, kbase, i) * (double)k[kbase + i];",
                           "bk[i] = (double)k[kbase + i];"),
    "write_gate_dropped": ("wv[j] = gate_at(w, w_kind, tok, vbase, j) * (double)v[vbase + j];",
                           "wv[j] = (double)v[vbase + j];"),
    "erase_reads_undecayed_state": ("e[j] += S[(size_t)i * dv + j] * ki;",
                                    "e[j] += S[(size_t)i * dv + j] * ki / ag[i];"),
    "erase_on_value_side": ("+= -bk[i] * e[j] + ki * wv[j];", "+= -ki * e[j] * (wv[j] / (double)v[vbase + j]) + ki * wv[j];"),
    "write_scaled_by_erase_gate": ("+= -bk[i] * e[j] + ki * wv[j];", "+= -bk[i] * e[j] + bk[i] * wv[j];"),
}


@pytest.fixture(scope="module")
def mutant_dir():
    d = tempfile.mkdtemp(prefix="gdr_oracle_mutants_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutants_are_caught(name, mutant_dir):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "gdr_oracle.c")).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, "mutation anchor not found: %s" % name
    path = os.path.join(mutant_dir, name + ".c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib = oracle.build(force=True, src=path, out=os.path.join(mutant_dir, name + ".so"))
    orc = oracle.Oracle(lib)
    errs = {p.__name__: p(orc) for p in PINS}
    assert max(errs.values()) > 1e-6, "mutant %s passed every pin: %s" % (name, errs)
