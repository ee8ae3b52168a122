"""The chunked gradient identities of the backward pass, checked in float64
against the oracle's step-by-step reverse-mode gradients.

The pages train the recurrence through its chunkwise WY form (FG^2-GDN page,
gist.science 2604.19021, section 2 "Methodology") but print no gradient; the
identities below are the reverse of the chunk form of test_chunk_identity.py
and are what the CUDA backward evaluates (in 32-token chunks).  This test pins
them independently of any GPU code.

Per chunk (n tokens, state S0 at its start, G_r = sum_{i<=r} log a_i per key
channel, G_C = G_{n-1}; Qh = e^G q, Kh = e^G k, Kt = e^{G_C-G} k, Bt = b Kt,
Kb = e^{-G_C} Kt, Bb = e^{-G_C} Bt, U = w v; A_qk = tril(Qh Kb^T),
A_qb = tril(Qh Bb^T), A_kk = tril_{-1}(Kh Kb^T), A_kb = tril_{-1}(Kh Bb^T),
T = (I + A_kb)^{-1}, Y = Kh S0 + A_kk U, E = T Y), given dO and dS_C:
  dE = -A_qb^T dO - Bt dS_C,  dY = T^T dE,  dU = A_qk^T dO + A_kk^T dY + Kt dS_C
  dA_qk = dO U^T, dA_qb = -dO E^T, dA_kk = dY U^T, dA_kb = -dY E^T   (masked)
  XQ = dO S0^T + e^{-G_C} (dA_qk Kt + dA_qb Bt)
  XK = dY S0^T + e^{-G_C} (dA_kk Kt + dA_kb Bt)
  YK = U dS_C^T + e^{-G_C} (dA_qk^T Qh + dA_kk^T Kh)
  YB = -E dS_C^T + e^{-G_C} (dA_qb^T Qh + dA_kb^T Kh)
  dq = e^G XQ, dk = e^G XK + e^{G_C-G} (YK + b YB), db = Kt YB, dv = w dU, dw = v dU
  dG = Qh XQ + Kh XK - Kt YK - Bt YB, and at row n-1 also
       e^{G_C} rowsum(dS_C * S0) + colsum(Kt * U dS_C^T - Bt * E dS_C^T)
  d log a_r = sum_{r' >= r} dG_r',  da = d log a / a,
  dS0 = e^{G_C} dS_C + Qh^T dO + Kh^T dY.
"""

import numpy as np
import pytest

import oracle


def _chunk_states(q, k, v, a, b, w, s0, C):
    """State at the start of every chunk, by the plain recurrence (float64)."""
    S, hs = s0.copy(), []
    for t in range(q.shape[0]):
        if t % C == 0:
            hs.append(S.copy())
        S = a[t][:, None] * S
        e = S.T @ k[t]
        S = S - np.outer(b[t] * k[t], e) + np.outer(k[t], w[t] * v[t])
    return hs


def chunked_backward_head(q, k, v, a, b, w, s0, do, dsT, C):
    """Gradients of one (batch, head) by the chunked identities above; gates
    given per channel (scalar gates broadcast by the caller)."""
    T, dk = q.shape
    dv = v.shape[1]
    hs = _chunk_states(q, k, v, a, b, w, s0, C)
    out = {n: np.zeros_like(x) for n, x in (("dq", q), ("dk", k), ("dv", v), ("da", a),
                                             ("db", b), ("dw", w))}
    dS = dsT.copy()
    incl = np.tril(np.ones((C, C)))
    strict = np.tril(np.ones((C, C)), -1)
    for ci in range(len(hs) - 1, -1, -1):
        t0 = ci * C
        n = min(C, T - t0)
        pad = lambda x, fill=0.0: np.concatenate(
            [x[t0:t0 + n], np.full((C - n,) + x.shape[1:], fill)], axis=0)
        Q, K, V, A, Bg, Wg, dO = pad(q), pad(k), pad(v), pad(a, 1.0), pad(b), pad(w), pad(do)
        S0 = hs[ci]
        G = np.cumsum(np.log(A), axis=0)
        GC = G[n - 1]
        eg, egi, igc = np.exp(G), np.exp(GC[None] - G), np.exp(-GC)
        Qh, Kh, Kt = eg * Q, eg * K, egi * K
        Bt = Bg * Kt
        Aqk = incl * (Qh @ (Kt * igc).T)
        Aqb = incl * (Qh @ (Bt * igc).T)
        Akk = strict * (Kh @ (Kt * igc).T)
        Akb = strict * (Kh @ (Bt * igc).T)
        Tm = np.linalg.inv(np.eye(C) + Akb)
        U = Wg * V
        E = Tm @ (Kh @ S0 + Akk @ U)
        dE = -Aqb.T @ dO - Bt @ dS
        dY = Tm.T @ dE
        dU = Aqk.T @ dO + Akk.T @ dY + Kt @ dS
        dAqk, dAqb = incl * (dO @ U.T), -incl * (dO @ E.T)
        dAkk, dAkb = strict * (dY @ U.T), -strict * (dY @ E.T)
        XQ, XK, YK, YB = dO @ S0.T, dY @ S0.T, U @ dS.T, -E @ dS.T
        dGC = np.exp(GC) * np.sum(dS * S0, axis=1) + np.sum(Kt * YK + Bt * YB, axis=0)
        dS_prev = np.exp(GC)[:, None] * dS + Qh.T @ dO + Kh.T @ dY
        XQ = XQ + igc * (dAqk @ Kt + dAqb @ Bt)
        XK = XK + igc * (dAkk @ Kt + dAkb @ Bt)
        YK = YK + igc * (dAqk.T @ Qh + dAkk.T @ Kh)
        YB = YB + igc * (dAqb.T @ Qh + dAkb.T @ Kh)
        dG = Qh * XQ + Kh * XK - Kt * YK - Bt * YB
        dG[n - 1] += dGC
        dlog = np.cumsum(dG[::-1], axis=0)[::-1]
        sl = slice(t0, t0 + n)
        out["dq"][sl] = (eg * XQ)[:n]
        out["dk"][sl] = (eg * XK + egi * (YK + Bg * YB))[:n]
        out["db"][sl] = (Kt * YB)[:n]
        out["da"][sl] = (dlog / A)[:n]
        out["dv"][sl] = (Wg * dU)[:n]
        out["dw"][sl] = (V * dU)[:n]
        dS = dS_prev
    out["ds0"] = dS
    return out


def _inputs(seed, T, dk, dv, scalar=False):
    rng = np.random.default_rng(seed)
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    q = unit(rng.standard_normal((T, dk)))
    k = unit(rng.standard_normal((T, dk)))
    v = rng.standard_normal((T, dv))
    sig = lambda x: 1 / (1 + np.exp(-x))
    if scalar:
        a = np.exp(-np.logaddexp(0.0, rng.normal(-4.0, 1.0, (T, 1)))) * np.ones((1, dk))
        b = sig(rng.standard_normal((T, 1))) * np.ones((1, dk))
        w = sig(rng.standard_normal((T, 1))) * np.ones((1, dv))
    else:
        a = np.exp(-np.logaddexp(0.0, rng.normal(-4.0, 1.0, (T, dk))))
        b = sig(rng.standard_normal((T, dk)))
        w = sig(rng.standard_normal((T, dv)))
    f32 = lambda z: z.astype(np.float32).astype(np.float64)
    s0 = rng.normal(0, 0.1, (dk, dv))
    do = rng.standard_normal((T, dv))
    dsT = rng.normal(0, 0.1, (dk, dv))
    return [f32(z) for z in (q, k, v, a, b, w)] + [s0, do, dsT]


def _rel(x, ref):
    return float(np.max(np.abs(x - ref)) / max(np.max(np.abs(ref)), 1e-300))


@pytest.mark.parametrize("C,T", [(32, 1), (32, 31), (32, 32), (32, 97), (16, 70), (64, 150)])
def test_chunked_gradients_equal_sequential(C, T):
    q, k, v, a, b, w, s0, do, dsT = _inputs(C * 1000 + T, T, 16, 12)
    ex = lambda x: x[None, :, None]
    ref = oracle.backward(*(ex(x).astype(np.float32) for x in (q, k, v, a, b, w)),
                          s0[None, None], ex(do), dsT[None, None])
    got = chunked_backward_head(q, k, v, a, b, w, s0, do, dsT, C)
    for name in ("dq", "dk", "dv", "da", "db", "dw"):
        assert _rel(got[name], ref[name][0, :, 0]) < 1e-11, name
    assert _rel(got["ds0"], ref["ds0"][0, 0]) < 1e-11


def test_chunked_gradients_scalar_gates():
    """Scalar gates broadcast over channels: the gate gradients are the sums
    over the channels they multiply."""
    q, k, v, a, b, w, s0, do, dsT = _inputs(7, 80, 8, 8, scalar=True)
    ex = lambda x: x[None, :, None]
    f = lambda x: ex(x).astype(np.float32)
    ref = oracle.backward(f(q), f(k), f(v), f(a[:, 0]), f(b[:, 0]), f(w[:, 0]), s0[None, None],
                          ex(do), dsT[None, None])
    got = chunked_backward_head(q, k, v, a, b, w, s0, do, dsT, 32)
    for name in ("dq", "dk", "dv"):
        assert _rel(got[name], ref[name][0, :, 0]) < 1e-11, name
    for name in ("da", "db", "dw"):
        assert _rel(got[name].sum(axis=1), ref[name][0, :, 0]) < 1e-11, name
    assert _rel(got["ds0"], ref["ds0"][0, 0]) < 1e-11
