"""The chunkwise-parallel form of the recurrence, checked in float64 against the
sequential oracle.

The pages name the chunkwise-parallel training algorithm (the WY
representation of a product of rank-1 Householder-like factors, with the
diagonal-plus-low-rank structure kept) without spelling it out: FG^2-GDN page
(gist.science 2604.19021), section 2 "Methodology" (symmetry keeps the rank-1
Householder structure for WY chunked training) and section 3 "Main
contributions" (DPLR structure compatible with KDA's chunked kernels).  The
CUDA kernels compute the identity below; this test pins that identity itself,
independent of any GPU code.

Within a chunk of C tokens with initial state S0, cumulative decay
gamma_r = prod_{i<=r} a_i (per key channel), U = w*V, and
  Qh = gamma*Q, Kh = gamma*K, Kc = K/gamma, Bc = (b*K)/gamma,
  Kt = (gamma_C/gamma)*K, Bt = (gamma_C/gamma)*b*K:
  E   = (I + tril_{-1}(Kh Bc^T))^{-1} (Kh S0 + tril_{-1}(Kh Kc^T) U)
  O   = Qh S0 + tril(Qh Kc^T) U - tril(Qh Bc^T) E
  S_C = Diag(gamma_C) S0 + Kt^T U - Bt^T E
Row r of E is e_r = S'_r^T k_r, the value the key reads before its erase.
"""

import numpy as np
import pytest

import oracle


def chunked_reference(q, k, v, a, b, w, s0, C):
    """float64 chunked evaluation; gates given as full vectors (broadcast)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    sT = np.zeros((B, H, dk, dv))
    for bi in range(B):
        for h in range(H):
            S = s0[bi, h].copy() if s0 is not None else np.zeros((dk, dv))
            for t0 in range(0, T, C):
                sl = slice(t0, min(t0 + C, T))
                Q, K, V = q[bi, sl, h], k[bi, sl, h], v[bi, sl, h]
                A, Bg, W = a[bi, sl, h], b[bi, sl, h], w[bi, sl, h]
                n = Q.shape[0]
                gam = np.exp(np.cumsum(np.log(A), axis=0))
                gC = gam[-1]
                U = W * V
                Qh, Kh = gam * Q, gam * K
                Kc, Bc = K / gam, Bg * K / gam
                Kt, Bt = (gC / gam) * K, (gC / gam) * Bg * K
                lo = np.tril(np.ones((n, n)), -1)
                li = np.tril(np.ones((n, n)))
                E = np.linalg.solve(np.eye(n) + lo * (Kh @ Bc.T), Kh @ S + (lo * (Kh @ Kc.T)) @ U)
                o[bi, sl, h] = Qh @ S + (li * (Qh @ Kc.T)) @ U - (li * (Qh @ Bc.T)) @ E
                S = gC[:, None] * S + Kt.T @ U - Bt.T @ E
            sT[bi, h] = S
    return o, sT


def _inputs(seed, B, T, H, dk, dv, scalar_decay=False):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, dk))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    x = rng.normal(-4.0, 1.0, (B, T, H) if scalar_decay else (B, T, H, dk))
    a = np.exp(-np.logaddexp(0.0, x))
    if scalar_decay:
        a = np.repeat(a[..., None], dk, axis=-1)
    b = 1 / (1 + np.exp(-rng.standard_normal((B, T, H, dk))))
    w = 1 / (1 + np.exp(-rng.standard_normal((B, T, H, dv))))
    s0 = rng.normal(0, 0.1, (B, H, dk, dv))
    f32 = lambda z: z.astype(np.float32).astype(np.float64)
    return [f32(z) for z in (q, k, v, a, b, w)] + [s0]


@pytest.mark.parametrize("C,T", [(8, 37), (16, 64), (64, 64), (64, 150), (32, 97)])
def test_chunked_equals_sequential(C, T):
    q, k, v, a, b, w, s0 = _inputs(C * 1000 + T, 1, T, 2, 16, 12)
    o_ref, s_ref = oracle.forward(q, k, v, a, b, w, s0)
    o, s = chunked_reference(q, k, v, a, b, w, s0, C)
    rel = lambda x, r: np.max(np.abs(x - r)) / np.max(np.abs(r))
    assert rel(o, o_ref) < 1e-12
    assert rel(s, s_ref) < 1e-12


def test_chunked_scalar_decay_and_shared_beta():
    q, k, v, a, b, w, s0 = _inputs(5, 1, 80, 2, 8, 8, scalar_decay=True)
    w = np.repeat(b[..., :1], 8, axis=-1)        # one scalar beta ...
    b = w.copy()                                  # ... for erase and write
    o_ref, s_ref = oracle.forward(q, k, v, a[..., 0], b[..., 0], w[..., 0], s0)
    o, s = chunked_reference(q, k, v, a, b, w, s0, 32)
    assert np.max(np.abs(o - o_ref)) / np.max(np.abs(o_ref)) < 1e-12
    assert np.max(np.abs(s - s_ref)) / np.max(np.abs(s_ref)) < 1e-12


def _block_inverse(N, n0):
    """T = (I + N)^{-1} for strictly lower N (size a power of two times n0)
    by the order the kernels use: forward substitution on the n0 x n0
    diagonal blocks, then the 2 x 2 block step T21 = -T2 (N21 T1) at every
    doubling of the block size."""
    n = N.shape[0]
    T = np.zeros_like(N)
    for i in range(0, n, n0):
        blk = N[i:i + n0, i:i + n0]
        for c in range(n0):
            x = np.zeros(n0)
            for r in range(n0):
                x[r] = (1.0 if r == c else 0.0) - blk[r, :r] @ x[:r]
            T[i:i + n0, i + c] = x
    m = n0
    while m < n:
        for i in range(0, n, 2 * m):
            T1, T2 = T[i:i + m, i:i + m], T[i + m:i + 2 * m, i + m:i + 2 * m]
            T[i + m:i + 2 * m, i:i + m] = -T2 @ (N[i + m:i + 2 * m, i:i + m] @ T1)
        m *= 2
    return T


@pytest.mark.parametrize("n0", [8, 16])
def test_ut_transform_block_recursion(n0):
    """The UT transform T = (I + A_kb)^{-1} of a 64-token chunk, evaluated as
    the kernels do (8 x 8 substitution and block steps at 8, 16 and 32 rows;
    16 x 16 substitution as before), equals the direct inverse, and T21 is
    the only block that changes per level (T stays unit lower triangular)."""
    rng = np.random.default_rng(5)
    k = rng.normal(size=(64, 128))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    gam = np.cumprod(np.exp(-np.log1p(np.exp(rng.normal(-4, 1, size=(64, 128))))), axis=0)
    beta = 1 / (1 + np.exp(-rng.normal(size=(64, 128))))
    N = np.tril((gam * k) @ (beta * k / gam).T, -1)
    T = _block_inverse(N, n0)
    assert np.allclose(T, np.linalg.inv(np.eye(64) + N), rtol=0, atol=1e-12)
    assert np.array_equal(np.triu(T, 1), np.zeros((64, 64)))
    assert np.allclose(np.diag(T), 1.0)
