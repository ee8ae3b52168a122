"""The sequence-split identity behind splitting one sequence across devices,
checked in float64 on the oracle.

The recurrence is affine in the state: every token maps S to
A_t S + k_t (w_t*v_t)^T with A_t = (I - (b_t*k_t) k_t^T) Diag(a_t) (FG^2-GDN page,
gist.science 2604.19021, section 2 "Methodology", update rule).  A segment of
tokens therefore maps its start state to S_end = M S_start + N, where M (the
product of its A_t) is what the segment makes of S_start = I with every value
zero, and N is what it makes of S_start = 0 with the real values.  Chaining the
(M, N) of consecutive segments gives each segment's start state; each segment
rerun from that state gives exactly the outputs and final state of the whole
sequence.  This is the exchange a sequence-parallel prefill needs (one (M, N)
per segment); the test pins the identity, not a parallel implementation.
"""

import numpy as np
import pytest

import oracle


def _inputs(seed, T, d):
    rng = np.random.default_rng(seed)
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    sig = lambda x: 1 / (1 + np.exp(-x))
    q = unit(rng.standard_normal((1, T, 1, d)))
    k = unit(rng.standard_normal((1, T, 1, d)))
    v = rng.standard_normal((1, T, 1, d))
    a = np.exp(-np.logaddexp(0.0, rng.normal(-4.0, 1.0, (1, T, 1, d))))
    b = sig(rng.standard_normal((1, T, 1, d)))
    w = sig(rng.standard_normal((1, T, 1, d)))
    s0 = rng.normal(0.0, 0.1, (1, 1, d, d))
    f32 = lambda z: z.astype(np.float32)
    return [f32(z) for z in (q, k, v, a, b, w)] + [s0]


@pytest.mark.parametrize("T,cuts", [(96, [40]), (150, [32, 64, 100]), (64, [1, 63])])
def test_segments_chained_by_affine_maps_equal_the_whole_sequence(T, cuts):
    d = 8
    q, k, v, a, b, w, s0 = _inputs(T + len(cuts), T, d)
    o_ref, s_ref = oracle.forward(q, k, v, a, b, w, s0)
    bounds = [0] + cuts + [T]
    S = s0[0, 0]
    outs = []
    for t0, t1 in zip(bounds[:-1], bounds[1:]):
        seg = lambda x: x[:, t0:t1]
        # the segment's transition M (from I with zero values) and offset N (from 0)
        _, M = oracle.forward(seg(q), seg(k), np.zeros_like(seg(v)), seg(a), seg(b), seg(w),
                              np.eye(d)[None, None], want_o=False)
        _, N = oracle.forward(seg(q), seg(k), seg(v), seg(a), seg(b), seg(w), None, want_o=False)
        o_seg, s_seg = oracle.forward(seg(q), seg(k), seg(v), seg(a), seg(b), seg(w), S[None, None])
        S_next = M[0, 0] @ S + N[0, 0]
        assert np.max(np.abs(S_next - s_seg[0, 0])) <= 1e-12 * max(1.0, np.max(np.abs(S_next)))
        outs.append(o_seg)
        S = S_next
    o = np.concatenate(outs, axis=1)
    assert np.max(np.abs(o - o_ref)) <= 1e-12 * np.max(np.abs(o_ref))
    assert np.max(np.abs(S - s_ref[0, 0])) <= 1e-12 * np.max(np.abs(s_ref))
