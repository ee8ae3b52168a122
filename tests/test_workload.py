"""Seeded synthetic inputs: determinism, per-head streams, bf16 rounding."""

import numpy as np

from gated_delta_rule_154_b200 import workload as wlmod


def test_bf16_round_to_nearest_even():
    x = np.array([1.0, 1.0 + 2**-8, 1.0 + 3 * 2**-8, -2.5, 3.0e-3, 1.0 + 2**-7], np.float32)
    bits = wlmod.f32_to_bf16_bits(x)
    back = wlmod.bf16_bits_to_f32(bits)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: even mantissa (1.0) wins;
    # 1 + 3*2^-8 ties between 1 + 2^-7 and 1 + 2^-6: even is 1 + 2^-6.
    assert back[0] == 1.0 and back[1] == 1.0 and back[2] == 1.0 + 2**-6
    assert back[3] == -2.5 and back[5] == 1.0 + 2**-7
    assert abs(back[4] - 3.0e-3) <= 3.0e-3 * 2**-8


def test_deterministic_and_subset_consistent():
    wl = wlmod.WORKLOADS["gdn2_bf16"].replace(B=2, T=70, H=3)
    full = wlmod.make_prefill(wl, seed=0)
    again = wlmod.make_prefill(wl, seed=0, threads=1)
    sub = wlmod.make_prefill(wl, seed=0, heads=[(1, 2)])
    for key in ("q", "k", "v", "a", "b", "w", "s0"):
        assert np.array_equal(full[key], again[key])
        assert np.array_equal(full[key][1, :, 2] if key != "s0" else full[key][1, 2],
                              sub[key][1, :, 2] if key != "s0" else sub[key][1, 2])
    other = wlmod.make_prefill(wl, seed=1)
    assert not np.array_equal(full["q"], other["q"])


def test_distributions_follow_recipe():
    wl = wlmod.WORKLOADS["gdn2_bf16"].replace(B=1, T=512, H=2)
    x = wlmod.make_prefill(wl, seed=0)
    f = lambda key: wlmod.as_f32(x[key], wl.dtype).astype(np.float64)
    qn = np.linalg.norm(f("q"), axis=-1)
    assert np.all(np.abs(qn - 1) < 1e-2)                # L2-normalised (bf16 rounding)
    a = f("a")
    assert np.all((a > 0) & (a <= 1))
    assert 0.95 < np.median(a) < 0.995                   # exp(-softplus(N(-4,1)))
    b = f("b")
    assert np.all((b > 0) & (b < 1)) and abs(np.median(b) - 0.5) < 0.05
    assert abs(np.std(x["s0"]) - 0.1) < 0.01


def test_shared_gate_and_scalar_shapes():
    wl = wlmod.WORKLOADS["kda_bf16"].replace(B=1, T=8, H=2)
    x = wlmod.make_prefill(wl)
    assert x["w"] is None and x["b"].shape == (1, 8, 2) and x["a"].shape == (1, 8, 2, 128)
    wl = wlmod.WORKLOADS["gdn_fp32"]
    x = wlmod.make_prefill(wl)
    assert x["q"].dtype == np.float32 and x["a"].shape == (1, 256, 2) and x["s0"] is None


def test_decode_steps_differ_and_subset_consistent():
    wl = wlmod.WORKLOADS["decode_bf16"].replace(B=2, H=3)
    s1 = wlmod.make_decode_step(wl, 1)
    s2 = wlmod.make_decode_step(wl, 2)
    assert not np.array_equal(s1["k"], s2["k"])
    sub = wlmod.make_decode_step(wl, 2, heads=[(1, 1)])
    assert np.array_equal(sub["v"][1, 1], s2["v"][1, 1])
    st = wlmod.make_decode_state(wl)
    assert st.shape == (2, 3, 128, 128) and abs(np.std(st) - 0.1) < 0.01


def test_upstream_gradients_seeded_and_independent_of_inputs():
    wl = wlmod.WORKLOADS["gdn2_bf16"].replace(B=2, T=40, H=3)
    up = wlmod.make_upstream(wl, seed=0)
    again = wlmod.make_upstream(wl, seed=0, threads=1)
    sub = wlmod.make_upstream(wl, seed=0, heads=[(1, 2)])
    assert up["do"].shape == (2, 40, 3, 128) and up["do"].dtype == np.uint16
    assert up["dsT"].shape == (2, 3, 128, 128) and up["dsT"].dtype == np.float32
    for key in ("do", "dsT"):
        assert np.array_equal(up[key], again[key])
    assert np.array_equal(sub["do"][1, :, 2], up["do"][1, :, 2])
    assert np.array_equal(sub["dsT"][1, 2], up["dsT"][1, 2])
    assert not sub["do"][0].any() and not sub["dsT"][0].any()      # undrawn heads stay zero
    inp = wlmod.make_prefill(wl, seed=0)                             # a stream of its own
    assert not np.array_equal(inp["v"], up["do"])
    do = wlmod.as_f32(up["do"], wl.dtype)
    assert abs(np.std(do) - 1.0) < 0.05 and abs(np.std(up["dsT"]) - 0.1) < 0.01
