"""Seeded synthetic workloads for the gated delta-rule recurrence.

This module only draws inputs.  It holds none of the recurrence's arithmetic
and imports nothing else from this package, so the CUDA path and the float64
oracle can both take their inputs from it.

Recipe (every workload, every step):

* one independent numpy PCG64 stream per (batch b, head h, decode step),
  ``SeedSequence(seed, spawn_key=(b, h, step))`` (step = 0 for prefill);
* draws in float64, in this order: q [T, dk], k [T, dk], v [T, dv],
  x_decay ([T, dk] or [T]), x_erase ([T, dk] or [T]), x_write ([T, dv] or [T],
  only when the write gate is decoupled), then s0 [dk, dv] when the workload
  has a random initial state;
* q, k ~ N(0, 1) then L2-normalised over dk per token; v ~ N(0, 1);
* decay a = exp(-softplus(x)), x ~ N(-4, 1); erase / write gates
  b, w = sigmoid(N(0, 1)); a shared gate (b = w = beta) is one tensor;
* s0 ~ N(0, 0.1) (standard deviation 0.1), kept in float32;
* float32 workloads keep float32 values; bf16 workloads round float32 to bf16
  with round-to-nearest-even.  The float32 images of the bf16 values are exact,
  so the oracle sees exactly the numbers the GPU sees.

The five named workloads carry the shapes and gate kinds of the gated
delta-rule family the pages describe: Gated DeltaNet (scalar decay, one scalar
beta for erase and write), KDA (per-channel decay, scalar beta), and
Gated DeltaNet-2 / FG^2-GDN+ (per-channel decay, decoupled per-channel erase
and write gates), plus a long-sequence prefill and a batched decode step.
"""

from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, Iterable, Optional, Sequence, Tuple

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    H: int
    dk: int
    dv: int
    chunk: int
    dtype: str          # "f32" or "bf16" (q, k, v, gates and o)
    decay: str          # "scalar" or "vector"
    erase: str          # "scalar" or "vector"
    write: str          # "scalar", "vector" or "shared" (the erase tensor)
    random_s0: bool     # s0 ~ N(0, 0.1) instead of zeros
    steps: int = 0      # decode steps (0 for prefill workloads)

    @property
    def token_heads(self) -> int:
        return self.B * self.T * self.H

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    # Gated DeltaNet, scalar gates, fp32: B=1 H=2 T=256 d=64, chunk 64.
    "gdn_fp32": Workload("gdn_fp32", 1, 256, 2, 64, 64, 64, "f32",
                         "scalar", "scalar", "shared", False),
    # KDA-style per-channel decay, scalar beta = erase = write, bf16.
    "kda_bf16": Workload("kda_bf16", 4, 4096, 16, 128, 128, 64, "bf16",
                         "vector", "scalar", "shared", False),
    # Decoupled per-channel erase and write gates, per-channel decay, bf16,
    # random initial state: the H=16, d=128, T=8k throughput workload.
    "gdn2_bf16": Workload("gdn2_bf16", 8, 8192, 16, 128, 128, 64, "bf16",
                          "vector", "vector", "vector", True),
    # Long-context prefill: B=1 H=32 T=65536, decoupled gates, zero s0.
    "long_bf16": Workload("long_bf16", 1, 65536, 32, 128, 128, 64, "bf16",
                          "vector", "vector", "vector", False),
    # Single-token decode: batch 256, H=32, d=128, state ~ N(0, 0.1),
    # 1000 consecutive steps with fresh inputs each step.
    "decode_bf16": Workload("decode_bf16", 256, 1, 32, 128, 128, 64, "bf16",
                            "vector", "vector", "vector", True, steps=1000),
}


# ---------------------------------------------------------------- bf16 helpers

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (round-to-nearest-even); returns uint16 bits."""
    u = np.array(x, dtype=np.float32, order="C").view(np.uint32)
    rounding = ((u >> 16) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + rounding) >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact float32 image of bf16 bit patterns."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32)
            << np.uint32(16)).view(np.float32)


# ------------------------------------------------------------------ drawing

def _stream(seed: int, b: int, h: int, step: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(
        np.random.SeedSequence(seed, spawn_key=(b, h, step))))


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def _l2norm(x):
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True))


def _draw_head(wl: Workload, T: int, seed: int, b: int, h: int, step: int):
    """All float64 draws of one (b, h, step) stream, in the fixed order."""
    g = _stream(seed, b, h, step)
    dk, dv = wl.dk, wl.dv
    q = _l2norm(g.standard_normal((T, dk)))
    k = _l2norm(g.standard_normal((T, dk)))
    v = g.standard_normal((T, dv))
    xa = g.normal(-4.0, 1.0, (T, dk) if wl.decay == "vector" else (T,))
    a = np.exp(-np.logaddexp(0.0, xa))           # exp(-softplus(x))
    xb = g.standard_normal((T, dk) if wl.erase == "vector" else (T,))
    bg = _sigmoid(xb)
    wg = None
    if wl.write != "shared":
        xw = g.standard_normal((T, dv) if wl.write == "vector" else (T,))
        wg = _sigmoid(xw)
    s0 = g.normal(0.0, 0.1, (dk, dv)) if wl.random_s0 else None
    return q, k, v, a, bg, wg, s0


def _gate_shape(kind: str, lead: Tuple[int, ...], d: int):
    return lead + ((d,) if kind == "vector" else ())


def _store(x64: np.ndarray, dtype: str) -> np.ndarray:
    x32 = x64.astype(np.float32)
    return x32 if dtype == "f32" else f32_to_bf16_bits(x32)


def make_prefill(wl: Workload, seed: int = 0, heads: Optional[Sequence[Tuple[int, int]]] = None,
                 threads: int = 8) -> Dict[str, np.ndarray]:
    """Draw q, k, v, a, b, w (and s0) for a prefill workload.

    Tensors come back in [B, T, H, ...] layout: float32 for "f32" workloads,
    uint16 bf16 bits for "bf16" workloads.  ``w`` is None when the write gate
    is shared with the erase gate.  ``s0`` is float32 [B, H, dk, dv] or None.
    If ``heads`` is given, only those (b, h) slices are drawn (the rest stay
    zero), which is enough to check a sample of heads.
    """
    B, T, H, dk, dv = wl.B, wl.T, wl.H, wl.dk, wl.dv
    st = np.float32 if wl.dtype == "f32" else np.uint16
    out = {
        "q": np.zeros((B, T, H, dk), st),
        "k": np.zeros((B, T, H, dk), st),
        "v": np.zeros((B, T, H, dv), st),
        "a": np.zeros(_gate_shape(wl.decay, (B, T, H), dk), st),
        "b": np.zeros(_gate_shape(wl.erase, (B, T, H), dk), st),
        "w": None if wl.write == "shared" else np.zeros(_gate_shape(wl.write, (B, T, H), dv), st),
        "s0": np.zeros((B, H, dk, dv), np.float32) if wl.random_s0 else None,
    }
    todo = list(heads) if heads is not None else [(b, h) for b in range(B) for h in range(H)]

    def one(bh):
        b, h = bh
        q, k, v, a, bg, wg, s0 = _draw_head(wl, T, seed, b, h, 0)
        out["q"][b, :, h] = _store(q, wl.dtype)
        out["k"][b, :, h] = _store(k, wl.dtype)
        out["v"][b, :, h] = _store(v, wl.dtype)
        out["a"][b, :, h] = _store(a, wl.dtype)
        out["b"][b, :, h] = _store(bg, wl.dtype)
        if wg is not None:
            out["w"][b, :, h] = _store(wg, wl.dtype)
        if s0 is not None:
            out["s0"][b, h] = s0.astype(np.float32)

    if threads > 1 and len(todo) > 1:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(one, todo))
    else:
        for bh in todo:
            one(bh)
    return out


def make_decode_state(wl: Workload, seed: int = 0,
                      heads: Optional[Iterable[Tuple[int, int]]] = None,
                      threads: int = 8) -> np.ndarray:
    """Initial decode state [B, H, dk, dv] float32, drawn from step 0's streams."""
    assert wl.random_s0
    st = np.zeros((wl.B, wl.H, wl.dk, wl.dv), np.float32)
    todo = list(heads) if heads is not None else [(b, h) for b in range(wl.B) for h in range(wl.H)]

    def one(bh):
        b, h = bh
        st[b, h] = _draw_head(wl, 1, seed, b, h, 0)[6].astype(np.float32)

    if threads > 1 and len(todo) > 1:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(one, todo))
    else:
        for bh in todo:
            one(bh)
    return st


def make_decode_step(wl: Workload, step: int, seed: int = 0,
                     heads: Optional[Sequence[Tuple[int, int]]] = None,
                     threads: int = 8) -> Dict[str, np.ndarray]:
    """Inputs of decode step ``step`` (1-based), [B, H, ...] layout.

    Same recipe as prefill with T = 1, drawn from the stream (b, h, step).
    """
    assert step >= 1
    B, H, dk, dv = wl.B, wl.H, wl.dk, wl.dv
    st = np.float32 if wl.dtype == "f32" else np.uint16
    out = {
        "q": np.zeros((B, H, dk), st),
        "k": np.zeros((B, H, dk), st),
        "v": np.zeros((B, H, dv), st),
        "a": np.zeros(_gate_shape(wl.decay, (B, H), dk), st),
        "b": np.zeros(_gate_shape(wl.erase, (B, H), dk), st),
        "w": None if wl.write == "shared" else np.zeros(_gate_shape(wl.write, (B, H), dv), st),
    }
    todo = list(heads) if heads is not None else [(b, h) for b in range(B) for h in range(H)]

    def one(bh):
        b, h = bh
        q, k, v, a, bg, wg, _ = _draw_head(wl.replace(random_s0=False), 1, seed, b, h, step)
        out["q"][b, h] = _store(q[0], wl.dtype)
        out["k"][b, h] = _store(k[0], wl.dtype)
        out["v"][b, h] = _store(v[0], wl.dtype)
        out["a"][b, h] = _store(a[0], wl.dtype)
        out["b"][b, h] = _store(bg[0], wl.dtype)
        if wg is not None:
            out["w"][b, h] = _store(wg[0], wl.dtype)

    if threads > 1 and len(todo) > 1:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(one, todo))
    else:
        for bh in todo:
            one(bh)
    return out


def as_f32(x: Optional[np.ndarray], dtype: str) -> Optional[np.ndarray]:
    """Exact float32 values of a drawn tensor (bf16 bits or float32)."""
    if x is None:
        return None
    return x if dtype == "f32" else bf16_bits_to_f32(x)


def make_upstream(wl: Workload, seed: int = 0,
                  heads: Optional[Sequence[Tuple[int, int]]] = None,
                  threads: int = 8) -> Dict[str, np.ndarray]:
    """Upstream gradients for the backward pass of a prefill workload: do
    [B, T, H, dv] ~ N(0, 1) in the workload's dtype (bf16 bits or float32) and
    dsT [B, H, dk, dv] ~ N(0, 0.1) float32, from streams of their own
    (spawn key (b, h, 2^20)), so they are independent of the inputs.  With
    ``heads`` only those (b, h) slices are drawn (the rest stay zero)."""
    B, T, H, dk, dv = wl.B, wl.T, wl.H, wl.dk, wl.dv
    st = np.float32 if wl.dtype == "f32" else np.uint16
    out = {"do": np.zeros((B, T, H, dv), st), "dsT": np.zeros((B, H, dk, dv), np.float32)}
    todo = list(heads) if heads is not None else [(b, h) for b in range(B) for h in range(H)]

    def one(bh):
        b, h = bh
        g = _stream(seed, b, h, 1 << 20)
        out["do"][b, :, h] = _store(g.standard_normal((T, dv)), wl.dtype)
        out["dsT"][b, h] = g.normal(0.0, 0.1, (dk, dv)).astype(np.float32)

    if threads > 1 and len(todo) > 1:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(one, todo))
    else:
        for bh in todo:
            one(bh)
    return out


# ------------------------------------------------- device-side draws (timing)

def _torch_draws(wl: Workload, lead: Tuple[int, ...], seed: int, device):
    """The same distributions as _draw_head, drawn by torch's generator on
    ``device`` for leading shape ``lead`` (a different random stream from the
    numpy one: used where host-side drawing would dominate a timing run)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    dk, dv = wl.dk, wl.dv
    dt = torch.float32 if wl.dtype == "f32" else torch.bfloat16

    def normal(shape, mean=0.0, std=1.0):
        return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std + mean

    def unit(shape):
        x = normal(shape)
        return x / x.norm(dim=-1, keepdim=True)

    cast = lambda x: x.to(dt).contiguous()   # each tensor leaves float32 at once
    out = {"q": cast(unit(lead + (dk,))), "k": cast(unit(lead + (dk,))),
           "v": cast(normal(lead + (dv,)))}
    xa = normal(lead + ((dk,) if wl.decay == "vector" else ()), -4.0, 1.0)
    out["a"] = cast(torch.exp(-torch.nn.functional.softplus(xa)))
    del xa
    out["b"] = cast(torch.sigmoid(normal(lead + ((dk,) if wl.erase == "vector" else ()))))
    out["w"] = None
    if wl.write != "shared":
        out["w"] = cast(torch.sigmoid(normal(lead + ((dv,) if wl.write == "vector" else ()))))
    return out


def make_prefill_device(wl: Workload, seed: int = 0, device="cuda"):
    """Prefill inputs of ``wl`` drawn on the device (torch tensors in the
    workload's dtype, [B, T, H, ...]); s0 ~ N(0, 0.1) float32 when the
    workload has a random initial state.  ``w`` is None for a shared gate."""
    import torch
    x = _torch_draws(wl, (wl.B, wl.T, wl.H), seed, device)
    x["s0"] = None
    if wl.random_s0:
        g = torch.Generator(device=device)
        g.manual_seed(seed + 7919)
        x["s0"] = torch.randn((wl.B, wl.H, wl.dk, wl.dv), generator=g, device=device) * 0.1
    return x


def make_decode_steps_device(wl: Workload, steps: int, seed: int = 0, device="cuda"):
    """Fresh inputs for ``steps`` consecutive decode steps, drawn on the
    device: tensors [steps, B, H, ...] in the workload's dtype."""
    return _torch_draws(wl, (steps, wl.B, wl.H), seed, device)
