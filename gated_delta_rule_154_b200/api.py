"""torch-facing calls of the gated delta-rule library.

Argument marshalling only: every step of the recurrence runs in libgdr.so's
CUDA kernels.  torch supplies device memory and the current stream.

Shapes (row-major, contiguous, on one CUDA device):
    prefill  q, k [B, T, H, dk]; v [B, T, H, dv]; a, b [B, T, H, dk] or
             [B, T, H] (scalar gate) or None (gate == 1); w [B, T, H, dv] or
             [B, T, H] or None; s0 [B, H, dk, dv] float32 or None (zeros)
    decode   the same without the T axis; state [B, H, dk, dv] float32,
             updated in place
q, k, v, the gates and o share one dtype (torch.float32 or torch.bfloat16).

FG^2-GDN / FG^2-GDN+ (forward_fg2, decode_step_fg2): per-channel learning
rates beta^k [.., dk] and beta^v [.., dv] (one tensor for both in FG^2-GDN),
entering through their square roots inside the kernels: key sqrt(beta^k) k,
erase gate 1, write gate sqrt(beta^v).
"""

from __future__ import annotations

from typing import Optional, Tuple

import torch

from . import _lib

_DT = {torch.float32: _lib.F32, torch.bfloat16: _lib.BF16}


def _ptr(t: Optional[torch.Tensor]) -> int:
    return 0 if t is None else int(t.data_ptr())


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _check(t: Optional[torch.Tensor], name: str, dtype, device, shapes):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if t.device != device:
        raise ValueError("%s is on %s, expected %s" % (name, t.device, device))
    if t.dtype != dtype:
        raise ValueError("%s has dtype %s, expected %s" % (name, t.dtype, dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if tuple(t.shape) not in [tuple(s) for s in shapes]:
        raise ValueError("%s has shape %s, expected one of %s" % (name, tuple(t.shape), shapes))


def _gate_kind(g: Optional[torch.Tensor], ndim_vector: int) -> int:
    if g is None:
        return _lib.GATE_ONE
    return _lib.GATE_VECTOR if g.dim() == ndim_vector else _lib.GATE_SCALAR


def make_desc(B, T, H, dk, dv, chunk, dtype, a_kind, b_kind, w_kind) -> _lib.GdrDesc:
    return _lib.GdrDesc(B, T, H, dk, dv, chunk, dtype, a_kind, b_kind, w_kind)


def desc_for(q, v, a, b, w, chunk: int = 64, decode: bool = False,
             fg2: bool = False) -> _lib.GdrDesc:
    if decode:
        B, H, dk = q.shape
        T = 1
        nd = 3
    else:
        B, T, H, dk = q.shape
        nd = 4
    dv = v.shape[-1]
    if fg2:
        return make_desc(B, T, H, dk, dv, chunk, _DT[q.dtype], _gate_kind(a, nd),
                         _lib.GATE_FG2, _lib.GATE_FG2)
    return make_desc(B, T, H, dk, dv, chunk, _DT[q.dtype], _gate_kind(a, nd),
                     _gate_kind(b, nd), _gate_kind(w, nd))


def workspace_size(desc: _lib.GdrDesc) -> int:
    return _lib.workspace_size(desc)


def forward_chunked(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                    a: Optional[torch.Tensor] = None, b: Optional[torch.Tensor] = None,
                    w: Optional[torch.Tensor] = None, s0: Optional[torch.Tensor] = None,
                    *, chunk: int = 64, out: Optional[torch.Tensor] = None,
                    s_final: Optional[torch.Tensor] = None, return_final: bool = True,
                    workspace: Optional[torch.Tensor] = None, stream=None,
                    fg2: bool = False,
                    split: bool = True) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Causal chunked prefill.  Returns (o [B, T, H, dv], S_T [B, H, dk, dv] or None).
    With fg2=True, b and w hold the vector learning rates beta^k, beta^v.
    Few heads with long sequences are split into segments that run side by
    side (the library's choice, when a workspace is given); split=False
    passes none and keeps the one-pass kernel."""
    if q.dtype not in _DT:
        raise ValueError("q must be float32 or bfloat16")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    _check(q, "q", dt, dev, [(B, T, H, dk)])
    _check(k, "k", dt, dev, [(B, T, H, dk)])
    _check(v, "v", dt, dev, [(B, T, H, dv)])
    _check(a, "a", dt, dev, [(B, T, H, dk), (B, T, H)])
    _check(b, "b", dt, dev, [(B, T, H, dk), (B, T, H)])
    _check(w, "w", dt, dev, [(B, T, H, dv), (B, T, H)])
    _check(s0, "s0", torch.float32, dev, [(B, H, dk, dv)])
    if fg2 and (b is None or w is None or b.dim() != 4 or w.dim() != 4):
        raise ValueError("fg2 needs vector beta^k [B, T, H, dk] and beta^v [B, T, H, dv]")
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=dt, device=dev)
    _check(out, "out", dt, dev, [(B, T, H, dv)])
    if s_final is None and return_final:
        s_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    _check(s_final, "s_final", torch.float32, dev, [(B, H, dk, dv)])
    desc = desc_for(q, v, a, b, w, chunk, fg2=fg2)
    need = _lib.workspace_size(desc) if split else 0
    if not split:
        workspace = None
    elif need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = _lib.forward_chunked(desc, _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(w),
                              _ptr(s0), _ptr(out), _ptr(s_final), _ptr(workspace), ws_bytes,
                              _stream_handle(stream))
    if st != _lib.OK:
        raise _lib.GdrError(st, "gdr_forward_chunked")
    return out, s_final


def backward_workspace_size(desc: _lib.GdrDesc) -> int:
    return _lib.backward_workspace_size(desc)


def backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
             a: Optional[torch.Tensor], b: Optional[torch.Tensor], w: Optional[torch.Tensor],
             s0: Optional[torch.Tensor], d_o: torch.Tensor,
             ds_final: Optional[torch.Tensor] = None, *,
             cu_seqlens: Optional[torch.Tensor] = None, fg2: bool = False,
             want_ds0: bool = True, out: Optional[dict] = None,
             workspace: Optional[torch.Tensor] = None, stream=None) -> dict:
    """Gradients of  L = sum_t <o_t, d_o_t> + <S_T, ds_final>  for the prefill
    of (q, k, v, a, b, w, s0).  Returns a dict with dq, dk, dv (input dtype),
    da, db, dw (shape and dtype of a, b, w; None for an absent gate) and ds0
    (float32, or None with want_ds0=False).  With b and w the same tensor
    (shared beta) its gradient is db + dw.  fg2=True: b and w are FG^2-GDN
    learning rates beta^k, beta^v and db, dw their gradients.  cu_seqlens
    (int32 [N + 1] on the device): packed sequences in q [1, T, H, dk] as in
    forward_varlen; s0, ds_final and ds0 are then [N, H, dk, dv] and tokens
    outside every sequence keep whatever `out` held.  `out` may supply any of
    the gradient tensors."""
    if q.dtype not in _DT:
        raise ValueError("q must be float32 or bfloat16")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    N = B
    if cu_seqlens is not None:
        if B != 1:
            raise ValueError("packed sequences take q as [1, T, H, dk]")
        _check(cu_seqlens, "cu_seqlens", torch.int32, dev, [tuple(cu_seqlens.shape)])
        if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
            raise ValueError("cu_seqlens must be int32 [N + 1], N >= 1")
        N = cu_seqlens.numel() - 1
    _check(q, "q", dt, dev, [(B, T, H, dk)])
    _check(k, "k", dt, dev, [(B, T, H, dk)])
    _check(v, "v", dt, dev, [(B, T, H, dv)])
    _check(a, "a", dt, dev, [(B, T, H, dk), (B, T, H)])
    _check(b, "b", dt, dev, [(B, T, H, dk), (B, T, H)])
    _check(w, "w", dt, dev, [(B, T, H, dv), (B, T, H)])
    _check(s0, "s0", torch.float32, dev, [(N, H, dk, dv)])
    _check(d_o, "d_o", dt, dev, [(B, T, H, dv)])
    _check(ds_final, "ds_final", torch.float32, dev, [(N, H, dk, dv)])
    if fg2 and (b is None or w is None or b.dim() != 4 or w.dim() != 4):
        raise ValueError("fg2 needs vector beta^k [B, T, H, dk] and beta^v [B, T, H, dv]")
    like = lambda t: None if t is None else torch.empty_like(t)
    g = {"dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v),
         "da": like(a), "db": like(b), "dw": like(w),
         "ds0": torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev) if want_ds0 else None}
    for name, t in (out or {}).items():
        if name not in g or g[name] is None:
            raise ValueError("unexpected output %s" % name)
        ref = g[name]
        _check(t, name, ref.dtype, dev, [tuple(ref.shape)])
        g[name] = t
    desc = desc_for(q, v, a, b, w, 32, fg2=fg2)
    need = (_lib.backward_varlen_workspace_size(desc, N) if cu_seqlens is not None
            else _lib.backward_workspace_size(desc))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size()
    grads = [_ptr(g[n]) for n in ("dq", "dk", "dv", "da", "db", "dw", "ds0")]
    ins = [_ptr(x) for x in (q, k, v, a, b, w, s0, d_o, ds_final)]
    if cu_seqlens is not None:
        st = _lib.backward_varlen(desc, _ptr(cu_seqlens), N, *ins, *grads, _ptr(workspace),
                                  ws_bytes, _stream_handle(stream))
        what = "gdr_backward_varlen"
    else:
        st = _lib.backward_chunked(desc, *ins, *grads, _ptr(workspace), ws_bytes,
                                   _stream_handle(stream))
        what = "gdr_backward_chunked"
    if st != _lib.OK:
        raise _lib.GdrError(st, what)
    return g


def decode_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                a: Optional[torch.Tensor], b: Optional[torch.Tensor],
                w: Optional[torch.Tensor], state: torch.Tensor, *,
                out: Optional[torch.Tensor] = None, stream=None,
                fg2: bool = False) -> torch.Tensor:
    """One decode step; `state` is updated in place.  Returns o [B, H, dv].
    With fg2=True, b and w hold the vector learning rates beta^k, beta^v."""
    if q.dtype not in _DT:
        raise ValueError("q must be float32 or bfloat16")
    B, H, dk = q.shape
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    _check(q, "q", dt, dev, [(B, H, dk)])
    _check(k, "k", dt, dev, [(B, H, dk)])
    _check(v, "v", dt, dev, [(B, H, dv)])
    _check(a, "a", dt, dev, [(B, H, dk), (B, H)])
    _check(b, "b", dt, dev, [(B, H, dk), (B, H)])
    _check(w, "w", dt, dev, [(B, H, dv), (B, H)])
    _check(state, "state", torch.float32, dev, [(B, H, dk, dv)])
    if fg2 and (b is None or w is None or b.dim() != 3 or w.dim() != 3):
        raise ValueError("fg2 needs vector beta^k [B, H, dk] and beta^v [B, H, dv]")
    if out is None:
        out = torch.empty((B, H, dv), dtype=dt, device=dev)
    _check(out, "out", dt, dev, [(B, H, dv)])
    desc = desc_for(q, v, a, b, w, decode=True, fg2=fg2)
    st = _lib.decode_step(desc, _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(w),
                          _ptr(state), _ptr(out), _stream_handle(stream))
    if st != _lib.OK:
        raise _lib.GdrError(st, "gdr_decode_step")
    return out


def forward_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                   a: Optional[torch.Tensor], b: Optional[torch.Tensor],
                   w: Optional[torch.Tensor], cu_seqlens: torch.Tensor,
                   s0: Optional[torch.Tensor] = None, *, chunk: int = 64,
                   out: Optional[torch.Tensor] = None, s_final: Optional[torch.Tensor] = None,
                   return_final: bool = True, stream=None,
                   fg2: bool = False) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Prefill of packed sequences: q, k, v, gates, o are [1, T, H, *]; sequence
    n is tokens [cu_seqlens[n], cu_seqlens[n + 1]) (int32 [N + 1] on the
    device); s0 and the returned final states are [N, H, dk, dv]."""
    if q.dtype not in _DT:
        raise ValueError("q must be float32 or bfloat16")
    B, T, H, dk = q.shape
    if B != 1:
        raise ValueError("packed sequences take q as [1, T, H, dk]")
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    _check(cu_seqlens, "cu_seqlens", torch.int32, dev, [tuple(cu_seqlens.shape)])
    if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
        raise ValueError("cu_seqlens must be int32 [N + 1], N >= 1")
    N = cu_seqlens.numel() - 1
    _check(q, "q", dt, dev, [(B, T, H, dk)])
    _check(k, "k", dt, dev, [(B, T, H, dk)])
    _check(v, "v", dt, dev, [(B, T, H, dv)])
    _check(a, "a", dt, dev, [(B, T, H, dk), (B, T, H)])
    _check(b, "b", dt, dev, [(B, T, H, dk), (B, T, H)])
    _check(w, "w", dt, dev, [(B, T, H, dv), (B, T, H)])
    _check(s0, "s0", torch.float32, dev, [(N, H, dk, dv)])
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=dt, device=dev)
    _check(out, "out", dt, dev, [(B, T, H, dv)])
    if s_final is None and return_final:
        s_final = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
    _check(s_final, "s_final", torch.float32, dev, [(N, H, dk, dv)])
    desc = desc_for(q, v, a, b, w, chunk, fg2=fg2)
    st = _lib.forward_varlen(desc, _ptr(cu_seqlens), N, _ptr(q), _ptr(k), _ptr(v), _ptr(a),
                             _ptr(b), _ptr(w), _ptr(s0), _ptr(out), _ptr(s_final), 0, 0,
                             _stream_handle(stream))
    if st != _lib.OK:
        raise _lib.GdrError(st, "gdr_forward_varlen")
    return out, s_final


def decode_step_paged(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                      a: Optional[torch.Tensor], b: Optional[torch.Tensor],
                      w: Optional[torch.Tensor], pool: torch.Tensor, slot: torch.Tensor, *,
                      out: Optional[torch.Tensor] = None, stream=None,
                      fg2: bool = False) -> torch.Tensor:
    """One decode step over a state pool [n_slots, H, dk, dv] float32: batch
    entry b updates pool[slot[b]] in place (slot int32 [B], distinct entries).
    Returns o [B, H, dv]; an out-of-range slot is skipped and reported by
    last_device_error() as ERR_INVALID_ARG."""
    if q.dtype not in _DT:
        raise ValueError("q must be float32 or bfloat16")
    B, H, dk = q.shape
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    _check(q, "q", dt, dev, [(B, H, dk)])
    _check(k, "k", dt, dev, [(B, H, dk)])
    _check(v, "v", dt, dev, [(B, H, dv)])
    _check(a, "a", dt, dev, [(B, H, dk), (B, H)])
    _check(b, "b", dt, dev, [(B, H, dk), (B, H)])
    _check(w, "w", dt, dev, [(B, H, dv), (B, H)])
    if pool.dim() != 4 or tuple(pool.shape[1:]) != (H, dk, dv):
        raise ValueError("pool must be [n_slots, %d, %d, %d]" % (H, dk, dv))
    _check(pool, "pool", torch.float32, dev, [tuple(pool.shape)])
    _check(slot, "slot", torch.int32, dev, [(B,)])
    if out is None:
        out = torch.empty((B, H, dv), dtype=dt, device=dev)
    _check(out, "out", dt, dev, [(B, H, dv)])
    desc = desc_for(q, v, a, b, w, decode=True, fg2=fg2)
    st = _lib.decode_step_paged(desc, _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(w),
                                _ptr(pool), _ptr(slot), pool.shape[0], _ptr(out),
                                _stream_handle(stream))
    if st != _lib.OK:
        raise _lib.GdrError(st, "gdr_decode_step_paged")
    return out


def forward_fg2(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, alpha: torch.Tensor,
                beta_k: torch.Tensor, beta_v: Optional[torch.Tensor] = None,
                s0: Optional[torch.Tensor] = None, **kw):
    """FG^2-GDN prefill (beta_v None: one beta for both, the symmetric form)
    or FG^2-GDN+ (separate beta_k, beta_v); alpha the per-channel (or scalar)
    decay.  Same kernels as forward_chunked."""
    return forward_chunked(q, k, v, alpha, beta_k, beta_k if beta_v is None else beta_v, s0,
                           fg2=True, **kw)


def decode_step_fg2(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, alpha: torch.Tensor,
                    beta_k: torch.Tensor, beta_v: Optional[torch.Tensor],
                    state: torch.Tensor, **kw) -> torch.Tensor:
    """One FG^2-GDN(+) decode step; `state` updated in place."""
    return decode_step(q, k, v, alpha, beta_k, beta_k if beta_v is None else beta_v, state,
                       fg2=True, **kw)


def last_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error status."""
    return _lib.last_device_error(_stream_handle(stream))


def test_skip_signal(enable: bool = True) -> None:
    """Test hook (gdr_test_skip_signal): the next bf16 tensor-core prefill
    launch leaves out one completion signal, so its bounded wait runs out and
    the launch ends with GDR_ERR_TIMEOUT in the device error word."""
    _lib.load().gdr_test_skip_signal(1 if enable else 0)


Desc = _lib.GdrDesc


# ------------------------------------------------- sequence-parallel prefill

def _desc_dk128(q, v, a, b, w, fg2):
    if q.shape[-1] != 128 or v.shape[-1] != 128:
        raise ValueError("segmented prefill needs dk = dv = 128")
    return desc_for(q, v, a, b, w, 64 if q.dtype == torch.bfloat16 else 32, fg2=fg2)


def forward_segmented(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                      a: Optional[torch.Tensor] = None, b: Optional[torch.Tensor] = None,
                      w: Optional[torch.Tensor] = None, s0: Optional[torch.Tensor] = None,
                      *, n_segments: int, out: Optional[torch.Tensor] = None,
                      s_final: Optional[torch.Tensor] = None, stream=None,
                      fg2: bool = False) -> Tuple[torch.Tensor, torch.Tensor]:
    """The prefill with every sequence split into n_segments segments that run
    side by side on this GPU (their affine maps, a scan, a second pass).
    Same arguments and results as forward_chunked; dk = dv = 128."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    for t, n, shp in ((q, "q", [(B, T, H, dk)]), (k, "k", [(B, T, H, dk)]),
                      (v, "v", [(B, T, H, dv)]), (a, "a", [(B, T, H, dk), (B, T, H)]),
                      (b, "b", [(B, T, H, dk), (B, T, H)]), (w, "w", [(B, T, H, dv), (B, T, H)])):
        _check(t, n, dt, dev, shp)
    _check(s0, "s0", torch.float32, dev, [(B, H, dk, dv)])
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=dt, device=dev)
    _check(out, "out", dt, dev, [(B, T, H, dv)])
    if s_final is None:
        s_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    _check(s_final, "s_final", torch.float32, dev, [(B, H, dk, dv)])
    desc = _desc_dk128(q, v, a, b, w, fg2)
    need = _lib.segmented_workspace_size(desc, n_segments)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    st = _lib.forward_segmented(desc, int(n_segments), _ptr(q), _ptr(k), _ptr(v), _ptr(a),
                                _ptr(b), _ptr(w), _ptr(s0), _ptr(out), _ptr(s_final), _ptr(ws),
                                need, _stream_handle(stream))
    if st != _lib.OK:
        raise _lib.GdrError(st, "gdr_forward_segmented")
    return out, s_final


def segment_maps(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                 a: Optional[torch.Tensor] = None, b: Optional[torch.Tensor] = None,
                 w: Optional[torch.Tensor] = None, *, stream=None,
                 fg2: bool = False) -> Tuple[torch.Tensor, torch.Tensor]:
    """Affine map of one segment per (batch, head): the state after the
    segment is M S_in + N.  Returns M [B, H, dk, dk] and N [B, H, dk, dv]
    (float32); dk = dv = 128."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    desc = _desc_dk128(q, v, a, b, w, fg2)
    m = torch.empty((B, H, dk, dk), dtype=torch.float32, device=q.device)
    n = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    need = _lib.segment_maps_workspace_size(desc)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    st = _lib.segment_maps(desc, _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(w), _ptr(m),
                           _ptr(n), _ptr(ws), need, _stream_handle(stream))
    if st != _lib.OK:
        raise _lib.GdrError(st, "gdr_segment_maps")
    return m, n


def segment_scan(m: torch.Tensor, n: torch.Tensor, s0: Optional[torch.Tensor] = None, *,
                 stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Start state of every segment and the final state from the maps of P
    consecutive segments, m [P, B, H, dk, dk] and n [P, B, H, dk, dv] (segment
    order first), starting from s0 [B, H, dk, dv] (None: zeros).  Returns
    (s_start [P, B, H, dk, dv], s_final [B, H, dk, dv])."""
    P, B, H, dk, _ = m.shape
    dv = n.shape[-1]
    dev = m.device
    _check(m, "m", torch.float32, dev, [(P, B, H, dk, dk)])
    _check(n, "n", torch.float32, dev, [(P, B, H, dk, dv)])
    _check(s0, "s0", torch.float32, dev, [(B, H, dk, dv)])
    s_start = torch.empty((P, B, H, dk, dv), dtype=torch.float32, device=dev)
    s_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    st = _lib.segment_scan(P, B, H, dk, dv, B * H, H, _ptr(m), _ptr(n), _ptr(s0), _ptr(s_start),
                           _ptr(s_final), _stream_handle(stream))
    if st != _lib.OK:
        raise _lib.GdrError(st, "gdr_segment_scan")
    return s_start, s_final
