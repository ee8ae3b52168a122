"""The sequence-parallel exchange on world-size-2 gloo process groups, without
a GPU: each rank holds one segment of a sequence, the segments' affine maps
are all-gathered, every rank scans them for its start state and runs its
segment from there (gated_delta_rule_154_b200.seqpar).  The three compute
steps are supplied here by the float64 oracle (the library's CUDA calls take
their place on GPUs), so what this checks is the plumbing: gather order,
rank indexing, the scan's use of the gathered maps and s0, and that every
rank ends with the whole sequence's final state."""

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from gated_delta_rule_154_b200 import seqpar  # noqa: E402

D, T, B, H = 8, 96, 2, 2


def _inputs(seed):
    rng = np.random.default_rng(seed)
    unit = lambda x: x / np.linalg.norm(x, axis=-1, keepdims=True)
    sig = lambda x: 1 / (1 + np.exp(-x))
    q = unit(rng.standard_normal((B, T, H, D)))
    k = unit(rng.standard_normal((B, T, H, D)))
    v = rng.standard_normal((B, T, H, D))
    a = np.exp(-np.logaddexp(0.0, rng.normal(-4.0, 1.0, (B, T, H, D))))
    b = sig(rng.standard_normal((B, T, H, D)))
    w = sig(rng.standard_normal((B, T, H, D)))
    s0 = rng.normal(0.0, 0.1, (B, H, D, D))
    f32 = lambda z: z.astype(np.float32)
    return [f32(z) for z in (q, k, v, a, b, w)] + [s0]


class OracleOps:
    """The three compute steps on the CPU, from the float64 oracle."""

    @staticmethod
    def maps(q, k, v, a, b, w, fg2=False):
        x = [t.numpy() for t in (q, k, v, a, b, w)]
        eye = np.broadcast_to(np.eye(D), (B, H, D, D)).copy()
        _, M = oracle.forward(x[0], x[1], np.zeros_like(x[2]), x[3], x[4], x[5], eye,
                              want_o=False)
        _, N = oracle.forward(*x, None, want_o=False)
        return torch.from_numpy(M), torch.from_numpy(N)

    @staticmethod
    def scan(m_all, n_all, s0):
        S = np.zeros((B, H, D, D)) if s0 is None else s0.numpy().copy()
        starts = []
        for p in range(m_all.shape[0]):
            starts.append(S.copy())
            S = np.einsum("bhik,bhkj->bhij", m_all[p].numpy(), S) + n_all[p].numpy()
        return torch.from_numpy(np.stack(starts)), torch.from_numpy(S)

    @staticmethod
    def forward(q, k, v, a, b, w, s_start, fg2=False):
        x = [t.numpy() for t in (q, k, v, a, b, w)]
        o, _ = oracle.forward(*x, s_start.numpy())
        return torch.from_numpy(o)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, seed, out_q):
    import datetime
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    x = _inputs(seed)
    L = T // world
    seg = [torch.from_numpy(np.ascontiguousarray(z[:, rank * L:(rank + 1) * L])) for z in x[:6]]
    o, s_final = seqpar.prefill(*seg, torch.from_numpy(x[6]), ops=OracleOps)
    out_q.put((rank, o.numpy(), s_final.numpy()))
    dist.destroy_process_group()


@pytest.mark.parametrize("seed", [1, 2])
def test_two_ranks_match_the_whole_sequence(seed):
    world = 2
    ctx = mp.get_context("spawn")
    out_q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, seed, out_q))
             for r in range(world)]
    for p in procs:
        p.start()
    got = sorted(out_q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    x = _inputs(seed)
    o_ref, s_ref = oracle.forward(*x[:6], x[6])
    o = np.concatenate([g[1] for g in got], axis=1)
    scale_o, scale_s = np.max(np.abs(o_ref)), np.max(np.abs(s_ref))
    assert np.max(np.abs(o - o_ref)) <= 1e-12 * scale_o
    for g in got:   # every rank has the whole sequence's final state
        assert np.max(np.abs(g[2] - s_ref)) <= 1e-12 * scale_s
