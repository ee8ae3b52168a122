"""bench.py's host-side logic without a GPU: the byte and flop counts behind
the roofline, and the multi-rank plumbing (barrier, max over ranks, per-rank
seeds, reference arm on rank 0 only) on world-size-2 gloo process groups."""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from gated_delta_rule_154_b200 import workload as W  # noqa: E402


def test_prefill_bytes_per_token_head():
    wl = W.WORKLOADS["gdn2_bf16"]
    th = wl.B * wl.T * wl.H
    state = 4 * wl.B * wl.H * 128 * 128
    # q, k, v, a, b, w read once (6 x 256 B) + o written once (256 B), s0 and S_T
    assert bench.prefill_bytes(wl) == th * 1792 + 2 * state
    assert bench.prefill_bytes(wl) == 1895825408
    kda = W.WORKLOADS["kda_bf16"]
    # shared scalar beta: q,k,v 768 + vector a 256 + beta 2 + o 256
    assert bench.prefill_bytes(kda) == kda.B * kda.T * kda.H * 1282 + 4 * kda.B * kda.H * 128 * 128


def test_capture_digest_follows_code_not_comments(tmp_path, monkeypatch):
    """The committed ncu counters stay attached to the kernel code they were
    taken from: comments and blank space do not change the digest, code does."""
    src = tmp_path / "k.cu"
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    src.write_text("int f(int x) {  // one\n  return x + 1; /* two */\n}\n")
    d0 = bench.code_digest(["k.cu"])
    src.write_text("// a header\nint f(int x)\n{\n    return x + 1;\n}\n")
    assert bench.code_digest(["k.cu"]) == d0
    src.write_text("int f(int x) { return x + 2; }\n")
    assert bench.code_digest(["k.cu"]) != d0


def test_committed_capture_matches_the_prefill_code():
    traffic, note = bench.measured_traffic()
    assert traffic is not None, note
    # within a few percent of the algorithmic bytes of the bench launch
    assert abs(traffic / bench.prefill_bytes(W.WORKLOADS["gdn2_bf16"]) - 1) < 0.05


def test_decode_bytes_per_head_step():
    wl = W.WORKLOADS["decode_bf16"]
    assert bench.decode_bytes(wl) == wl.B * wl.H * 132864


def test_flops_formula():
    wl = W.WORKLOADS["gdn2_bf16"]
    assert bench.prefill_flops(wl) == wl.B * wl.T * wl.H * (8 * 128 ** 2 + 16 * 64 * 128 + 64 ** 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    r = bench.Ranks(world, device="cpu")
    r.barrier()
    m = r.max(float(10 * rank + 1))
    r.barrier()
    q.put((rank, m, bench.rank_seed(rank)))
    dist.destroy_process_group()


def test_max_over_ranks_and_seeds_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(world))
    assert [g[1] for g in got] == [11.0, 11.0]       # the max over ranks on every rank
    assert [g[2] for g in got] == [0, 1]              # each rank draws its own batch


def test_reference_arm_non_zero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""


@pytest.mark.slow
def test_reference_arm_prints_one_json_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3", "--ref-seconds", "0.5"], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
