"""The multi-process (N > 1) host paths on CPU with world size 2: every rank
runs its own replica of the workload, the step time is the maximum over ranks
(gloo here, NCCL on GPUs), and under torchrun rank 0 alone prints the bench
line.  The path shards into independent (sequence, head) units, so there is
no data-path collective to test."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        got = bench.max_over_ranks(1.5 * (rank + 1), dist, torch, "cpu")
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(repr(got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    vals = [float(open(tmp_path / f"rank{r}.txt").read()) for r in range(2)]
    assert vals == [3.0, 3.0]


def test_max_over_ranks_without_a_group_is_the_value():
    import torch
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.5, None, torch, "cpu") == 2.5


def test_reference_arm_under_torchrun_world2():
    """bench.py --impl reference launched like the driver's N = 2 run: rank 0
    times the oracle and prints one JSON line, rank 1 exits 0 without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
           "--ref-step-seconds", "0.5"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT,
                       env=dict(os.environ, OMP_NUM_THREADS="2"))
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


def _ring_main(rank, world, port, out_dir, causal):
    import datetime

    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from flashattention_attention_b200 import ring
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        B, hq, hkv, S, d = 2, 4, 2, 24 * world, 16
        rng = np.random.default_rng(7)
        q = torch.from_numpy(rng.standard_normal((B * hq, S, d)))
        k = torch.from_numpy(rng.standard_normal((B * hkv, S, d)))
        v = torch.from_numpy(rng.standard_normal((B * hkv, S, d)))
        blk = S // world
        sl = slice(rank * blk, (rank + 1) * blk)

        calls = []

        def step(q, k, v, acc, *, hq, hkv, causal, scale, first, last, epilogue):
            calls.append((first, last, acc is None))
            o, lse = oracle.attention_lse(q.numpy(), k.numpy(), v.numpy(), hq=hq, hkv=hkv, causal=causal, scale=scale)
            if acc is not None:
                o, lse = oracle.merge(acc[0], acc[1], o, lse)
            out = None
            if last:
                out = o.copy()
                for op, val in epilogue:
                    out = out * val if op == "mul" else out + val
                out = torch.from_numpy(out)
            return (o, lse), out

        out = ring.ring_attention_fwd(q[:, sl].contiguous(), k[:, sl].contiguous(), v[:, sl].contiguous(), hq=hq,
                                      hkv=hkv, causal=causal, epilogue=[("mul", 2.0), ("add", 0.5)],
                                      group=dist.group.WORLD, step=step)
        n = rank + 1 if causal else world
        assert calls == [(c == 0, c == n - 1, c == 0) for c in range(n)], calls
        ref = oracle.attention(q.numpy(), k.numpy(), v.numpy(), hq=hq, hkv=hkv, causal=causal,
                               epilogue=[("mul", 2.0), ("add", 0.5)])[:, sl]
        err = float(np.abs(out.numpy() - ref).max())
        with open(os.path.join(out_dir, f"ring{rank}.txt"), "w") as f:
            f.write(repr(err))
    finally:
        dist.destroy_process_group()


def test_ring_schedule_pairs_every_send_with_a_receive():
    """Every transfer of ring_schedule has its receive on the next rank, and
    rank r attends to exactly blocks 0..r (causal) or all blocks, each once."""
    sys.path.insert(0, ROOT)
    from flashattention_attention_b200.ring import ring_schedule
    for world in range(1, 9):
        for causal in (False, True):
            held = list(range(world))  # block held by each rank
            seen = [[] for _ in range(world)]
            for s in range(world):
                for r in range(world):
                    seen[r].append(held[r])
                sched = [ring_schedule(r, world, causal, s) for r in range(world)]
                for r in range(world):
                    assert sched[r][0] == sched[(r + 1) % world][1], (world, causal, s, r)
                held = [held[(r - 1) % world] if sched[r][1] else held[r] for r in range(world)]
            for r in range(world):
                want = list(range(r + 1)) if causal else list(range(world))
                got = [b for b in seen[r][:len(want)]]
                assert sorted(got) == want, (world, causal, r, seen[r])
            if causal and world > 1:
                n_sends = sum(ring_schedule(r, world, True, s)[0] for r in range(world) for s in range(world))
                assert n_sends == world * (world - 1) // 2


@pytest.mark.parametrize("world,causal", [(2, True), (2, False), (3, True), (4, True)])
def test_ring_schedule_gloo(tmp_path, world, causal):
    """The ring schedule of ring_attention_fwd (blocks passed to the next
    rank while each step computes, future blocks skipped under causal
    masking, the diagonal block causal, partial results merged) over gloo
    ranks with the oracle's per-step computations: every rank's block equals
    the oracle's attention over the whole sequence."""
    port = _free_port()
    mp.start_processes(_ring_main, args=(world, port, str(tmp_path), causal), nprocs=world, join=True,
                       start_method="spawn")
    errs = [float(open(tmp_path / f"ring{r}.txt").read()) for r in range(world)]
    assert max(errs) < 1e-12, errs


def test_ring_job_flops_counts_the_whole_band():
    """The N-GPU ring line counts the causal band over all ranks' positions:
    one rank is the single-GPU headline step; N ranks is the same tile rule
    over N * 4096 positions (a triangle of 32 N (32 N + 1) / 2 tiles per
    head plane)."""
    sys.path.insert(0, ROOT)
    import bench
    from flashattention_attention_b200 import inputs
    w = inputs.gqa_causal_prefill()
    assert bench.ring_job_flops(1) == bench.prefill_flops(w)[0]
    for n in (2, 4, 8):
        t = 32 * n
        assert bench.ring_job_flops(n) == 4 * 32 * 4 * 128 * 128 * 128 * (t * (t + 1) // 2)
