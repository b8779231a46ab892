"""The multi-GPU path on the CPU: two ranks over gloo.

The benchmark runs one independent replica per GPU: each rank draws its own
seeded inputs, the slowest rank's device time decides the job's time, and
the job's throughput counts every rank's work.  These tests run that
scaffolding (exact_io_aware_73_b200.replicas) with world size 2 on gloo,
plus the reference arm of bench.py under torchrun, where only rank 0 works.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    from exact_io_aware_73_b200 import replicas as R
    from exact_io_aware_73_b200 import workloads as W
    w_, r_, l_ = R.env_ranks()
    R.init("gloo", w_, timeout_s=60)
    R.barrier(w_)
    # rank-dependent "device times": the job time must be the slowest
    local_ms = 10.0 + 5.0 * rank
    job_ms = R.max_over_ranks(local_ms, w_)
    wl = W.shape_case(1, 2, 64, 64, False, seed=R.rank_seed(500, rank))
    q, _, _ = W.make_qkv(wl)
    tput = R.job_throughput(1000.0, w_, job_ms * 1e-3)
    R.barrier(w_)
    R.finish(w_)
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"world": w_, "rank": r_, "local": l_, "job_ms": job_ms,
                   "seed": R.rank_seed(500, rank), "q_sum": float(q.float().sum()),
                   "tput": tput}, f)


def test_two_gloo_ranks_share_max_time_and_draw_distinct_inputs(tmp_path):
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, 2, port, str(tmp_path)))
             for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    assert [r["rank"] for r in res] == [0, 1]
    assert all(r["world"] == 2 for r in res)
    # both ranks agree on the slowest rank's time
    assert res[0]["job_ms"] == res[1]["job_ms"] == 15.0
    # whole-job throughput = both ranks' work over the slowest time
    assert res[0]["tput"] == pytest.approx(2 * 1000.0 / 0.015)
    # independent replicas: distinct seeds, distinct inputs
    assert res[0]["seed"] != res[1]["seed"]
    assert res[0]["q_sum"] != res[1]["q_sum"]


def test_single_rank_needs_no_process_group():
    from exact_io_aware_73_b200 import replicas as R
    R.init("gloo", 1)
    assert not torch.distributed.is_initialized()
    assert R.max_over_ranks(3.5, 1) == 3.5
    assert R.job_throughput(10.0, 1, 2.0) == 5.0


def test_reference_arm_under_torchrun_prints_on_rank0_only(tmp_path):
    """bench.py --impl reference with two CPU ranks: rank 0 times the oracle
    and prints one JSON line, rank 1 exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           "--nproc-per-node=2", "--master-addr=127.0.0.1",
           f"--master-port={port}", os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup",
           "3", "--workload", "small_b1h1n256d64", "--cpu-budget-s", "0.3"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=300,
                         cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["value"] > 0


# --------------------------------------------------------------------------
# one problem split by heads over ranks (bench.py --split heads)
# --------------------------------------------------------------------------

def test_head_shard_tiles_every_head_exactly_once():
    from exact_io_aware_73_b200 import replicas as R
    for bh in (1, 2, 5, 12, 32, 48, 97):
        for world in (1, 2, 3, 4, 8):
            ranges = [R.head_shard(bh, world, r) for r in range(world)]
            covered = [h for h0, n in ranges for h in range(h0, h0 + n)]
            assert covered == list(range(bh)), (bh, world, ranges)
            counts = [n for _, n in ranges]
            assert max(counts) - min(counts) <= 1


def _head_worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import numpy as np
    import oracle
    from exact_io_aware_73_b200 import replicas as R
    from exact_io_aware_73_b200 import workloads as W
    R.init("gloo", world, timeout_s=60)
    # every rank draws the same problem and computes its own range of heads;
    # the oracle stands in for the kernel (each head is computed alone)
    w = W.shape_case(2, 3, 50, 64, True, seed=321)
    f = [oracle.bf16_bits_to_f64(oracle.bf16_bits(t)) for t in W.make_qkv(w)]
    h0, nh = R.head_shard(w.B * w.H, world, rank)
    part = [x.reshape(w.B * w.H, w.N, w.d)[h0:h0 + nh][None] for x in f]
    O, L = oracle.attention(*part, w.causal, w.scale)
    # test-side gather of the shards (the benchmark itself exchanges nothing)
    outs = [None] * world
    torch.distributed.all_gather_object(outs, (h0, nh, O[0], L[0]))
    R.finish(world)
    if rank == 0:
        O_all = np.concatenate([o for _, _, o, _ in outs])
        L_all = np.concatenate([l for _, _, _, l in outs])
        O_ref, L_ref = oracle.attention(*f, w.causal, w.scale)
        np.save(os.path.join(out_dir, "o.npy"), O_all)
        np.save(os.path.join(out_dir, "o_ref.npy"), O_ref.reshape(O_all.shape))
        np.save(os.path.join(out_dir, "l.npy"), L_all)
        np.save(os.path.join(out_dir, "l_ref.npy"), L_ref.reshape(L_all.shape))


@pytest.mark.parametrize("world", [2, 3])
def test_heads_split_over_gloo_ranks_reassemble_the_whole_problem(tmp_path, world):
    import numpy as np
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_head_worker, args=(r, world, port, str(tmp_path)))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    o, o_ref = np.load(tmp_path / "o.npy"), np.load(tmp_path / "o_ref.npy")
    l, l_ref = np.load(tmp_path / "l.npy"), np.load(tmp_path / "l_ref.npy")
    assert np.array_equal(o, o_ref) and np.array_equal(l, l_ref)
