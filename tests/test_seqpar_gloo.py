"""The sequence-sharded ring (exact_io_aware_73_b200.seqpar) on the CPU:
world sizes 2 and 3 over gloo.

Each rank holds one contiguous shard of Q, K, V; the K/V shards travel
around the ring while each rank attends its queries to the shard it holds
and folds the partial (O, lse) into an accumulator.  The block attention and
the merge are injected here as fp64 CPU stand-ins (the fp64 oracle for a
block, the log-sum-exp merge written out in numpy), so that the test checks
the distributed part: the schedule (which shard at which step, which blocks
are skipped under the causal mask) and the exchange (every rank sees every
shard once).  The merged result must equal the oracle's attention over the
whole sequence for the rank's rows.
"""
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _CpuOps:
    """fp64 stand-ins: the oracle for a block, the log-sum-exp merge in
    torch (the same fold the kernel's epilogue performs)."""

    def __init__(self, oracle):
        self.oracle = oracle

    def block(self, q, k, v, causal, scale, state, i, n):
        import torch
        O, lse = self.oracle.attention(q.double().numpy(), k.double().numpy(),
                                       v.double().numpy(), causal, scale, threads=1)
        O, lse = torch.from_numpy(O), torch.from_numpy(lse)
        if i == 0:
            state["o"], state["lse"] = O, lse
        else:
            m = torch.maximum(state["lse"], lse)
            wa, wp = torch.exp(state["lse"] - m), torch.exp(lse - m)
            t = wa + wp
            state["o"] = (wa / t)[..., None] * state["o"] + (wp / t)[..., None] * O
            state["lse"] = m + torch.log(t)
        return (state["o"], state["lse"]) if i == n - 1 else None


def _worker(rank, world, port, causal, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch
    import torch.distributed as dist
    import oracle
    from exact_io_aware_73_b200 import seqpar
    from exact_io_aware_73_b200 import workloads as W
    dist.init_process_group("gloo", rank=rank, world_size=world)
    N = 40 * world
    w = W.shape_case(1, 2, N, 16, causal, seed=31)
    q, k, v = (t.double() for t in W.make_qkv(w))
    n = N // world
    sl = slice(rank * n, (rank + 1) * n)
    stats = seqpar.RingStats()
    O, lse = seqpar.ring_attention(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(),
                                   v[:, :, sl].contiguous(), causal, w.scale,
                                   ops=_CpuOps(oracle), stats=stats)
    Of, lf = oracle.attention(q.numpy(), k.numpy(), v.numpy(), causal, w.scale, threads=1)
    err_o = float(np.abs(O.numpy() - Of[:, :, sl]).max())
    err_l = float(np.abs(lse.numpy() - lf[:, :, sl]).max())
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
        json.dump({"err_o": err_o, "err_l": err_l, "blocks": stats.blocks,
                   "skipped": stats.skipped, "steps": stats.steps,
                   "bytes": stats.bytes_sent}, f)


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_over_gloo_equals_full_attention(tmp_path, world, causal):
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, causal, str(tmp_path)))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    for r in range(world):
        res = json.load(open(tmp_path / f"r{r}.json"))
        assert res["err_o"] <= 1e-12 and res["err_l"] <= 1e-12, res
        assert res["steps"] == world
        # causal: rank r attends shards 0..r (r + 1 blocks), skips the rest
        assert res["blocks"] == (r + 1 if causal else world)
        assert res["skipped"] == world - res["blocks"]
        # every step but the last passes a K/V pair (2 x 1 x 2 x 40 x 16 doubles) on
        assert res["bytes"] == (world - 1) * 2 * 2 * 40 * 16 * 8


def test_shard_plan_visits_every_shard_once():
    sys.path.insert(0, ROOT)
    from exact_io_aware_73_b200 import seqpar
    for world in (1, 2, 5):
        for rank in range(world):
            for causal in (False, True):
                plan = seqpar.shard_plan(rank, world, causal)
                assert sorted(s for s, _ in plan) == list(range(world))
                assert plan[0] == (rank, "causal" if causal else "full")
                for s, how in plan:
                    assert (how is None) == (causal and s > rank)
