"""Multi-process host logic of bench.py on CPU (gloo, world size 2).

The path partitions over independent sequences with no data-path collective;
what crosses ranks is the barrier around the timed region and the max over
ranks of the timed total.  These run without a GPU.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    ws, r, local = bench.dist_setup()
    assert ws == world and r == rank
    bench.barrier(ws)
    got = bench.max_over_ranks(10.0 + rank, ws)
    import torch.distributed as dist
    dist.destroy_process_group()
    q.put((rank, got))


def test_max_over_ranks_and_barrier_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res == {0: 11.0, 1: 11.0}


def test_reference_arm_under_torchrun_only_rank0_prints():
    """`bench.py --impl reference` under two ranks: rank 0 runs the oracle on a
    bounded sample and prints one JSON line; rank 1 exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    import json
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle"
    # tokens of the whole workload: a 16-of-96-head sample of 4096 tokens of the sweep counts
    # as 4096 * 16 / 96 tokens
    assert abs(d["value"] * d["ms_per_step"] * 1e-3 - 4096 * 16 / 96) < 1e-6 * 4096
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["host_cores"] >= d["cpu_baseline"]["cores"]
    assert "T=65536" in d["config"]["workload"]


def _cp_worker(rank, world, port, q, cuts):
    """One rank of the context-parallel forward on CPU (gloo).  The three library calls are
    replaced by FP64 oracle functions (the exchange and the ordering are what runs here)."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch
    import torch.distributed as dist
    import kda_workloads as W
    import oracle
    from gated_delta_rule_73_b200.context_parallel import chunk_fwd_context_parallel

    class OracleOps:
        def segment_pair(self, q, k, v, g, beta):
            a = [x.double().numpy() for x in (q, k, v, g, beta)]
            M = oracle.transition_product_np(a[1], a[3], a[4])
            Bm = oracle.recurrence_c(*a, None)[1]
            return torch.from_numpy(M), torch.from_numpy(Bm)

        def affine_combine(self, Ms, Bs, n, S0):
            s0 = None if S0 is None else S0.double().numpy()
            return torch.from_numpy(oracle.affine_combine_np(Ms[:n].numpy(), Bs[:n].numpy(), s0))

        def segment_forward(self, q, k, v, g, beta, S0):
            a = [x.double().numpy() for x in (q, k, v, g, beta)]
            o, s = oracle.recurrence_c(*a, S0.numpy())
            return torch.from_numpy(o), torch.from_numpy(s)

    dist.init_process_group("gloo")
    x = W.chunk_inputs(2, cuts[-1], 2, 8, 4, dtype=torch.float32, seed=5)
    a, b = cuts[rank], cuts[rank + 1]
    seg = [x[n][:, a:b].contiguous() for n in ("q", "k", "v", "g", "beta")]
    out, S_T, S_start = chunk_fwd_context_parallel(*seg, x["S0"].double(), ops=OracleOps())
    dist.destroy_process_group()
    q.put((rank, out.numpy(), S_T.numpy(), S_start.numpy()))


@pytest.mark.parametrize("cuts", [[0, 9, 23], [0, 16, 16]], ids=["ragged", "empty-last"])
def test_context_parallel_exchange_gloo(cuts):
    """Two ranks each hold one segment of the same sequences; after the all-gather of the
    segment pairs and the ordered fold, rank r's outputs and start state, and the final
    state on every rank, equal the oracle's run over the whole sequence."""
    import numpy as np
    sys.path.insert(0, ROOT)
    import torch
    import kda_workloads as W
    import oracle
    ctx = mp.get_context("spawn")
    qq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_cp_worker, args=(r, 2, port, qq, cuts)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        r, o, s, s0 = qq.get(timeout=180)
        res[r] = (o, s, s0)
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    x = W.chunk_inputs(2, cuts[-1], 2, 8, 4, dtype=torch.float32, seed=5)
    a = [x[n].double().numpy() for n in ("q", "k", "v", "g", "beta")]
    S0 = x["S0"].double().numpy()
    ref_o, ref_s = oracle.recurrence_c(*a, S0)
    full = np.concatenate([res[0][0], res[1][0]], axis=1)
    assert np.max(np.abs(full - ref_o)) <= 1e-10 * np.max(np.abs(ref_o))
    for r in range(2):
        assert np.max(np.abs(res[r][1] - ref_s)) <= 1e-10 * np.max(np.abs(ref_s))
    start1 = oracle.recurrence_c(*[t[:, :cuts[1]] for t in a], S0)[1]
    assert np.max(np.abs(res[1][2] - start1)) <= 1e-10 * np.max(np.abs(start1))
    assert np.array_equal(res[0][2], S0)
