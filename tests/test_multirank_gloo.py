"""Multi-rank host logic on the CPU with the gloo backend (world size 2).

The routing path shards by tokens: every rank routes its own tokens and no
data-path collective is needed.  These tests check, with the CPU oracle, that
per-token results do not depend on the sharding, and that the benchmark's
aggregation (max over ranks of the timed interval, whole-job tokens/s) works
across processes."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import oracle as O
        from combine_moe_topk_gate_b200.workloads import Workload, make_inputs
        # aggregation: the max over ranks and the whole-job rate
        local_ms = 10.0 + 5.0 * rank
        m = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        rate = bench.whole_job_rate(100, world, 4, m)
        # sharded routing of one batch: each rank takes a contiguous token shard
        w = Workload("shard", 96, 256, 32, 4, 4, "sigmoid_group", "fp8", "random", 4, 2, 2)
        inp = make_inputs(w, 7)
        lo, hi = rank * w.N // world, (rank + 1) * w.N // world
        idx, wts = O.topk_gate(inp.logits[lo:hi].numpy(), w.k, w.gate_kind, w.n_groups, w.topk_groups,
                               w.group_topn)
        L = O.get_layout(idx, w.E, w.R)
        x = inp.x[lo:hi].contiguous().view(torch.int16).numpy().view(np.uint16)
        recv, scale, _ = O.dispatch(x, L.token_slot, w.dtype_code)
        # expert outputs of this shard: the shard's own tokens' rows of the seeded y
        yb = inp.y.view(torch.int16).numpy().view(np.uint16).reshape(w.N, w.k, w.H)[lo:hi]
        y_local = np.empty(((hi - lo) * w.k, w.H), np.uint16)
        y_local[L.token_slot.reshape(-1)] = yb.reshape(-1, w.H)
        out, _ = O.combine(y_local, L.token_slot, wts)
        # gloo has no 16-bit all_gather: carry the bf16 bit patterns as int32
        outs = [torch.empty((hi - lo, w.H), dtype=torch.int32) for _ in range(world)]
        dist.all_gather(outs, torch.from_numpy(out.astype(np.int32)))
        idxs = [torch.empty((hi - lo, w.k), dtype=torch.int32) for _ in range(world)]
        dist.all_gather(idxs, torch.from_numpy(idx))
        if rank == 0:
            q.put(dict(m=m, rate=rate, out=torch.cat(outs).numpy().astype(np.uint16),
                       idx=torch.cat(idxs).numpy()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_tokens_and_aggregate():
    import oracle as O
    from combine_moe_topk_gate_b200.workloads import Workload, make_inputs
    O.build()
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res["m"] == 15.0
    assert res["rate"] == pytest.approx(100 * 2 * 4 / 15e-3)
    # the unsharded batch gives the same per-token routing and outputs
    w = Workload("shard", 96, 256, 32, 4, 4, "sigmoid_group", "fp8", "random", 4, 2, 2)
    inp = make_inputs(w, 7)
    idx, wts = O.topk_gate(inp.logits.numpy(), w.k, w.gate_kind, w.n_groups, w.topk_groups, w.group_topn)
    L = O.get_layout(idx, w.E, w.R)
    yb = inp.y.view(torch.int16).numpy().view(np.uint16).reshape(w.N * w.k, w.H)
    y_full = np.empty_like(yb)
    y_full[L.token_slot.reshape(-1)] = yb
    out, _ = O.combine(y_full, L.token_slot, wts)
    assert np.array_equal(res["idx"], idx)
    assert np.array_equal(res["out"], out)


def test_reference_arm_rank0_prints_other_ranks_exit_quietly():
    """The comparison arm (the CPU oracle) under a 2-rank launch: rank 0 prints
    the one JSON line, rank 1 exits 0 without work or output."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--workload", "tiny",
           "--steps", "2", "--warmup", "3"]
    outs = []
    for rank in (0, 1):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
        r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env, cwd=root)
        assert r.returncode == 0, r.stderr[-2000:]
        outs.append(r.stdout.strip())
    line = json.loads(outs[0].splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["host_cores"] == os.cpu_count()
    assert outs[1] == ""
    # the comparison arm describes the workload exactly as our arm does
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_cfg", os.path.join(root, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    from combine_moe_topk_gate_b200.workloads import WORKLOADS as W
    assert line["config"] == bench.config_of(W["tiny"], 2)
    assert line["metric"] == bench.METRIC and line["unit"] == "tokens/s" and line["higher_is_better"] is True
