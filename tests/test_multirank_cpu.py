"""The N > 1 plumbing of bench.py on the CPU: two ranks over gloo.

Planes are independent, so ranks share no data; the only cross-rank steps
are the barriers around the timed region and the max-over-ranks reduction of
the step time.  The reference arm runs on rank 0 alone and the other ranks
leave without work.  Nothing here touches a GPU.
"""
import contextlib
import io
import json
import os
import socket
import sys
import types

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    from linear_spatial_propagation_line_b200.inputs import WORKLOADS

    r, local, w = bench.dist_init("gloo")
    out = {"rank": r, "local": local, "world": w}
    bench.barrier(w)
    out["max"] = bench.max_over_ranks(1.5 * (r + 1), w, torch.device("cpu"))
    out["config"] = bench.config_dict(WORKLOADS["hires2048x1024_global_bf16"], w)
    bench.dist_close(w)
    # reference arm launched the way torchrun would launch it
    args = types.SimpleNamespace(gpus=w, steps=1, warmup=0)
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(args, WORKLOADS["tiny16_global_f32"])
    out["ref_stdout"] = buf.getvalue()
    q.put(out)


def test_two_gloo_ranks_time_as_max_and_reference_on_rank0_only():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
        assert p.exitcode == 0
    res = sorted([q.get() for _ in range(world)], key=lambda o: o["rank"])
    assert [o["rank"] for o in res] == [0, 1]
    assert all(o["world"] == world for o in res)
    # every rank sees the slowest rank's time
    assert all(o["max"] == pytest.approx(3.0) for o in res)
    cfg = res[0]["config"]
    assert cfg["global_batch"] == 1 * world and cfg["planes_per_gpu"] == 64
    assert "no collective" in cfg["parallelism"]
    # one JSON line from rank 0, nothing from rank 1
    lines = [ln for ln in res[0]["ref_stdout"].splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == world and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert res[1]["ref_stdout"].strip() == ""
