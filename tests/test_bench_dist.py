"""bench.py's multi-process logic on CPU: world size 2 over gloo.

The layer runs as independent replicas (no data-path collective); what the
benchmark adds for N > 1 is rank/world parsing from the launcher's
environment, barriers around the timed region, the max over ranks of the
device time, and, for the reference arm, rank 0 alone printing one JSON
line. Each is checked here with two spawned processes on 127.0.0.1."""
import json
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, outdir):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import argparse
    import contextlib
    import io

    import bench
    args = argparse.Namespace(gpus=world, steps=1, warmup=0, workload="decode", impl="reference",
                              cpu_seconds=0.5, no_cpu_baseline=False, copies=1)
    w, r, local = bench.setup_dist(args)
    res = {"world": w, "rank": r, "local": local}
    res["max"] = bench.dist_max(float(10 + r), w)
    bench.barrier(w)
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(args, w, r)
    res["printed"] = buf.getvalue()
    bench.barrier(w)
    import torch.distributed as dist
    dist.destroy_process_group()
    with open(os.path.join(outdir, f"rank{rank}.json"), "w") as fh:
        json.dump(res, fh)


def test_two_rank_replicas_over_gloo(tmp_path):
    import torch.multiprocessing as mp
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    r0 = json.load(open(tmp_path / "rank0.json"))
    r1 = json.load(open(tmp_path / "rank1.json"))
    assert (r0["world"], r0["rank"], r1["world"], r1["rank"]) == (2, 0, 2, 1)
    assert r0["max"] == r1["max"] == 11.0          # max over ranks, seen by both
    assert r1["printed"] == ""                      # only rank 0 reports
    line = json.loads(r0["printed"].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["unit"] == "tokens/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
