"""The N > 1 bench path on CPU: two processes under gloo (the GPU runs use NCCL with the same calls).

Replicas only: the process group carries the barrier and the max-over-ranks timing, nothing of the layer.
Each rank checks that the max over ranks is the largest rank's value, that every rank passes the barrier,
that the reference arm prints on rank 0 only, and that ranks build different decode layers (weak scaling).
"""
import io
import json
import os
import socket
import sys
import contextlib

import pytest

torch = pytest.importorskip("torch")
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, ws, port, outdir):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(ws), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "CUDA_VISIBLE_DEVICES": ""})
    sys.path.insert(0, ROOT)
    import bench
    from bit_quantized_moe_02_b200 import synth
    import torch.distributed as dist

    got_ws, got_rank, _ = bench.dist_setup()
    res = {"ws": got_ws, "rank": got_rank, "backend": dist.get_backend()}
    res["max"] = bench.max_over_ranks(float(rank + 1), got_ws)
    bench.barrier(got_ws)
    # the reference arm prints its JSON line on rank 0 only; other ranks return without work
    buf = io.StringIO()
    if rank != 0:
        with contextlib.redirect_stdout(buf):
            bench.run_reference(type("A", (), {"steps": 1, "warmup": 0, "gpus": ws})(), got_ws, got_rank)
    res["ref_output"] = buf.getvalue()
    # replicas hold different layers (seeded by rank), so per-GPU work is fixed as N grows
    wl = synth.WORKLOADS["tiny"]
    res["wr0"] = float(synth.make_layer(wl, layer=16 * rank).wr.view("float16")[0, 0])
    bench.barrier(got_ws)
    dist.destroy_process_group()
    with open(os.path.join(outdir, "r%d.json" % rank), "w") as f:
        json.dump(res, f)


def test_two_rank_gloo_barrier_and_max(tmp_path):
    ws, port = 2, _free_port()
    mp.spawn(_worker, args=(ws, port, str(tmp_path)), nprocs=ws, join=True)
    res = [json.load(open(tmp_path / ("r%d.json" % r))) for r in range(ws)]
    assert [r["rank"] for r in res] == [0, 1]
    assert all(r["ws"] == 2 and r["backend"] == "gloo" for r in res)
    assert all(r["max"] == 2.0 for r in res)
    assert res[1]["ref_output"] == ""
    assert res[0]["wr0"] != res[1]["wr0"]
