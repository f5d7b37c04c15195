"""The multi-GPU path on the CPU: two gloo ranks, no GPU.

On N GPUs the decode step runs as N independent replicas (one process per GPU,
each with its own full batch; the path has no exchange step, so there is no
data-path collective). What the ranks share is host logic, checked here with
world_size 2 on the gloo backend:

* every rank builds the same split plan from the same lengths (the partition is
  a pure function of the lengths and the worker count),
* the step time is the maximum over ranks and every rank sees that maximum,
* the whole-job value counts the bytes of all ranks against that time,
* only rank 0 prints the JSON line, and the reference arm does no work on the
  other ranks.
"""

import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, out_dir):
    sys.path.insert(0, ROOT)
    import bench
    from mla_latent_kv_21_b200 import _lib as L
    import mla_latent_kv_21_b200 as M

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=WORLD)
    res = {}
    # replicas plan identically
    dims = M.dims_for(128, 512, 64, 128, 128, 1, 192 ** -0.5, "bf16", 1)
    lens = [32768, 1000, 65, 4096] * 4
    plan, ws = L.mla_decode_plan_ex(dims, lens, num_sms=148, kernel=L.MLA_KERNEL_TCGEN05,
                                    num_workers=0)
    segs = L.mla_plan_segments(plan)
    L.mla_plan_destroy(plan)
    gathered = [None] * WORLD
    dist.all_gather_object(gathered, (segs, ws))
    res["plans_equal"] = all(g == gathered[0] for g in gathered)
    # max over ranks: rank r timed 10 + r ms
    res["max"] = bench.max_over_ranks(10.0 + rank, dist, "cpu")
    res["value"] = bench.whole_job_value(WORLD, 1.0e9, res["max"])
    # only rank 0 prints
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.emit({"metric": "m", "value": res["value"]}, rank)
    res["printed"] = buf.getvalue()
    # the reference arm returns at once on ranks other than 0
    if rank != 0:
        class A:
            steps = 1
            warmup = 1
        buf = io.StringIO()
        with redirect_stdout(buf):
            r = bench.reference_arm(A(), None, WORLD, rank)
        res["ref_other_rank"] = (r, buf.getvalue())
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


def test_two_gloo_ranks(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(port, str(tmp_path)), nprocs=WORLD, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(WORLD)]
    for r in res:
        assert r["plans_equal"]
        assert r["max"] == pytest.approx(10.0 + WORLD - 1)
        assert r["value"] == pytest.approx(WORLD * 1.0e9 / ((10.0 + WORLD - 1) * 1e-3) / 1e9)
    line = json.loads(res[0]["printed"])
    assert line["value"] == pytest.approx(res[0]["value"])
    assert all(r["printed"] == "" for r in res[1:])
    assert res[1]["ref_other_rank"] == [None, ""]
