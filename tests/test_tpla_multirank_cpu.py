"""TPLA across GPUs, host side, on two gloo ranks (no GPU).

Each rank of a two-way TPLA group holds one latent shard. What the ranks do on
the host is checked here with world_size 2: the rank-to-group layout bench.py
uses, the per-rank input slicing (layout only), the per-rank plan (a one-shard
plan of half the latent rank on the tensor-core kernel), and the group's sum
through TplaShardPlan.allreduce. The shard outputs are the oracle's (an MLA
decode over the rank's slice), standing in for the GPU kernels; their
all-reduced sum must equal the oracle's TPLA definition over the full inputs,
which pins both the slicing and the exchange step.
"""

import json
import os
import socket
import sys

import numpy as np
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
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import bench
    import mla_latent_kv_21_b200 as M
    from mla_workloads import WORKLOADS, generate, tpla_shard_inputs
    from oracle import mla_oracle

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=WORLD)
    res = {}
    wl = WORKLOADS["tpla_dsv3"]
    tp = wl.latent_shards
    layout = bench.tpla_layout(WORLD, tp)
    groups = [dist.new_group(r) for r in layout["groups"]]
    my = layout["group_of"][rank]
    tp_rank = layout["tp_rank"][rank]
    res["layout"] = layout

    lens = [70, 200, 1, 129]
    inputs = generate(wl, seq_lens=lens)
    sh = tpla_shard_inputs(inputs, wl, tp, tp_rank)
    dims = M.dims_for(wl.heads, wl.latent_rank, wl.rope_dim, wl.nope_dim, wl.v_dim, wl.q_len,
                      wl.softmax_scale, wl.dtype, wl.latent_shards, wl.page_size)
    plan = M.TplaShardPlan(dims, lens, tp=tp, group=groups[my], num_sms=148)
    res["kernel"] = plan.info.kernel
    res["shard_width"] = list(sh["kv_pool"].shape)
    # the shard's output: the oracle's MLA decode over this rank's slice
    width = wl.latent_rank // tp
    ckv, kr = {}, {}
    for b, L in enumerate(lens):
        n = -(-L // wl.page_size)
        rows = sh["kv_pool"][sh["block_table"][b, :n].long()].reshape(n * wl.page_size, -1)[:L]
        ckv[b], kr[b] = rows[:, :width].double().numpy(), rows[:, width:].double().numpy()
    out = mla_oracle.mla_decode(sh["q_nope"].double().numpy(), sh["q_rope"].double().numpy(), ckv, kr,
                                sh["w_uk"].double().numpy(), sh["w_uv"].double().numpy(),
                                wl.softmax_scale, 1)
    t = torch.from_numpy(out)
    plan.allreduce(t)
    plan.close()
    if rank == 0:
        # the full inputs, the TPLA definition
        ckv, kr = {}, {}
        for b in range(len(lens)):
            from mla_workloads import logical_cache
            c, k = logical_cache(inputs, b, wl)
            ckv[b], kr[b] = c.double().numpy(), k.double().numpy()
        ref = mla_oracle.mla_decode(inputs["q_nope"].double().numpy(), inputs["q_rope"].double().numpy(),
                                    ckv, kr, inputs["w_uk"].double().numpy(), inputs["w_uv"].double().numpy(),
                                    wl.softmax_scale, wl.latent_shards)
        res["max_diff"] = float(np.abs(t.numpy() - ref).max())
        res["ref_scale"] = float(np.abs(ref).max())
    gathered = [None] * WORLD
    dist.all_gather_object(gathered, float(t.sum()))
    res["same_sum_on_all_ranks"] = len(set(gathered)) == 1
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


def test_tpla_two_gloo_ranks(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(port, str(tmp_path)), nprocs=WORLD, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(WORLD)]
    import mla_latent_kv_21_b200 as M
    for r in res:
        assert r["kernel"] == M.MLA_KERNEL_TCGEN05
        assert r["shard_width"][-1] == 256 + 64
        assert r["same_sum_on_all_ranks"]
        assert r["layout"]["groups"] == [[0, 1]]
    assert res[0]["layout"]["tp_rank"] == [0, 1]
    assert res[0]["max_diff"] <= 1e-12 * max(1.0, res[0]["ref_scale"])


def test_tpla_layout_of_eight_ranks():
    sys.path.insert(0, ROOT)
    import bench
    lay = bench.tpla_layout(8, 2)
    assert lay["groups"] == [[0, 1], [2, 3], [4, 5], [6, 7]]
    assert lay["tp_rank"] == [0, 1] * 4
    assert lay["group_of"] == [0, 0, 1, 1, 2, 2, 3, 3]
    try:
        bench.tpla_layout(3, 2)
    except ValueError:
        pass
    else:
        raise AssertionError("an odd world size cannot hold two-way groups")
