"""TPLA across GPUs, emulated on one GPU: the per-GPU shard plans summed.

A tp-way TPLA group runs, on each GPU, the plain decode over that GPU's latent
shard (latent_rank = r / tp, one shard, the full RoPE key) and sums the bf16
outputs with an all-reduce. Here both shards of the two-way TPLA workload run
one after the other on one GPU through the C ABI (the r = 256 tensor-core
kernels), and their outputs are summed as the all-reduce would (bf16 inputs,
one rounding of the sum) and compared with the oracle's TPLA definition.
"""

import pytest
import torch

import mla_latent_kv_21_b200 as M
from mla_workloads import WORKLOADS, generate, tpla_shard_inputs

from harness import assert_close, dims_of, oracle_out, to_device
from test_gpu_parity import full_size_pairs

pytestmark = pytest.mark.gpu

WL = WORKLOADS["tpla_dsv3"]
TP = WL.latent_shards


def _shard_sum(inputs, lens, device, num_workers=0):
    outs = []
    for g in range(TP):
        sh = to_device(tpla_shard_inputs(inputs, WL, TP, g), device)
        plan = M.TplaShardPlan(dims_of(WL), lens, tp=TP, num_workers=num_workers).allocate_workspace(device)
        assert plan.info.kernel == M.MLA_KERNEL_TCGEN05
        out = torch.full((len(lens), WL.q_len, WL.heads, WL.v_dim), float("nan"), dtype=torch.bfloat16,
                         device=device)
        plan.run_shard(sh["q_nope"], sh["q_rope"], sh["kv_pool"], sh["block_table"], sh["seq_lens"],
                       sh["w_uk"], sh["w_uv"], out)
        torch.cuda.synchronize(device)
        assert plan.read_status() == 0
        plan.close()
        outs.append(out.float())
        del sh
    # the all-reduce: bf16 shard outputs summed, the sum rounded to bf16 once
    return sum(outs).to(torch.bfloat16).double().cpu().numpy()


@pytest.mark.parametrize("lens,workers", [([1, 63, 65, 130, 640], 0), ([2048, 300, 64], 5)])
def test_shard_plans_sum_to_the_tpla_oracle(cuda_device, lens, workers):
    inputs = generate(WL, seq_lens=lens)
    got = _shard_sum(inputs, lens, cuda_device, workers)
    assert_close(got, oracle_out(WL, inputs), "bf16", f"tpla shards {lens}")


def test_shard_plans_full_size(cuda_device, parity_report):
    inputs = generate(WL)
    lens = inputs["seq_lens"].tolist()
    got = _shard_sum(inputs, lens, cuda_device)
    pairs = full_size_pairs(WL, n_min=32)
    by_seq = {}
    for b, h in pairs:
        by_seq.setdefault(b, []).append(h)
    g, r = [], []
    for b, hs in sorted(by_seq.items()):
        r.append(oracle_out(WL, inputs, [b], hs)[0].reshape(-1, WL.v_dim))
        g.append(got[b][:, hs].reshape(-1, WL.v_dim))
    import numpy as np
    max_abs, rel = assert_close(np.concatenate(g), np.concatenate(r), "bf16", "tpla shards full size")
    parity_report.append(("tpla_dsv3 as 2 per-GPU shards", f"{len(pairs)} pairs", max_abs, rel))
