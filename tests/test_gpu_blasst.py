"""Decode with threshold skipping (mla_decode_run_blasst, through the C ABI)
against the oracle's definition of the skip rule (mla_oracle.mla_decode_blasst).

The oracle takes the plan's split segments from an independent recomputation of
the partition (tests/harness_partition.py), so both sides form the same blocks
of 256 keys. Each test checks that every block decision is far from the
threshold (the GPU decides in fp32 from bf16 operands, the oracle in fp64), that
the skipped / total group counters equal the oracle's, and the outputs within
the bf16 tolerance. With no threshold (-inf) the skipping kernel must match the
dense kernel bit for bit.
"""

import numpy as np
import pytest
import torch

import mla_latent_kv_21_b200 as M
from mla_workloads import WORKLOADS, generate, logical_cache
from oracle import mla_oracle

from harness import assert_close, dims_of, to_device
from harness_partition import segment_key_ranges

pytestmark = pytest.mark.gpu

WL = WORKLOADS["deepseek_v3_peaked"]
THR = -6.0


def _gpu(wl, inputs, device, thr, num_workers=0, dense=False):
    dev = to_device(inputs, device)
    lens = inputs["seq_lens"].tolist()
    plan = M.DecodePlan(dims_of(wl), lens, num_workers=num_workers).allocate_workspace(device)
    out = torch.full((len(lens), wl.q_len, wl.heads, wl.v_dim), float("nan"), dtype=torch.bfloat16,
                     device=device)
    args = (dev["q_nope"], dev["q_rope"], dev["kv_pool"], dev["block_table"], dev["seq_lens"], dev["w_uk"],
            dev["w_uv"], out)
    if dense:
        plan.run(*args)
        counts = None
    else:
        plan.run_blasst(*args, thr)
        counts = plan.skip_counts()
    torch.cuda.synchronize(device)
    assert plan.read_status() == 0
    W = plan.info.num_workers
    plan.close()
    return out.cpu(), counts, W


def _oracle(wl, inputs, lens, W, thr, seqs):
    outs, kept_all, margins = [], [], []
    for b in seqs:
        c, k = logical_cache(inputs, b, wl)
        o, kept, mg = mla_oracle.mla_decode_blasst(
            inputs["q_nope"][b].double().numpy(), inputs["q_rope"][b].double().numpy(), c.double().numpy(),
            k.double().numpy(), inputs["w_uk"].double().numpy(), inputs["w_uv"].double().numpy(),
            wl.softmax_scale, segment_key_ranges(lens, wl.page_size, W, b), thr)
        outs.append(o)
        kept_all.append(kept)
        margins.append(mg)
    kept = np.concatenate(kept_all)
    mg = np.concatenate(margins)
    fin = np.abs(mg[np.isfinite(mg)])
    # inf where every block opens its segment (always kept): no decision near the threshold
    return np.stack(outs), int((~kept).sum()), len(kept), float(fin.min()) if fin.size else float("inf")


@pytest.mark.parametrize("lens,workers", [([4096, 2500, 1200], 5), ([4096, 2500, 1200], 0), ([9000, 300], 3)])
def test_skip_decisions_counts_and_parity(cuda_device, lens, workers):
    inputs = generate(WL, seq_lens=lens)
    got, (skipped, total), W = _gpu(WL, inputs, cuda_device, THR, workers)
    ref, o_skipped, o_total, margin = _oracle(WL, inputs, lens, W, THR, range(len(lens)))
    assert margin > 0.1, f"a block decision lies within {margin} of the threshold"
    assert (skipped, total) == (o_skipped, o_total)
    assert o_skipped > 0 or workers == 0   # 74 workers on 123 pages: every block opens a segment
    assert_close(got.double().numpy(), ref, "bf16", f"blasst {lens} W={W}")


def test_no_threshold_matches_the_dense_kernel_bit_for_bit(cuda_device):
    lens = [4096, 2500, 1200]
    inputs = generate(WL, seq_lens=lens)
    a, (skipped, total), _ = _gpu(WL, inputs, cuda_device, float("-inf"), 5)
    b, _, _ = _gpu(WL, inputs, cuda_device, 0.0, 5, dense=True)
    assert skipped == 0 and total > 0
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_flat_attention_skips_nothing(cuda_device):
    wl = WORKLOADS["deepseek_v3"]
    lens = [3000, 700]
    inputs = generate(wl, seq_lens=lens)
    a, (skipped, total), _ = _gpu(wl, inputs, cuda_device, THR, 4)
    b, _, _ = _gpu(wl, inputs, cuda_device, 0.0, 4, dense=True)
    assert skipped == 0 and total > 0
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_full_size_first_and_last_sequence(cuda_device, parity_report):
    inputs = generate(WL)
    lens = inputs["seq_lens"].tolist()
    got, (skipped, total), W = _gpu(WL, inputs, cuda_device, THR)
    seqs = [0, len(lens) - 1]
    ref, _, _, margin = _oracle(WL, inputs, lens, W, THR, seqs)
    assert margin > 0.1
    max_abs, rel = assert_close(got[seqs].double().numpy(), ref, "bf16", "blasst full size")
    parity_report.append(("deepseek_v3_peaked, threshold -6", f"sequences 0 and 31, all heads; "
                          f"{skipped} of {total} groups skipped", max_abs, rel))
