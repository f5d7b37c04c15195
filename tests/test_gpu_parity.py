"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

* reduced sizes: every output element, lengths that span several pages and
  ragged tails (1, 63, 64, 65 ... tokens);
* the five full workload sizes, in the launch configuration bench.py times,
  on sampled (sequence, head) outputs that the oracle computes one by one;
* invariants: permuted vs contiguous block table (bit-identical), split-count
  independence, repeated runs;
* device-side error paths: bad block ids and lengths are reported, not faulted.
"""

import numpy as np
import pytest
import torch

import mla_latent_kv_21_b200 as M
from mla_workloads import WORKLOADS, generate

from harness import assert_close, errors, oracle_out, run_gpu

pytestmark = pytest.mark.gpu

REDUCED = {
    "tiny": [[256], [1, 63, 64, 65, 130, 200]],
    "llama2_7b": [[1, 63, 64, 65, 300, 1000]],
    "deepseek_v3": [[1, 64, 65, 129, 700], [2048]],
    "kimi_k2_mtp": [[2, 3, 64, 65, 66, 129, 500]],
    "tpla_dsv3": [[1, 63, 65, 130, 640]],
}


KERNELS = {"auto": M.MLA_KERNEL_AUTO, "simt": M.MLA_KERNEL_SIMT}


def _cases():
    for name, lens_sets in REDUCED.items():
        for lens in lens_sets:
            yield name, lens


@pytest.mark.parametrize("name,lens", list(_cases()))
@pytest.mark.parametrize("kernel", ["auto", "simt"])
def test_reduced_size_parity(cuda_device, name, lens, kernel):
    wl = WORKLOADS[name]
    k = KERNELS[kernel]
    inputs = generate(wl, seq_lens=lens)
    got, info = run_gpu(wl, inputs, cuda_device, kernel=k)
    ref = oracle_out(wl, inputs)
    assert_close(got.double().numpy(), ref, wl.dtype, f"{name} {lens} kernel={info.kernel}")


FULL_SAMPLES = {
    "tiny": None,  # every output
    "llama2_7b": [(0, 0), (7, 13), (15, 31)],
    "deepseek_v3": [(0, 0), (13, 77), (31, 127)],
    "kimi_k2_mtp": [(0, 0), (21, 40), (63, 63)],
    "tpla_dsv3": [(0, 5), (16, 64), (31, 127)],
}


@pytest.mark.parametrize("name,kernel", [(n, "auto") for n in FULL_SAMPLES])
def test_full_size_sampled_parity(cuda_device, name, kernel):
    wl = WORKLOADS[name]
    inputs = generate(wl)
    got, info = run_gpu(wl, inputs, cuda_device, kernel=KERNELS[kernel])
    got = got.double().numpy()
    assert np.isfinite(got).all()
    samples = FULL_SAMPLES[name]
    if samples is None:
        assert_close(got, oracle_out(wl, inputs), wl.dtype, name)
        return
    for b, h in samples:
        ref = oracle_out(wl, inputs, [b], [h])[0, :, 0]
        assert_close(got[b, :, h], ref, wl.dtype, f"{name} b={b} h={h}")


def test_block_table_permutation_is_bit_identical(cuda_device):
    wl = WORKLOADS["deepseek_v3"]
    lens = [65, 700, 1, 300]
    paged = generate(wl, seq_lens=lens)
    contiguous = generate(wl.with_(paged=False), seq_lens=lens)
    assert not torch.equal(paged["block_table"], contiguous["block_table"])
    a, _ = run_gpu(wl, paged, cuda_device)
    b, _ = run_gpu(wl, contiguous, cuda_device)
    assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a,
                       b.view(torch.int16) if b.dtype == torch.bfloat16 else b)


@pytest.mark.parametrize("name", ["deepseek_v3", "tpla_dsv3", "kimi_k2_mtp", "tiny"])
def test_split_count_independence(cuda_device, name):
    wl = WORKLOADS[name]
    lens = [1200, 70, 3] if wl.q_len == 1 else [1200, 70, 4]
    inputs = generate(wl, seq_lens=lens)
    ref = oracle_out(wl, inputs)
    outs = []
    for nw in (1, 3, 17, 0):
        got, info = run_gpu(wl, inputs, cuda_device, num_workers=nw)
        outs.append(got.double().numpy())
        assert_close(outs[-1], ref, wl.dtype, f"{name} workers={info.num_workers}")
    for o in outs[1:]:
        _, rel = errors(o, outs[0])
        assert rel <= (2e-3 if wl.dtype == "bf16" else 2e-6)


def test_repeated_runs_are_deterministic(cuda_device):
    wl = WORKLOADS["kimi_k2_mtp"]
    inputs = generate(wl, seq_lens=[500, 64, 2, 1000])
    a, _ = run_gpu(wl, inputs, cuda_device, repeat=1)
    b, _ = run_gpu(wl, inputs, cuda_device, repeat=3)
    assert torch.equal(a.float(), b.float())


def test_plan_lengths_only_affect_balance(cuda_device):
    """The device recomputes the partition from this run's lengths."""
    wl = WORKLOADS["deepseek_v3"]
    inputs = generate(wl, seq_lens=[700, 65, 300])
    got, _ = run_gpu(wl, inputs, cuda_device, plan_lens=[64, 64, 64])
    assert_close(got.double().numpy(), oracle_out(wl, inputs), wl.dtype)


@pytest.mark.parametrize("bad", ["block_high", "block_negative", "length_high"])
def test_device_errors_are_reported_not_faulted(cuda_device, bad):
    wl = WORKLOADS["deepseek_v3"]
    inputs = generate(wl, seq_lens=[300, 130])
    if bad == "block_high":
        inputs["block_table"][1, 1] = inputs["num_blocks"] + 5
    elif bad == "block_negative":
        inputs["block_table"][0, 2] = -7
    else:
        inputs["seq_lens"][1] = inputs["block_table"].shape[1] * 64 + 1
    run_gpu(wl, inputs, cuda_device, plan_lens=[300, 130], expect_status=M.MLA_ERR_BOUNDS)
    # the context is still usable afterwards
    good = generate(wl, seq_lens=[300, 130])
    got, _ = run_gpu(wl, good, cuda_device)
    assert_close(got.double().numpy(), oracle_out(wl, good), wl.dtype)
