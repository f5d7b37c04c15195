"""Parity of the FP8-cache decode (mla_decode_run_fp8) with the CPU oracle.

The oracle decodes the cache's E4M3 codes from the format definition and runs
the non-absorbed fp64 attention on the dequantised values, so the comparison
measures the GPU path's own error (the query as e4m3 + e5m2 and P * s_t as two
e4m3 terms, the fp16 partials, bf16 output) against the FP8 tolerance.
"""

import dataclasses

import pytest
import torch

from mla_workloads import WORKLOADS, generate

from harness import assert_close, oracle_out, run_gpu

pytestmark = pytest.mark.gpu

WL = WORKLOADS["deepseek_v3_fp8"]
# the Kimi-K2 MTP shape (64 heads, two query tokens with the causal rule) over the FP8 cache
MTP = dataclasses.replace(WORKLOADS["kimi_k2_mtp"], name="kimi_k2_mtp_fp8", dtype="fp8")


@pytest.mark.parametrize("lens", [[1, 63, 64, 65, 130, 200, 700], [2048], [3000, 1, 257]])
def test_reduced_size_parity(cuda_device, lens):
    inputs = generate(WL, seq_lens=lens)
    got, info = run_gpu(WL, inputs, cuda_device)
    assert_close(got.double().numpy(), oracle_out(WL, inputs), WL.dtype, f"fp8 {lens}")


@pytest.mark.parametrize("workers", [1, 5, 0])
def test_split_counts(cuda_device, workers):
    inputs = generate(WL, seq_lens=[1200, 70, 3])
    got, info = run_gpu(WL, inputs, cuda_device, num_workers=workers)
    assert_close(got.double().numpy(), oracle_out(WL, inputs), WL.dtype, f"workers={info.num_workers}")


@pytest.mark.parametrize("lens", [[2, 65, 300, 1030], [129, 3]])
def test_mtp_parity(cuda_device, lens):
    # row t of a sequence sees keys j <= L - 2 + t: a segment holding only the
    # last key has a row that sees nothing there
    inputs = generate(MTP, seq_lens=lens)
    got, _ = run_gpu(MTP, inputs, cuda_device, num_workers=5)
    assert_close(got.double().numpy(), oracle_out(MTP, inputs), MTP.dtype, f"mtp fp8 {lens}")


def _poison_tail_slots(inputs, wl):
    """Slots past each sequence's length in its last page: codes set to the
    largest finite e4m3 value (0x7E = 448), RoPE keys and scales to NaN."""
    P = wl.page_size
    codes, rope, scale = inputs["kv_codes"].clone(), inputs["kv_rope"].clone(), inputs["kv_scale"].clone()
    for b, L in enumerate(inputs["seq_lens"].tolist()):
        npg = -(-L // P)
        blk = int(inputs["block_table"][b, npg - 1])
        t0 = L - (npg - 1) * P
        codes[blk, t0:] = 0x7E
        rope[blk, t0:] = float("nan")
        scale[blk, t0:] = float("nan")
    return dict(inputs, kv_codes=codes, kv_rope=rope, kv_scale=scale)


def test_tail_slots_may_hold_any_scale_and_rope(cuda_device):
    # a key past the sequence is weighted by exactly 0, its scale is replaced
    # by 0 in the kernel, its score is masked: the output cannot change
    inputs = generate(WL, seq_lens=[1, 63, 65, 200])
    clean, _ = run_gpu(WL, inputs, cuda_device)
    dirty, _ = run_gpu(WL, _poison_tail_slots(inputs, WL), cuda_device)
    assert torch.isfinite(dirty.float()).all()
    assert torch.equal(clean, dirty)

