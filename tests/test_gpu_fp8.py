"""Parity of the FP8-cache decode (mla_decode_run_fp8) with the CPU oracle.

The oracle decodes the cache's E4M3 codes from the format definition and runs
the non-absorbed fp64 attention on the dequantised values, so the comparison
measures the GPU path's own error (the query and P split into e4m3 + e5m2
operands, the fp16 partials, bf16 output) against the bf16 tolerance.
"""

import numpy as np
import pytest

from mla_workloads import WORKLOADS, generate

from harness import assert_close, oracle_out, run_gpu

pytestmark = pytest.mark.gpu

WL = WORKLOADS["deepseek_v3_fp8"]


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


def test_full_size_sampled_parity(cuda_device):
    inputs = generate(WL)
    got, _ = run_gpu(WL, inputs, cuda_device)
    got = got.double().numpy()
    assert np.isfinite(got).all()
    for b, h in [(0, 0), (13, 77), (31, 127)]:
        ref = oracle_out(WL, inputs, [b], [h])[0, :, 0]
        assert_close(got[b, :, h], ref, WL.dtype, f"b={b} h={h}")
