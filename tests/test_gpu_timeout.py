"""The decode kernel's bounded-wait error path, driven on the GPU.

Every mbarrier wait of the split-KV decode kernel gives up after a time limit,
records MLA_ERR_DEVICE_TIMEOUT in the workspace status word, raises the CTA's
abort flag and lets every role unwind to the kernel's exit (tensor memory
released, no trap). mla_decode_selftest_timeout runs one step with that limit
cut to 1 ms and the softmax warps withholding the release of their score
buffers, so the QK issuer waits on a barrier that nothing completes (no copy is
in flight on it). The test checks that the call returns quickly, that the
status word reports the timeout, and that a normal step on the same plan and
workspace afterwards is correct against the oracle.
"""

import time

import pytest
import torch

import mla_latent_kv_21_b200 as M
from mla_latent_kv_21_b200 import _lib as L
from mla_workloads import WORKLOADS, generate

from harness import assert_close, dims_of, oracle_out, to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["deepseek_v3", "tpla_dsv3"])
def test_device_timeout_is_reported_and_the_context_stays_usable(cuda_device, name):
    wl = WORKLOADS[name]
    lens = [2048, 700]                       # one worker: 11 groups of 256 keys, two segments
    inputs = generate(wl, seq_lens=lens)
    dev = to_device(inputs, cuda_device)
    plan = M.DecodePlan(dims_of(wl), lens, num_workers=1).allocate_workspace(cuda_device)
    shape = (len(lens), wl.q_len, wl.heads, wl.v_dim)
    out = torch.zeros(shape, dtype=wl.torch_dtype, device=cuda_device)
    stream = torch.cuda.current_stream(cuda_device).cuda_stream
    torch.cuda.synchronize(cuda_device)

    t0 = time.perf_counter()
    L.mla_decode_selftest_timeout(plan.handle, dev["q_nope"].data_ptr(), dev["q_rope"].data_ptr(),
                                  dev["kv_pool"].data_ptr(), dev["kv_pool"].shape[0],
                                  dev["block_table"].data_ptr(), dev["block_table"].shape[1],
                                  dev["seq_lens"].data_ptr(), dev["w_uk"].data_ptr(),
                                  dev["w_uv"].data_ptr(), out.data_ptr(), plan.workspace.data_ptr(),
                                  plan.workspace_bytes, 1_000_000, stream)
    torch.cuda.synchronize(cuda_device)
    elapsed = time.perf_counter() - t0
    assert plan.read_status() == M.MLA_ERR_DEVICE_TIMEOUT
    # a few 1 ms waits ran out, far below the normal 2 s limit
    assert elapsed < 1.0, elapsed

    # the context, the plan and the workspace are still usable
    out.fill_(float("nan"))
    plan.run(dev["q_nope"], dev["q_rope"], dev["kv_pool"], dev["block_table"], dev["seq_lens"],
             dev["w_uk"], dev["w_uv"], out)
    torch.cuda.synchronize(cuda_device)
    assert plan.read_status() == 0
    assert_close(out.double().cpu().numpy(), oracle_out(wl, inputs), wl.dtype, f"{name} after timeout")
    plan.close()
