"""The decode entry point for callers that cannot allocate device memory.

mla_decode_run_no_alloc serves callers that cannot call cudaMalloc where they
run decode steps (an engine whose memory pool owns the whole device, or a
latency-critical loop that cannot afford allocation's implicit device
synchronisation). It takes no workspace: its scratch is a fixed 32 MiB array
inside the library. These tests call it through the C ABI and check that two
calls in a row reproduce the output of mla_decode_run with a caller-allocated
workspace bit for bit (both launch the same deterministic kernels on the same
plan and inputs; only where the scratch lives differs, so any difference would
be a scratch-layout fault), and that plans needing more scratch than the array
holds are refused.

The file name makes pytest collect it last; each test also passes when the
file runs alone in a fresh process.
"""

import pytest
import torch

import mla_latent_kv_21_b200 as M
from mla_latent_kv_21_b200 import _lib as L
from mla_workloads import WORKLOADS, generate

from harness import dims_of, errors, to_device

pytestmark = pytest.mark.gpu


def _run_no_alloc(plan, wl, dev, out, stream):
    L.mla_decode_run_no_alloc(plan.handle, dev["q_nope"].data_ptr(), dev["q_rope"].data_ptr(),
                              dev["kv_pool"].data_ptr(), dev["kv_pool"].shape[0],
                              dev["block_table"].data_ptr(), dev["block_table"].shape[1],
                              dev["seq_lens"].data_ptr(), dev["w_uk"].data_ptr(),
                              dev["w_uv"].data_ptr(), out.data_ptr(), stream)


@pytest.mark.parametrize("name,lens", [
    ("deepseek_v3", [700, 65, 1, 300, 2048]),
    ("kimi_k2_mtp", [2, 129, 500, 66]),
    ("tpla_dsv3", [640, 63, 1000]),
    ("tiny", [256, 70]),
])
def test_no_alloc_matches_workspace_entry_point(cuda_device, name, lens):
    wl = WORKLOADS[name]
    inputs = generate(wl, seq_lens=lens)
    dev = to_device(inputs, cuda_device)
    plan = M.DecodePlan(dims_of(wl), lens).allocate_workspace(cuda_device)
    shape = (len(lens), wl.q_len, wl.heads, wl.v_dim)
    stream = torch.cuda.current_stream(cuda_device).cuda_stream

    ref = torch.full(shape, float("nan"), dtype=wl.torch_dtype, device=cuda_device)
    plan.run(dev["q_nope"], dev["q_rope"], dev["kv_pool"], dev["block_table"], dev["seq_lens"],
             dev["w_uk"], dev["w_uv"], ref)
    torch.cuda.synchronize(cuda_device)
    assert plan.read_status() == 0
    ref = ref.cpu()
    assert torch.isfinite(ref.float()).all()

    for call in range(2):
        got = torch.full(shape, float("nan"), dtype=wl.torch_dtype, device=cuda_device)
        _run_no_alloc(plan, wl, dev, got, stream)
        torch.cuda.synchronize(cuda_device)
        got = got.cpu()
        assert torch.isfinite(got.float()).all(), f"call {call}: non-finite output"
        same = torch.equal(got.view(torch.int16), ref.view(torch.int16)) if got.dtype == torch.bfloat16 \
            else torch.equal(got.view(torch.int32), ref.view(torch.int32))
        if not same:
            _, rel = errors(got.double().numpy(), ref.double().numpy())
            raise AssertionError(f"call {call}: not bit-identical to mla_decode_run (rel_fro {rel:.3e})")
    plan.close()


def test_no_alloc_refuses_plans_larger_than_its_scratch(cuda_device):
    wl = WORKLOADS["deepseek_v3"]
    lens = [32768] * 64  # twice the 32 x 32K batch: about 64 MB of scratch
    plan = M.DecodePlan(dims_of(wl), lens)
    assert plan.workspace_bytes > 32 << 20
    fake = 1 << 20  # never dereferenced: the size check comes before any device work
    with pytest.raises(L.MlaError) as e:
        L.mla_decode_run_no_alloc(plan.handle, fake, fake, fake, 1, fake, 512, fake, fake, fake,
                                  fake, 0)
    assert e.value.status == L.MLA_ERR_WORKSPACE_TOO_SMALL
    plan.close()
