"""mla_decode_run inside a CUDA graph.

The header states that mla_decode_run allocates nothing, does not synchronise
and reads nothing back on the host, so a stream can be captured around it (its
kernels are launched with programmatic stream serialization, which a captured
graph keeps as programmatic edges). Captured once and replayed, the step must
reproduce the eager output bit for bit (the decode is deterministic) and stay
within the oracle tolerance.
"""

import pytest
import torch

import mla_latent_kv_21_b200 as M
from mla_workloads import WORKLOADS, generate

from harness import assert_close, dims_of, oracle_out, to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,lens", [
    ("deepseek_v3", [700, 65, 1, 300, 2048]),
    ("kimi_k2_mtp", [2, 129, 500, 66]),
    ("tpla_dsv3", [640, 63, 1000]),
    ("tiny", [256]),
])
def test_graph_replay_matches_eager(cuda_device, name, lens):
    wl = WORKLOADS[name]
    inputs = generate(wl, seq_lens=lens)
    dev = to_device(inputs, cuda_device)
    plan = M.DecodePlan(dims_of(wl), lens).allocate_workspace(cuda_device)
    shape = (len(lens), wl.q_len, wl.heads, wl.v_dim)

    def step(out, stream):
        plan.run(dev["q_nope"], dev["q_rope"], dev["kv_pool"], dev["block_table"],
                 dev["seq_lens"], dev["w_uk"], dev["w_uv"], out, stream)

    eager = torch.full(shape, float("nan"), dtype=wl.torch_dtype, device=cuda_device)
    step(eager, torch.cuda.current_stream(cuda_device).cuda_stream)
    torch.cuda.synchronize(cuda_device)

    out = torch.full(shape, float("nan"), dtype=wl.torch_dtype, device=cuda_device)
    side = torch.cuda.Stream(cuda_device)
    side.wait_stream(torch.cuda.current_stream(cuda_device))
    with torch.cuda.stream(side):
        step(out, side.cuda_stream)  # warm-up outside the capture
    torch.cuda.synchronize(cuda_device)
    out.fill_(float("nan"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        step(out, side.cuda_stream)
    for _ in range(2):
        out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize(cuda_device)
        assert plan.read_status() == 0
        assert torch.equal(out, eager), "graph replay differs from the eager run"
    got = out.double().cpu().numpy()
    ref = oracle_out(wl, inputs)
    assert_close(got, ref, wl.dtype, f"{wl.name} graph replay")
    del g
    plan.close()
