"""More parity edge cases of the CUDA path (through the C ABI) against the oracle.

* one 32K-token sequence: every worker of the plan holds a segment of the same
  sequence, so the combine merges 74 partials per row (many rounds of its
  four-segment load loop);
* many short sequences of random lengths, with the default worker count and
  with 8 workers that each cross several sequence ends (segments of one or
  two pages, partial groups, query reloads);
* two plans of different workloads run concurrently on two streams with their
  own workspaces: results equal the same runs made one after the other;
* seeded random shapes (heads, query tokens, latent shards, worker count and
  lengths drawn together) on the tensor-core path, every element.
"""

import random

import numpy as np
import pytest
import torch

import mla_latent_kv_21_b200 as M
from mla_workloads import WORKLOADS, generate

from harness import assert_close, dims_of, oracle_out, run_gpu, to_device

pytestmark = pytest.mark.gpu


def test_single_long_sequence_all_workers(cuda_device):
    wl = WORKLOADS["deepseek_v3"]
    inputs = generate(wl, seq_lens=[32768])
    got, info = run_gpu(wl, inputs, cuda_device)
    assert info.num_workers == 74 and info.num_split_slots == 74
    got = got.double().numpy()
    assert np.isfinite(got).all()
    for h in (0, 77, 127):
        ref = oracle_out(wl, inputs, [0], [h])[0, :, 0]
        assert_close(got[0, :, h], ref, wl.dtype, f"h={h}")


@pytest.mark.parametrize("workers", [0, 8])
@pytest.mark.parametrize("name", ["deepseek_v3", "kimi_k2_mtp", "tpla_dsv3"])
def test_many_short_sequences(cuda_device, name, workers):
    wl = WORKLOADS[name]
    rng = random.Random(7)
    lens = [rng.randint(wl.q_len, 300) for _ in range(40)]
    inputs = generate(wl, seq_lens=lens)
    got, info = run_gpu(wl, inputs, cuda_device, num_workers=workers)
    if workers:
        assert info.num_workers == workers  # each worker crosses several sequence ends
    assert_close(got.double().numpy(), oracle_out(wl, inputs), wl.dtype, f"{name} workers={workers}")


def test_two_plans_on_two_streams(cuda_device):
    cases = []
    for name, lens in (("deepseek_v3", [700, 65, 3000, 1]), ("kimi_k2_mtp", [2, 900, 129, 4000])):
        wl = WORKLOADS[name]
        inputs = generate(wl, seq_lens=lens)
        solo, _ = run_gpu(wl, inputs, cuda_device)
        dev = to_device(inputs, cuda_device)
        plan = M.DecodePlan(dims_of(wl), lens).allocate_workspace(cuda_device)
        out = torch.full((len(lens), wl.q_len, wl.heads, wl.v_dim), float("nan"),
                         dtype=wl.torch_dtype, device=cuda_device)
        cases.append((wl, dev, plan, out, solo, torch.cuda.Stream(cuda_device)))
    torch.cuda.synchronize(cuda_device)
    for _ in range(3):
        for wl, dev, plan, out, solo, stream in cases:
            plan.run(dev["q_nope"], dev["q_rope"], dev["kv_pool"], dev["block_table"],
                     dev["seq_lens"], dev["w_uk"], dev["w_uv"], out, stream=stream.cuda_stream)
    torch.cuda.synchronize(cuda_device)
    for wl, dev, plan, out, solo, stream in cases:
        assert plan.read_status() == 0
        assert torch.equal(out.cpu().view(torch.int16), solo.view(torch.int16)), wl.name
        plan.close()


def test_tail_slots_may_hold_any_rope_and_finite_ckv(cuda_device):
    # slots past a sequence's length in its last page are read (whole pages
    # move) but weighted by exactly 0: NaN RoPE keys (masked scores) and large
    # finite cKV there leave the output bit-identical
    wl = WORKLOADS["deepseek_v3"]
    inputs = generate(wl, seq_lens=[1, 63, 65, 200])
    pool = inputs["kv_pool"].clone()
    P, r = wl.page_size, wl.latent_rank
    for b, L in enumerate(inputs["seq_lens"].tolist()):
        npg = -(-L // P)
        blk = int(inputs["block_table"][b, npg - 1])
        t0 = L - (npg - 1) * P
        pool[blk, t0:, :r] = 3.0e4
        pool[blk, t0:, r:] = float("nan")
    clean, _ = run_gpu(wl, inputs, cuda_device)
    dirty, _ = run_gpu(wl, dict(inputs, kv_pool=pool), cuda_device)
    assert torch.isfinite(dirty.float()).all()
    assert torch.equal(clean, dirty)



def _random_shapes(n=8, seed=2024):
    rng = random.Random(seed)
    cases = []
    for _ in range(n):
        shards = rng.choice([1, 2])
        q_len = rng.choice([1, 1, 2])
        heads = rng.choice([h for h in (8, 16, 24, 40, 64, 96, 128) if h * q_len <= 128])
        lens = [rng.randint(q_len, rng.choice([70, 700, 3000])) for _ in range(rng.randint(1, 6))]
        workers = rng.choice([0, 0, 5, 33])
        cases.append((shards, q_len, heads, lens, workers))
    return cases


@pytest.mark.parametrize("shards,q_len,heads,lens,workers", _random_shapes())
def test_random_shapes(cuda_device, shards, q_len, heads, lens, workers):
    """Heads x query tokens from 8 to 128 rows, one or two latent shards,
    default and small worker counts, ragged lengths: the tensor-core path
    against the oracle, every element."""
    base = WORKLOADS["tpla_dsv3" if shards == 2 else "deepseek_v3"]
    wl = base.with_(heads=heads, q_len=q_len)
    inputs = generate(wl, seq_lens=lens)
    got, info = run_gpu(wl, inputs, cuda_device, num_workers=workers)
    assert info.kernel == M.MLA_KERNEL_TCGEN05
    ref = oracle_out(wl, inputs)
    assert_close(got.double().numpy(), ref, wl.dtype,
                 f"S={shards} H={heads} Lq={q_len} workers={info.num_workers} {lens}")
