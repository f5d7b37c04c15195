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


@pytest.mark.parametrize("heads,q_len,lens", [
    (64, 2, [2, 3, 65, 66, 130, 700]),   # two query tokens: causal limit per query row
    (16, 1, [1, 64, 65, 257, 900]),      # 16 real rows of each CTA pair's 128
    (128, 1, [4096, 33]),                # several segments per sequence
])
def test_two_shard_shapes(cuda_device, heads, q_len, lens):
    """The two-shard (TPLA) decode on shapes beyond its workload: MTP rows,
    few heads, long sequences split over several workers; every element."""
    wl = WORKLOADS["tpla_dsv3"].with_(heads=heads, q_len=q_len)
    inputs = generate(wl, seq_lens=lens)
    got, info = run_gpu(wl, inputs, cuda_device)
    assert info.kernel == M.MLA_KERNEL_TCGEN05
    ref = oracle_out(wl, inputs)
    assert_close(got.double().numpy(), ref, wl.dtype, f"two shards H={heads} Lq={q_len} {lens}")


@pytest.mark.parametrize("heads,q_len,lens", [
    (40, 1, [1, 65, 300, 2000]),     # 40 rows: the second CTA of each pair holds only padding rows
    (96, 1, [3, 64, 129, 1500]),     # 96 rows: the second CTA holds 32 real rows
    (48, 2, [2, 5, 190, 777]),       # 96 rows over two query tokens
])
def test_one_shard_row_counts(cuda_device, heads, q_len, lens):
    """The one-shard decode at row counts (heads x query tokens) between the
    workloads' 32, 128: every element."""
    wl = WORKLOADS["deepseek_v3"].with_(heads=heads, q_len=q_len)
    inputs = generate(wl, seq_lens=lens)
    got, info = run_gpu(wl, inputs, cuda_device)
    assert info.kernel == M.MLA_KERNEL_TCGEN05
    ref = oracle_out(wl, inputs)
    assert_close(got.double().numpy(), ref, wl.dtype, f"one shard H={heads} Lq={q_len} {lens}")


def full_size_pairs(wl, n_min=64):
    """(sequence, head) pairs checked at full size: every sequence (so every
    split segment, including those of workers whose range crosses a sequence
    end), heads cycling through both CTAs' query-row halves (rows [0, 64) and
    [64, 128): row = t H + h), the first and the last head, at least n_min
    pairs. Every query token of a pair is compared (both MTP rows)."""
    B, H = wl.batch, wl.heads
    per_seq = max(1, -(-n_min // B))
    pairs = {(0, 0), (B - 1, H - 1), (0, H - 1), (B - 1, 0)}
    for b in range(B):
        for k in range(per_seq):
            # k-th head of sequence b: alternate the halves [0, H/2) and [H/2, H)
            base = (37 * b + 11 * k) % max(1, H // 2)
            pairs.add((b, base + (H // 2 if (b + k) % 2 else 0)))
    return sorted(pairs)


@pytest.mark.parametrize("name", ["tiny", "llama2_7b", "deepseek_v3", "kimi_k2_mtp", "tpla_dsv3",
                                  "deepseek_v3_fp8"])
def test_full_size_parity(cuda_device, name, parity_report):
    """Every workload at its full size, in the launch configuration bench.py
    times; tiny: every output; the others: >= 64 (sequence, head) pairs, every
    element of each compared at the tolerance of the workload's dtype."""
    wl = WORKLOADS[name]
    inputs = generate(wl)
    got, info = run_gpu(wl, inputs, cuda_device)
    got = got.double().numpy()
    assert np.isfinite(got).all()
    if name == "tiny":
        max_abs, rel = assert_close(got, oracle_out(wl, inputs), wl.dtype, name)
        parity_report.append((name, "all outputs", max_abs, rel))
        return
    pairs = full_size_pairs(wl)
    assert len(pairs) >= 64 and {b for b, _ in pairs} == set(range(wl.batch))
    rows = wl.heads * wl.q_len
    if rows > 64:  # both CTAs of a pair own query rows
        assert {(t * wl.heads + h) // 64 for _, h in pairs for t in range(wl.q_len)} == {0, 1}
    by_seq = {}
    for b, h in pairs:
        by_seq.setdefault(b, []).append(h)
    g, r = [], []
    for b, hs in sorted(by_seq.items()):
        ref = oracle_out(wl, inputs, [b], hs)[0]           # [Lq, len(hs), dv]
        g.append(got[b][:, hs])
        r.append(ref)
    g = np.concatenate([x.reshape(-1, wl.v_dim) for x in g])
    r = np.concatenate([x.reshape(-1, wl.v_dim) for x in r])
    max_abs, rel = assert_close(g, r, wl.dtype, name)
    parity_report.append((name, f"{len(pairs)} pairs x {wl.q_len} rows, {info.num_workers} workers",
                          max_abs, rel))


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
