"""Parity of the MLA-form prefill (mla_prefill_run, through the C ABI) with
the oracle's causal prefill.

* short prompts around the 128-token tiles (1, 64, 127, 128, 129, 300 tokens)
  with 16 heads: every output element;
* longer prompts (1000 and 2500 tokens, 16 heads): every head of sampled
  tokens (the first, the last, those around tile edges, random ones);
* the DeepSeek-V3 prefill shape at full size (2 prompts x 8192 tokens, 128
  heads): >= 64 sampled (token, head) rows;
* repeated runs are bit-identical; device errors are not raised.
"""

import random

import numpy as np
import pytest
import torch

import mla_latent_kv_21_b200 as M
from mla_workloads import PREFILL_WORKLOADS, generate_prefill
from oracle import mla_oracle

from harness import assert_close_prefill, dims_of, to_device

pytestmark = pytest.mark.gpu

WL = PREFILL_WORKLOADS["deepseek_v3_prefill"]


def _run(wl, inputs, device, repeat=1):
    d = to_device(inputs, device)
    lens = inputs["seq_lens"].tolist()
    plan = M.PrefillPlan(dims_of(wl), lens).allocate_workspace(device)
    T = sum(lens)
    out = torch.full((T, wl.heads, wl.v_dim), float("nan"), dtype=torch.bfloat16, device=device)
    for _ in range(repeat):
        plan.run(d["q_nope"], d["q_rope"], d["kv_rows"], d["cu_seqlens"], d["w_uk"], d["w_uv"], out)
    torch.cuda.synchronize(device)
    assert plan.read_status() == 0
    plan.close()
    return out.double().cpu().numpy()


def _oracle(wl, inputs, pairs):
    return mla_oracle.mla_prefill(inputs["q_nope"].double().numpy(), inputs["q_rope"].double().numpy(),
                                  inputs["kv_rows"].double().numpy(), inputs["cu_seqlens"].tolist(),
                                  inputs["w_uk"].double().numpy(), inputs["w_uv"].double().numpy(),
                                  wl.softmax_scale, pairs, abs_weighted=True)


def _sample_tokens(cu, rng, n_random):
    toks = set()
    for b in range(len(cu) - 1):
        s, e = cu[b], cu[b + 1]
        for t in (s, s + 1, e - 1, e - 2):
            if s <= t < e:
                toks.add(t)
        for edge in range(s + 127, e, 128):   # both sides of every 128-token tile edge
            toks.update(x for x in (edge, edge + 1) if x < e)
    toks.update(rng.randrange(0, cu[-1]) for _ in range(n_random))
    return sorted(toks)


@pytest.mark.parametrize("lens", [[1, 64, 127, 128, 129, 300], [257, 2, 130]])
def test_short_prompts_every_output(cuda_device, lens):
    wl = WL.with_(heads=16)
    inputs = generate_prefill(wl, seq_lens=lens)
    got = _run(wl, inputs, cuda_device)
    T = sum(lens)
    pairs = [(t, h) for t in range(T) for h in range(wl.heads)]
    ref, aw = _oracle(wl, inputs, pairs)
    assert_close_prefill(got.reshape(-1, wl.v_dim), ref, aw, f"prefill {lens}")


def test_longer_prompts_sampled_tokens(cuda_device):
    wl = WL.with_(heads=16)
    lens = [1000, 2500]
    inputs = generate_prefill(wl, seq_lens=lens)
    got = _run(wl, inputs, cuda_device)
    toks = _sample_tokens(inputs["cu_seqlens"].tolist(), random.Random(3), 24)
    pairs = [(t, h) for t in toks for h in range(wl.heads)]
    ref, aw = _oracle(wl, inputs, pairs)
    assert_close_prefill(np.stack([got[t, h] for t, h in pairs]), ref, aw, "prefill 1000 + 2500")


def test_full_size_sampled(cuda_device, parity_report):
    inputs = generate_prefill(WL)
    got = _run(WL, inputs, cuda_device)
    rng = random.Random(5)
    cu = inputs["cu_seqlens"].tolist()
    toks = _sample_tokens(cu, rng, 8)
    toks = sorted(set(toks[:6] + toks[-6:] + rng.sample(toks, min(len(toks), 40))))
    heads = [0, WL.heads - 1, 64, 63]
    pairs = [(t, heads[i % len(heads)] if i % 3 else rng.randrange(WL.heads)) for i, t in enumerate(toks)]
    pairs += [(cu[1] - 1, 5), (cu[-1] - 1, 77), (0, 3), (cu[1], 100)]
    assert len(pairs) >= 48
    ref, aw = _oracle(WL, inputs, pairs)
    max_abs, rel = assert_close_prefill(np.stack([got[t, h] for t, h in pairs]), ref, aw, "prefill full size")
    parity_report.append(("deepseek_v3_prefill", f"{len(pairs)} (token, head) rows", max_abs, rel))


def test_repeated_runs_are_deterministic(cuda_device):
    wl = WL.with_(heads=8)
    inputs = generate_prefill(wl, seq_lens=[300, 129])
    a = _run(wl, inputs, cuda_device)
    b = _run(wl, inputs, cuda_device, repeat=2)
    assert np.array_equal(a, b)
