"""The Python binding's argument checks (dtype and shape against the plan),
run on CPU tensors: the C ABI sees bare pointers, so a mismatch has to be
caught before the call. Every workload's own inputs pass the checks and stop
only at the device-tensor check; a wrong dtype or shape names the argument."""

import dataclasses

import pytest
import torch

import mla_latent_kv_21_b200 as M
from mla_workloads import WORKLOADS, generate

from harness import dims_of


def _call(wl, plan, inputs, **override):
    a = dict(inputs, **override)
    B = len(inputs["seq_lens"])
    out = a.get("out", torch.zeros((B, wl.q_len, wl.heads, wl.v_dim), dtype=wl.torch_dtype))
    if wl.dtype == "fp8":
        plan.run_fp8(a["q_nope"], a["q_rope"], a["kv_codes"], a["kv_rope"], a["kv_scale"],
                     a["block_table"], a["seq_lens"], a["w_uk"], a["w_uv"], out)
    else:
        plan.run(a["q_nope"], a["q_rope"], a["kv_pool"], a["block_table"], a["seq_lens"],
                 a["w_uk"], a["w_uv"], out)


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_workload_inputs_pass_the_checks(name):
    wl = WORKLOADS[name]
    lens = [max(wl.q_len, 70), max(wl.q_len, 5)]
    inputs = generate(wl, seq_lens=lens)
    plan = M.DecodePlan(dims_of(wl), lens, num_sms=148)
    try:
        with pytest.raises(ValueError, match="contiguous CUDA tensor"):
            _call(wl, plan, inputs)
    finally:
        plan.close()


@pytest.mark.parametrize("arg,bad,msg", [
    ("q_nope", lambda t: t.float(), "q_nope: dtype"),
    ("q_rope", lambda t: t[:, :, :, :32].contiguous(), "q_rope: shape"),
    ("kv_pool", lambda t: t[:, :, :512].contiguous(), "kv_pool: shape"),
    ("block_table", lambda t: t.long(), "block_table: dtype"),
    ("seq_lens", lambda t: t[:1], "seq_lens: shape"),
    ("w_uv", lambda t: t.transpose(1, 2).contiguous(), "w_uv: shape"),
    ("out", lambda t: t.float(), "out: dtype"),
])
def test_mismatches_are_named(arg, bad, msg):
    wl = WORKLOADS["deepseek_v3"]
    lens = [100, 7]
    inputs = generate(wl, seq_lens=lens)
    inputs["out"] = torch.zeros((2, 1, wl.heads, wl.v_dim), dtype=torch.bfloat16)
    plan = M.DecodePlan(dims_of(wl), lens, num_sms=148)
    try:
        with pytest.raises(ValueError, match=msg):
            _call(wl, plan, inputs, **{arg: bad(inputs[arg])})
    finally:
        plan.close()


def test_fp8_cache_tensors_are_checked_and_plans_not_mixed():
    wl = WORKLOADS["deepseek_v3_fp8"]
    lens = [100, 7]
    inputs = generate(wl, seq_lens=lens)
    plan = M.DecodePlan(dims_of(wl), lens, num_sms=148)
    try:
        with pytest.raises(ValueError, match="kv_scale: shape"):
            _call(wl, plan, inputs, kv_scale=inputs["kv_scale"][:-1].contiguous())
        with pytest.raises(ValueError, match="kv_codes: dtype"):
            _call(wl, plan, inputs, kv_codes=inputs["kv_codes"].to(torch.int8))
        with pytest.raises(ValueError, match="run_fp8"):
            plan.run(*(inputs[k] for k in ("q_nope", "q_rope", "kv_codes", "block_table", "seq_lens",
                                             "w_uk", "w_uv")), torch.zeros(1))
    finally:
        plan.close()
    bf = dataclasses.replace(wl, name="bf16_plan", dtype="bf16")
    plan = M.DecodePlan(dims_of(bf), lens, num_sms=148)
    try:
        with pytest.raises(ValueError, match="plan made with dtype 'fp8'"):
            _call(wl, plan, inputs)
    finally:
        plan.close()
