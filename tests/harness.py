"""Shared test helpers: run the CUDA path through the C ABI and the CPU oracle
on the same seeded inputs, and compare them with the stated tolerances."""

from __future__ import annotations

import numpy as np
import torch

import mla_latent_kv_21_b200 as M
from mla_workloads import Workload, generate, logical_cache, stored_rows_fp8
from oracle import fp8_cache, mla_oracle

# bf16 inputs with fp32 accumulation: max-abs <= 2e-2 and rel-Frobenius <= 5e-3;
# the fp32 workload: rel-Frobenius <= 1e-5.
# FP8 cache, against its dequantised values: the absorbed query reaches the
# tensor cores as an e4m3 + e5m2 pair carrying 7 significant bits against
# bf16's 8 (P * s_t, an e4m3 pair scaled per group, keeps 8 for its largest
# weights), so the relative rounding bound of the scores doubles, and so do
# the bf16 tolerances
TOL = {"bf16": dict(max_abs=2e-2, rel_fro=5e-3), "fp32": dict(max_abs=1e-4, rel_fro=1e-5),
       "fp8": dict(max_abs=4e-2, rel_fro=1e-2)}


def dims_of(wl: Workload):
    return M.dims_for(wl.heads, wl.latent_rank, wl.rope_dim, wl.nope_dim, wl.v_dim, wl.q_len,
                      wl.softmax_scale, wl.dtype, wl.latent_shards, wl.page_size)


def to_device(inputs: dict, device) -> dict:
    return {k: (v.to(device) if torch.is_tensor(v) else v) for k, v in inputs.items()}


def run_gpu(wl: Workload, inputs: dict, device, kernel=M.MLA_KERNEL_AUTO, num_workers=0,
            plan_lens=None, repeat=1, expect_status=0):
    """Runs the decode through the C ABI; returns (out on CPU, plan info)."""
    dev = to_device(inputs, device)
    lens = inputs["seq_lens"].tolist() if plan_lens is None else plan_lens
    plan = M.DecodePlan(dims_of(wl), lens, kernel=kernel, num_workers=num_workers)
    plan.allocate_workspace(device)
    B = len(inputs["seq_lens"])
    out = torch.full((B, wl.q_len, wl.heads, wl.v_dim), float("nan"), dtype=wl.torch_dtype,
                     device=device)
    for _ in range(repeat):
        if wl.dtype == "fp8":
            plan.run_fp8(dev["q_nope"], dev["q_rope"], dev["kv_codes"], dev["kv_rope"], dev["kv_scale"],
                         dev["block_table"], dev["seq_lens"], dev["w_uk"], dev["w_uv"], out)
        else:
            plan.run(dev["q_nope"], dev["q_rope"], dev["kv_pool"], dev["block_table"],
                     dev["seq_lens"], dev["w_uk"], dev["w_uv"], out)
    torch.cuda.synchronize(device)
    status = plan.read_status()
    assert status == expect_status, M.mla_status_string(status)
    info = plan.info
    plan.close()
    return out.cpu(), info


def oracle_out(wl: Workload, inputs: dict, batch_indices=None, heads=None) -> np.ndarray:
    """fp64 oracle on the same (bf16 or fp32) values, widened exactly."""
    B = len(inputs["seq_lens"])
    bs = list(range(B)) if batch_indices is None else list(batch_indices)
    ckv, kr = {}, {}
    for b in bs:
        if wl.dtype == "fp8":
            codes, rope, scale = stored_rows_fp8(inputs, b, wl)
            ckv[b], kr[b] = fp8_cache.logical_cache_fp8(codes.numpy(), rope.double().numpy(),
                                                        scale.double().numpy())
        else:
            c, k = logical_cache(inputs, b, wl)
            ckv[b], kr[b] = c.double().numpy(), k.double().numpy()
    return mla_oracle.mla_decode(inputs["q_nope"].double().numpy(),
                                 inputs["q_rope"].double().numpy(), ckv, kr,
                                 inputs["w_uk"].double().numpy(), inputs["w_uv"].double().numpy(),
                                 wl.softmax_scale, wl.latent_shards, bs, heads)


def errors(got: np.ndarray, ref: np.ndarray):
    got = np.asarray(got, dtype=np.float64)
    diff = got - ref
    return float(np.abs(diff).max()), float(np.linalg.norm(diff) / np.linalg.norm(ref))


def assert_close(got, ref, dtype: str, what: str = ""):
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    max_abs, rel = errors(got, ref)
    tol = TOL[dtype]
    assert max_abs <= tol["max_abs"] and rel <= tol["rel_fro"], (
        f"{what}: max_abs {max_abs:.3e} (tol {tol['max_abs']}), rel_fro {rel:.3e} "
        f"(tol {tol['rel_fro']})")
    return max_abs, rel
