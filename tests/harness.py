"""Shared test helpers: run the CUDA path through the C ABI and the CPU oracle
on the same seeded inputs, and compare them with the stated tolerances."""

from __future__ import annotations

import math

import numpy as np
import torch

import mla_latent_kv_21_b200 as M
from mla_workloads import Workload, generate, logical_cache, stored_rows_fp8
from oracle import fp8_cache, mla_oracle

# ---------------------------------------------------------------------------
# Error model of the tensor-core paths (bf16 cache and FP8 cache), from the
# precision of each rounding step alone. Round-to-nearest-even with unit
# roundoff u (2^-8 bf16, 2^-11 f16, 2^-4 e4m3, 2^-3 e5m2) has an rms relative
# error of RHO * u for significands spread log-uniformly over [1, 2):
# E[(err/x)^2] = u^2 E[1/m^2] / 3 with E[1/m^2] = 3 / (8 ln 2). Each step's
# rms relative error reaches the output at most at that size (the score
# perturbation of a rounded query moves the output by W_UV^T (scale * error),
# the same fraction of the output as of the query; the value-side roundings
# move it through the W_UV contraction), and independent steps add in
# quadrature:
#   query operand   bf16: RHO u_bf16      FP8: e4m3 + e5m2 of its residual,
#                                              split_rms(4, 3)
#   P operand       bf16: RHO u_bf16      FP8: two e4m3 terms for P' in
#                                              [1/4, 448], p_split_rms(), and
#                                              the f16 step before the split,
#                                              RHO u_f16
#   fp16 partials   RHO u_f16             o_lat (bf16 MMA operand) RHO u_bf16
#   output (bf16)   RHO u_bf16 (rms), at most u_bf16 |out| per element
# Relative Frobenius bound: 1.5x the model's rms (the bf16 bound of 5e-3 that
# the task states is 1.50x its model value). Element-wise bound: the output
# rounding at its worst, u_bf16 |ref|, plus 6 standard deviations of the other
# steps, taken relative to the rms of the reference row (the 128 outputs of
# one sequence, query token and head), which sets their scale.
# ---------------------------------------------------------------------------
E_INV_M2 = 3.0 / (8.0 * math.log(2.0))   # E[1/m^2], m log-uniform on [1, 2)
RHO = math.sqrt(E_INV_M2 / 3.0)
U = {"bf16": 2.0 ** -8, "f16": 2.0 ** -11, "e4m3": 2.0 ** -4, "e5m2": 2.0 ** -3}


def split_rms(p1: int, p2: int) -> float:
    """rms relative error of x ~ hi + lo, hi = x rounded to p1 significant bits
    and lo = the residual rounded to p2 bits (in its normal range). The
    residual is uniform on (-h, h), h = 2^(e - p1) for x in [2^e, 2^(e+1)); a
    residual in binade k (probability 2^k / h) is rounded with an error uniform
    on +-2^(k - p2), so E[err^2] = sum_k (2^k / h) 4^(k - p2) / 3 = 4^-p2 h^2 / 21,
    and relative to x = m 2^e: 2^-(p1 + p2) sqrt(E[1/m^2] / 21)."""
    return 2.0 ** -(p1 + p2) * math.sqrt(E_INV_M2 / 21.0)


def p_split_rms(lo: float = 0.25, hi: float = 448.0, n: int = 20000) -> float:
    """rms relative error of the FP8 path's P' split (hi = e4m3(x), lo =
    e4m3(x - hi)) for x log-uniform on [lo, hi]: as split_rms(4, 4), except
    that a residual below e4m3's smallest normal 2^-6 is rounded on the
    subnormal grid (spacing 2^-9, error uniform on +-2^-10). Midpoint sum over
    log2 x of E[err^2 | binade of x] / x^2."""
    a, b = math.log2(lo), math.log2(hi)
    acc = 0.0
    for i in range(n):
        x = 2.0 ** (a + (b - a) * (i + 0.5) / n)
        e = math.floor(math.log2(x))
        h = 2.0 ** (e - 4)
        m2 = min(h, 2.0 ** -6) / h * 4.0 ** -10 / 3.0
        for k in range(-6, e - 4):
            m2 += (2.0 ** k / h) * 4.0 ** (k - 4) / 3.0
        acc += m2 / (x * x)
    return math.sqrt(acc / n)


MODEL_STEPS = {
    "bf16": {"query": RHO * U["bf16"], "p": RHO * U["bf16"], "partials": RHO * U["f16"],
             "o_lat": RHO * U["bf16"]},
    "fp8": {"query": split_rms(4, 3),
            "p": math.hypot(p_split_rms(), RHO * U["f16"]), "partials": RHO * U["f16"],
            "o_lat": RHO * U["bf16"]},
}
ELEMENT_Z = 6.0


def model_sigma_inner(dtype: str) -> float:
    """rms relative output error of every step but the output rounding."""
    return math.sqrt(sum(v * v for v in MODEL_STEPS[dtype].values()))


def model_rel_rms(dtype: str) -> float:
    """The model's rms relative output error, output rounding included."""
    return math.hypot(model_sigma_inner(dtype), RHO * U["bf16"])


# bf16 inputs with fp32 accumulation: max-abs <= 2e-2 and rel-Frobenius <= 5e-3
# (the stated tolerance; the model predicts 3.3e-3 rms) and, from the model,
# the element-wise bound; the fp32 workload: rel-Frobenius <= 1e-5. FP8 cache,
# against its dequantised values: rel-Frobenius <= 1.5x its model rms (2.8e-3)
# and the element-wise bound; its largest errors sit on rows with few keys and
# |out| of order 1, where the bf16 output rounding alone is u_bf16 |out|, so it
# has no absolute max-abs bound.
TOL = {"bf16": dict(max_abs=2e-2, rel_fro=5e-3, elementwise=True),
       "fp32": dict(max_abs=1e-4, rel_fro=1e-5, elementwise=False),
       "fp8": dict(max_abs=None, rel_fro=1.5 * model_rel_rms("fp8"), elementwise=True)}


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


def elementwise_ratio(got, ref, dtype: str) -> float:
    """max over elements of |got - ref| / (u_bf16 |ref| + z sigma rms_row(ref)),
    rows along the last axis; <= 1 passes the model's element-wise bound."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms_row = np.sqrt(np.mean(ref * ref, axis=-1, keepdims=True))
    bound = U["bf16"] * np.abs(ref) + ELEMENT_Z * model_sigma_inner(dtype) * rms_row
    return float(np.max(np.abs(got - ref) / bound))


def assert_close(got, ref, dtype: str, what: str = ""):
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    max_abs, rel = errors(got, ref)
    tol = TOL[dtype]
    ok = rel <= tol["rel_fro"] and (tol["max_abs"] is None or max_abs <= tol["max_abs"])
    ratio = elementwise_ratio(got, ref, dtype) if tol["elementwise"] else 0.0
    assert ok and ratio <= 1.0, (
        f"{what}: max_abs {max_abs:.3e} (tol {tol['max_abs']}), rel_fro {rel:.3e} "
        f"(tol {tol['rel_fro']:.3e}), element-wise bound ratio {ratio:.3f} (tol 1)")
    return max_abs, rel


# Prefill (MLA form) has its own rounding steps: K_nope and V are materialised
# in bf16 (the scores' and the values' roundings, key by key), P is bf16 and
# the output bf16; q, k_rope and the latent rows are exact inputs. Rounding V
# key by key moves an output element by at most u_bf16 sum_j p_j |V_j| (the
# oracle's abs_weighted); the K_nope and P roundings are random terms of rms
# RHO u_bf16 each relative to the row (as in the decode model). Element-wise
# bound: u_bf16 |ref| + u_bf16 sum_j p_j |V_j| + ELEMENT_Z sigma rms(ref row),
# sigma = hypot(RHO u, RHO u). Relative Frobenius and max-abs: the stated bf16
# bounds.
PREFILL_SIGMA = math.hypot(RHO * U["bf16"], RHO * U["bf16"])


def assert_close_prefill(got, ref, abs_weighted, what: str = ""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    max_abs, rel = errors(got, ref)
    rms_row = np.sqrt(np.mean(ref * ref, axis=-1, keepdims=True))
    bound = U["bf16"] * (np.abs(ref) + np.asarray(abs_weighted)) + ELEMENT_Z * PREFILL_SIGMA * rms_row
    ratio = float(np.max(np.abs(got - ref) / bound))
    tol = TOL["bf16"]
    assert rel <= tol["rel_fro"] and max_abs <= tol["max_abs"] and ratio <= 1.0, (
        f"{what}: max_abs {max_abs:.3e} (tol {tol['max_abs']}), rel_fro {rel:.3e} (tol {tol['rel_fro']}), "
        f"element-wise bound ratio {ratio:.3f} (tol 1)")
    return max_abs, rel
