"""Seeded synthetic inputs for MLA latent-cache decode.

This module only draws random numbers and lays them out in memory (a paged
latent pool plus a block table). It holds none of the attention arithmetic, so
both the CPU oracle (via the tests) and the CUDA path can consume the same
inputs without sharing any of the method's code.

Workloads (shapes as the TransMLA / TPLA pages describe the models; values are
synthetic because no trained weights are available):

* ``tiny``        fp32, 8 heads, r=64, rope 16, nope 32, v 32, L=256, contiguous
* ``llama2_7b``   bf16, TransMLA-converted LLaMA-2-7B shape: 32 heads, r=512,
                  rope 64, nope 128, v 128 (576 cached values per token against
                  8192 for the GQA original), B=16, L=8192, paged
* ``deepseek_v3`` bf16, 128 heads, r=512, rope 64, nope 128, v 128, B=32,
                  L=32768, paged
* ``kimi_k2_mtp`` bf16, 64 heads, same dims, 64 sequences with L uniform in
                  [1024, 32768], 2 causal query tokens per sequence, paged
* ``tpla_dsv3``   bf16, DeepSeek-V3 shape with the latent split into 2 shards
                  (TPLA), B=32, L=32768, paged
* ``deepseek_v3_peaked`` the DeepSeek-V3 shape with peaked attention (a quarter
                  of the tokens, in runs of 1024, relevant to every query;
                  PEAK_* below): the threshold-skipping workload
* ``deepseek_v3_fp8`` the DeepSeek-V3 shape over an FP8 latent cache: cKV as
                  E4M3 codes with one fp32 scale per token, the RoPE key bf16
                  stored divided by the token's scale; activations and weights
                  bf16

Recipe (every draw is float32 N(0, 1) from ``torch.Generator`` seeded per
tensor, then scaled and cast to the workload dtype with round-to-nearest-even):

* per-tensor seeds: ``seed * 1_000_003 + tag`` with a fixed tag per tensor;
  the latent rows of sequence ``b`` use tag ``100 + b`` so that any subset of
  sequences can be regenerated on its own;
* lengths (varlen only): integers uniform in [lo, hi] inclusive;
* q_nope [B, Lq, H, dn], q_rope [B, Lq, H, dr] ~ N(0, 1) (q_rope stands for the
  query after RoPE; decode applies no rotation);
* per sequence, one [L_b, r + dr] block ~ N(0, 1): columns [0, r) are cKV,
  columns [r, r + dr) are the (already rotated) decoupled RoPE key;
* W_UK [H, dn, r] and W_UV [H, r, dv] ~ N(0, 1/r) with r the full latent rank;
* the pool has sum_b ceil(L_b / P) blocks of P = 64 tokens; paged workloads
  place logical page (b, i) at a block chosen by a seeded random permutation,
  contiguous ones at the identity position. Unused table entries are -1 and
  the tail of a partial page is zero.

FP8 cache (``dtype="fp8"``): the same per-sequence N(0, 1) block, times 32, is
cast to E4M3 codes with torch's own conversion (columns [0, r)) and to bf16
(columns [r, r + dr), the stored RoPE key); each token's scale is uniform in
[1/48, 1/24] (tag ``200 + b``). The logical cache is s_t * code and
s_t * stored RoPE key; the CPU oracle decodes it (``oracle/fp8_cache.py``).
The pool is three tensors: kv_codes uint8 [blocks, P, r], kv_rope bf16
[blocks, P, dr] and kv_scale float32 [blocks, P] (zero in unused slots).
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import torch

__all__ = ["Workload", "WORKLOADS", "generate", "logical_cache", "pages_of", "stored_rows_fp8",
           "tpla_shard_columns", "tpla_shard_inputs", "PREFILL_WORKLOADS", "generate_prefill"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    batch: int
    q_len: int
    heads: int
    latent_rank: int
    rope_dim: int
    nope_dim: int
    v_dim: int
    context: int            # fixed length, or the upper bound when varlen
    context_min: int = 0    # > 0 selects uniform integer lengths in [context_min, context]
    latent_shards: int = 1
    dtype: str = "bf16"     # "bf16", "fp32" or "fp8" (FP8 cache, bf16 activations)
    paged: bool = True      # False: identity block table (contiguous cache)
    page_size: int = 64
    peaked: bool = False    # True: clustered relevant keys (see PEAK_* below)

    @property
    def softmax_scale(self) -> float:
        # 1/sqrt(d_qk) with d_qk = nope + rope dims of the non-absorbed head
        return 1.0 / math.sqrt(self.nope_dim + self.rope_dim)

    @property
    def row_width(self) -> int:
        return self.latent_rank + self.rope_dim

    @property
    def torch_dtype(self) -> torch.dtype:
        """Activations, weights and output."""
        return torch.float32 if self.dtype == "fp32" else torch.bfloat16

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", seed=0, batch=1, q_len=1, heads=8, latent_rank=64,
                     rope_dim=16, nope_dim=32, v_dim=32, context=256,
                     dtype="fp32", paged=False),
    "llama2_7b": Workload("llama2_7b", seed=1, batch=16, q_len=1, heads=32,
                          latent_rank=512, rope_dim=64, nope_dim=128, v_dim=128,
                          context=8192),
    "deepseek_v3": Workload("deepseek_v3", seed=2, batch=32, q_len=1, heads=128,
                            latent_rank=512, rope_dim=64, nope_dim=128, v_dim=128,
                            context=32768),
    "kimi_k2_mtp": Workload("kimi_k2_mtp", seed=3, batch=64, q_len=2, heads=64,
                            latent_rank=512, rope_dim=64, nope_dim=128, v_dim=128,
                            context=32768, context_min=1024),
    "tpla_dsv3": Workload("tpla_dsv3", seed=4, batch=32, q_len=1, heads=128,
                          latent_rank=512, rope_dim=64, nope_dim=128, v_dim=128,
                          context=32768, latent_shards=2),
    "deepseek_v3_fp8": Workload("deepseek_v3_fp8", seed=5, batch=32, q_len=1, heads=128,
                                latent_rank=512, rope_dim=64, nope_dim=128, v_dim=128,
                                context=32768, dtype="fp8"),
    "deepseek_v3_peaked": Workload("deepseek_v3_peaked", seed=7, batch=32, q_len=1, heads=128,
                                   latent_rank=512, rope_dim=64, nope_dim=128, v_dim=128,
                                   context=32768, peaked=True),
}

# Peaked attention (threshold-skipping workload). Synthetic N(0, 1) data gives
# nearly flat attention; the pages' workloads are peaked. Here the tokens at
# positions j with (j // PEAK_RUN) % PEAK_PERIOD == 0 (a quarter, in runs of
# 1024) are relevant: their RoPE key is PEAK_KEEP * N(0, 1) + PEAK_GAIN * u,
# every other token's RoPE key stays N(0, 1), and every query's RoPE part is
# N(0, 1) + PEAK_GAIN * u, with u a seeded +-1 vector. A relevant key then
# scores about scale * PEAK_GAIN^2 * d_rope (~10.4 at d_rope = 64, scale
# 1/sqrt(192)) above an irrelevant one, for every head.
PEAK_RUN, PEAK_PERIOD, PEAK_GAIN, PEAK_KEEP = 1024, 4, 1.5, 0.5
_TAG_PEAK = 9


def peak_direction(wl: Workload) -> torch.Tensor:
    g = _gen(wl.seed, _TAG_PEAK)
    return (torch.randint(0, 2, (wl.rope_dim,), generator=g) * 2 - 1).to(torch.float32)


def relevant_tokens(length: int) -> torch.Tensor:
    return (torch.arange(length) // PEAK_RUN) % PEAK_PERIOD == 0

_TAG_LENS, _TAG_QN, _TAG_QR, _TAG_WUK, _TAG_WUV, _TAG_PERM = 1, 2, 3, 4, 5, 6
_TAG_SEQ0 = 100
_TAG_SCALE0 = 200
FP8_CODE_STD = 32.0                      # std of the values cast to E4M3 codes
FP8_SCALE_RANGE = (1.0 / 48.0, 1.0 / 24.0)


def _gen(seed: int, tag: int) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed(seed * 1_000_003 + tag)
    return g


def pages_of(length: int, page_size: int) -> int:
    return (length + page_size - 1) // page_size


def draw_lengths(wl: Workload) -> torch.Tensor:
    if wl.context_min > 0:
        g = _gen(wl.seed, _TAG_LENS)
        return torch.randint(wl.context_min, wl.context + 1, (wl.batch,),
                             generator=g, dtype=torch.int64).to(torch.int32)
    return torch.full((wl.batch,), wl.context, dtype=torch.int32)


def draw_sequence_rows(wl: Workload, b: int, length: int) -> torch.Tensor:
    """[length, r + dr] latent rows of sequence b in the workload dtype."""
    g = _gen(wl.seed, _TAG_SEQ0 + b)
    x = torch.randn((length, wl.row_width), generator=g, dtype=torch.float32)
    if wl.peaked:
        rel = relevant_tokens(length)
        x[rel, wl.latent_rank:] = PEAK_KEEP * x[rel, wl.latent_rank:] + PEAK_GAIN * peak_direction(wl)
    return x.to(wl.torch_dtype)


def generate(wl: Workload, seq_lens: Optional[Sequence[int]] = None,
             with_pool: bool = True) -> dict:
    """All decode inputs as CPU tensors.

    ``seq_lens`` overrides the workload's lengths (reduced-size parity cases).
    Returns q_nope, q_rope, w_uk, w_uv, seq_lens (int32), and when
    ``with_pool``: kv_pool [num_blocks, P, r + dr], block_table [B, max_pages]
    (int32, -1 where unused), num_blocks.
    """
    if seq_lens is None:
        lens = draw_lengths(wl)
    else:
        lens = torch.as_tensor(list(seq_lens), dtype=torch.int32)
    B = int(lens.numel())
    dt = wl.torch_dtype
    r, dr, dn, dv, H, Lq = (wl.latent_rank, wl.rope_dim, wl.nope_dim, wl.v_dim,
                            wl.heads, wl.q_len)
    out = {"seq_lens": lens}
    out["q_nope"] = torch.randn((B, Lq, H, dn), generator=_gen(wl.seed, _TAG_QN)).to(dt)
    qr = torch.randn((B, Lq, H, dr), generator=_gen(wl.seed, _TAG_QR))
    if wl.peaked:
        qr = qr + PEAK_GAIN * peak_direction(wl)
    out["q_rope"] = qr.to(dt)
    wstd = 1.0 / math.sqrt(r)
    out["w_uk"] = (torch.randn((H, dn, r), generator=_gen(wl.seed, _TAG_WUK)) * wstd).to(dt)
    out["w_uv"] = (torch.randn((H, r, dv), generator=_gen(wl.seed, _TAG_WUV)) * wstd).to(dt)
    if not with_pool:
        return out

    P = wl.page_size
    if wl.dtype == "fp8":
        return _fp8_pool(wl, lens, out)
    npages = [pages_of(int(L), P) for L in lens.tolist()]
    total = sum(npages)
    max_pages = max(npages) if npages else 0
    if wl.paged:
        perm = torch.randperm(total, generator=_gen(wl.seed, _TAG_PERM)).to(torch.int32)
    else:
        perm = torch.arange(total, dtype=torch.int32)
    table = torch.full((B, max(max_pages, 1)), -1, dtype=torch.int32)
    pool = torch.zeros((total, P, wl.row_width), dtype=dt)
    base = 0
    for b, L in enumerate(lens.tolist()):
        n = npages[b]
        ids = perm[base:base + n]
        table[b, :n] = ids
        rows = draw_sequence_rows(wl, b, L)
        padded = torch.zeros((n * P, wl.row_width), dtype=dt)
        padded[:L] = rows
        pool[ids.long()] = padded.view(n, P, wl.row_width)
        base += n
    out["kv_pool"] = pool
    out["block_table"] = table
    out["num_blocks"] = total
    return out


def _fp8_pool(wl: Workload, lens: torch.Tensor, out: dict) -> dict:
    P, r, dr = wl.page_size, wl.latent_rank, wl.rope_dim
    B = int(lens.numel())
    npages = [pages_of(int(L), P) for L in lens.tolist()]
    total = sum(npages)
    perm = torch.randperm(total, generator=_gen(wl.seed, _TAG_PERM)).to(torch.int32)
    table = torch.full((B, max(max(npages) if npages else 0, 1)), -1, dtype=torch.int32)
    codes = torch.zeros((total, P, r), dtype=torch.uint8)
    rope = torch.zeros((total, P, dr), dtype=torch.bfloat16)
    scale = torch.zeros((total, P), dtype=torch.float32)
    lo, hi = FP8_SCALE_RANGE
    base = 0
    for b, L in enumerate(lens.tolist()):
        n = npages[b]
        ids = perm[base:base + n]
        table[b, :n] = ids
        x = torch.randn((L, wl.row_width), generator=_gen(wl.seed, _TAG_SEQ0 + b),
                        dtype=torch.float32) * FP8_CODE_STD
        c = torch.zeros((n * P, r), dtype=torch.uint8)
        c[:L] = x[:, :r].to(torch.float8_e4m3fn).view(torch.uint8)
        k = torch.zeros((n * P, dr), dtype=torch.bfloat16)
        k[:L] = x[:, r:].to(torch.bfloat16)
        sc = torch.zeros(n * P, dtype=torch.float32)
        sc[:L] = lo + (hi - lo) * torch.rand(L, generator=_gen(wl.seed, _TAG_SCALE0 + b))
        codes[ids.long()] = c.view(n, P, r)
        rope[ids.long()] = k.view(n, P, dr)
        scale[ids.long()] = sc.view(n, P)
        base += n
    out["kv_codes"], out["kv_rope"], out["kv_scale"] = codes, rope, scale
    out["block_table"] = table
    out["num_blocks"] = total
    return out


def stored_rows_fp8(inputs: dict, b: int, wl: Workload):
    """(codes uint8 [L_b, r], stored RoPE key bf16 [L_b, dr], scales [L_b]) of
    sequence b, gathered from the FP8 pool (layout only, no arithmetic)."""
    L = int(inputs["seq_lens"][b])
    P = wl.page_size
    n = pages_of(L, P)
    ids = inputs["block_table"][b, :n].long()
    codes = inputs["kv_codes"][ids].reshape(n * P, wl.latent_rank)[:L]
    rope = inputs["kv_rope"][ids].reshape(n * P, wl.rope_dim)[:L]
    scale = inputs["kv_scale"][ids].reshape(n * P)[:L]
    return codes, rope, scale


def logical_cache(inputs: dict, b: int, wl: Workload):
    """(cKV [L_b, r], k_rope [L_b, dr]) of sequence b, gathered from the pool."""
    L = int(inputs["seq_lens"][b])
    P = wl.page_size
    n = pages_of(L, P)
    ids = inputs["block_table"][b, :n].long()
    rows = inputs["kv_pool"][ids].reshape(n * P, wl.row_width)[:L]
    return rows[:, :wl.latent_rank], rows[:, wl.latent_rank:]


def tpla_shard_columns(latent_rank: int, tp: int, g: int) -> slice:
    """Latent columns of shard g of tp equal shards."""
    w = latent_rank // tp
    return slice(g * w, (g + 1) * w)


def tpla_shard_inputs(inputs: dict, wl: Workload, tp: int, g: int) -> dict:
    """The inputs one GPU of a tp-way TPLA group holds (layout only): the pool
    rows with cKV narrowed to shard g's latent columns, followed by the full
    RoPE key, [blocks, P, r / tp + dr]; W_UK[h][:, cols] and W_UV[h][cols, :];
    queries, block table and lengths unchanged."""
    cols = tpla_shard_columns(wl.latent_rank, tp, g)
    pool = inputs["kv_pool"]
    out = dict(inputs)
    out["kv_pool"] = torch.cat([pool[..., cols], pool[..., wl.latent_rank:]], dim=-1).contiguous()
    out["w_uk"] = inputs["w_uk"][:, :, cols].contiguous()
    out["w_uv"] = inputs["w_uv"][:, cols, :].contiguous()
    return out


# Prefill workloads (MLA form; the prompt attends to itself causally): the
# DeepSeek-V3 attention shape on prompts of 8K tokens.
PREFILL_WORKLOADS = {
    "deepseek_v3_prefill": Workload("deepseek_v3_prefill", seed=6, batch=2, q_len=1, heads=128,
                                    latent_rank=512, rope_dim=64, nope_dim=128, v_dim=128,
                                    context=8192),
}
_TAG_PQN, _TAG_PQR = 7, 8


def generate_prefill(wl: Workload, seq_lens: Optional[Sequence[int]] = None) -> dict:
    """Prefill inputs as CPU tensors: the prompts' tokens concatenated.

    q_nope [T, H, dn], q_rope [T, H, dr] ~ N(0, 1); kv_rows [T, r + dr] (the
    prompts' latent rows: per sequence the same N(0, 1) draw as a decode
    workload's cache rows); W_UK, W_UV ~ N(0, 1/r); seq_lens int32 [B];
    cu_seqlens int32 [B + 1] (prefix sums)."""
    lens = draw_lengths(wl) if seq_lens is None else torch.as_tensor(list(seq_lens), dtype=torch.int32)
    T = int(lens.sum())
    dt = wl.torch_dtype
    r, dr, dn, dv, H = wl.latent_rank, wl.rope_dim, wl.nope_dim, wl.v_dim, wl.heads
    out = {"seq_lens": lens}
    cu = torch.zeros(len(lens) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(lens, 0)
    out["cu_seqlens"] = cu
    out["q_nope"] = torch.randn((T, H, dn), generator=_gen(wl.seed, _TAG_PQN)).to(dt)
    out["q_rope"] = torch.randn((T, H, dr), generator=_gen(wl.seed, _TAG_PQR)).to(dt)
    wstd = 1.0 / math.sqrt(r)
    out["w_uk"] = (torch.randn((H, dn, r), generator=_gen(wl.seed, _TAG_WUK)) * wstd).to(dt)
    out["w_uv"] = (torch.randn((H, r, dv), generator=_gen(wl.seed, _TAG_WUV)) * wstd).to(dt)
    out["kv_rows"] = torch.cat([draw_sequence_rows(wl, b, int(L)) for b, L in enumerate(lens.tolist())], 0)
    return out
