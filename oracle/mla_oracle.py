"""CPU oracle for MLA decode over a compressed latent KV cache.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may use it.

What it computes is the plain, non-absorbed definition of one MLA decode step
(numpy, float64 throughout):

* Multi-Head Latent Attention caches only a low-rank latent cKV per token plus
  a decoupled RoPE key shared by all heads (TPLA abstract, on the
  taxoreview listing pages; "TransMLA: Multi-Head Latent Attention Is All You
  Need", abstract; pith.science verdict record for 2502.07864, core_discovery:
  one RoPE key per token, common to every head as in multi-query attention).
* Per head h the keys and values are recovered through up-projections,
  K_h = [cKV . W_UK[h]^T || k_rope] and V_h = cKV . W_UV[h] (TransMLA v1
  abstract on the kk6lht.com listing: keys and values are recovered from the
  latent by an up-projection).
  W_UK[h] is stored [d_nope, r] and W_UV[h] is stored [r, d_v].
* Scores are scale * q . K_h[j] with q = [q_nope || q_rope]; query token t of
  Lq sees keys j <= L - Lq + t (the Lq query tokens are the newest Lq cache
  rows, multi-token-prediction style; Lq = 1 sees every key).
* Softmax over the visible keys, then out = p . V_h.
* TPLA: the latent dimension (and each head's W_UK / W_UV along it) is split
  into shards, attention runs independently per shard with the full RoPE term
  in every shard, and the shard outputs are summed (TPLA abstract).

The absorbed form that the GPU path uses reaches the same function by
associativity (q_nope . (cKV W_UK^T)^T = (q_nope W_UK) . cKV^T and
(p . cKV) W_UV = p . (cKV W_UV)); TransMLA's abstract names this the Absorb
operation and the verdict record's key_machinery calls it exact. The oracle
deliberately does not use it: it materialises K and V.

Pins (tests/test_oracle_pins.py): brute-force scalar loops on tiny inputs,
the absorb identity, GQA as an MLA with selector up-projections, RoPE-pair and
cross-head rotation invariance, closed forms (zero query, single key, one
dominant key), the MTP causal reduction and the TPLA shard sum.
"""

from __future__ import annotations

from typing import Iterable, Optional, Sequence

import numpy as np

__all__ = [
    "materialise_kv",
    "softmax_attention",
    "mla_decode",
    "mla_decode_rows",
    "mla_prefill",
    "mla_decode_blasst",
]


def materialise_kv(ckv: np.ndarray, k_rope: np.ndarray, w_uk_h: np.ndarray,
                   w_uv_h: np.ndarray):
    """Up-project one sequence's latent cache for one head.

    ckv [L, r], k_rope [L, dr], w_uk_h [dn, r], w_uv_h [r, dv]
    -> K [L, dn + dr], V [L, dv]
    """
    k_nope = ckv @ w_uk_h.T
    k = np.concatenate([k_nope, k_rope], axis=1)
    v = ckv @ w_uv_h
    return k, v


def softmax_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                      n_visible: int) -> np.ndarray:
    """Textbook softmax attention of one query over the first n_visible keys."""
    s = scale * (k[:n_visible] @ q)
    s = s - s.max()
    p = np.exp(s)
    p = p / p.sum()
    return p @ v[:n_visible]


def _shard_columns(r: int, shards: int, s: int) -> slice:
    w = r // shards
    return slice(s * w, (s + 1) * w)


def mla_decode_rows(q_nope_b: np.ndarray, q_rope_b: np.ndarray, ckv: np.ndarray,
                    k_rope: np.ndarray, w_uk: np.ndarray, w_uv: np.ndarray,
                    scale: float, heads: Iterable[int], latent_shards: int = 1
                    ) -> np.ndarray:
    """Decode of one sequence for the listed heads.

    q_nope_b [Lq, H, dn], q_rope_b [Lq, H, dr], ckv [L, r], k_rope [L, dr],
    w_uk [H, dn, r], w_uv [H, r, dv]  ->  [Lq, len(heads), dv]
    """
    heads = list(heads)
    Lq = q_nope_b.shape[0]
    L, r = ckv.shape
    dv = w_uv.shape[2]
    out = np.zeros((Lq, len(heads), dv), dtype=np.float64)
    for hi, h in enumerate(heads):
        for s in range(latent_shards):
            cols = _shard_columns(r, latent_shards, s)
            k, v = materialise_kv(ckv[:, cols], k_rope, w_uk[h][:, cols], w_uv[h][cols, :])
            for t in range(Lq):
                q = np.concatenate([q_nope_b[t, h], q_rope_b[t, h]])
                n_visible = L - Lq + t + 1
                out[t, hi] += softmax_attention(q, k, v, scale, n_visible)
    return out


def mla_decode(q_nope: np.ndarray, q_rope: np.ndarray, ckv_seqs: Sequence[np.ndarray],
               krope_seqs: Sequence[np.ndarray], w_uk: np.ndarray, w_uv: np.ndarray,
               scale: float, latent_shards: int = 1,
               batch_indices: Optional[Iterable[int]] = None,
               heads: Optional[Iterable[int]] = None) -> np.ndarray:
    """Non-absorbed MLA (or TPLA when latent_shards > 1) decode.

    q_nope [B, Lq, H, dn], q_rope [B, Lq, H, dr]; ckv_seqs[b] [L_b, r] and
    krope_seqs[b] [L_b, dr] are indexed by the batch position b;
    w_uk [H, dn, r], w_uv [H, r, dv].
    Returns [len(batch_indices), Lq, len(heads), dv] (all of them by default).
    """
    B, Lq, H, _ = q_nope.shape
    bs = list(range(B)) if batch_indices is None else list(batch_indices)
    hs = list(range(H)) if heads is None else list(heads)
    out = np.zeros((len(bs), Lq, len(hs), w_uv.shape[2]), dtype=np.float64)
    for bi, b in enumerate(bs):
        out[bi] = mla_decode_rows(q_nope[b], q_rope[b], ckv_seqs[b], krope_seqs[b],
                                  w_uk, w_uv, scale, hs, latent_shards)
    return out


def mla_prefill(q_nope: np.ndarray, q_rope: np.ndarray, kv_rows: np.ndarray,
                cu_seqlens: Sequence[int], w_uk: np.ndarray, w_uv: np.ndarray, scale: float,
                pairs: Optional[Iterable] = None, abs_weighted: bool = False):
    """Causal prefill in the MLA (non-absorbed) form over concatenated prompts.

    TPLA abstract: prefill keeps the MLA form. Every prompt token is a query
    over the prompt's own tokens up to itself; per head the keys and values
    are materialised from the latent rows exactly as in mla_decode.

    q_nope [T, H, dn], q_rope [T, H, dr], kv_rows [T, r + dr] (cKV columns
    [0, r), the RoPE key after them), cu_seqlens [B + 1] (sequence b owns rows
    [cu[b], cu[b+1])), w_uk [H, dn, r], w_uv [H, r, dv]. pairs: (token row,
    head) pairs to compute, all of them by default. Returns [len(pairs), dv];
    with abs_weighted, also sum_j p_j |V_j| per row (the scale of any error
    that rounds the values key by key), [len(pairs), dv].
    """
    T, H, _ = q_nope.shape
    r = w_uk.shape[2]
    cu = [int(x) for x in cu_seqlens]
    if pairs is None:
        pairs = [(t, h) for t in range(T) for h in range(H)]
    pairs = list(pairs)
    out = np.zeros((len(pairs), w_uv.shape[2]), dtype=np.float64)
    aw = np.zeros_like(out)
    groups = {}
    for i, (t, h) in enumerate(pairs):
        b = max(k for k in range(len(cu) - 1) if cu[k] <= t)
        groups.setdefault((b, h), []).append((i, t))
    for (b, h), items in groups.items():
        rows = kv_rows[cu[b]:cu[b + 1]]
        k, v = materialise_kv(rows[:, :r], rows[:, r:], w_uk[h], w_uv[h])
        for i, t in items:
            q = np.concatenate([q_nope[t, h], q_rope[t, h]])
            n = t - cu[b] + 1
            out[i] = softmax_attention(q, k, v, scale, n)
            if abs_weighted:
                aw[i] = softmax_attention(q, k, np.abs(v), scale, n)
    return (out, aw) if abs_weighted else out


def mla_decode_blasst(q_nope_b: np.ndarray, q_rope_b: np.ndarray, ckv: np.ndarray,
                      k_rope: np.ndarray, w_uk: np.ndarray, w_uv: np.ndarray, scale: float,
                      segments: Sequence, skip_log2: float, group_keys: int = 256):
    """Decode of one sequence (every head) with threshold skipping of key blocks.

    BLASST abstract (kk6lht.com "GQA-to-MLA" listing): a fixed threshold and the
    running maximum that the online softmax keeps identify negligible scores;
    for them the exponentials, the value loads and the products with the values
    are skipped. Read here for a blocked decode:

    * the keys of the sequence are split into segments (``segments``: (first
      key, end key) pairs, in key order, covering [0, L)), each processed with
      its own running maxima; a segment's blocks are its consecutive runs of
      ``group_keys`` keys from its first key (the last one shorter);
    * for every query row (t, h), s_j = scale * q . K_h[j] over the keys it
      may see (j <= L - Lq + t); its block maximum and running maximum are taken
      in log2 units (s * log2 e);
    * a row keeps a block when it sees a key there and either its running
      maximum is still -inf or the block maximum is at least the running
      maximum + skip_log2; a block is skipped when no row keeps it;
    * every row's running maximum then takes the block maximum (a skipped
      block's maxima are below it, so skipping leaves it unchanged);
    * out = softmax over the row's visible keys in kept blocks, times V_h.

    q_nope_b [Lq, H, dn], q_rope_b [Lq, H, dr], ckv [L, r], k_rope [L, dr],
    w_uk [H, dn, r], w_uv [H, r, dv]. Returns (out [Lq, H, dv], kept [blocks],
    margin [blocks]) with margin = the largest row value of block max - running
    max - skip_log2 (the decision's distance from the threshold; +inf where a row
    with no running maximum yet keeps the block).
    """
    Lq, H, _ = q_nope_b.shape
    L = ckv.shape[0]
    dv = w_uv.shape[2]
    log2e = 1.0 / np.log(2.0)
    scores = np.full((Lq, H, L), -np.inf)
    values = []
    for h in range(H):
        k, v = materialise_kv(ckv, k_rope, w_uk[h], w_uv[h])
        values.append(v)
        for t in range(Lq):
            n = L - Lq + t + 1
            q = np.concatenate([q_nope_b[t, h], q_rope_b[t, h]])
            scores[t, h, :n] = scale * (k[:n] @ q)
    s2 = scores * log2e
    included = np.zeros(L, dtype=bool)
    kept, margins = [], []
    for k0, k1 in segments:
        runmax = np.full((Lq, H), -np.inf)
        for g0 in range(k0, k1, group_keys):
            g1 = min(g0 + group_keys, k1)
            bm = s2[:, :, g0:g1].max(axis=2)
            seen = np.isfinite(bm)
            first = seen & np.isneginf(runmax)
            cmp = np.where(seen & ~first, bm - runmax - skip_log2, -np.inf)
            keep = bool(first.any() or (cmp >= 0).any())
            kept.append(keep)
            margins.append(np.inf if first.any() else float(cmp.max()))
            runmax = np.maximum(runmax, bm)
            if keep:
                included[g0:g1] = True
    out = np.zeros((Lq, H, dv))
    for t in range(Lq):
        n = L - Lq + t + 1
        mask = included[:n]
        for h in range(H):
            s = scores[t, h, :n][mask]
            p = np.exp(s - s.max())
            out[t, h] = (p / p.sum()) @ values[h][:n][mask]
    return out, np.array(kept), np.array(margins)
