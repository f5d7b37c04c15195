"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test ties the oracle to something the pages or plain mathematics fix:
brute-force scalar evaluation on tiny inputs, the absorb identity (TransMLA
abstract; verdict record key_machinery), GQA as a special case of MLA (TransMLA
v1 abstract; verdict record core_discovery), rotation invariance inside RoPE
frequency subspaces (verdict record skeptic_critique.rationale on Appendix B),
closed forms, the multi-token-prediction causal reduction and the TPLA shard
sum (TPLA abstract). A mutation test at the end plants plausible mistakes in
the oracle and checks that these pins catch each one.
"""

import json
import math
import os

import numpy as np
import torch
import pytest

from oracle import mla_oracle as mo

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_problem(rng, B=2, Lq=2, H=3, r=8, dr=2, dn=3, dv=4, lens=(7, 5)):
    q_nope = rng.standard_normal((B, Lq, H, dn))
    q_rope = rng.standard_normal((B, Lq, H, dr))
    ckv = [rng.standard_normal((L, r)) for L in lens]
    kr = [rng.standard_normal((L, dr)) for L in lens]
    w_uk = rng.standard_normal((H, dn, r)) / math.sqrt(r)
    w_uv = rng.standard_normal((H, r, dv)) / math.sqrt(r)
    return q_nope, q_rope, ckv, kr, w_uk, w_uv


def _brute(q_nope, q_rope, ckv, kr, w_uk, w_uv, scale, shards=1):
    """Scalar loops straight from the definition (pure Python floats)."""
    B, Lq, H, dn = q_nope.shape
    dr = q_rope.shape[3]
    r, dv = w_uv.shape[1], w_uv.shape[2]
    out = np.zeros((B, Lq, H, dv))
    for b in range(B):
        L = ckv[b].shape[0]
        for t in range(Lq):
            for h in range(H):
                acc = [0.0] * dv
                for s in range(shards):
                    lo, hi = s * r // shards, (s + 1) * r // shards
                    nvis = L - Lq + t + 1
                    scores = []
                    for j in range(nvis):
                        x = 0.0
                        for d in range(dn):
                            kd = 0.0
                            for c in range(lo, hi):
                                kd += float(ckv[b][j, c]) * float(w_uk[h, d, c])
                            x += float(q_nope[b, t, h, d]) * kd
                        for e in range(dr):
                            x += float(q_rope[b, t, h, e]) * float(kr[b][j, e])
                        scores.append(scale * x)
                    mx = max(scores)
                    wts = [math.exp(v - mx) for v in scores]
                    z = sum(wts)
                    for e in range(dv):
                        y = 0.0
                        for j in range(nvis):
                            vj = 0.0
                            for c in range(lo, hi):
                                vj += float(ckv[b][j, c]) * float(w_uv[h, c, e])
                            y += wts[j] / z * vj
                        acc[e] += y
                out[b, t, h] = acc
    return out


@pytest.mark.parametrize("shards", [1, 2])
@pytest.mark.parametrize("Lq", [1, 2])
def test_oracle_matches_brute_force(shards, Lq):
    rng = np.random.default_rng(10 + shards + 3 * Lq)
    prob = _rand_problem(rng, Lq=Lq)
    scale = 1.0 / math.sqrt(3 + 2)
    got = mo.mla_decode(*prob, scale=scale, latent_shards=shards)
    want = _brute(*prob, scale=scale, shards=shards)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-13)


def _absorbed(q_nope, q_rope, ckv, kr, w_uk, w_uv, scale):
    """Absorbed (MQA) form: W_UK folded into the query, P.cKV then W_UV."""
    B, Lq, H, _ = q_nope.shape
    out = np.zeros((B, Lq, H, w_uv.shape[2]))
    for b in range(B):
        L = ckv[b].shape[0]
        q_lat = np.einsum("thd,hdr->thr", q_nope[b], w_uk)
        s = scale * (np.einsum("thr,lr->thl", q_lat, ckv[b])
                     + np.einsum("the,le->thl", q_rope[b], kr[b]))
        for t in range(Lq):
            nvis = L - Lq + t + 1
            st = s[t, :, :nvis]
            p = np.exp(st - st.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            o_lat = p @ ckv[b][:nvis]
            out[b, t] = np.einsum("hr,hrv->hv", o_lat, w_uv)
    return out


def test_absorb_identity():
    rng = np.random.default_rng(1)
    prob = _rand_problem(rng, B=2, Lq=2, H=4, r=32, dr=4, dn=8, dv=6, lens=(40, 33))
    scale = 0.3
    np.testing.assert_allclose(mo.mla_decode(*prob, scale=scale), _absorbed(*prob, scale=scale),
                               rtol=1e-11, atol=1e-13)


def test_gqa_is_mla_with_selector_up_projections():
    """GQA with g KV groups of dim d is an MLA with r = 2gd and 0/1 W_UK/W_UV."""
    rng = np.random.default_rng(2)
    g, d, rep, L, B = 2, 4, 3, 9, 2
    H, r = g * rep, 2 * g * d
    q = rng.standard_normal((B, 1, H, d))
    ks = rng.standard_normal((B, L, g, d))
    vs = rng.standard_normal((B, L, g, d))
    scale = 1.0 / math.sqrt(d)
    # textbook GQA: repeat the KV heads to the query heads
    k_rep = np.repeat(ks, rep, axis=2)
    v_rep = np.repeat(vs, rep, axis=2)
    s = scale * np.einsum("bhd,blhd->bhl", q[:, 0], k_rep)
    p = np.exp(s - s.max(-1, keepdims=True))
    p /= p.sum(-1, keepdims=True)
    gqa = np.einsum("bhl,blhd->bhd", p, v_rep)[:, None]
    # the same layer as MLA: cKV = [k_1..k_g, v_1..v_g], selector up-projections
    ckv = [np.concatenate([ks[b].reshape(L, g * d), vs[b].reshape(L, g * d)], axis=1)
           for b in range(B)]
    w_uk = np.zeros((H, d, r))
    w_uv = np.zeros((H, r, d))
    for h in range(H):
        grp = h // rep
        for i in range(d):
            w_uk[h, i, grp * d + i] = 1.0
            w_uv[h, g * d + grp * d + i, i] = 1.0
    mla = mo.mla_decode(q, np.zeros((B, 1, H, 0)), ckv, [np.zeros((L, 0))] * B,
                        w_uk, w_uv, scale)
    np.testing.assert_allclose(mla, gqa, rtol=1e-13, atol=1e-15)


def test_rope_pair_rotation_invariance():
    rng = np.random.default_rng(3)
    prob = list(_rand_problem(rng, B=2, Lq=1, H=3, r=16, dr=6, dn=4, dv=5, lens=(11, 6)))
    base = mo.mla_decode(*prob, scale=0.4)
    q_rope, kr = prob[1].copy(), [k.copy() for k in prob[3]]
    for i in range(q_rope.shape[-1] // 2):
        th = rng.uniform(0, 2 * math.pi)
        rot = np.array([[math.cos(th), -math.sin(th)], [math.sin(th), math.cos(th)]])
        q_rope[..., 2 * i:2 * i + 2] = q_rope[..., 2 * i:2 * i + 2] @ rot.T
        for k in kr:
            k[:, 2 * i:2 * i + 2] = k[:, 2 * i:2 * i + 2] @ rot.T
    prob[1], prob[3] = q_rope, kr
    np.testing.assert_allclose(mo.mla_decode(*prob, scale=0.4), base, rtol=1e-12, atol=1e-14)


def _apply_rope(x_re, x_im, theta, pos):
    """RoPE on complex pairs: (re + i im) * exp(i theta pos), theta per frequency."""
    c, s = np.cos(theta * pos), np.sin(theta * pos)
    return x_re * c - x_im * s, x_re * s + x_im * c


def _pack(re, im):
    # [..., F, g] -> rope dims ordered (frequency, copy, re/im)
    return np.stack([re, im], axis=-1).reshape(*re.shape[:-2], -1)


def test_cross_head_rotation_within_rope_frequency():
    """One orthogonal U_l per frequency, applied across the g head copies of
    both query and key before RoPE, leaves every score unchanged."""
    rng = np.random.default_rng(4)
    F, g, H, L, r, dn, dv = 3, 4, 2, 10, 8, 3, 4
    theta = 10000.0 ** (-np.arange(F) / F)
    qre, qim = rng.standard_normal((2, 1, 1, H, F, g))
    kre, kim = rng.standard_normal((2, L, F, g))
    ckv = [rng.standard_normal((L, r))]
    w_uk = rng.standard_normal((H, dn, r))
    w_uv = rng.standard_normal((H, r, dv))
    q_nope = rng.standard_normal((1, 1, H, dn))
    pos_q = L - 1
    pos_k = np.arange(L)[:, None, None]
    th = theta[None, :, None]

    def run(qre, qim, kre, kim):
        a, b = _apply_rope(qre, qim, theta[:, None], pos_q)
        c, d = _apply_rope(kre, kim, th, pos_k)
        return mo.mla_decode(q_nope, _pack(a, b), ckv, [_pack(c, d)], w_uk, w_uv, 0.2)

    base = run(qre, qim, kre, kim)
    U = [np.linalg.qr(rng.standard_normal((g, g)))[0] for _ in range(F)]

    def rot(x):
        return np.stack([x[..., l, :] @ U[l].T for l in range(F)], axis=-2)

    np.testing.assert_allclose(run(rot(qre), rot(qim), rot(kre), rot(kim)), base,
                               rtol=1e-11, atol=1e-13)
    # control: rotating only the keys must change the output
    assert np.abs(run(qre, qim, rot(kre), rot(kim)) - base).max() > 1e-3


def test_zero_query_gives_mean_of_values():
    rng = np.random.default_rng(5)
    q_nope, q_rope, ckv, kr, w_uk, w_uv = _rand_problem(rng, B=1, Lq=2, lens=(9,))
    q_nope[:] = 0
    q_rope[:] = 0
    out = mo.mla_decode(q_nope, q_rope, ckv, kr, w_uk, w_uv, scale=0.5)
    for t in range(2):
        nvis = 9 - 2 + t + 1
        for h in range(w_uk.shape[0]):
            v_mean = np.mean([[sum(ckv[0][j, c] * w_uv[h, c, e] for c in range(8))
                               for e in range(4)] for j in range(nvis)], axis=0)
            np.testing.assert_allclose(out[0, t, h], v_mean, rtol=1e-12, atol=1e-14)


def test_single_key_returns_its_value():
    rng = np.random.default_rng(6)
    q_nope, q_rope, ckv, kr, w_uk, w_uv = _rand_problem(rng, B=1, Lq=1, lens=(1,))
    out = mo.mla_decode(q_nope, q_rope, ckv, kr, w_uk, w_uv, scale=3.0)
    for h in range(w_uk.shape[0]):
        v0 = [sum(ckv[0][0, c] * w_uv[h, c, e] for c in range(8)) for e in range(4)]
        np.testing.assert_allclose(out[0, 0, h], v0, rtol=1e-12)


def test_dominant_key_is_selected():
    rng = np.random.default_rng(7)
    q_nope, q_rope, ckv, kr, w_uk, w_uv = _rand_problem(rng, B=1, Lq=1, H=1, lens=(12,))
    q_nope[:] = 0
    kr[0][5] = 60.0 * q_rope[0, 0, 0] / np.linalg.norm(q_rope[0, 0, 0])
    out = mo.mla_decode(q_nope, q_rope, ckv, kr, w_uk, w_uv, scale=1.0)
    v5 = ckv[0][5] @ w_uv[0]
    np.testing.assert_allclose(out[0, 0, 0], v5, rtol=1e-9, atol=1e-9)


def test_mtp_rows_reduce_to_single_query_decodes():
    rng = np.random.default_rng(8)
    q_nope, q_rope, ckv, kr, w_uk, w_uv = _rand_problem(rng, B=1, Lq=2, lens=(10,))
    both = mo.mla_decode(q_nope, q_rope, ckv, kr, w_uk, w_uv, scale=0.7)
    row0 = mo.mla_decode(q_nope[:, :1], q_rope[:, :1], [ckv[0][:9]], [kr[0][:9]],
                         w_uk, w_uv, scale=0.7)
    row1 = mo.mla_decode(q_nope[:, 1:], q_rope[:, 1:], ckv, kr, w_uk, w_uv, scale=0.7)
    np.testing.assert_allclose(both[:, :1], row0, rtol=1e-13)
    np.testing.assert_allclose(both[:, 1:], row1, rtol=1e-13)


def test_tpla_is_sum_of_independent_shard_attentions():
    rng = np.random.default_rng(9)
    q_nope, q_rope, ckv, kr, w_uk, w_uv = _rand_problem(rng, B=2, Lq=1, r=16, lens=(13, 4))
    tpla = mo.mla_decode(q_nope, q_rope, ckv, kr, w_uk, w_uv, scale=0.5, latent_shards=2)
    halves = [mo.mla_decode(q_nope, q_rope, [c[:, sl] for c in ckv], kr, w_uk[:, :, sl],
                            w_uv[:, sl, :], scale=0.5)
              for sl in (slice(0, 8), slice(8, 16))]
    np.testing.assert_allclose(tpla, halves[0] + halves[1], rtol=1e-13)
    # and it is a different function from MLA on the full latent
    mla = mo.mla_decode(q_nope, q_rope, ckv, kr, w_uk, w_uv, scale=0.5)
    assert np.abs(tpla - mla).max() > 1e-3


def test_cache_compression_golden():
    """The converted LLaMA-2-7B row width is 576 values against 8192 (92.97%)."""
    with open(os.path.join(GOLDEN, "cache_compression.json")) as f:
        gold = json.load(f)
    from mla_workloads import WORKLOADS
    wl = WORKLOADS["llama2_7b"]
    assert wl.row_width == gold["mla_values_per_token"]
    assert 2 * 32 * 128 == gold["gqa_values_per_token"]
    pct = 100.0 * (1.0 - wl.row_width / gold["gqa_values_per_token"])
    assert round(pct, 2) == gold["compression_percent_printed"]
    assert round(pct) == gold["compression_percent_abstract"]


# ---- planted mistakes: every one must be caught by the brute-force pin ----

_orig_softmax = mo.softmax_attention
_orig_mkv = mo.materialise_kv

def _mut_drop_rope(ckv, k_rope, w_uk_h, w_uv_h):
    k, v = _orig_mkv(ckv, k_rope, w_uk_h, w_uv_h)
    k[:, w_uk_h.shape[0]:] = 0.0
    return k, v


def _mut_rope_sign(ckv, k_rope, w_uk_h, w_uv_h):
    return _orig_mkv(ckv, -k_rope, w_uk_h, w_uv_h)


def _mut_wuk_index(ckv, k_rope, w_uk_h, w_uv_h):
    return _orig_mkv(ckv, k_rope, w_uk_h[::-1], w_uv_h)


def _mut_wuv_latent_index(ckv, k_rope, w_uk_h, w_uv_h):
    return _orig_mkv(ckv, k_rope, w_uk_h, w_uv_h[::-1])


def _mut_no_causal(q, k, v, scale, n_visible):
    return _orig_softmax(q, k, v, scale, k.shape[0])


def _mut_scale(q, k, v, scale, n_visible):
    return _orig_softmax(q, k, v, scale * scale, n_visible)




@pytest.mark.parametrize("target,mutant", [
    ("materialise_kv", _mut_drop_rope),
    ("materialise_kv", _mut_rope_sign),
    ("materialise_kv", _mut_wuk_index),
    ("materialise_kv", _mut_wuv_latent_index),
    ("softmax_attention", _mut_no_causal),
    ("softmax_attention", _mut_scale),
])
def test_planted_mistakes_are_caught(monkeypatch, target, mutant):
    rng = np.random.default_rng(11)
    prob = _rand_problem(rng, Lq=2)
    scale = 0.45
    want = _brute(*prob, scale=scale, shards=2)
    monkeypatch.setattr(mo, target, mutant)
    got = mo.mla_decode(*prob, scale=scale, latent_shards=2)
    assert np.abs(got - want).max() > 1e-6


# ---------------------------------------------------------------------------
# FP8 cache format: the oracle's E4M3 decoder (written from the bit fields)
# against torch's own float8_e4m3fn conversion, every code.
# ---------------------------------------------------------------------------
def test_e4m3_decoder_matches_torch_on_every_code():
    from oracle.fp8_cache import e4m3_table
    ours = e4m3_table()
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan) and nan.sum() == 2  # 0x7F and 0xFF
    assert np.array_equal(ours[~nan], ref[~nan])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x38] == 1.0


def test_fp8_logical_cache_scales_codes_and_rope():
    from oracle.fp8_cache import logical_cache_fp8
    codes = np.array([[0x38, 0xC0, 0x00], [0x40, 0x01, 0xB8]], dtype=np.uint8)   # 1, -2, 0 / 2, 2^-9, -1
    rope = np.array([[1.0, -3.0], [0.5, 2.0]])
    scales = np.array([0.25, 4.0])
    ckv, kr = logical_cache_fp8(codes, rope, scales)
    assert np.array_equal(ckv, [[0.25, -0.5, 0.0], [8.0, 4.0 * 2.0 ** -9, -4.0]])
    assert np.array_equal(kr, [[0.25, -0.75], [2.0, 8.0]])


def test_prefill_matches_brute_force_and_is_causal():
    """The prefill oracle against scalar loops (every token of two short
    prompts, every head): query t of a prompt attends to the prompt's tokens
    j <= t only, so each row is the brute-force decode of the prefix that ends
    at t. Changing a later token must leave earlier rows unchanged."""
    rng = np.random.default_rng(77)
    H, r, dr, dn, dv = 2, 8, 2, 3, 4
    lens = [5, 3]
    T = sum(lens)
    cu = [0, 5, 8]
    q_nope = rng.standard_normal((T, H, dn))
    q_rope = rng.standard_normal((T, H, dr))
    kv_rows = rng.standard_normal((T, r + dr))
    w_uk = rng.standard_normal((H, dn, r)) / math.sqrt(r)
    w_uv = rng.standard_normal((H, r, dv)) / math.sqrt(r)
    scale = 0.37
    got = mo.mla_prefill(q_nope, q_rope, kv_rows, cu, w_uk, w_uv, scale)
    i = 0
    for t in range(T):
        b = 0 if t < 5 else 1
        n = t - cu[b] + 1
        prefix = kv_rows[cu[b]:cu[b] + n]
        ref = _brute(q_nope[None, t:t + 1], q_rope[None, t:t + 1], [prefix[:, :r]], [prefix[:, r:]],
                     w_uk, w_uv, scale)[0, 0]
        for h in range(H):
            assert np.allclose(got[i], ref[h], rtol=1e-12, atol=1e-13)
            i += 1
    # causality: the last token of prompt 0 changes, earlier rows do not
    kv2 = kv_rows.copy()
    kv2[4] += 3.0
    got2 = mo.mla_prefill(q_nope, q_rope, kv2, cu, w_uk, w_uv, scale)
    assert np.array_equal(got2[:8], got[:8])       # tokens 0..3 of prompt 0, both heads
    assert not np.allclose(got2[8:10], got[8:10])  # token 4 sees its own change
    assert np.array_equal(got2[10:], got[10:])     # prompt 1 is independent


def _blasst_problem(rng, L=12, Lq=1, H=2, r=8, dr=2, dn=3, dv=4):
    q_nope = rng.standard_normal((Lq, H, dn))
    q_rope = np.zeros((Lq, H, dr))
    q_rope[:, :, 0] = 10.0
    ckv = rng.standard_normal((L, r))
    kr = np.zeros((L, dr))
    kr[:, 0] = 1.0
    w_uk = rng.standard_normal((H, dn, r)) / math.sqrt(r) * 0.1
    w_uv = rng.standard_normal((H, r, dv)) / math.sqrt(r)
    return q_nope, q_rope, ckv, kr, w_uk, w_uv


def test_blasst_without_threshold_is_the_dense_decode():
    rng = np.random.default_rng(90)
    prob = _rand_problem(rng, B=1, Lq=2, lens=(23,))
    q_nope, q_rope, ckv, kr, w_uk, w_uv = prob
    dense = mo.mla_decode(q_nope, q_rope, ckv, kr, w_uk, w_uv, 0.4)[0]
    for segs in ([(0, 23)], [(0, 9), (9, 23)]):
        got, kept, _ = mo.mla_decode_blasst(q_nope[0], q_rope[0], ckv[0], kr[0], w_uk, w_uv, 0.4, segs,
                                            -np.inf, group_keys=4)
        assert kept.all()
        assert np.allclose(got, dense, rtol=1e-12, atol=1e-14)


def test_blasst_skips_exactly_the_negligible_block():
    """Keys 4..7 score ~60 log2 units below the others for every row: with a
    threshold of -10 that block (and only it) is skipped, and the output is the
    brute-force attention over the kept keys. With the block's keys moved into
    a segment of their own it is that segment's first block and is kept."""
    rng = np.random.default_rng(91)
    q_nope, q_rope, ckv, kr, w_uk, w_uv = _blasst_problem(rng)
    kr[4:8, 0] = -5.0
    scale = 0.5
    got, kept, margin = mo.mla_decode_blasst(q_nope, q_rope, ckv, kr, w_uk, w_uv, scale, [(0, 12)],
                                             -10.0, group_keys=4)
    assert kept.tolist() == [True, False, True]
    assert margin[1] < -20 and margin[2] > 5
    keep = np.r_[0:4, 8:12]
    ref = _brute(q_nope[None], q_rope[None], [ckv[keep]], [kr[keep]], w_uk, w_uv, scale)[0]
    assert np.allclose(got, ref, rtol=1e-11, atol=1e-13)
    # a segment that starts at key 4 keeps its first block
    _, kept2, _ = mo.mla_decode_blasst(q_nope, q_rope, ckv, kr, w_uk, w_uv, scale, [(0, 4), (4, 12)],
                                       -10.0, group_keys=4)
    assert kept2.tolist() == [True, True, True]


def test_blasst_keeps_a_block_that_one_row_needs():
    """Only head 1 scores high on keys 4..7 (head 0 scores them very low): the
    block is kept for both heads (the decision covers every row)."""
    rng = np.random.default_rng(92)
    q_nope, q_rope, ckv, kr, w_uk, w_uv = _blasst_problem(rng)
    q_rope[0, 1, 1] = 10.0       # head 1 also reads the second RoPE column
    kr[4:8, 0] = -5.0
    kr[4:8, 1] = 8.0             # ... where keys 4..7 score high
    _, kept, _ = mo.mla_decode_blasst(q_nope, q_rope, ckv, kr, w_uk, w_uv, 0.5, [(0, 12)], -10.0, group_keys=4)
    assert kept.tolist() == [True, True, True]
