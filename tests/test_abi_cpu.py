"""Host-side checks of the C ABI that need no GPU: the library loads and
exports every declared symbol, argument validation, and the split partition
against an independent recomputation (integer-exact)."""

import os
import random
import re
import subprocess

import pytest

import mla_latent_kv_21_b200 as M
from mla_latent_kv_21_b200 import _lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    inc = os.path.join(ROOT, "include")
    for fn in os.listdir(inc):
        if fn.endswith(".h"):
            text = open(os.path.join(inc, fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names.update(re.findall(r"\b(mla_[a-z_0-9]+)\s*\(", text))
    return names


def test_library_exports_every_declared_symbol():
    declared = _declared_functions()
    assert declared, "no declarations found"
    out = subprocess.run(["nm", "-D", "--defined-only", M.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\b[TW]\s+(mla_\w+)", out))
    assert declared <= exported, declared - exported
    assert declared == set(L.EXPORTED)
    assert L.mla_abi_version() == 1


def _dims(**kw):
    d = dict(heads=128, latent_rank=512, rope_dim=64, nope_dim=128, v_dim=128, q_len=1,
             softmax_scale=192 ** -0.5, dtype="bf16", latent_shards=1)
    d.update(kw)
    return M.dims_for(**d)


def test_status_strings():
    for s in range(8):
        assert L.mla_status_string(s) and L.mla_status_string(s) != "unknown status"
    assert L.mla_status_string(99) == "unknown status"


@pytest.mark.parametrize("kw,status", [
    (dict(heads=0), L.MLA_ERR_INVALID_ARG),
    (dict(softmax_scale=float("nan")), L.MLA_ERR_INVALID_ARG),
    (dict(page_size=32), L.MLA_ERR_UNSUPPORTED),
    (dict(latent_shards=3), L.MLA_ERR_UNSUPPORTED),
    (dict(latent_rank=1024), L.MLA_ERR_UNSUPPORTED),
    (dict(nope_dim=256), L.MLA_ERR_UNSUPPORTED),
])
def test_plan_rejects_bad_dims(kw, status):
    with pytest.raises(L.MlaError) as e:
        L.mla_decode_plan(_dims(**kw), [100, 200], num_sms=148)
    assert e.value.status == status


def test_plan_rejects_short_sequences():
    with pytest.raises(L.MlaError) as e:
        L.mla_decode_plan(_dims(q_len=2), [5, 1], num_sms=148)
    assert e.value.status == L.MLA_ERR_INVALID_ARG


def test_run_rejects_null_and_small_workspace():
    plan, ws = L.mla_decode_plan_ex(_dims(), [100], num_sms=148, kernel=L.MLA_KERNEL_SIMT)
    try:
        with pytest.raises(L.MlaError) as e:
            L.mla_decode_run(plan, 0, 0, 0, 1, 0, 1, 0, 0, 0, 0, 0, ws, 0)
        assert e.value.status == L.MLA_ERR_INVALID_ARG
        fake = 1 << 20  # never dereferenced: the size check comes first
        with pytest.raises(L.MlaError) as e:
            L.mla_decode_run(plan, fake, fake, fake, 1, fake, 2, fake, fake, fake, fake, fake,
                             ws - 1, 0)
        assert e.value.status == L.MLA_ERR_WORKSPACE_TOO_SMALL
    finally:
        L.mla_plan_destroy(plan)


from harness_partition import reference_segments as _reference_segments  # noqa: E402


@pytest.mark.parametrize("seed", range(12))
def test_split_partition_matches_independent_recomputation(seed):
    rng = random.Random(seed)
    B = rng.choice([1, 2, 3, 7, 32, 64])
    q_len = rng.choice([1, 2])
    lens = [rng.randint(q_len, rng.choice([64, 65, 300, 5000, 32768])) for _ in range(B)]
    kernel = rng.choice([L.MLA_KERNEL_SIMT, L.MLA_KERNEL_AUTO])
    workers = rng.choice([0, 0, 1, 5, 74, 1000])
    plan, ws = L.mla_decode_plan_ex(_dims(q_len=q_len), lens, num_sms=148, kernel=kernel,
                                    num_workers=workers)
    try:
        info = L.mla_plan_get_info(plan)
        W = info.num_workers
        got = L.mla_plan_segments(plan)
        want, pages = _reference_segments(lens, 64, W)
        assert got == want
        assert info.total_pages == sum(pages)
        assert 1 <= W <= sum(pages)
        assert info.num_split_slots == W + B - 1
        # each sequence covered exactly once, in order, by its segments
        for b in range(B):
            mine = [s for s in got if s[1] == b]
            assert mine[0][2] == 0 and mine[-1][3] == pages[b]
            for s0, s1 in zip(mine, mine[1:]):
                assert s0[3] == s1[2]
        slots = [s[4] for s in got]
        assert len(set(slots)) == len(slots) and max(slots) < W + B - 1
        assert slots == sorted(slots)
        assert ws == info.workspace_bytes
    finally:
        L.mla_plan_destroy(plan)


@pytest.mark.parametrize("batch", [32, 200000])
def test_workspace_holds_partials_for_every_slot(batch):
    # 200000 x 32K tokens: 1e8 pages and a workspace of ~100 GB, past every
    # 32-bit count; the plan must size it without wrapping
    lens = [32768] * batch
    plan, ws = L.mla_decode_plan_ex(_dims(), lens, num_sms=148, kernel=L.MLA_KERNEL_SIMT)
    try:
        info = L.mla_plan_get_info(plan)
        rows, slots = 128, info.num_split_slots
        assert slots == info.num_workers + batch - 1
        assert info.total_pages == batch * 512
        need = slots * rows * 512 * 4 + slots * rows * 4 + batch * 128 * 576 * 2 + (batch + 1) * 8
        assert ws >= need
    finally:
        L.mla_plan_destroy(plan)


@pytest.mark.parametrize("kw,kernel,status", [
    # the tensor-core kernels need r = 512 bf16; the fp32 tiny shape is SIMT only
    (dict(latent_rank=64, rope_dim=16, nope_dim=32, v_dim=32, dtype="fp32"),
     L.MLA_KERNEL_TCGEN05, L.MLA_ERR_UNSUPPORTED),
    # unknown kernel kinds (3 was a removed latent-split variant)
    (dict(), 3, L.MLA_ERR_INVALID_ARG),
    (dict(), 7, L.MLA_ERR_INVALID_ARG),
    # the FP8 cache runs on the tcgen05 decode kernel only, with one latent shard
    (dict(dtype="fp8"), L.MLA_KERNEL_SIMT, L.MLA_ERR_UNSUPPORTED),
    (dict(dtype="fp8", latent_shards=2), L.MLA_KERNEL_AUTO, L.MLA_ERR_UNSUPPORTED),
])
def test_plan_rejects_unsupported_kernel_choices(kw, kernel, status):
    with pytest.raises(L.MlaError) as e:
        L.mla_decode_plan_ex(_dims(**kw), [100, 200], num_sms=148, kernel=kernel)
    assert e.value.status == status


@pytest.mark.parametrize("kernel", [L.MLA_KERNEL_AUTO, L.MLA_KERNEL_TCGEN05, L.MLA_KERNEL_SIMT])
def test_plan_reports_kernel_and_launches(kernel):
    plan, ws = L.mla_decode_plan_ex(_dims(), [4000, 65], num_sms=148, kernel=kernel)
    try:
        info = L.mla_plan_get_info(plan)
        want = L.MLA_KERNEL_TCGEN05 if kernel == L.MLA_KERNEL_AUTO else kernel
        assert info.kernel == want
        assert info.launches_per_run == 3
        assert info.workspace_bytes == ws > 0
    finally:
        L.mla_plan_destroy(plan)


def test_plan_rejects_an_empty_batch():
    with pytest.raises(L.MlaError) as e:
        L.mla_decode_plan(_dims(), [], num_sms=148)
    assert e.value.status == L.MLA_ERR_INVALID_ARG


def test_fp8_plan_uses_tcgen05_and_bf16_run_refuses_it():
    plan, ws = L.mla_decode_plan_ex(_dims(dtype="fp8"), [4000, 65], num_sms=148, kernel=L.MLA_KERNEL_AUTO)
    try:
        info = L.mla_plan_get_info(plan)
        assert info.kernel == L.MLA_KERNEL_TCGEN05 and info.launches_per_run == 3
        fake = 1 << 20  # never dereferenced: the dtype check comes before any launch
        with pytest.raises(L.MlaError) as e:
            L.mla_decode_run(plan, fake, fake, fake, 1, fake, 1, fake, fake, fake, fake, fake, ws, 0)
        assert e.value.status == L.MLA_ERR_INVALID_ARG
    finally:
        L.mla_plan_destroy(plan)


def _kimi_lens():
    from mla_workloads import WORKLOADS, draw_lengths
    return draw_lengths(WORKLOADS["kimi_k2_mtp"]).tolist()


@pytest.mark.parametrize("name,fits", [("tiny", True), ("llama2_7b", True), ("deepseek_v3", True),
                                       ("tpla_dsv3", True), ("kimi_k2_mtp", False)])
def test_no_alloc_scratch_covers_the_documented_plans(name, fits):
    """The no-allocation entry point's fixed 32 MiB scratch holds the plans the
    header lists (148 SMs, the default kernel) and refuses the larger one."""
    from mla_workloads import WORKLOADS
    wl = WORKLOADS[name]
    lens = _kimi_lens() if wl.context_min else [wl.context] * wl.batch
    dims = M.dims_for(wl.heads, wl.latent_rank, wl.rope_dim, wl.nope_dim, wl.v_dim, wl.q_len,
                      wl.softmax_scale, wl.dtype, wl.latent_shards, wl.page_size)
    plan, ws = L.mla_decode_plan(dims, lens, num_sms=148)
    try:
        assert (ws <= 32 << 20) == fits, ws
        if not fits:
            fake = 1 << 20  # never dereferenced: the size check comes before any device work
            with pytest.raises(L.MlaError) as e:
                L.mla_decode_run_no_alloc(plan, fake, fake, fake, 1, fake, 512, fake, fake, fake,
                                          fake, 0)
            assert e.value.status == L.MLA_ERR_WORKSPACE_TOO_SMALL
    finally:
        L.mla_plan_destroy(plan)


def test_no_alloc_refuses_fp8_plans_before_any_device_work():
    plan, _ = L.mla_decode_plan(_dims(dtype="fp8"), [4000, 65], num_sms=148)
    try:
        fake = 1 << 20  # never dereferenced: the dtype check comes before any device work
        with pytest.raises(L.MlaError) as e:
            L.mla_decode_run_no_alloc(plan, fake, fake, fake, 1, fake, 512, fake, fake, fake, fake, 0)
        assert e.value.status == L.MLA_ERR_UNSUPPORTED
    finally:
        L.mla_plan_destroy(plan)


@pytest.mark.parametrize("kw,kernel,limit,status", [
    (dict(), L.MLA_KERNEL_SIMT, 1_000_000, L.MLA_ERR_UNSUPPORTED),
    (dict(dtype="fp8"), L.MLA_KERNEL_TCGEN05, 1_000_000, L.MLA_ERR_UNSUPPORTED),
    (dict(), L.MLA_KERNEL_TCGEN05, 999, L.MLA_ERR_INVALID_ARG),
    (dict(), L.MLA_KERNEL_TCGEN05, 3_000_000_000, L.MLA_ERR_INVALID_ARG),
])
def test_timeout_selftest_argument_checks(kw, kernel, limit, status):
    """The timeout self-test takes bf16 tensor-core plans and a limit in
    [1 us, 2 s]; the checks come before any device work."""
    plan, ws = L.mla_decode_plan_ex(_dims(**kw), [4000, 65], num_sms=148, kernel=kernel)
    try:
        fake = 1 << 20  # never dereferenced
        with pytest.raises(L.MlaError) as e:
            L.mla_decode_selftest_timeout(plan, fake, fake, fake, 1, fake, 64, fake, fake, fake, fake,
                                          fake, ws, limit, 0)
        assert e.value.status == status
    finally:
        L.mla_plan_destroy(plan)


@pytest.mark.parametrize("kw,thr,status", [
    (dict(), 0.5, L.MLA_ERR_INVALID_ARG),            # a threshold above the running max
    (dict(), float("nan"), L.MLA_ERR_INVALID_ARG),
    (dict(dtype="fp8"), -6.0, L.MLA_ERR_UNSUPPORTED),
    (dict(latent_shards=2), -6.0, L.MLA_ERR_UNSUPPORTED),
])
def test_blasst_argument_checks(kw, thr, status):
    """Threshold skipping takes bf16, one latent shard and a threshold <= 0;
    the checks come before any device work."""
    plan, ws = L.mla_decode_plan_ex(_dims(**kw), [4000, 65], num_sms=148, kernel=L.MLA_KERNEL_AUTO)
    try:
        fake = 1 << 20  # never dereferenced
        with pytest.raises(L.MlaError) as e:
            L.mla_decode_run_blasst(plan, fake, fake, fake, 1, fake, 64, fake, fake, fake, fake, fake, ws, thr)
        assert e.value.status == status
    finally:
        L.mla_plan_destroy(plan)
