"""ctypes binding of libmla_decode.so (argument marshalling only).

Every function keeps the C name from include/mla_decode.h. Device buffers are
passed as integer addresses (e.g. ``tensor.data_ptr()``), streams as integer
handles (``torch.cuda.current_stream().cuda_stream``). A non-OK status raises
MlaError. There is no fallback: if the library is missing, importing this
module raises.
"""

from __future__ import annotations

import ctypes
import os
from typing import Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmla_decode.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m mla_latent_kv_21_b200.build` "
        "(nvcc, sm_100a). There is no CPU fallback.")

_lib = ctypes.CDLL(LIB_PATH)

MLA_OK = 0
MLA_ERR_INVALID_ARG = 1
MLA_ERR_UNSUPPORTED = 2
MLA_ERR_WORKSPACE_TOO_SMALL = 3
MLA_ERR_CUDA = 4
MLA_ERR_DEVICE_TIMEOUT = 5
MLA_ERR_BOUNDS = 6
MLA_ERR_NO_DEVICE = 7

MLA_BF16 = 0
MLA_FP32 = 1
MLA_FP8_CACHE = 2

MLA_KERNEL_AUTO = 0
MLA_KERNEL_SIMT = 1
MLA_KERNEL_TCGEN05 = 2

# symbols declared in include/mla_decode.h
EXPORTED = (
    "mla_decode_plan", "mla_decode_plan_ex", "mla_decode_run", "mla_decode_run_ex",
    "mla_decode_run_fp8", "mla_decode_run_no_alloc", "mla_decode_selftest_timeout", "mla_decode_run_blasst",
    "mla_workspace_init",
    "mla_decode_read_status", "mla_plan_get_info", "mla_plan_segments", "mla_plan_destroy",
    "mla_status_string", "mla_abi_version", "mla_prefill_plan", "mla_prefill_run",
    "mla_prefill_run_ex", "mla_prefill_plan_destroy",
)


class mla_dims_t(ctypes.Structure):
    _fields_ = [("num_heads", ctypes.c_int32), ("latent_rank", ctypes.c_int32),
                ("rope_dim", ctypes.c_int32), ("nope_dim", ctypes.c_int32),
                ("v_dim", ctypes.c_int32), ("q_len", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("latent_shards", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("dtype", ctypes.c_int32)]


class mla_plan_options_t(ctypes.Structure):
    _fields_ = [("num_sms", ctypes.c_int32), ("kernel", ctypes.c_int32),
                ("num_workers", ctypes.c_int32)]


class mla_run_options_t(ctypes.Structure):
    _fields_ = [("decode_start_event", ctypes.c_void_p), ("decode_stop_event", ctypes.c_void_p)]


class mla_plan_info_t(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("rows", ctypes.c_int32), ("kernel", ctypes.c_int32),
                ("num_workers", ctypes.c_int32), ("num_split_slots", ctypes.c_int32),
                ("launches_per_run", ctypes.c_int32), ("total_pages", ctypes.c_int64),
                ("workspace_bytes", ctypes.c_uint64)]


_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_i32p = ctypes.POINTER(ctypes.c_int32)

_lib.mla_status_string.restype = ctypes.c_char_p
_lib.mla_status_string.argtypes = [ctypes.c_int]
_lib.mla_abi_version.restype = _i32
_lib.mla_abi_version.argtypes = []
_lib.mla_decode_plan.restype = ctypes.c_int
_lib.mla_decode_plan.argtypes = [ctypes.POINTER(mla_dims_t), _i32, _i32p, _i32,
                                 ctypes.POINTER(_vp), ctypes.POINTER(_sz)]
_lib.mla_decode_plan_ex.restype = ctypes.c_int
_lib.mla_decode_plan_ex.argtypes = [ctypes.POINTER(mla_dims_t), _i32, _i32p,
                                    ctypes.POINTER(mla_plan_options_t), ctypes.POINTER(_vp),
                                    ctypes.POINTER(_sz)]
_lib.mla_decode_run.restype = ctypes.c_int
_lib.mla_decode_run.argtypes = [_vp, _vp, _vp, _vp, _i64, _vp, _i32, _vp, _vp, _vp, _vp, _vp,
                                _sz, _vp]
_lib.mla_decode_run_ex.restype = ctypes.c_int
_lib.mla_decode_run_ex.argtypes = [_vp, _vp, _vp, _vp, _i64, _vp, _i32, _vp, _vp, _vp, _vp, _vp,
                                   _sz, _vp, ctypes.POINTER(mla_run_options_t)]
_lib.mla_decode_run_fp8.restype = ctypes.c_int
_lib.mla_decode_run_fp8.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _i32, _vp, _vp, _vp, _vp,
                                    _vp, _sz, _vp, ctypes.POINTER(mla_run_options_t)]
_lib.mla_decode_run_no_alloc.restype = ctypes.c_int
_lib.mla_decode_run_no_alloc.argtypes = [_vp, _vp, _vp, _vp, _i64, _vp, _i32, _vp, _vp, _vp, _vp,
                                         _vp]
_lib.mla_decode_run_blasst.restype = ctypes.c_int
_lib.mla_decode_run_blasst.argtypes = [_vp, _vp, _vp, _vp, _i64, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _sz,
                                       ctypes.c_float, _vp, ctypes.POINTER(mla_run_options_t)]
_lib.mla_decode_selftest_timeout.restype = ctypes.c_int
_lib.mla_decode_selftest_timeout.argtypes = [_vp, _vp, _vp, _vp, _i64, _vp, _i32, _vp, _vp, _vp, _vp,
                                             _vp, _sz, ctypes.c_uint64, _vp]
_lib.mla_prefill_plan.restype = ctypes.c_int
_lib.mla_prefill_plan.argtypes = [ctypes.POINTER(mla_dims_t), _i32, _i32p, ctypes.POINTER(_vp),
                                  ctypes.POINTER(_sz)]
_lib.mla_prefill_run.restype = ctypes.c_int
_lib.mla_prefill_run.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.mla_prefill_run_ex.restype = ctypes.c_int
_lib.mla_prefill_run_ex.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp,
                                    ctypes.POINTER(mla_run_options_t)]
_lib.mla_prefill_plan_destroy.restype = None
_lib.mla_prefill_plan_destroy.argtypes = [_vp]
_lib.mla_workspace_init.restype = ctypes.c_int
_lib.mla_workspace_init.argtypes = [_vp, _sz, _vp]
_lib.mla_decode_read_status.restype = ctypes.c_int
_lib.mla_decode_read_status.argtypes = [_vp, _vp, _i32p]
_lib.mla_plan_get_info.restype = ctypes.c_int
_lib.mla_plan_get_info.argtypes = [_vp, ctypes.POINTER(mla_plan_info_t)]
_lib.mla_plan_segments.restype = ctypes.c_int
_lib.mla_plan_segments.argtypes = [_vp, _i32p, _i64, ctypes.POINTER(_i64)]
_lib.mla_plan_destroy.restype = None
_lib.mla_plan_destroy.argtypes = [_vp]


class MlaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {mla_status_string(status)} (status {status})")


def _check(status: int, where: str) -> None:
    if status != MLA_OK:
        raise MlaError(status, where)


def mla_status_string(status: int) -> str:
    return _lib.mla_status_string(int(status)).decode()


def mla_abi_version() -> int:
    return int(_lib.mla_abi_version())


def make_dims(num_heads, latent_rank, rope_dim, nope_dim, v_dim, q_len, page_size,
              latent_shards, softmax_scale, dtype) -> mla_dims_t:
    return mla_dims_t(num_heads, latent_rank, rope_dim, nope_dim, v_dim, q_len, page_size,
                      latent_shards, softmax_scale, dtype)


def _lens_array(seq_lens_host: Sequence[int]):
    arr = (ctypes.c_int32 * len(seq_lens_host))(*[int(x) for x in seq_lens_host])
    return arr


def mla_decode_plan(dims: mla_dims_t, seq_lens_host: Sequence[int], num_sms: int = 0):
    """Returns (plan handle, workspace bytes)."""
    plan, ws = _vp(), _sz()
    lens = _lens_array(seq_lens_host)
    _check(_lib.mla_decode_plan(ctypes.byref(dims), len(seq_lens_host), lens, num_sms,
                                ctypes.byref(plan), ctypes.byref(ws)), "mla_decode_plan")
    return plan.value, ws.value


def mla_decode_plan_ex(dims: mla_dims_t, seq_lens_host: Sequence[int], num_sms: int = 0,
                       kernel: int = MLA_KERNEL_AUTO, num_workers: int = 0):
    plan, ws = _vp(), _sz()
    lens = _lens_array(seq_lens_host)
    opts = mla_plan_options_t(num_sms, kernel, num_workers)
    _check(_lib.mla_decode_plan_ex(ctypes.byref(dims), len(seq_lens_host), lens,
                                   ctypes.byref(opts), ctypes.byref(plan), ctypes.byref(ws)),
           "mla_decode_plan_ex")
    return plan.value, ws.value


def mla_decode_run(plan, q_nope, q_rope, kv_cache, num_blocks, block_table, block_table_stride,
                   seq_lens_dev, w_uk, w_uv, out, workspace, workspace_bytes, stream=0) -> None:
    _check(_lib.mla_decode_run(plan, q_nope, q_rope, kv_cache, num_blocks, block_table,
                               block_table_stride, seq_lens_dev, w_uk, w_uv, out, workspace,
                               workspace_bytes, stream), "mla_decode_run")


def mla_decode_run_ex(plan, q_nope, q_rope, kv_cache, num_blocks, block_table,
                      block_table_stride, seq_lens_dev, w_uk, w_uv, out, workspace,
                      workspace_bytes, stream=0, decode_start_event=None,
                      decode_stop_event=None) -> None:
    opts = mla_run_options_t(decode_start_event, decode_stop_event)
    _check(_lib.mla_decode_run_ex(plan, q_nope, q_rope, kv_cache, num_blocks, block_table,
                                  block_table_stride, seq_lens_dev, w_uk, w_uv, out, workspace,
                                  workspace_bytes, stream, ctypes.byref(opts)),
           "mla_decode_run_ex")


def mla_decode_run_fp8(plan, q_nope, q_rope, kv_codes, kv_rope, kv_scale, num_blocks, block_table,
                       block_table_stride, seq_lens_dev, w_uk, w_uv, out, workspace,
                       workspace_bytes, stream=0, decode_start_event=None,
                       decode_stop_event=None) -> None:
    """One decode step over an FP8 latent cache (codes, RoPE key / scale, scales)."""
    opts = mla_run_options_t(decode_start_event, decode_stop_event)
    _check(_lib.mla_decode_run_fp8(plan, q_nope, q_rope, kv_codes, kv_rope, kv_scale, num_blocks,
                                   block_table, block_table_stride, seq_lens_dev, w_uk, w_uv, out,
                                   workspace, workspace_bytes, stream, ctypes.byref(opts)),
           "mla_decode_run_fp8")


def mla_decode_run_no_alloc(plan, q_nope, q_rope, kv_cache, num_blocks, block_table,
                            block_table_stride, seq_lens_dev, w_uk, w_uv, out, stream=0) -> None:
    """mla_decode_run without a workspace (for callers that cannot allocate
    device memory); the scratch is a fixed 32 MiB array inside the library."""
    _check(_lib.mla_decode_run_no_alloc(plan, q_nope, q_rope, kv_cache, num_blocks, block_table,
                                        block_table_stride, seq_lens_dev, w_uk, w_uv, out,
                                        stream), "mla_decode_run_no_alloc")


def mla_decode_run_blasst(plan, q_nope, q_rope, kv_cache, num_blocks, block_table, block_table_stride,
                          seq_lens_dev, w_uk, w_uv, out, workspace, workspace_bytes, skip_log2,
                          stream=0, decode_start_event=None, decode_stop_event=None) -> None:
    """One decode step skipping key groups whose scores fall below the running
    max + skip_log2 (log2 units) for every query row (see the C header)."""
    opts = mla_run_options_t(decode_start_event, decode_stop_event)
    _check(_lib.mla_decode_run_blasst(plan, q_nope, q_rope, kv_cache, num_blocks, block_table,
                                      block_table_stride, seq_lens_dev, w_uk, w_uv, out, workspace,
                                      workspace_bytes, float(skip_log2), stream, ctypes.byref(opts)),
           "mla_decode_run_blasst")


def mla_decode_selftest_timeout(plan, q_nope, q_rope, kv_cache, num_blocks, block_table,
                                block_table_stride, seq_lens_dev, w_uk, w_uv, out, workspace,
                                workspace_bytes, wait_limit_ns, stream=0) -> None:
    """Diagnostics: a decode step whose decode kernel withholds one barrier
    arrival with every wait bounded by wait_limit_ns (see the C header)."""
    _check(_lib.mla_decode_selftest_timeout(plan, q_nope, q_rope, kv_cache, num_blocks, block_table,
                                            block_table_stride, seq_lens_dev, w_uk, w_uv, out,
                                            workspace, workspace_bytes, wait_limit_ns, stream),
           "mla_decode_selftest_timeout")


def mla_prefill_plan(dims: mla_dims_t, seq_lens_host: Sequence[int]):
    """-> (plan handle, workspace bytes) of a causal MLA-form prefill."""
    plan = _vp()
    ws = _sz()
    arr = _lens_array(seq_lens_host)
    _check(_lib.mla_prefill_plan(ctypes.byref(dims), len(seq_lens_host), arr, ctypes.byref(plan),
                                 ctypes.byref(ws)), "mla_prefill_plan")
    return plan.value, ws.value


def mla_prefill_run(plan, q_nope, q_rope, kv_rows, cu_seqlens, w_uk, w_uv, out, workspace,
                    workspace_bytes, stream=0, attn_start_event=None, attn_stop_event=None) -> None:
    if attn_start_event is None and attn_stop_event is None:
        _check(_lib.mla_prefill_run(plan, q_nope, q_rope, kv_rows, cu_seqlens, w_uk, w_uv, out, workspace,
                                    workspace_bytes, stream), "mla_prefill_run")
        return
    opts = mla_run_options_t(attn_start_event, attn_stop_event)
    _check(_lib.mla_prefill_run_ex(plan, q_nope, q_rope, kv_rows, cu_seqlens, w_uk, w_uv, out, workspace,
                                   workspace_bytes, stream, ctypes.byref(opts)), "mla_prefill_run_ex")


def mla_prefill_plan_destroy(plan) -> None:
    _lib.mla_prefill_plan_destroy(plan)


def mla_workspace_init(workspace, workspace_bytes, stream=0) -> None:
    _check(_lib.mla_workspace_init(workspace, workspace_bytes, stream), "mla_workspace_init")


def mla_decode_read_status(workspace, stream=0) -> int:
    st = ctypes.c_int32()
    _check(_lib.mla_decode_read_status(workspace, stream, ctypes.byref(st)),
           "mla_decode_read_status")
    return int(st.value)


def mla_plan_get_info(plan) -> mla_plan_info_t:
    info = mla_plan_info_t()
    _check(_lib.mla_plan_get_info(plan, ctypes.byref(info)), "mla_plan_get_info")
    return info


def mla_plan_segments(plan):
    """List of (worker, sequence, first page, end page, slot) tuples."""
    n = _i64()
    _check(_lib.mla_plan_segments(plan, None, 0, ctypes.byref(n)), "mla_plan_segments")
    buf = (ctypes.c_int32 * (5 * max(n.value, 1)))()
    _check(_lib.mla_plan_segments(plan, buf, n.value, ctypes.byref(n)), "mla_plan_segments")
    return [tuple(buf[5 * i:5 * i + 5]) for i in range(n.value)]


def mla_plan_destroy(plan) -> None:
    if plan:
        _lib.mla_plan_destroy(plan)
