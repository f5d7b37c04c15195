"""Torch-tensor convenience over the C ABI (marshalling only: every step of the
decode runs inside libmla_decode.so; torch provides device memory and streams)."""

from __future__ import annotations

from typing import Optional, Sequence

from . import _lib as L


def dims_for(heads: int, latent_rank: int, rope_dim: int, nope_dim: int, v_dim: int,
             q_len: int, softmax_scale: float, dtype: str = "bf16", latent_shards: int = 1,
             page_size: int = 64) -> L.mla_dims_t:
    code = {"bf16": L.MLA_BF16, "fp32": L.MLA_FP32, "fp8": L.MLA_FP8_CACHE}[dtype]
    return L.make_dims(heads, latent_rank, rope_dim, nope_dim, v_dim, q_len, page_size,
                       latent_shards, float(softmax_scale), code)


class DecodePlan:
    """Owns one plan handle and (once bound) its device workspace tensor."""

    def __init__(self, dims: L.mla_dims_t, seq_lens_host: Sequence[int], num_sms: int = 0,
                 kernel: int = L.MLA_KERNEL_AUTO, num_workers: int = 0):
        self.dims = dims
        self.batch = len(seq_lens_host)
        self.handle, self.workspace_bytes = L.mla_decode_plan_ex(
            dims, list(seq_lens_host), num_sms, kernel, num_workers)
        self.info = L.mla_plan_get_info(self.handle)
        self.workspace = None

    def allocate_workspace(self, device) -> "DecodePlan":
        import torch
        self.workspace = torch.empty(self.workspace_bytes, dtype=torch.uint8, device=device)
        L.mla_workspace_init(self.workspace.data_ptr(), self.workspace_bytes,
                             torch.cuda.current_stream(device).cuda_stream)
        return self

    def segments(self):
        return L.mla_plan_segments(self.handle)

    def _check(self, name, t, dtype, shape) -> None:
        """One argument's dtype and shape against the plan (None: any extent).
        The C ABI sees bare pointers, so this is where a mismatch is caught."""
        if t.dtype != dtype:
            raise ValueError(f"{name}: dtype {t.dtype}, the plan needs {dtype}")
        if t.dim() != len(shape) or any(e is not None and e != n for e, n in zip(shape, t.shape)):
            want = tuple("*" if e is None else e for e in shape)
            raise ValueError(f"{name}: shape {tuple(t.shape)}, the plan needs {want}")

    def _check_common(self, act, q_nope, q_rope, block_table, seq_lens, w_uk, w_uv, out) -> None:
        import torch
        d, B = self.dims, self.batch
        H, Lq, r, dr, dn, dv = d.num_heads, d.q_len, d.latent_rank, d.rope_dim, d.nope_dim, d.v_dim
        self._check("q_nope", q_nope, act, (B, Lq, H, dn))
        self._check("q_rope", q_rope, act, (B, Lq, H, dr))
        self._check("block_table", block_table, torch.int32, (B, None))
        self._check("seq_lens", seq_lens, torch.int32, (B,))
        self._check("w_uk", w_uk, act, (H, dn, r))
        self._check("w_uv", w_uv, act, (H, r, dv))
        self._check("out", out, act, (B, Lq, H, dv))

    def run(self, q_nope, q_rope, kv_pool, block_table, seq_lens, w_uk, w_uv, out,
            stream: Optional[int] = None, decode_events=None) -> None:
        """All arguments are device tensors laid out as in include/mla_decode.h."""
        import torch
        d = self.dims
        if d.dtype == L.MLA_FP8_CACHE:
            raise ValueError("a plan over the FP8 cache runs with run_fp8")
        act = torch.float32 if d.dtype == L.MLA_FP32 else torch.bfloat16
        self._check_common(act, q_nope, q_rope, block_table, seq_lens, w_uk, w_uv, out)
        self._check("kv_pool", kv_pool, act, (None, d.page_size, d.latent_rank + d.rope_dim))
        for name, t in (("q_nope", q_nope), ("q_rope", q_rope), ("kv_pool", kv_pool),
                        ("block_table", block_table), ("seq_lens", seq_lens), ("w_uk", w_uk),
                        ("w_uv", w_uv), ("out", out)):
            if not t.is_cuda or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous CUDA tensor")
        if self.workspace is None:
            self.allocate_workspace(q_nope.device)
        if stream is None:
            stream = torch.cuda.current_stream(q_nope.device).cuda_stream
        # decode_events: optional (start, stop) raw cudaEvent_t handles (ints)
        ev0, ev1 = (None, None) if decode_events is None else decode_events
        L.mla_decode_run_ex(self.handle, q_nope.data_ptr(), q_rope.data_ptr(),
                            kv_pool.data_ptr(), kv_pool.shape[0], block_table.data_ptr(),
                            block_table.shape[1], seq_lens.data_ptr(), w_uk.data_ptr(),
                            w_uv.data_ptr(), out.data_ptr(), self.workspace.data_ptr(),
                            self.workspace_bytes, stream, ev0, ev1)

    def run_fp8(self, q_nope, q_rope, kv_codes, kv_rope, kv_scale, block_table, seq_lens, w_uk,
                w_uv, out, stream: Optional[int] = None, decode_events=None) -> None:
        """As run, over an FP8 latent cache (include/mla_decode.h, mla_decode_run_fp8)."""
        import torch
        d = self.dims
        if d.dtype != L.MLA_FP8_CACHE:
            raise ValueError("run_fp8 needs a plan made with dtype 'fp8'")
        self._check_common(torch.bfloat16, q_nope, q_rope, block_table, seq_lens, w_uk, w_uv, out)
        nb = kv_codes.shape[0] if kv_codes.dim() == 3 else None
        self._check("kv_codes", kv_codes, torch.uint8, (nb, d.page_size, d.latent_rank))
        self._check("kv_rope", kv_rope, torch.bfloat16, (nb, d.page_size, d.rope_dim))
        self._check("kv_scale", kv_scale, torch.float32, (nb, d.page_size))
        for name, t in (("q_nope", q_nope), ("q_rope", q_rope), ("kv_codes", kv_codes),
                        ("kv_rope", kv_rope), ("kv_scale", kv_scale), ("block_table", block_table),
                        ("seq_lens", seq_lens), ("w_uk", w_uk), ("w_uv", w_uv), ("out", out)):
            if not t.is_cuda or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous CUDA tensor")
        if self.workspace is None:
            self.allocate_workspace(q_nope.device)
        if stream is None:
            stream = torch.cuda.current_stream(q_nope.device).cuda_stream
        ev0, ev1 = (None, None) if decode_events is None else decode_events
        L.mla_decode_run_fp8(self.handle, q_nope.data_ptr(), q_rope.data_ptr(), kv_codes.data_ptr(),
                             kv_rope.data_ptr(), kv_scale.data_ptr(), kv_codes.shape[0],
                             block_table.data_ptr(), block_table.shape[1], seq_lens.data_ptr(),
                             w_uk.data_ptr(), w_uv.data_ptr(), out.data_ptr(),
                             self.workspace.data_ptr(), self.workspace_bytes, stream, ev0, ev1)

    def run_blasst(self, q_nope, q_rope, kv_pool, block_table, seq_lens, w_uk, w_uv, out, skip_log2: float,
                   stream: Optional[int] = None, decode_events=None) -> None:
        """A decode step with threshold skipping (mla_decode_run_blasst); the
        arguments are those of run plus the threshold in log2 units (<= 0)."""
        import torch
        d = self.dims
        act = torch.bfloat16
        self._check_common(act, q_nope, q_rope, block_table, seq_lens, w_uk, w_uv, out)
        self._check("kv_pool", kv_pool, act, (None, d.page_size, d.latent_rank + d.rope_dim))
        for name, t in (("q_nope", q_nope), ("q_rope", q_rope), ("kv_pool", kv_pool),
                        ("block_table", block_table), ("seq_lens", seq_lens), ("w_uk", w_uk),
                        ("w_uv", w_uv), ("out", out)):
            if not t.is_cuda or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous CUDA tensor")
        if self.workspace is None:
            self.allocate_workspace(q_nope.device)
        if stream is None:
            stream = torch.cuda.current_stream(q_nope.device).cuda_stream
        ev0, ev1 = (None, None) if decode_events is None else decode_events
        L.mla_decode_run_blasst(self.handle, q_nope.data_ptr(), q_rope.data_ptr(), kv_pool.data_ptr(),
                                kv_pool.shape[0], block_table.data_ptr(), block_table.shape[1],
                                seq_lens.data_ptr(), w_uk.data_ptr(), w_uv.data_ptr(), out.data_ptr(),
                                self.workspace.data_ptr(), self.workspace_bytes, skip_log2, stream, ev0, ev1)

    def skip_counts(self):
        """(skipped groups, groups) of the last threshold-skipping step (the
        workspace header's counters; synchronises the device)."""
        import torch
        torch.cuda.synchronize(self.workspace.device)
        c = self.workspace[8:16].view(torch.int32).cpu().tolist()
        return c[0], c[1]

    def read_status(self, stream: Optional[int] = None) -> int:
        import torch
        if stream is None:
            stream = torch.cuda.current_stream(self.workspace.device).cuda_stream
        return L.mla_decode_read_status(self.workspace.data_ptr(), stream)

    def close(self) -> None:
        if self.handle:
            L.mla_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class PrefillPlan:
    """Owns one prefill plan handle and its device workspace tensor (the
    up-projected per-head keys and values)."""

    def __init__(self, dims: L.mla_dims_t, seq_lens_host: Sequence[int]):
        self.dims = dims
        self.lens = [int(x) for x in seq_lens_host]
        self.handle, self.workspace_bytes = L.mla_prefill_plan(dims, self.lens)
        self.workspace = None

    def allocate_workspace(self, device) -> "PrefillPlan":
        import torch
        self.workspace = torch.empty(self.workspace_bytes, dtype=torch.uint8, device=device)
        L.mla_workspace_init(self.workspace.data_ptr(), self.workspace_bytes,
                             torch.cuda.current_stream(device).cuda_stream)
        return self

    def run(self, q_nope, q_rope, kv_rows, cu_seqlens, w_uk, w_uv, out, stream: Optional[int] = None,
            attn_events=None) -> None:
        """q_nope [T, H, dn], q_rope [T, H, dr], kv_rows [T, r + dr], cu_seqlens int32 [B + 1],
        w_uk [H, dn, r], w_uv [H, r, dv], out [T, H, dv]: contiguous CUDA tensors."""
        import torch
        d, T = self.dims, sum(self.lens)
        H, r, dr, dn, dv = d.num_heads, d.latent_rank, d.rope_dim, d.nope_dim, d.v_dim
        bf = torch.bfloat16
        for name, t, dtype, shape in (("q_nope", q_nope, bf, (T, H, dn)), ("q_rope", q_rope, bf, (T, H, dr)),
                                      ("kv_rows", kv_rows, bf, (T, r + dr)),
                                      ("cu_seqlens", cu_seqlens, torch.int32, (len(self.lens) + 1,)),
                                      ("w_uk", w_uk, bf, (H, dn, r)), ("w_uv", w_uv, bf, (H, r, dv)),
                                      ("out", out, bf, (T, H, dv))):
            if t.dtype != dtype or tuple(t.shape) != shape:
                raise ValueError(f"{name}: {t.dtype} {tuple(t.shape)}, the plan needs {dtype} {shape}")
            if not t.is_cuda or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous CUDA tensor")
        if self.workspace is None:
            self.allocate_workspace(q_nope.device)
        if stream is None:
            stream = torch.cuda.current_stream(q_nope.device).cuda_stream
        ev0, ev1 = (None, None) if attn_events is None else attn_events
        L.mla_prefill_run(self.handle, q_nope.data_ptr(), q_rope.data_ptr(), kv_rows.data_ptr(),
                          cu_seqlens.data_ptr(), w_uk.data_ptr(), w_uv.data_ptr(), out.data_ptr(),
                          self.workspace.data_ptr(), self.workspace_bytes, stream, ev0, ev1)

    def read_status(self, stream: Optional[int] = None) -> int:
        import torch
        if stream is None:
            stream = torch.cuda.current_stream(self.workspace.device).cuda_stream
        return L.mla_decode_read_status(self.workspace.data_ptr(), stream)

    def close(self) -> None:
        if self.handle:
            L.mla_prefill_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
