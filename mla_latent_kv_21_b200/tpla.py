"""TPLA across GPUs: one latent shard per GPU and one all-reduce of the output.

TPLA partitions the latent cKV (and each head's W_UK / W_UV along the latent
axis) across the devices of a tensor-parallel group; every device attends with
its own shard, adding the full RoPE score and running its own softmax, and the
per-device outputs are summed by an all-reduce (TPLA abstract, on the
taxoreview listing pages for dblp:408/6122 and dblp:256/5536-3). On one GPU
the library computes the same function in one launch (latent_shards = 2); here
each GPU of a group runs the plain decode over its shard (latent_rank = r / tp,
one shard) and the group sums the bf16 outputs with NCCL.

Marshalling only: the decode runs in libmla_decode.so, the sum in NCCL (the one
exchange step of the method); torch.distributed provides the group.
"""

from __future__ import annotations

from typing import Optional, Sequence

from . import _lib as L
from .api import DecodePlan


def shard_dims(dims: L.mla_dims_t, tp: int) -> L.mla_dims_t:
    """Dims of one GPU's shard of a tp-way TPLA decode whose full form is
    `dims` (latent_shards == tp): latent_rank / tp columns, one shard, the same
    scale (the full RoPE term is in every shard)."""
    if dims.latent_shards != tp or dims.latent_rank % tp:
        raise ValueError(f"dims hold {dims.latent_shards} latent shards of rank {dims.latent_rank}, "
                         f"not {tp}")
    return L.make_dims(dims.num_heads, dims.latent_rank // tp, dims.rope_dim, dims.nope_dim, dims.v_dim,
                       dims.q_len, dims.page_size, 1, dims.softmax_scale, dims.dtype)


class TplaShardPlan:
    """This GPU's part of a tp-way TPLA decode: a DecodePlan over its latent
    shard, and the all-reduce that sums the group's outputs."""

    def __init__(self, dims: L.mla_dims_t, seq_lens_host: Sequence[int], tp: int, group=None,
                 num_sms: int = 0, num_workers: int = 0):
        self.tp = tp
        self.group = group
        self.plan = DecodePlan(shard_dims(dims, tp), seq_lens_host, num_sms=num_sms, num_workers=num_workers)

    @property
    def info(self):
        return self.plan.info

    def allocate_workspace(self, device) -> "TplaShardPlan":
        self.plan.allocate_workspace(device)
        return self

    def run_shard(self, q_nope, q_rope, kv_shard, block_table, seq_lens, w_uk_shard, w_uv_shard, out,
                  stream: Optional[int] = None, decode_events=None) -> None:
        """This shard's attention output (not yet summed) into `out`."""
        self.plan.run(q_nope, q_rope, kv_shard, block_table, seq_lens, w_uk_shard, w_uv_shard, out,
                      stream, decode_events)

    def allreduce(self, out) -> None:
        """Sum of the group's shard outputs, in place (NCCL on the current
        stream; every rank of the group calls it once per step)."""
        import torch.distributed as dist
        dist.all_reduce(out, op=dist.ReduceOp.SUM, group=self.group)

    def run(self, q_nope, q_rope, kv_shard, block_table, seq_lens, w_uk_shard, w_uv_shard, out,
            stream: Optional[int] = None, decode_events=None) -> None:
        """One TPLA decode step: this shard's attention, then the group sum."""
        self.run_shard(q_nope, q_rope, kv_shard, block_table, seq_lens, w_uk_shard, w_uv_shard, out,
                       stream, decode_events)
        self.allreduce(out)

    def read_status(self, stream: Optional[int] = None) -> int:
        return self.plan.read_status(stream)

    def close(self) -> None:
        self.plan.close()
