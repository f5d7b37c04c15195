"""CPU oracle package (test infrastructure only; see mla_oracle.py)."""
from .mla_oracle import materialise_kv, softmax_attention, mla_decode, mla_decode_rows  # noqa: F401
