"""Float64 CPU oracle (test infrastructure only; see ``paged_attention``)."""
from .paged_attention import attend, decode, decode_step, gather, prefill, reshape_and_cache, slot_of_position, widen

__all__ = ["attend", "decode", "decode_step", "gather", "prefill", "reshape_and_cache", "slot_of_position", "widen"]
