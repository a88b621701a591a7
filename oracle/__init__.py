"""fp64 CPU oracle for paged-KV attention. Test infrastructure only (see paged_attention.py)."""
from .paged_attention import (  # noqa: F401
    attention, copy_blocks, gather_sequence, merge, num_partitions, reshape_and_cache, slot_mapping,
    softmax_attention, splitkv_partials, step,
)
