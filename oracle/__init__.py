"""fp64 CPU oracle for paged decode attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  It shares no code with the CUDA library.
"""
from .oracle import (  # noqa: F401
    bytes_kv, bytes_mla, decode_gqa, decode_gqa_vis, decode_mla, dequantize_e4m3,
    e4m3_encode, e4m3_table, quantize_rows_e4m3, mla_absorb_q, mla_explicit,
    mla_project_out, set_threads, get_threads, slot_offset, visible_range,
)
