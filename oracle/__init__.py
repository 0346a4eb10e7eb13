"""CPU oracle for the ternary linear layer: test infrastructure only (see tern_oracle)."""
from .tern_oracle import (  # noqa: F401
    GROUP, pack_exec, unpack_exec, pack_store, unpack_store, store_row_bytes,
    slot_map, row_bitmap, dequant, linear, round_fp16, rel_err, bits,
    ELEM_BLOCK, elem_blocks, pack_elem, unpack_elem, bits_elem, rotate, ternarize, fit_groups,
)
