"""fp64 CPU oracle (test infrastructure only; see oracle.py's header)."""
from .oracle import (Geom, attention, block_len, block_probs, build_mask, forward, lpt_order,
                     pool, reorder, select_row, slot_of_token, slot_of_token_loops, slot_valid,
                     unreorder)

__all__ = ["Geom", "attention", "block_len", "block_probs", "build_mask", "forward", "lpt_order",
           "pool", "reorder", "select_row", "slot_of_token", "slot_of_token_loops", "slot_valid",
           "unreorder"]
