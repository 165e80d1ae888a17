"""fp64 CPU oracle (test infrastructure only; see oracle.py's header)."""
from .oracle import (Geom, attention, block_coords, block_len, block_probs, build_mask,
                     csr_from_keep, forward, in_stripe, lpt_order, pool, reorder, select_row,
                     slot_of_token, slot_of_token_loops, slot_valid, stripe_keep,
                     stripe_keep_loops, stripe_mask, unreorder)

__all__ = ["Geom", "attention", "block_coords", "block_len", "block_probs", "build_mask",
           "csr_from_keep", "forward", "in_stripe", "lpt_order", "pool", "reorder", "select_row",
           "slot_of_token", "slot_of_token_loops", "slot_valid", "stripe_keep",
           "stripe_keep_loops", "stripe_mask", "unreorder"]
