"""fp64 CPU oracle (test infrastructure only; see oracle.py's header)."""
from .oracle import (E4M3_MAX, EXPCAST_BIAS, EXPCAST_TAU, Geom, attention, attention_fp8,
                     block_coords, block_len, block_probs, build_mask, csr_from_keep,
                     e4m3_decode, e4m3_encode, expcast_code, forward, in_stripe, lpt_order, pool,
                     reorder, select_row, slot_of_token, slot_of_token_loops, slot_valid,
                     stripe_keep, stripe_keep_loops, stripe_mask, unreorder, v_smooth,
                     v_smooth_dequant)

__all__ = ["E4M3_MAX", "EXPCAST_BIAS", "EXPCAST_TAU", "attention_fp8", "e4m3_decode",
           "e4m3_encode", "expcast_code", "v_smooth", "v_smooth_dequant",
           "Geom", "attention", "block_coords", "block_len", "block_probs", "build_mask",
           "csr_from_keep", "forward", "in_stripe", "lpt_order", "pool", "reorder", "select_row",
           "slot_of_token", "slot_of_token_loops", "slot_valid", "stripe_keep",
           "stripe_keep_loops", "stripe_mask", "unreorder"]
