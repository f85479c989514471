"""fp64 CPU oracles (test infrastructure only; see moe_oracle and gdn_oracle)."""
from .moe_oracle import (GROUP, SECTION_NAMES, SLOT_POLICIES, SlotCache, bf16_to_f64, blob_layout, dequantize,
                         expert_forward, expert_hidden, f64_to_bf16_bits, group_pairs,
                         layer_forward, layer_forward_by_expert, layer_forward_dense_masked, read_expert, route,
                         router_logits, sigmoid, silu, unpack_codes)
from .gdn_oracle import gdn_step, gdn_steps, l2_normalize
