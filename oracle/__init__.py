"""CPU oracle for the LSA decode hot path -- test infrastructure only (see lsa_oracle)."""
from .lsa_oracle import (bf16_to_f64, query_projection, block_logits, kept_blocks, index_pass,
                         n_candidates, attended_positions, softmax_attention, step_output,
                         decode_sequence, softmax_f64, top_p_set, denoise_labels, BLOCK)
