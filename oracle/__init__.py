"""CPU oracle for the LSA decode hot path -- test infrastructure only (see lsa_oracle)."""
from .lsa_oracle import (bf16_to_f64, query_projection, query_projection_lowrank, block_logits,
                         kept_blocks, index_pass, index_pass_lowrank, n_candidates,
                         attended_positions, softmax_attention, softmax_attention_bits,
                         step_output, decode_sequence, softmax_f64, top_p_set, denoise_labels,
                         BLOCK)
