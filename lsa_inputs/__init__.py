"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the CPU oracle."""
from .configs import (BLOCK, TAU, N_LAYERS, D_INDEX, LsaConfig, tiny, mid_batch, long_ctx,
                      one_million, ragged_mix, one_million_layer_keys, one_million_latent,
                      one_million_lowrank,
                      all_configs, by_name, scaled_down, DenoiseConfig, denoise_1m,
                      denoise_tiny)
from .generate import Workload, bf16_bits, stream_seed, denoise_logits, denoise_batch
