"""The five synthetic LSA decode workloads, as plain data.

Shapes follow the decode loop of "FlashMemory-DeepSeek-V4 Explained" (zhichai.net,
section 2): an indexer pass every tau = 64 decode steps, 64-token KV blocks, three
indexer layers (section 4) whose outputs are OR-ed. The pages give no block size,
window, head count or d_head; those numbers are the workload's own.

This module holds no arithmetic of the method: it only names sizes and seeds.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

BLOCK = 64          # tokens per KV block (one page of the HBM pool)
TAU = 64            # decode steps per indexer pass
N_LAYERS = 3        # indexer layers (at backbone depths 10, 12 and 20 on the pages)
D_INDEX = 128       # width of the indexer query / compressed block key


@dataclasses.dataclass
class LsaConfig:
    name: str
    B: int                       # sequences in the batch
    D: int                       # d_model of the hidden state the indexer reads
    W: int                       # recent window, tokens (multiple of BLOCK)
    H: int                       # query heads sharing one KV head (MQA)
    d: int                       # head dimension
    passes: int                  # indexer passes to run (each followed by TAU steps)
    seed: int
    ctx_tokens: Optional[List[int]] = None   # per-sequence context at pass 0
    ctx_uniform_blocks: Optional[tuple] = None  # (lo, hi) blocks, inclusive, drawn per sequence
    bias: Optional[List[float]] = None       # per-sequence indexer bias (shared by layers)
    bias_uniform: Optional[tuple] = None     # (lo, hi), drawn per sequence
    kidx_per_layer: bool = False             # one compressed key table per indexer layer
    rank: int = 0                            # > 0: factorised query encoders W_2 (W_1 h)
                                             #   through a rank-`rank` latent
    L: int = N_LAYERS
    d_i: int = D_INDEX
    block: int = BLOCK
    tau: int = TAU

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def wq_std(self) -> float:
        # variance-preserving projection: N(0, 1/D) entries
        return 1.0 / math.sqrt(self.D)

    @property
    def wb(self) -> int:
        return self.W // self.block


def _fixed(name, B, ctx, D, W, H, d, bias, passes, seed):
    return LsaConfig(name=name, B=B, D=D, W=W, H=H, d=d, passes=passes, seed=seed,
                     ctx_tokens=[ctx] * B, bias=[bias] * B)


def tiny() -> LsaConfig:
    """B=1, 16,384-token context, D=1024, 8 heads of 128, window 1,024, bias -2."""
    return _fixed("tiny_16k", 1, 16384, 1024, 1024, 8, 128, -2.0, 1, 0)


def mid_batch() -> LsaConfig:
    """B=8 x 131,072 tokens, D=4096, 64 heads of 512, window 4,096, bias -2."""
    return _fixed("mid_b8_128k", 8, 131072, 4096, 4096, 64, 512, -2.0, 1, 0)


def long_ctx() -> LsaConfig:
    """B=4 x 524,288 tokens, window 8,192, bias -2, four indexer passes."""
    return _fixed("long_b4_512k", 4, 524288, 4096, 8192, 64, 512, -2.0, 4, 0)


def one_million(bias: float = -2.0) -> LsaConfig:
    """B=1 x 1,048,576 tokens, window 8,192, bias swept over -1.5 / -2.0 / -2.5."""
    tag = {-1.5: "b15", -2.0: "b20", -2.5: "b25"}.get(bias, "b%g" % bias)
    return _fixed("1m_" + tag, 1, 1 << 20, 4096, 8192, 64, 512, bias, 1, 0)


def one_million_layer_keys() -> LsaConfig:
    """1M-token sequence at bias -2 whose three indexer layers each score against their
    own compressed key table (K_idx [3][blocks][128])."""
    c = _fixed("1m_b20_lk", 1, 1 << 20, 4096, 8192, 64, 512, -2.0, 1, 0)
    c.kidx_per_layer = True
    return c


def one_million_latent() -> LsaConfig:
    """1M-token sequence at bias -2 whose query encoders read a rank-2048 query latent
    of the backbone instead of the 4096-wide hidden state (W_q [3][128][2048])."""
    return _fixed("1m_b20_r2048", 1, 1 << 20, 2048, 8192, 64, 512, -2.0, 1, 0)


def one_million_lowrank() -> LsaConfig:
    """1M-token sequence at bias -2 whose query encoders are factorised through a rank-2048
    latent: q = W_2 (W_1 h), W_1 [3][2048][4096], W_2 [3][128][2048]."""
    c = _fixed("1m_b20_lr2048", 1, 1 << 20, 4096, 8192, 64, 512, -2.0, 1, 0)
    c.rank = 2048
    return c


def ragged_mix() -> LsaConfig:
    """B=64, context U{512..4096} blocks per sequence, bias U(-3,-1) per sequence, seed 7."""
    return LsaConfig(name="ragged_b64", B=64, D=4096, W=4096, H=64, d=512, passes=1, seed=7,
                     ctx_uniform_blocks=(512, 4096), bias_uniform=(-3.0, -1.0))


def all_configs() -> List[LsaConfig]:
    return [tiny(), mid_batch(), long_ctx(), one_million(-1.5), one_million(-2.0),
            one_million(-2.5), ragged_mix(), one_million_layer_keys(), one_million_latent(),
            one_million_lowrank()]


def by_name(name: str) -> LsaConfig:
    for c in all_configs():
        if c.name == name:
            return c
    raise KeyError(name)


def scaled_down(cfg: LsaConfig, ctx_blocks: int, B: Optional[int] = None,
                passes: Optional[int] = None, W: Optional[int] = None) -> LsaConfig:
    """Same head geometry and distributions at a context the CPU oracle finishes quickly."""
    B = cfg.B if B is None else B
    W = cfg.W if W is None else W
    out = dataclasses.replace(cfg, name=cfg.name + "_small", B=B, W=W,
                              passes=cfg.passes if passes is None else passes)
    if cfg.ctx_uniform_blocks is not None:
        lo = max(W // cfg.block + 1, ctx_blocks // 2)
        out.ctx_uniform_blocks = (lo, ctx_blocks)
        out.ctx_tokens = None
    else:
        out.ctx_tokens = [ctx_blocks * cfg.block] * B
    if cfg.bias is not None:
        out.bias = [cfg.bias[0]] * B
    return out



@dataclasses.dataclass
class DenoiseConfig:
    """Synthetic Lightning-Indexer logits for the label-denoising workload: per token
    window, `layers` CSA layers score `blocks` KV blocks. Logits are N(0, sigma^2) with
    `relevant` blocks per window raised by `boost` in each layer with probability 1/2."""
    name: str
    windows: int
    layers: int = 21
    blocks: int = 16384
    sigma: float = 1.0
    boost: float = 5.0
    relevant: int = 300
    top_p: float = 0.6
    min_votes: int = 3
    seed: int = 0


def denoise_1m() -> DenoiseConfig:
    """64 token windows of a 1M-token context (16,384 blocks), 21 CSA layers."""
    return DenoiseConfig(name="denoise_1m", windows=64)


def denoise_tiny() -> DenoiseConfig:
    """4 windows over 1,000 blocks (a row that is not a multiple of 32)."""
    return DenoiseConfig(name="denoise_tiny", windows=4, blocks=1000, relevant=30, seed=3)
