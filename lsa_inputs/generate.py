"""Seeded synthetic inputs for the LSA decode workloads.

Both the CUDA path and the CPU oracle are fed from here; this module holds no
arithmetic of the method (no projection, scoring, selection or attention), only
random draws and their bf16 casts (round to nearest even, torch's fp32 -> bf16 copy).

Every tensor is drawn from its own named stream (a torch CPU generator seeded by a
hash of the workload seed and the stream's name), so any piece -- one pass's hidden
states, one step's queries, one chunk of the cold pool -- can be regenerated alone,
and the draws do not depend on the device or the number of threads used.

Distributions (all i.i.d.): W_q ~ N(0, 1/D); h, K_idx, K, V, q ~ N(0, 1); all cast
to bf16. The KV history of a sequence is drawn for its final context (pass-0
context plus 64 tokens per pass), so the token decode step s of pass p appends is
simply history position N_p + s.
"""
from __future__ import annotations

import dataclasses
import hashlib
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Optional, Sequence

import numpy as np
import torch

from .configs import LsaConfig

POOL_CHUNK_BLOCKS = 256


def stream_seed(base: int, *keys) -> int:
    h = hashlib.blake2b(repr((int(base),) + tuple(keys)).encode(), digest_size=8)
    return int.from_bytes(h.digest(), "little") & ((1 << 63) - 1)


def _gen(base: int, *keys) -> torch.Generator:
    return torch.Generator().manual_seed(stream_seed(base, *keys))


def _randn_bf16(shape, gen: torch.Generator, std: float = 1.0) -> torch.Tensor:
    x = torch.randn(shape, generator=gen, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


class Workload:
    """All inputs of one LSA decode run (one config)."""

    def __init__(self, cfg: LsaConfig, pin: bool = False, threads: Optional[int] = None,
                 with_pool: bool = True, seqs: Optional[Sequence[int]] = None):
        """seqs: restrict the run to these sequences of the batch (a shard). Every tensor
        holds exactly the values the whole-batch workload draws for those sequences."""
        self.cfg = cfg
        B, blk = cfg.B, cfg.block
        # context lengths (tokens at pass 0) and per-sequence bias
        if cfg.ctx_tokens is not None:
            ctx = np.asarray(cfg.ctx_tokens, dtype=np.int64)
        else:
            lo, hi = cfg.ctx_uniform_blocks
            g = _gen(cfg.seed, "ctx_blocks")
            ctx = torch.randint(lo, hi + 1, (B,), generator=g).numpy().astype(np.int64) * blk
        assert ctx.shape == (B,) and np.all(ctx % blk == 0) and np.all(ctx > 0)
        if cfg.bias is not None:
            bias = np.asarray(cfg.bias, dtype=np.float32)
        else:
            lo, hi = cfg.bias_uniform
            g = _gen(cfg.seed, "bias")
            bias = (lo + (hi - lo) * torch.rand((B,), generator=g, dtype=torch.float64)).numpy()
            bias = bias.astype(np.float32)
        # the whole batch's block offsets fix the cold pool's draws (chunks of blocks)
        off_all = np.zeros(B + 1, dtype=np.int64)
        off_all[1:] = np.cumsum(ctx // blk + cfg.passes)
        self.seqs = np.arange(B) if seqs is None else np.asarray(list(seqs), dtype=np.int64)
        if seqs is not None:
            ctx, bias = ctx[self.seqs], bias[self.seqs]
            self.cfg = cfg = dataclasses.replace(
                cfg, name="%s_seqs%d-%d" % (cfg.name, int(self.seqs[0]), int(self.seqs[-1])),
                B=len(self.seqs), ctx_tokens=[int(x) for x in ctx], ctx_uniform_blocks=None,
                bias=[float(x) for x in bias], bias_uniform=None)
            B = cfg.B
        self._off_all = off_all
        self._full_B = len(off_all) - 1
        self.ctx0 = ctx
        self.nb0 = ctx // blk
        self.nb_final = self.nb0 + cfg.passes
        self.bias = bias
        off = np.zeros(B + 1, dtype=np.int64)
        off[1:] = np.cumsum(self.nb_final)
        self.blk_off = off            # first block of sequence b in k_idx and in the host pool
        self.total_blocks = int(off[-1])

        self.w_q = _randn_bf16((cfg.L, cfg.d_i, cfg.D), _gen(cfg.seed, "w_q"), cfg.wq_std)
        self.w_1 = self.w_2 = None
        if cfg.rank > 0:
            # factorised encoders: W_1 ~ N(0, 1/D), W_2 ~ N(0, 1/rank) (variance-preserving)
            self.w_1 = _randn_bf16((cfg.L, cfg.rank, cfg.D), _gen(cfg.seed, "w_1"),
                                   cfg.D ** -0.5)
            self.w_2 = _randn_bf16((cfg.L, cfg.d_i, cfg.rank), _gen(cfg.seed, "w_2"),
                                   cfg.rank ** -0.5)
        gb = [int(x) for x in self.seqs]          # global sequence index of each row
        if cfg.kidx_per_layer:
            # one table per layer: [L][blocks][d_i]
            self.k_idx = torch.empty((cfg.L, self.total_blocks, cfg.d_i), dtype=torch.bfloat16)
            for l in range(cfg.L):
                for b in range(B):
                    self.k_idx[l, off[b]:off[b + 1]] = _randn_bf16(
                        (int(self.nb_final[b]), cfg.d_i), _gen(cfg.seed, "k_idx_layer", l, gb[b]))
        else:
            self.k_idx = torch.empty((self.total_blocks, cfg.d_i), dtype=torch.bfloat16)
            for b in range(B):
                self.k_idx[off[b]:off[b + 1]] = _randn_bf16(
                    (int(self.nb_final[b]), cfg.d_i), _gen(cfg.seed, "k_idx", gb[b]))
        self.host_pool = None
        if with_pool:
            self.host_pool = torch.empty((self.total_blocks, 2, blk, cfg.d), dtype=torch.bfloat16,
                                         pin_memory=pin)
            self._fill_pool(threads)

    # -- cold pool ---------------------------------------------------------------
    def _fill_pool(self, threads):
        n = self.total_blocks
        flat = self.host_pool.view(n, -1)
        seed = self.cfg.seed
        n_all = int(self._off_all[-1])
        # (global chunk, [global block range wanted], local destination of its first block)
        chunks = []
        for b, g in enumerate(int(x) for x in self.seqs):
            g0, g1 = int(self._off_all[g]), int(self._off_all[g + 1])
            c0 = (g0 // POOL_CHUNK_BLOCKS) * POOL_CHUNK_BLOCKS
            for lo in range(c0, g1, POOL_CHUNK_BLOCKS):
                hi = min(lo + POOL_CHUNK_BLOCKS, n_all)
                a0, a1 = max(lo, g0), min(hi, g1)
                chunks.append((lo, hi, a0, a1, int(self.blk_off[b]) + a0 - g0))

        def work(c):
            lo, hi, a0, a1, dst = c
            x = torch.randn((hi - lo, flat.shape[1]), generator=_gen(seed, "pool", lo),
                            dtype=torch.float32)
            flat[dst:dst + a1 - a0].copy_(x[a0 - lo:a1 - lo])

        nthr = threads or min(32, os.cpu_count() or 1)
        if len(chunks) == 1 or nthr == 1:
            for c in chunks:
                work(c)
            return
        old = torch.get_num_threads()
        torch.set_num_threads(1)
        try:
            with ThreadPoolExecutor(nthr) as ex:
                list(ex.map(work, chunks))
        finally:
            torch.set_num_threads(old)

    # -- per pass / per step draws -------------------------------------------------
    def ctx_at(self, p: int) -> np.ndarray:
        """Tokens of each sequence's context when pass p starts."""
        return self.ctx0 + self.cfg.tau * p

    def h(self, p: int) -> torch.Tensor:
        """Hidden states the indexer reads at the start of pass p: bf16 [L][B][D]."""
        c = self.cfg
        x = _randn_bf16((c.L, self._full_B, c.D), _gen(c.seed, "h", p))
        return x if c.B == self._full_B else x[:, torch.from_numpy(self.seqs)].contiguous()

    def q(self, p: int, s: int) -> torch.Tensor:
        """Queries of decode step s of pass p: bf16 [B][H][d]."""
        c = self.cfg
        x = _randn_bf16((self._full_B, c.H, c.d), _gen(c.seed, "q", p, s))
        return x if c.B == self._full_B else x[torch.from_numpy(self.seqs)].contiguous()

    def token_kv(self, b: int, pos: int):
        """(K, V) bf16 [d] of history position pos of sequence b."""
        blk = self.cfg.block
        page = self.host_pool[self.blk_off[b] + pos // blk]
        return page[0, pos % blk], page[1, pos % blk]

    def kv_new(self, p: int, s: int):
        """The token appended at step s of pass p: (k, v) bf16 [B][d] each."""
        pos = self.ctx_at(p) + s
        ks = torch.stack([self.token_kv(b, int(pos[b]))[0] for b in range(self.cfg.B)])
        vs = torch.stack([self.token_kv(b, int(pos[b]))[1] for b in range(self.cfg.B)])
        return ks, vs

    def seq_kv(self, b: int):
        """Views K, V bf16 [tokens][d] over the whole drawn history of sequence b."""
        pages = self.host_pool[self.blk_off[b]:self.blk_off[b + 1]]
        d = self.cfg.d
        return pages[:, 0].reshape(-1, d), pages[:, 1].reshape(-1, d)

    def seq_k_idx(self, b: int) -> torch.Tensor:
        """Compressed keys of sequence b: [blocks][d_i], or [L][blocks][d_i] per layer."""
        if self.k_idx.dim() == 3:
            return self.k_idx[:, self.blk_off[b]:self.blk_off[b + 1]]
        return self.k_idx[self.blk_off[b]:self.blk_off[b + 1]]


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The raw bf16 bit patterns of a tensor, as a numpy uint16 array (no conversion)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def denoise_logits(cfg, w: int) -> torch.Tensor:
    """Lightning-Indexer logits of token window w: float32 [layers][blocks]."""
    x = torch.randn((cfg.layers, cfg.blocks), generator=_gen(cfg.seed, "dn_noise", w),
                    dtype=torch.float32)
    if cfg.sigma != 1.0:
        x.mul_(cfg.sigma)
    rel = torch.randperm(cfg.blocks, generator=_gen(cfg.seed, "dn_relevant", w))[:cfg.relevant]
    active = torch.rand((cfg.layers, cfg.relevant), generator=_gen(cfg.seed, "dn_active", w)) < 0.5
    for l in range(cfg.layers):
        x[l, rel[active[l]]] += cfg.boost
    return x


def denoise_batch(cfg) -> torch.Tensor:
    """All windows: float32 [windows][layers][blocks]."""
    return torch.stack([denoise_logits(cfg, w) for w in range(cfg.windows)])
