"""CPU oracle of the Lookahead Sparse Attention (LSA) decode hot path.

TEST INFRASTRUCTURE ONLY. Nothing in the product library imports, links or runs this
module; only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use it. It shares no code with the CUDA path: the only thing both sides
have in common is the seeded input generator (``lsa_inputs``), which holds none of
the method's arithmetic.

What it computes, step by step, following the inference loop of
"FlashMemory-DeepSeek-V4 Explained: Replacing Memory Sponge with a Fortune Teller via
Lookahead Sparse Attention" (zhichai.net), section 2 "Core Idea of LSA", steps 1-5:

  1. every tau = 64 decode steps the Neural Memory Indexer runs;
  2. each indexer layer's query encoder projects the current hidden state,
     q_l = W_q,l . h_l (section 3: only the small query projections are trained;
     section 4: independent indexers at three backbone layers);
  3. each historical block is scored against its frozen compressed key K_idx[c]
     (section 3, "KIComp"; the dual-encoder formulation of the abstract on the
     1kpapers.com page), z_l[c] = q_l . K_idx[c] / sqrt(d_i) + bias, and a block is
     kept when sigmoid(z) > 0.5, i.e. z > 0; the three layers are OR-ed
     (section 4, union strategy);
  4. the next 64 decode steps attend only over the kept blocks (plus the recent
     window and the tokens decoded since the pass started);
  5. after 64 steps the indexer runs again.

Readings where the pages are silent:
  * blocks are 64 tokens; the recent window W is part of the workload;
  * only blocks that end before the window are candidates;
  * the window grows with the decoded tokens inside a pass and is re-based at the
    next pass; the current token attends to itself;
  * the threshold is strict: z == 0 is not kept;
  * attention is exact softmax attention with scale 1/sqrt(d), one KV head shared by
    all query heads, no mask beyond the attended token set.

Precision: every input is bf16 (given as raw uint16 bit patterns, decoded here
exactly); all arithmetic is float64, with numpy matmul as the only library step.
The selection decision is taken on the float64 logit.

Parity status: pinned by tests/test_oracle.py (closed forms, brute force on tiny
inputs, special cases that reduce to textbook softmax attention, selection rates
against their closed form). Absolute values on the full-size synthetic workloads
have no printed worked example on the pages; they are pinned only through those
checks.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

BLOCK = 64


# ---------------------------------------------------------------------------------
# bf16 decoding
# ---------------------------------------------------------------------------------
def bf16_to_f64(bits) -> np.ndarray:
    """Exact value of bf16 bit patterns: bf16 is the upper half of an IEEE float32."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------------
# indexer
# ---------------------------------------------------------------------------------
def query_projection(w_q: np.ndarray, h: np.ndarray) -> np.ndarray:
    """q_l = W_q,l . h_l for every indexer layer l.

    w_q: [L][d_i][D] (row j of layer l is the weight vector of query component j)
    h:   [L][D]      (the hidden state read at layer l)
    returns q: [L][d_i]
    Query encoder of section 3 of the zhichai.net explainer; one per layer (section 4).
    """
    L = w_q.shape[0]
    assert h.shape == (L, w_q.shape[2])
    return np.stack([w_q[l] @ h[l] for l in range(L)])


def query_projection_lowrank(w_1: np.ndarray, w_2: np.ndarray, h: np.ndarray) -> np.ndarray:
    """q_l = W_2,l . (W_1,l . h_l): each layer's query encoder factorised through a rank-r
    latent (the "low-rank query projection (r=2048)" of section 4 of the zhichai.net
    explainer, read as two stacked linear maps).

    w_1: [L][r][D] (down-projection), w_2: [L][d_i][r] (up-projection), h: [L][D].
    returns q: [L][d_i]. The latent W_1,l . h_l is kept exact (float64), not rounded.
    """
    L = w_1.shape[0]
    assert w_2.shape[0] == L and w_2.shape[2] == w_1.shape[1] and h.shape == (L, w_1.shape[2])
    return np.stack([w_2[l] @ (w_1[l] @ h[l]) for l in range(L)])


def block_logits(q: np.ndarray, k_idx: np.ndarray, bias: float) -> np.ndarray:
    """z_l[c] = q_l . K_idx[c] / sqrt(d_i) + bias, for every layer l and block c.

    q: [L][d_i]; k_idx: [n][d_i] (one frozen compressed key per candidate block,
    shared by the layers) or [L][n][d_i] (each indexer layer with its own keys: the
    "three small projection matrices" of section 3 paired with per-layer key tables).
    returns z: [L][n]. Scoring of step 3 of section 2.
    """
    d_i = k_idx.shape[-1]
    assert q.shape[1] == d_i
    if k_idx.ndim == 3:
        assert k_idx.shape[0] == q.shape[0]
        return np.stack([k_idx[l] @ q[l] for l in range(q.shape[0])]) / math.sqrt(d_i) + bias
    return (q @ k_idx.T) / math.sqrt(d_i) + bias


def kept_blocks(z: np.ndarray) -> np.ndarray:
    """Ids of blocks kept by at least one layer (sigmoid(z) > 0.5 <=> z > 0), ascending.

    Sigmoid threshold of step 3 of section 2 and the OR-union of section 4.
    """
    keep_any = np.zeros(z.shape[1], dtype=bool)
    for l in range(z.shape[0]):
        keep_any |= z[l] > 0.0
    return np.flatnonzero(keep_any).astype(np.int64)


def index_pass(w_q_bits, h_bits, k_idx_bits, bias: float):
    """One indexer pass for one sequence.

    w_q_bits [L][d_i][D], h_bits [L][D], k_idx_bits [n_cand][d_i] or, with per-layer
    keys, [L][n_cand][d_i] (bf16 bit patterns of the candidate blocks only). Returns
    (ids, z) with z float64 [L][n_cand].
    """
    q = query_projection(bf16_to_f64(w_q_bits), bf16_to_f64(h_bits))
    z = block_logits(q, bf16_to_f64(k_idx_bits), float(bias))
    return kept_blocks(z), z


def index_pass_lowrank(w_1_bits, w_2_bits, h_bits, k_idx_bits, bias: float):
    """index_pass with the factorised query encoder: w_1_bits [L][r][D], w_2_bits
    [L][d_i][r] (bf16 bit patterns); the rest as index_pass. Returns (ids, z)."""
    q = query_projection_lowrank(bf16_to_f64(w_1_bits), bf16_to_f64(w_2_bits),
                                 bf16_to_f64(h_bits))
    z = block_logits(q, bf16_to_f64(k_idx_bits), float(bias))
    return kept_blocks(z), z


def n_candidates(n_ctx: int, window: int, block: int = BLOCK) -> int:
    """Blocks that end at or before the start of the window (context n_ctx tokens)."""
    return max(0, (n_ctx - window) // block)


# ---------------------------------------------------------------------------------
# attended set and attention
# ---------------------------------------------------------------------------------
def attended_positions(ids: Sequence[int], n_ctx: int, window: int, s: int,
                       block: int = BLOCK) -> np.ndarray:
    """History positions attended at decode step s of a pass that started at n_ctx.

    The kept blocks' tokens, then the window [n_ctx - W, n_ctx) and the tokens decoded
    since the pass started, [n_ctx, n_ctx + s] (the current token included).
    """
    parts = [np.arange(int(c) * block, int(c) * block + block, dtype=np.int64) for c in ids]
    parts.append(np.arange(max(0, n_ctx - window), n_ctx + s + 1, dtype=np.int64))
    pos = np.concatenate(parts)
    return np.unique(pos)


def softmax_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """Exact single-query softmax attention for each query head, one shared KV head.

    q: [H][d]; K, V: [T][d]. out[h] = sum_t softmax_t(scale * q_h . K_t) V_t.
    """
    if K.shape[0] == 0:
        return np.zeros((q.shape[0], V.shape[1]))
    s = scale * (q @ K.T)                       # [H][T]
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    return (p @ V) / p.sum(axis=1, keepdims=True)


def softmax_attention_bits(q: np.ndarray, K_bits, V_bits, scale: float,
                           chunk: int = 65536) -> np.ndarray:
    """softmax_attention over keys and values given as bf16 bit patterns [T][d], decoded
    a chunk of rows at a time, so that a context of a million tokens fits in memory.

    Two passes: every score scale * q_h . K_t (float64), then the exact softmax weights
    exp(score - max) applied to V chunk by chunk. Equal to softmax_attention on the
    decoded arrays up to the order of the float64 sums.
    """
    T = K_bits.shape[0]
    if T == 0:
        return np.zeros((q.shape[0], V_bits.shape[1]))
    scores = np.empty((q.shape[0], T))
    for t0 in range(0, T, chunk):
        scores[:, t0:t0 + chunk] = scale * (q @ bf16_to_f64(K_bits[t0:t0 + chunk]).T)
    p = np.exp(scores - scores.max(axis=1, keepdims=True))
    out = np.zeros((q.shape[0], V_bits.shape[1]))
    for t0 in range(0, T, chunk):
        out += p[:, t0:t0 + chunk] @ bf16_to_f64(V_bits[t0:t0 + chunk])
    return out / p.sum(axis=1, keepdims=True)


def step_output(q_bits, K_bits, V_bits, ids, n_ctx: int, window: int, s: int, scale: float,
                heads: Optional[Sequence[int]] = None, block: int = BLOCK) -> np.ndarray:
    """Attention output of one decode step of one sequence, float64 [H'][d].

    K_bits / V_bits: bf16 bit patterns [tokens][d] of the sequence's history (any
    array supporting fancy row indexing, e.g. a numpy view of the host pool).
    heads: optional subset of query heads (sampled checks at full size).
    """
    pos = attended_positions(ids, n_ctx, window, s, block)
    q = bf16_to_f64(q_bits)
    if heads is not None:
        q = q[np.asarray(heads)]
    K = bf16_to_f64(K_bits[pos])
    V = bf16_to_f64(V_bits[pos])
    return softmax_attention(q, K, V, scale)


def decode_sequence(w_q_bits, k_idx_bits, K_bits, V_bits, bias: float, n_ctx0: int,
                    window: int, scale: float, h_of_pass, q_of_step, passes: int,
                    steps: int = 64, block: int = BLOCK):
    """The whole loop of section 2 for one sequence.

    h_of_pass(p) -> bf16 bits [L][D]; q_of_step(p, s) -> bf16 bits [H][d].
    k_idx_bits: [blocks][d_i] for the sequence's whole history.
    Returns a list over passes of (ids, z, [out_s for s in range(steps)]).
    """
    result = []
    for p in range(passes):
        n_ctx = n_ctx0 + steps * p
        nc = n_candidates(n_ctx, window, block)
        ids, z = index_pass(w_q_bits, h_of_pass(p), k_idx_bits[:nc], bias)
        outs = [step_output(q_of_step(p, s), K_bits, V_bits, ids, n_ctx, window, s, scale,
                            block=block) for s in range(steps)]
        result.append((ids, z, outs))
    return result


# ---------------------------------------------------------------------------------
# Label denoising (training labels for the indexer)
# ---------------------------------------------------------------------------------
# "FlashMemory-DeepSeek-V4 Explained" (zhichai.net), section 3, "Label Denoising
# Pipeline": the raw Lightning Indexer logits of each CSA layer are softmax-normalised
# over the blocks; each layer keeps the smallest set of blocks whose cumulative
# probability reaches p = 0.6 (top-p instead of a fixed top-k); a block is a positive
# label of the token window when at least 3 of the 21 layers keep it.
def softmax_f64(x: np.ndarray) -> np.ndarray:
    """Softmax of one row in float64 (max-shifted)."""
    x = np.asarray(x, dtype=np.float64)
    e = np.exp(x - x.max())
    return e / e.sum()


def top_p_set(probs: np.ndarray, p: float) -> np.ndarray:
    """Ids (ascending) of the smallest set of entries whose probabilities sum to >= p,
    taking entries in decreasing probability, equal probabilities in increasing id."""
    order = np.argsort(-probs, kind="stable")
    cum = np.cumsum(probs[order])
    k = int(np.searchsorted(cum, p, side="left"))    # first k with cum[k] >= p
    k = min(k, len(order) - 1)
    return np.sort(order[:k + 1])


def denoise_labels(logits: np.ndarray, p: float = 0.6, min_votes: int = 3):
    """logits float [n_layers][n_blocks] of one token window. Returns (labels, sets):
    labels = ascending ids kept by at least min_votes layers; sets = each layer's
    top-p set."""
    sets = [top_p_set(softmax_f64(row), p) for row in logits]
    votes = np.zeros(logits.shape[1], dtype=np.int64)
    for s in sets:
        votes[s] += 1
    return np.flatnonzero(votes >= min_votes).astype(np.int64), sets
