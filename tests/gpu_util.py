"""Helpers shared by the GPU parity tests: tolerances, comparisons, oracle adapters."""
import math

import numpy as np
import torch

from lsa_inputs import bf16_bits
import oracle

# Attention output tolerance for bf16 inputs with fp32 accumulation (bf16 output).
ATTN_MAX_ABS = 1e-2
ATTN_REL_L2 = 5e-3
# Logit tolerance: the kernel's fp32 q (D-term sums) and fp32 z (128-term dot) differ from
# the oracle's fp64 values by at most a few ulp of the partial sums' magnitudes; with
# |w_q . h| ~ 1 and |q . k| ~ 11 that is ~1e-5. 1e-4 leaves margin.
LOGIT_ABS = 1e-4
# Blocks whose oracle logit is this close to 0 in some layer may legitimately flip.
NEAR_TIE = 1e-3


def compare_attention(got: torch.Tensor, ref: np.ndarray, what: str = ""):
    g = got.float().cpu().numpy().astype(np.float64)
    err = np.abs(g - ref)
    max_abs = float(err.max()) if err.size else 0.0
    denom = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(g - ref) / denom) if denom > 0 else float(np.linalg.norm(g))
    assert np.all(np.isfinite(g)), "%s: non-finite output" % what
    assert max_abs <= ATTN_MAX_ABS, "%s: max abs err %.3g > %.3g" % (what, max_abs, ATTN_MAX_ABS)
    assert rel <= ATTN_REL_L2, "%s: rel L2 err %.3g > %.3g" % (what, rel, ATTN_REL_L2)
    return max_abs, rel


def compare_selection(gpu_ids, ref_ids, ref_z, what=""):
    """Ids must match exactly except blocks with min_l |z_l| < NEAR_TIE (returned)."""
    g, r = set(int(x) for x in gpu_ids), set(int(x) for x in ref_ids)
    diff = sorted(g ^ r)
    near = [c for c in diff if float(np.min(np.abs(ref_z[:, c]))) < NEAR_TIE]
    bad = [c for c in diff if c not in near]
    assert not bad, "%s: selection differs outside the near-tie band at %s" % (what, bad[:10])
    assert list(gpu_ids) == sorted(g), "%s: ids not ascending/unique" % what
    return near


def bits(t: torch.Tensor) -> np.ndarray:
    return bf16_bits(t.cpu() if t.is_cuda else t)


def paged_oracle_out(pool, bt, q, entries, tails, scale):
    """The oracle's attention over paged KV: sequence b attends to the tokens of pages
    bt[b][0 .. entries[b]-1], all 64 tokens of each except tails[b] of the last one.
    Returns float64 [B][H][d] (zero for a sequence without pages)."""
    B, H, d = q.shape
    pb = bits(pool)
    out = np.zeros((B, H, d))
    for b in range(B):
        if entries[b] == 0:
            continue
        Ks, Vs = [], []
        for e in range(entries[b]):
            page = int(bt[b, e])
            n = 64 if e < entries[b] - 1 else tails[b]
            Ks.append(pb[page, 0, :n])
            Vs.append(pb[page, 1, :n])
        K = oracle.bf16_to_f64(np.concatenate(Ks))
        V = oracle.bf16_to_f64(np.concatenate(Vs))
        out[b] = oracle.softmax_attention(oracle.bf16_to_f64(bits(q[b])), K, V, scale)
    return out
