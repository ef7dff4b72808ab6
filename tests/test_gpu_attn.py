"""GPU parity of lsa_decode_attn (split-K tcgen05 decode attention + LSE merge) against
the oracle's exact softmax attention, on synthetic paged KV with ragged block tables."""
import math
import zlib

import numpy as np
import pytest
import torch

import lookahead_sparse_kv_lsa_b200 as lsa
import oracle
from gpu_util import compare_attention, bits, paged_oracle_out

pytestmark = pytest.mark.gpu


def make_case(seed, B, H, d, entries, tails, n_pages=None, q_scale=1.0, garbage=100.0):
    """Random pool, random distinct pages per sequence; tokens past tail_len hold `garbage`."""
    g = torch.Generator().manual_seed(seed)
    total = int(sum(entries))
    n_pages = n_pages or max(1, total + 3)
    pool = torch.randn((n_pages, 2, 64, d), generator=g).to(torch.bfloat16)
    perm = torch.randperm(n_pages, generator=g)
    bt_stride = max(1, max(entries))
    bt = torch.full((B, bt_stride), -7, dtype=torch.int32)
    k = 0
    for b in range(B):
        for e in range(entries[b]):
            bt[b, e] = int(perm[k]); k += 1
        if entries[b] > 0:
            last = int(bt[b, entries[b] - 1])
            pool[last, :, tails[b]:, :] = garbage
    q = (torch.randn((B, H, d), generator=g) * q_scale).to(torch.bfloat16)
    return pool, bt, q


oracle_out = paged_oracle_out


def run_gpu(pool, bt, q, entries, tails, scale):
    dev = torch.device("cuda")
    B, H, d = q.shape
    pool_d, bt_d, q_d = pool.to(dev), bt.to(dev), q.to(dev)
    ne = torch.tensor(entries, dtype=torch.int32, device=dev)
    tl = torch.tensor(tails, dtype=torch.int32, device=dev)
    out = torch.full((B, H, d), float("nan"), dtype=torch.bfloat16, device=dev)
    ws = torch.zeros(lsa.decode_attn_workspace_size(B, H, d), dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    lsa.lsa_decode_attn(q_d, pool_d, bt_d, ne, tl, scale, out, ws, err)
    torch.cuda.synchronize()
    return out, int(err.item())


CASES = [
    # (name, B, H, d, entries, tails, q_scale)
    ("single_token", 1, 8, 128, [1], [1], 1.0),
    ("one_page_partial", 1, 8, 128, [1], [37], 1.0),
    ("two_pages", 1, 64, 512, [2], [64], 1.0),
    ("odd_pages_tail33", 1, 64, 512, [5], [33], 1.0),
    ("tail32_boundary", 2, 64, 512, [3, 4], [32, 31], 1.0),
    ("h8_d128_many", 1, 8, 128, [300], [17], 1.0),
    ("h64_d512_many", 1, 64, 512, [700], [64], 1.0),
    ("ragged_batch", 6, 64, 512, [1, 40, 3, 0, 97, 250], [5, 64, 1, 1, 49, 12], 1.0),
    ("h20_d256", 3, 20, 256, [10, 11, 12], [7, 8, 9], 1.0),
    ("h64_d384", 2, 64, 384, [30, 2], [60, 3], 1.0),
    ("large_scores_rescale", 2, 64, 512, [200, 150], [64, 20], 8.0),
    ("h8_large_scores", 1, 8, 128, [400], [64], 10.0),
    ("tiny_batch_many_seqs", 40, 8, 128, [1 + (i * 7) % 13 for i in range(40)],
     [1 + (i * 11) % 64 for i in range(40)], 1.0),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_decode_attn_matches_oracle(cuda_ok, case):
    name, B, H, d, entries, tails, qs = case
    scale = 1.0 / math.sqrt(d)
    pool, bt, q = make_case(zlib.crc32(name.encode()) & 0xFFFF, B, H, d, entries, tails, q_scale=qs)
    out, err = run_gpu(pool, bt, q, entries, tails, scale)
    assert err == 0, "device error word %d" % err
    ref = oracle_out(pool, bt, q, entries, tails, scale)
    compare_attention(out, ref, name)


def test_single_token_returns_v(cuda_ok):
    pool, bt, q = make_case(3, 1, 8, 128, [1], [1])
    out, err = run_gpu(pool, bt, q, [1], [1], 1 / math.sqrt(128))
    v = pool[int(bt[0, 0]), 1, 0].float()
    assert err == 0
    assert torch.equal(out[0].float().cpu(), v.expand(8, 128))


def test_bad_page_is_flagged_not_read(cuda_ok):
    pool, bt, q = make_case(4, 1, 8, 128, [3], [64])
    bt[0, 1] = 10_000_000  # far outside the pool
    out, err = run_gpu(pool, bt, q, [3], [64], 1 / math.sqrt(128))
    assert err & lsa._lib.DEVERR_BAD_PAGE
    assert torch.isfinite(out.float()).all()


def test_malformed_sizes_flagged(cuda_ok):
    pool, bt, q = make_case(5, 2, 8, 128, [2, 2], [10, 10])
    out, err = run_gpu(pool, bt, q, [2, 2], [0, 65], 1 / math.sqrt(128))
    assert err & lsa._lib.DEVERR_BAD_SIZE
    assert torch.count_nonzero(out.float()) == 0
