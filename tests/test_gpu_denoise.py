"""GPU parity of label denoising (lsa_denoise_labels) against the oracle.

Every row's kept set must be a prefix of the oracle's order (probability descending, equal
probabilities by increasing id), which involves no tolerance: ties in probability are ties
in the fp32 logit on both sides. Only the prefix length may differ, and only on rows where
the oracle's running mass passes top_p within EPS of it. The kernel's probabilities carry
fp32 rounding (at most about 6e-7 relative per block, from the exponent's fma and exp2),
and its sums are fp64 over fp32 partials. So its running mass differs from the exact one
by at most about 4e-7 of the total; EPS = 2e-6 gives a factor 5 of margin. Labels must
equal the oracle's on every block whose membership no near-tie row can change. They must
also equal, exactly, the vote over the kernel's own sets.
"""
import numpy as np
import pytest
import torch

import lookahead_sparse_kv_lsa_b200 as lsa
import lsa_inputs as LI
import oracle

pytestmark = pytest.mark.gpu

EPS = 2e-6


def run(logits: torch.Tensor, p=0.6, v=3, cap=4096, repeat=1):
    dev = torch.device("cuda")
    W, L, N = logits.shape
    NW = (N + 31) // 32
    x = logits.to(dev).contiguous()
    set_mask = torch.full((W, L, NW), -1, dtype=torch.int32, device=dev)
    set_cnt = torch.full((W, L), -1, dtype=torch.int32, device=dev)
    label_mask = torch.full((W, NW), -1, dtype=torch.int32, device=dev)
    label_ids = torch.full((W, max(cap, 1)), -7, dtype=torch.int32, device=dev)[:, :cap]
    label_ids = label_ids.contiguous()
    label_cnt = torch.full((W,), -1, dtype=torch.int32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    for _ in range(repeat):
        lsa.lsa_denoise_labels(x, set_mask, label_cnt, err, top_p=p, min_votes=v,
                               set_cnt=set_cnt, label_mask=label_mask,
                               label_ids=label_ids if cap > 0 else None)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return dict(set_mask=set_mask.cpu().numpy().view(np.uint32),
                set_cnt=set_cnt.cpu().numpy(), label_mask=label_mask.cpu().numpy().view(np.uint32),
                label_ids=label_ids.cpu().numpy(), label_cnt=label_cnt.cpu().numpy())


def bits(words: np.ndarray, N: int) -> np.ndarray:
    """[..., NW] u32 words -> [..., N] bool (bit c % 32 of word c // 32)."""
    b = np.unpackbits(words.view(np.uint8).reshape(*words.shape, 4), axis=-1, bitorder="little")
    return b.reshape(*words.shape[:-1], -1)[..., :N].astype(bool)


def check(logits: torch.Tensor, out, p=0.6, v=3, cap=4096):
    """Returns the number of near-tie rows."""
    x = logits.numpy()
    W, L, N = x.shape
    NW = (N + 31) // 32
    sets = bits(out["set_mask"], N)                      # [W][L][N]
    assert not bits(out["set_mask"], 32 * NW)[..., N:].any(), "bits past n_blocks set"
    assert not bits(out["label_mask"], 32 * NW)[..., N:].any(), "bits past n_blocks set"
    np.testing.assert_array_equal(out["set_cnt"], sets.sum(-1))
    near = 0
    for w in range(W):
        uncertain = np.zeros(N, dtype=bool)
        o_labels, o_sets = oracle.denoise_labels(x[w], p=p, min_votes=v)
        for l in range(L):
            probs = oracle.softmax_f64(x[w, l])
            order = np.argsort(-probs, kind="stable")
            cum = np.cumsum(probs[order])
            k = len(o_sets[l])
            assert np.array_equal(np.sort(order[:k]), o_sets[l])
            got = sets[w, l]
            n = int(got.sum())
            # a prefix of the oracle's order, whatever its length
            assert got[order[:n]].all(), (w, l, "not a prefix of the probability order")
            ok = np.flatnonzero((cum >= p - EPS) &
                                np.concatenate([[True], cum[:-1] < p + EPS])) + 1
            assert k in ok
            if len(ok) > 1:
                near += 1
                uncertain[order[ok.min() - 1:ok.max()]] = True
            assert n in ok, (w, l, n, k, cum[k - 2:k + 1] if k > 1 else cum[:2])
        # labels: the vote over the kernel's own sets, exactly
        votes = sets[w].sum(0)
        lab = bits(out["label_mask"][w], N)
        np.testing.assert_array_equal(lab, votes >= v)
        # and the oracle's labels wherever no near-tie can reach
        o_lab = np.zeros(N, dtype=bool)
        o_lab[o_labels] = True
        np.testing.assert_array_equal(lab[~uncertain], o_lab[~uncertain])
        ids = np.flatnonzero(lab)
        assert out["label_cnt"][w] == len(ids)
        np.testing.assert_array_equal(out["label_ids"][w][:min(cap, len(ids))], ids[:cap])
    return near


def test_small_windows(cuda_ok):
    """4 windows x 21 layers over 1,000 blocks (the last mask word is partial)."""
    cfg = LI.denoise_tiny()
    x = LI.denoise_batch(cfg)
    check(x, run(x))


def test_full_size_windows(cuda_ok):
    """64 windows x 21 layers x 16,384 blocks (a 1M-token context), every row."""
    cfg = LI.denoise_1m()
    x = LI.denoise_batch(cfg)
    near = check(x, run(x, repeat=2))
    assert near < 0.05 * cfg.windows * cfg.layers


@pytest.mark.parametrize("p", [0.05, 0.3, 0.95])
def test_other_top_p(cuda_ok, p):
    cfg = LI.DenoiseConfig(name="dn_p", windows=3, blocks=3000, relevant=60, seed=11)
    x = LI.denoise_batch(cfg)
    check(x, run(x, p=p), p=p)


@pytest.mark.parametrize("v", [-1, 0, 1, 2, 4, 8, 9, 21, 22])
def test_vote_thresholds(cuda_ok, v):
    cfg = LI.DenoiseConfig(name="dn_v", windows=2, blocks=700, relevant=40, seed=5)
    x = LI.denoise_batch(cfg)
    check(x, run(x, v=v), v=v)


def _edge_rows(N: int) -> torch.Tensor:
    g = torch.Generator().manual_seed(1234)
    rows = []
    rows.append(torch.zeros(N))                                   # all equal: first m by id
    r = torch.zeros(N); r[N // 2] = 10.0; rows.append(r)          # one block dominates
    r = torch.randn(N, generator=g) - 4.0; r[100:400] = 2.0       # 300 ties at the boundary
    rows.append(r)
    r = torch.randn(N, generator=g) - 4.0; r[::7] = 1.5           # ~140 ties, fits the list
    rows.append(r)
    rows.append(torch.randn(N, generator=g) * 300.0)              # wide spread, most mass 0
    rows.append(torch.randn(N, generator=g) * 3.0)                # wide spread
    r = torch.randn(N, generator=g) * 1e-3                        # a narrow band: splits
    rows.append(r)
    r = torch.randn(N, generator=g); r[r.abs() < 0.3] = 0.0       # +0 and -0 ties
    r[::2] = torch.where(r[::2] == 0, torch.tensor(-0.0), r[::2])
    rows.append(r)
    rows.append(torch.arange(N, dtype=torch.float32) * -1e-4)      # strictly decreasing
    return torch.stack(rows)


def test_edge_rows(cuda_ok):
    """Ties beyond the candidate list, one dominant block, spread and narrow rows, signed
    zeros, over an odd block count; the vote across these 9 rows with min_votes 2."""
    x = _edge_rows(1001).unsqueeze(0)
    out = run(x, v=2)
    near = check(x, out, v=2)
    assert out["set_cnt"][0][1] == 1
    assert out["set_cnt"][0][0] == 601            # 0.6 * 1001 = 600.6 -> 601 equal blocks
    sets = bits(out["set_mask"], 1001)[0]
    assert sets[0][:601].all() and not sets[0][601:].any()
    assert near <= 1


def test_edge_rows_bulk_copied(cuda_ok):
    """The same rows over 8,192 blocks, a count the kernel copies in with bulk copies: the
    all-equal and the narrow rows put more blocks in the boundary bin than the candidate
    list holds, so they are split over the whole row first."""
    N = 8192
    x = _edge_rows(N).unsqueeze(0)
    out = run(x, v=2)
    near = check(x, out, v=2)
    want = int(np.ceil(0.6 * N))                  # 4915.2 -> 4916 equal blocks, by id
    assert out["set_cnt"][0][0] == want
    sets = bits(out["set_mask"], N)[0]
    assert sets[0][:want].all() and not sets[0][want:].any()
    assert near <= 1


def test_misaligned_logits(cuda_ok):
    """Logits that start 4 bytes past a 16-byte boundary: the rows are read with plain
    loads instead of bulk copies, with the same result."""
    cfg = LI.DenoiseConfig(name="dn_m", windows=2, layers=5, blocks=4096, relevant=50, seed=21)
    x = LI.denoise_batch(cfg)
    W, L, N = x.shape
    flat = torch.empty(W * L * N + 4, dtype=torch.float32)
    flat[1:1 + W * L * N] = x.reshape(-1)
    dev = torch.device("cuda")
    big = flat.to(dev)
    xv = big[1:1 + W * L * N].view(W, L, N)
    assert xv.data_ptr() % 16 == 4
    a = run(xv, v=1)
    b = run(x, v=1)
    for k in a:
        np.testing.assert_array_equal(a[k], b[k])
    check(x, a, v=1)


def test_large_magnitude_logits(cuda_ok):
    """Rows whose maximum exceeds 2^22 in magnitude: the kernel bins by the rounded
    difference to ceil(max) there instead of the exact one-add floor. At 3e7 the fp32
    logits are multiples of 2, so most blocks tie with others."""
    g = torch.Generator().manual_seed(77)
    N = 4096
    rows = [5.0e6 + torch.randn(N, generator=g) * 50.0,
            -5.0e6 + torch.randn(N, generator=g) * 50.0,
            3.0e7 + torch.randn(N, generator=g) * 1000.0,
            4.0e6 + torch.randn(N, generator=g) * 3.0]
    x = torch.stack(rows).to(torch.float32).unsqueeze(0)
    out = run(x, v=2)
    check(x, out, v=2)


def test_single_block_and_single_layer(cuda_ok):
    x = torch.tensor([[[0.25]]])
    out = run(x, v=1)
    assert out["set_cnt"][0][0] == 1 and out["label_cnt"][0] == 1
    assert out["label_ids"][0][0] == 0
    check(x, out, v=1)


def test_label_cap_smaller_than_count(cuda_ok):
    cfg = LI.denoise_tiny()
    x = LI.denoise_batch(cfg)
    out = run(x, cap=5)
    check(x, out, cap=5)
    assert (out["label_cnt"] > 5).all()


def test_unaligned_rows_and_largest_row(cuda_ok):
    """A block count not divisible by 4 (scalar loads) and the largest supported row."""
    for N, W, L in ((1003, 2, 5), (lsa.DENOISE_MAX_BLOCKS, 1, 3)):
        cfg = LI.DenoiseConfig(name="dn_n", windows=W, layers=L, blocks=N, relevant=50, seed=N)
        x = LI.denoise_batch(cfg)
        check(x, run(x, v=1), v=1)
