"""GPU parity of lsa_index (projection, scoring, sign test, OR, compaction) against the
oracle, at the full sizes of every workload (the indexer is cheap for the oracle)."""
import numpy as np
import pytest
import torch

import lookahead_sparse_kv_lsa_b200 as lsa
import lsa_inputs as LI
import oracle
from gpu_util import LOGIT_ABS, NEAR_TIE, bits, compare_selection

pytestmark = pytest.mark.gpu

CONFIGS = {
    "tiny_16k": LI.tiny,
    "mid_b8_128k": LI.mid_batch,
    "long_b4_512k": LI.long_ctx,
    "1m_b15": lambda: LI.one_million(-1.5),
    "1m_b20": lambda: LI.one_million(-2.0),
    "1m_b25": lambda: LI.one_million(-2.5),
    "ragged_b64": LI.ragged_mix,
    "1m_b20_lk": LI.one_million_layer_keys,
    "1m_b20_r2048": LI.one_million_latent,
}


def cand_keys(wl, b, nc):
    """bf16 bits of sequence b's first nc compressed keys ([nc][d_i] or [L][nc][d_i])."""
    k = wl.seq_k_idx(b)
    return bits(k[:, :nc] if k.dim() == 3 else k[:nc])


def run_index(wl, p, cap=None, n_cand=None):
    dev = torch.device("cuda")
    c = wl.cfg
    B, L = c.B, c.L
    if n_cand is None:
        n_cand = [oracle.n_candidates(int(x), c.W) for x in wl.ctx_at(p)]
    max_cand = max(1, max(n_cand))
    cap = max_cand if cap is None else cap
    h = wl.h(p).to(dev)
    sel_ids = torch.full((B, max(1, cap)), -1, dtype=torch.int32, device=dev)
    sel_cnt = torch.full((B,), -1, dtype=torch.int32, device=dev)
    logits = torch.full((L, B, max_cand), float("nan"), device=dev)
    mask = torch.zeros((L + 1, B, (max_cand + 31) // 32), dtype=torch.int32, device=dev)
    ws = torch.zeros(lsa.index_workspace_size(B, L, c.d_i, max_cand), dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    lsa.lsa_index(h, wl.w_q.to(dev), torch.from_numpy(wl.bias).to(dev), wl.k_idx.to(dev),
                  torch.from_numpy(wl.blk_off[:B]).to(dev),
                  torch.tensor(n_cand, dtype=torch.int32, device=dev), max_cand, sel_ids, sel_cnt,
                  ws, err, logits=logits, layer_mask=mask)
    torch.cuda.synchronize()
    return (sel_ids.cpu(), sel_cnt.cpu(), logits.cpu().numpy(), mask.cpu().numpy().view(np.uint32),
            int(err.item()), n_cand)


@pytest.mark.parametrize("name", sorted(CONFIGS))
def test_index_matches_oracle(cuda_ok, name):
    wl = LI.Workload(CONFIGS[name](), with_pool=False)
    c = wl.cfg
    for p in range(c.passes):
        ids, cnt, z_gpu, mask, err, n_cand = run_index(wl, p)
        assert err == 0
        hb = bits(wl.h(p))
        n_near = 0
        for b in range(c.B):
            nc = n_cand[b]
            ref_ids, z_ref = oracle.index_pass(bits(wl.w_q), hb[:, b], cand_keys(wl, b, nc),
                                               float(wl.bias[b]))
            dz = np.abs(z_gpu[:, b, :nc] - z_ref)
            assert dz.max(initial=0.0) <= LOGIT_ABS, (name, b, dz.max())
            got = ids[b, :int(cnt[b])].tolist()
            n_near += len(compare_selection(got, ref_ids, z_ref, "%s p%d b%d" % (name, p, b)))
            # per-layer bits and the OR word agree with the kernel's own logits exactly
            for l in range(c.L + 1):
                bitv = np.unpackbits(mask[l, b].view(np.uint8), bitorder="little")[:nc].astype(bool)
                zz = z_gpu[:, b, :nc]
                expect = (zz > 0).any(axis=0) if l == c.L else zz[l] > 0
                assert np.array_equal(bitv, expect)
            assert got == np.flatnonzero((z_gpu[:, b, :nc] > 0).any(axis=0)).tolist()
        # near ties are rare: ~2e-3 * phi(bias) * 3 per candidate
        assert n_near <= max(3, 0.01 * sum(n_cand))


def test_capacity_overflow_flagged(cuda_ok):
    wl = LI.Workload(LI.tiny(), with_pool=False)
    ids_full, cnt_full, *_ = run_index(wl, 0)
    n = int(cnt_full[0])
    assert n > 4
    ids, cnt, _, _, err, _ = run_index(wl, 0, cap=4)
    assert err & lsa._lib.DEVERR_SEL_CAPACITY
    assert int(cnt[0]) == 4 and ids[0, :4].tolist() == ids_full[0, :4].tolist()


def test_no_candidates(cuda_ok):
    wl = LI.Workload(LI.tiny(), with_pool=False)
    ids, cnt, _, _, err, _ = run_index(wl, 0, n_cand=[0])
    assert err == 0 and int(cnt[0]) == 0


def test_all_and_none_kept(cuda_ok):
    cfg = LI.tiny()
    for bias, expect_all in ((1e4, True), (-1e4, False)):
        cfg.bias = [bias]
        wl = LI.Workload(cfg, with_pool=False)
        ids, cnt, _, _, err, n_cand = run_index(wl, 0)
        assert err == 0
        if expect_all:
            assert ids[0, :int(cnt[0])].tolist() == list(range(n_cand[0]))
        else:
            assert int(cnt[0]) == 0


def test_many_short_sequences(cuda_ok):
    """Hundreds of sequences of 0..90 candidates: many sequences share a CTA's range of
    keep words, some have none, word boundaries fall inside and between sequences."""
    dev = torch.device("cuda")
    g = torch.Generator().manual_seed(11)
    B, L, D, d_i = 300, 3, 1024, 128
    n_cand = torch.randint(0, 91, (B,), generator=g)
    n_cand[::7] = 0
    rows = int(n_cand.sum())
    off = torch.zeros(B, dtype=torch.int64)
    off[1:] = torch.cumsum(n_cand, 0)[:-1]
    w_q = (torch.randn(L, d_i, D, generator=g) / D ** 0.5).to(torch.bfloat16)
    h = torch.randn(L, B, D, generator=g).to(torch.bfloat16)
    k_idx = torch.randn(max(1, rows), d_i, generator=g).to(torch.bfloat16)
    bias = (torch.rand(B, generator=g) * 2.0 - 3.0).float()
    max_cand = int(n_cand.max())
    sel_ids = torch.full((B, max_cand), -1, dtype=torch.int32, device=dev)
    sel_cnt = torch.full((B,), -1, dtype=torch.int32, device=dev)
    logits = torch.full((L, B, max_cand), float("nan"), device=dev)
    ws = torch.zeros(lsa.index_workspace_size(B, L, d_i, max_cand), dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    wb, hb, kb = bits(w_q), bits(h), bits(k_idx)
    G = min(torch.cuda.get_device_properties(dev).multi_processor_count, 1024)
    for call in range(2):   # the workspace is reusable as left
        lsa.lsa_index(h.to(dev), w_q.to(dev), bias.to(dev), k_idx.to(dev), off.to(dev),
                      n_cand.to(torch.int32).to(dev), max_cand, sel_ids, sel_cnt, ws, err,
                      logits=logits)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        ids, cnt, z_gpu = sel_ids.cpu(), sel_cnt.cpu(), logits.cpu().numpy()
        for b in range(B):
            nc = int(n_cand[b])
            ref_ids, z_ref = oracle.index_pass(wb, hb[:, b], kb[int(off[b]):int(off[b]) + nc],
                                               float(bias[b]))
            assert np.abs(z_gpu[:, b, :nc] - z_ref).max(initial=0.0) <= LOGIT_ABS
            got = ids[b, :int(cnt[b])].tolist()
            compare_selection(got, ref_ids, z_ref, "short b%d" % b)
            assert got == np.flatnonzero((z_gpu[:, b, :nc] > 0).any(axis=0)).tolist()
        # the barrier counter (first 8 bytes) grew by two rounds of the grid per call
        assert int(ws[:8].cpu().view(torch.int64)[0]) == 2 * G * (call + 1)
        assert not ws[8:256].any()


def run_index_lowrank(wl, p, calls=1):
    """lsa_index_lowrank on pass p of a workload with factorised encoders; returns the
    last call's (ids, counts, logits, err, n_cand, workspace)."""
    dev = torch.device("cuda")
    c = wl.cfg
    B, L = c.B, c.L
    n_cand = [oracle.n_candidates(int(x), c.W) for x in wl.ctx_at(p)]
    max_cand = max(1, max(n_cand))
    sel_ids = torch.full((B, max_cand), -1, dtype=torch.int32, device=dev)
    sel_cnt = torch.full((B,), -1, dtype=torch.int32, device=dev)
    logits = torch.full((L, B, max_cand), float("nan"), device=dev)
    ws = torch.zeros(lsa.index_lowrank_workspace_size(B, L, c.d_i, c.rank, max_cand),
                     dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    args = (wl.h(p).to(dev), wl.w_1.to(dev), wl.w_2.to(dev), torch.from_numpy(wl.bias).to(dev),
            wl.k_idx.to(dev), torch.from_numpy(wl.blk_off[:B]).to(dev),
            torch.tensor(n_cand, dtype=torch.int32, device=dev), max_cand, sel_ids, sel_cnt, ws, err)
    for _ in range(calls):
        lsa.lsa_index_lowrank(*args, logits=logits)
    torch.cuda.synchronize()
    return sel_ids.cpu(), sel_cnt.cpu(), logits.cpu().numpy(), int(err.item()), n_cand, ws


def check_lowrank(wl, calls=1):
    c = wl.cfg
    ids, cnt, z_gpu, err, n_cand, ws = run_index_lowrank(wl, 0, calls)
    assert err == 0
    w1, w2, hb = bits(wl.w_1), bits(wl.w_2), bits(wl.h(0))
    n_near = 0
    for b in range(c.B):
        nc = n_cand[b]
        ref_ids, z_ref = oracle.index_pass_lowrank(w1, w2, hb[:, b], cand_keys(wl, b, nc),
                                                   float(wl.bias[b]))
        dz = np.abs(z_gpu[:, b, :nc] - z_ref)
        assert dz.max(initial=0.0) <= LOGIT_ABS, (c.name, b, dz.max())
        got = ids[b, :int(cnt[b])].tolist()
        n_near += len(compare_selection(got, ref_ids, z_ref, "%s b%d" % (c.name, b)))
        assert got == np.flatnonzero((z_gpu[:, b, :nc] > 0).any(axis=0)).tolist()
    assert n_near <= max(3, 0.01 * sum(n_cand))
    return ws


def test_lowrank_encoder_full_size(cuda_ok):
    """Factorised query encoders q = W_2 (W_1 h), r = 2048, D = 4096, at the 1M-token
    context: logits within the tolerance of the oracle's float64 values, ids exact
    outside the near-tie band."""
    check_lowrank(LI.Workload(LI.one_million_lowrank(), with_pool=False))


def test_lowrank_encoder_batch_and_small_rank(cuda_ok):
    """Five sequences (more than one staged group of hidden states), D = 1024, r = 512
    (a CTA's latent rows span two layers), two calls on one workspace: the barrier
    counter grows by three rounds of the grid per call."""
    import dataclasses
    cfg = LI.scaled_down(LI.one_million_lowrank(), ctx_blocks=300, B=5)
    cfg = dataclasses.replace(cfg, D=1024, rank=512)
    cfg.bias = [-2.0, -1.0, -3.0, -1.5, -2.5]
    wl = LI.Workload(cfg, with_pool=False)
    ws = check_lowrank(wl, calls=2)
    G = min(torch.cuda.get_device_properties(0).multi_processor_count, 1024)
    assert int(ws[:8].cpu().view(torch.int64)[0]) == 3 * G * 2
