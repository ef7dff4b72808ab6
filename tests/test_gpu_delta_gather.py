"""GPU checks of the delta gather (resident-page reuse across passes): the decode loop's
outputs match the oracle as with the plain gather, only blocks new to a pass are copied,
reused blocks keep their page, and every kept page holds its block bit for bit."""
import numpy as np
import pytest
import torch

import lookahead_sparse_kv_lsa_b200 as lsa
import lsa_inputs as LI
import oracle
from gpu_util import bits

from test_gpu_step import check_loop

pytestmark = pytest.mark.gpu


def build(wl, delta=True):
    dev = torch.device("cuda")
    c = wl.cfg
    max_cand = max(1, max(oracle.n_candidates(int(x), c.W) for x in wl.ctx_at(c.passes - 1)))
    return lsa.LsaDecoder(wl.w_q.to(dev), wl.k_idx.to(dev), wl.blk_off[:c.B],
                          torch.from_numpy(wl.bias).to(dev), wl.host_pool, wl.blk_off, wl.nb0,
                          W=c.W, H=c.H, cap=max_cand, max_cand=max_cand, scale=c.scale,
                          delta_gather=delta)


def test_loop_matches_oracle_with_delta_gather(cuda_ok, monkeypatch):
    """The 4-pass loop through lsa_step with resident-page reuse, against the oracle."""
    import test_gpu_step
    monkeypatch.setattr(test_gpu_step, "build_decoder", lambda wl: build(wl, True))
    wl = LI.Workload(LI.scaled_down(LI.long_ctx(), ctx_blocks=200, B=2), pin=True)
    check_loop(wl, {0, 1, 32, 63})


def _pass(dec, wl, p, h):
    """The head of pass p as lsa_step composes it: set-up, indexer, (delta) gather."""
    dev = torch.device("cuda")
    c = wl.cfg
    dec.pass_setup(p)
    dec.index(h.to(dev))
    dec.gather()
    torch.cuda.synchronize()
    cnt = dec.sel_cnt.cpu()
    ids = [dec.sel_ids[b, :int(cnt[b])].cpu().tolist() for b in range(c.B)]
    pages = [dec.block_table[b, :int(cnt[b])].cpu().tolist() for b in range(c.B)]
    return ids, pages


def _check_pages_hold_blocks(dec, wl, ids, pages):
    for b, (ib, pb) in enumerate(zip(ids, pages)):
        for c_id, pg in zip(ib, pb):
            assert pg >= 0
            got = dec.hbm_pool[pg].cpu()
            ref = wl.host_pool[int(wl.blk_off[b]) + c_id]
            assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), (b, c_id, pg)


@pytest.mark.parametrize("same_h", [False, True], ids=["fresh_hidden_state", "same_hidden_state"])
def test_only_new_blocks_are_copied(cuda_ok, same_h):
    """Passes 0..2 of a scaled 4-pass workload. With a fresh hidden state per pass the kept
    sets overlap a little; with the same one they overlap almost entirely. Either way the
    copy count is the number of blocks not kept by the previous pass, reused blocks keep
    their page, and every kept page holds its block."""
    wl = LI.Workload(LI.scaled_down(LI.long_ctx(), ctx_blocks=400, B=3), pin=True)
    dec = build(wl)
    dec.load_window(0)
    prev_ids, prev_pages = None, None
    for p in range(3):
        h = wl.h(0 if same_h else p)
        before = int(dec.copied.item())
        ids, pages = _pass(dec, wl, p, h)
        copied = int(dec.copied.item()) - before
        assert dec.read_err() == 0
        if prev_ids is None:
            expect = sum(len(x) for x in ids)
        else:
            expect = 0
            for b in range(wl.cfg.B):
                old = dict(zip(prev_ids[b], prev_pages[b]))
                for c_id, pg in zip(ids[b], pages[b]):
                    if c_id in old:
                        assert pg == old[c_id], "reused block moved"
                    else:
                        expect += 1
        assert copied == expect, (p, copied, expect)
        if same_h and p > 0:
            assert copied <= 0.1 * sum(len(x) for x in ids) + wl.cfg.B
        _check_pages_hold_blocks(dec, wl, ids, pages)
        # distinct pages within the pass
        flat = [pg for pb in pages for pg in pb]
        assert len(flat) == len(set(flat))
        prev_ids, prev_pages = ids, pages
