"""GPU parity of the whole decode loop (lsa_step: index + gather every 64 steps, append +
attention every step) against the oracle's loop, on every workload: in full at the tiny
size and scaled-down sizes, and on sampled steps and heads at the full 1M-token size."""
import math

import numpy as np
import pytest
import torch

import lookahead_sparse_kv_lsa_b200 as lsa
import lsa_inputs as LI
import oracle
from gpu_util import bits, compare_attention, compare_selection

pytestmark = pytest.mark.gpu


def build_decoder(wl):
    dev = torch.device("cuda")
    c = wl.cfg
    max_cand = max(1, max(oracle.n_candidates(int(x), c.W) for x in wl.ctx_at(c.passes - 1)))
    return lsa.LsaDecoder(wl.w_q.to(dev), wl.k_idx.to(dev), wl.blk_off[:c.B],
                          torch.from_numpy(wl.bias).to(dev), wl.host_pool, wl.blk_off, wl.nb0,
                          W=c.W, H=c.H, cap=max_cand, max_cand=max_cand, scale=c.scale)


def run_loop(wl, keep_steps):
    """Runs every step of every pass; returns {(p, s): out}, [per-pass (ids, cnt)]."""
    dev = torch.device("cuda")
    c = wl.cfg
    dec = build_decoder(wl)
    dec.load_window(0)
    outs, sels = {}, []
    out = torch.empty((c.B, c.H, c.d), dtype=torch.bfloat16, device=dev)
    for p in range(c.passes):
        h = wl.h(p).to(dev)
        for s in range(c.tau):
            k, v = wl.kv_new(p, s)
            dec.step(p * c.tau + s, h if s == 0 else None, wl.q(p, s).to(dev), k.to(dev),
                     v.to(dev), out)
            if s == 0:
                sels.append((dec.sel_ids.cpu().clone(), dec.sel_cnt.cpu().clone()))
            if s in keep_steps:
                outs[(p, s)] = out.cpu().clone()
    torch.cuda.synchronize()
    assert dec.read_err() == 0, "device error word %d" % dec.read_err()
    return outs, sels


def check_loop(wl, keep_steps, heads=None, seqs=None):
    """Selection of every sequence in every pass against the oracle (exact outside the
    near-tie band); attention of the sequences `seqs` (all by default) on the kept steps
    and heads. Returns the near-tie flips per pass."""
    c = wl.cfg
    outs, sels = run_loop(wl, keep_steps)
    check_b = set(range(c.B)) if seqs is None else set(seqs)
    flips = []
    wq = bits(wl.w_q)
    for p in range(c.passes):
        hb = bits(wl.h(p))
        ids_gpu, cnt_gpu = sels[p]
        for b in range(c.B):
            n_ctx = int(wl.ctx_at(p)[b])
            nc = oracle.n_candidates(n_ctx, c.W)
            kb = wl.seq_k_idx(b)
            kb = kb[:, :nc] if kb.dim() == 3 else kb[:nc]
            ref_ids, z = oracle.index_pass(wq, hb[:, b], bits(kb), float(wl.bias[b]))
            got = ids_gpu[b, :int(cnt_gpu[b])].tolist()
            near = compare_selection(got, ref_ids, z, "%s p%d b%d" % (c.name, p, b))
            flips.append(len(near))
            if b not in check_b:
                continue
            # with near-tie flips, attention is checked over the GPU's own selection
            use_ids = got if near else ref_ids
            K, V = wl.seq_kv(b)
            Kb, Vb = bits(K), bits(V)
            for s in sorted(keep_steps):
                ref = oracle.step_output(bits(wl.q(p, s)[b]), Kb, Vb, use_ids, n_ctx, c.W, s,
                                         c.scale, heads=heads)
                got_o = outs[(p, s)][b]
                if heads is not None:
                    got_o = got_o[list(heads)]
                compare_attention(got_o, ref, "%s p%d s%d b%d" % (c.name, p, s, b))
    print("%s: near-tie flips %d over %d sequence passes" % (c.name, sum(flips), len(flips)))
    return flips


def test_tiny_every_step(cuda_ok):
    wl = LI.Workload(LI.tiny(), pin=True)
    check_loop(wl, set(range(64)))


STEPS = {0, 1, 31, 32, 33, 63}


@pytest.mark.parametrize("name,cfg", [
    ("mid_batch_small", lambda: LI.scaled_down(LI.mid_batch(), ctx_blocks=160)),
    ("long_4pass_small", lambda: LI.scaled_down(LI.long_ctx(), ctx_blocks=200, B=2)),
    ("ragged_small", lambda: LI.scaled_down(LI.ragged_mix(), ctx_blocks=160, B=12)),
    ("one_million_geometry_small", lambda: LI.scaled_down(LI.one_million(-1.5), ctx_blocks=300)),
    ("window_covers_context", lambda: LI.scaled_down(LI.tiny(), ctx_blocks=12, W=1024)),
    ("layer_keys_2pass_small", lambda: LI.scaled_down(LI.one_million_layer_keys(), ctx_blocks=300,
                                                      passes=2)),
    ("latent_input_small", lambda: LI.scaled_down(LI.one_million_latent(), ctx_blocks=300)),
])
def test_scaled_loops(cuda_ok, name, cfg):
    wl = LI.Workload(cfg(), pin=True)
    check_loop(wl, STEPS)


@pytest.mark.slow
def test_one_million_full_sampled(cuda_ok):
    """1,048,576-token context, bias -2: steps 0 and 63 on four sampled heads."""
    wl = LI.Workload(LI.one_million(-2.0), pin=True)
    check_loop(wl, {0, 63}, heads=[0, 21, 42, 63])


@pytest.mark.slow
def test_mid_batch_full_sampled(cuda_ok):
    """B=8 x 131,072 tokens: steps 0 and 63 on two sampled heads of every sequence."""
    wl = LI.Workload(LI.mid_batch(), pin=True)
    check_loop(wl, {0, 63}, heads=[5, 60])


@pytest.mark.slow
@pytest.mark.parametrize("bias", [-1.5, -2.5])
def test_one_million_other_biases_full_sampled(cuda_ok, bias):
    """1M tokens at bias -1.5 (~3,000 kept blocks, 416 MB per step) and -2.5: steps 0
    and 63 on four heads."""
    wl = LI.Workload(LI.one_million(bias), pin=True)
    check_loop(wl, {0, 63}, heads=[0, 21, 42, 63])


@pytest.mark.slow
def test_long_context_four_passes_full_sampled(cuda_ok):
    """B=4 x 524,288 tokens, all four indexer passes: steps 0 and 63 of every pass on two
    heads of every sequence (the window slides and the candidates grow each pass)."""
    wl = LI.Workload(LI.long_ctx(), pin=True)
    check_loop(wl, {0, 63}, heads=[7, 56])


@pytest.mark.slow
def test_ragged_mix_full_sampled(cuda_ok):
    """B=64 sequences of 32K..256K tokens with per-sequence bias: the selection of all 64,
    attention of 8 sampled sequences (the shortest, the longest and six spread over the
    batch) at steps 0 and 63 on two heads."""
    wl = LI.Workload(LI.ragged_mix(), pin=True)
    ctx = wl.ctx0
    spread = [int(x) for x in np.linspace(0, wl.cfg.B - 1, 6).round()]
    seqs = sorted(set([int(np.argmin(ctx)), int(np.argmax(ctx))] + spread))
    check_loop(wl, {0, 63}, heads=[3, 50], seqs=seqs)


@pytest.mark.slow
def test_dense_one_million_full(cuda_ok):
    """Dense decode at 1M tokens: lsa_decode_attn over every block of the context (16,385
    pages, the last one full), with the queries of steps 0 and 63, on four heads, against
    the oracle's softmax over all 1,048,640 tokens."""
    dev = torch.device("cuda")
    wl = LI.Workload(LI.one_million(-2.0), pin=True)
    c = wl.cfg
    n = int(wl.nb0[0]) + 1
    pool = wl.host_pool[:n].to(dev)
    bt = torch.arange(n, dtype=torch.int32, device=dev).view(1, n)
    ne = torch.tensor([n], dtype=torch.int32, device=dev)
    tl = torch.tensor([64], dtype=torch.int32, device=dev)
    ws = torch.zeros(lsa.decode_attn_workspace_size(1, c.H, c.d), dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    K, V = wl.seq_kv(0)
    T = n * 64
    Kb, Vb = bits(K[:T]), bits(V[:T])
    heads = [0, 21, 42, 63]
    for s in (0, 63):
        q = wl.q(0, s).to(dev)
        out = torch.full_like(q, float("nan"))
        lsa.lsa_decode_attn(q, pool, bt, ne, tl, c.scale, out, ws, err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        qf = oracle.bf16_to_f64(bits(wl.q(0, s)[0]))[heads]
        ref = oracle.softmax_attention_bits(qf, Kb, Vb, c.scale)
        compare_attention(out[0][heads], ref, "dense 1M s%d" % s)


def test_shard_is_the_same_computation(cuda_ok):
    """A rank's shard of a batch (sequences 4..8 of a scaled-down ragged batch of 12)
    decoded alone on one GPU equals the oracle fed from the whole batch's draws for
    those sequences: sharding by sequence changes nothing in what is computed."""
    full = LI.Workload(LI.scaled_down(LI.ragged_mix(), ctx_blocks=160, B=12), pin=True)
    shard = LI.Workload(LI.scaled_down(LI.ragged_mix(), ctx_blocks=160, B=12), pin=True,
                        seqs=range(4, 9))
    c = shard.cfg
    steps = {0, 31, 63}
    outs, sels = run_loop(shard, steps)
    wq = bits(full.w_q)
    hb = bits(full.h(0))
    for i, b in enumerate(range(4, 9)):
        n_ctx = int(full.ctx_at(0)[b])
        assert n_ctx == int(shard.ctx_at(0)[i])
        nc = oracle.n_candidates(n_ctx, c.W)
        ref_ids, z = oracle.index_pass(wq, hb[:, b], bits(full.seq_k_idx(b)[:nc]),
                                       float(full.bias[b]))
        ids_gpu, cnt_gpu = sels[0]
        got = ids_gpu[i, :int(cnt_gpu[i])].tolist()
        near = compare_selection(got, ref_ids, z, "shard seq %d" % b)
        use_ids = got if near else ref_ids
        K, V = full.seq_kv(b)
        Kb, Vb = bits(K), bits(V)
        for s in sorted(steps):
            qf = bits(full.q(0, s)[b])
            ref = oracle.step_output(qf, Kb, Vb, use_ids, n_ctx, c.W, s, c.scale)
            compare_attention(outs[(0, s)][i], ref, "shard seq %d s%d" % (b, s))
