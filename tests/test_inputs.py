"""The seeded input generator: determinism, shapes and the drawn distributions."""
import numpy as np
import torch

import lsa_inputs as LI


def small_cfg():
    return LI.scaled_down(LI.tiny(), ctx_blocks=40, W=512)


def test_deterministic_and_independent_streams():
    a, b = LI.Workload(small_cfg()), LI.Workload(small_cfg(), threads=1)
    assert torch.equal(a.w_q, b.w_q) and torch.equal(a.k_idx, b.k_idx)
    assert torch.equal(a.host_pool, b.host_pool)
    assert torch.equal(a.h(0), b.h(0)) and torch.equal(a.q(0, 5), b.q(0, 5))
    assert not torch.equal(a.q(0, 5), a.q(0, 6))


def test_shapes_and_offsets():
    w = LI.Workload(small_cfg())
    c = w.cfg
    assert w.w_q.shape == (3, 128, c.D) and w.w_q.dtype == torch.bfloat16
    assert w.k_idx.shape == (w.total_blocks, 128)
    assert w.host_pool.shape == (w.total_blocks, 2, 64, c.d)
    assert list(w.nb_final) == [40 + c.passes]
    k, v = w.kv_new(0, 3)
    K, V = w.seq_kv(0)
    assert torch.equal(k[0], K[int(w.ctx0[0]) + 3]) and torch.equal(v[0], V[int(w.ctx0[0]) + 3])


def test_ragged_mix_draws():
    cfg = LI.scaled_down(LI.ragged_mix(), ctx_blocks=100, B=16, W=256)
    w = LI.Workload(cfg)
    assert np.all(w.nb0 >= 50) and np.all(w.nb0 <= 100)
    assert np.all(w.bias >= -3.0) and np.all(w.bias <= -1.0)
    assert len(set(w.nb0.tolist())) > 1


def test_distributions():
    w = LI.Workload(LI.scaled_down(LI.mid_batch(), ctx_blocks=80, B=1, W=1024))
    wq = w.w_q.float()
    assert abs(wq.std().item() * np.sqrt(4096) - 1.0) < 0.02
    pool = w.host_pool.float()
    assert abs(pool.mean().item()) < 0.01 and abs(pool.std().item() - 1.0) < 0.01


def test_shard_holds_the_batch_draws():
    """A workload restricted to some sequences holds exactly the whole batch's values for
    them (the sequence-sharded multi-GPU run splits one workload, not a new one)."""
    cfg = LI.scaled_down(LI.ragged_mix(), ctx_blocks=200, B=6)
    full = LI.Workload(cfg)
    part = LI.Workload(cfg, seqs=[2, 3, 4])
    assert part.cfg.B == 3
    for lb, gb in enumerate([2, 3, 4]):
        assert torch.equal(part.seq_k_idx(lb), full.seq_k_idx(gb))
        K1, V1 = part.seq_kv(lb)
        K2, V2 = full.seq_kv(gb)
        assert torch.equal(K1, K2) and torch.equal(V1, V2)
        assert int(part.ctx0[lb]) == int(full.ctx0[gb])
        assert float(part.bias[lb]) == float(full.bias[gb])
    assert torch.equal(part.h(0), full.h(0)[:, 2:5])
    assert torch.equal(part.q(0, 5), full.q(0, 5)[2:5])
    k1, v1 = part.kv_new(0, 3)
    k2, v2 = full.kv_new(0, 3)
    assert torch.equal(k1, k2[2:5]) and torch.equal(v1, v2[2:5])
