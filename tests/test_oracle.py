"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each check ties one part of the oracle to a closed form, a brute-force evaluation in
exact integer / rational arithmetic, a library routine that computes the same textbook
quantity another way, or an invariant the pages fix (the loop of section 2 and the
OR-union of section 4 of "FlashMemory-DeepSeek-V4 Explained", zhichai.net). The
mutation tests at the end plant plausible mistakes in the oracle (on the CPU) and
require that at least one pin fails for each.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle import lsa_oracle as O


def f64_to_bf16_bits(x):
    """Exact bf16 bits of values that are exactly representable in bf16."""
    t = torch.as_tensor(np.asarray(x, dtype=np.float64)).to(torch.bfloat16)
    back = t.to(torch.float64).numpy()
    assert np.array_equal(back, np.asarray(x, dtype=np.float64)), "value not bf16-exact"
    return t.view(torch.int16).numpy().view(np.uint16)


# ----------------------------------------------------------------------------- pins
def check_bf16_decode(O=O):
    bits = np.array([0x3F80, 0xC000, 0x0001, 0x7F80, 0xFF80, 0x4049, 0x8000, 0x3E00],
                    dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = O.bf16_to_f64(bits)
    assert np.array_equal(got, ref)
    assert got[0] == 1.0 and got[1] == -2.0 and got[2] == 2.0 ** -133


def check_projection_unit_rows(O=O):
    rng = np.random.default_rng(1)
    L, d_i, D = 3, 16, 40
    perms = [rng.permutation(D)[:d_i] for _ in range(L)]
    w = np.zeros((L, d_i, D))
    for l in range(L):
        w[l, np.arange(d_i), perms[l]] = 1.0
    h = rng.standard_normal((L, D))
    q = O.query_projection(w, h)
    for l in range(L):
        assert np.array_equal(q[l], h[l][perms[l]])


def check_projection_bruteforce(O=O):
    rng = np.random.default_rng(2)
    L, d_i, D = 3, 5, 12
    w = rng.integers(-8, 9, (L, d_i, D)).astype(np.float64)
    h = rng.integers(-8, 9, (L, D)).astype(np.float64) / 4.0
    w_bits, h_bits = f64_to_bf16_bits(w), f64_to_bf16_bits(h)
    q = O.query_projection(O.bf16_to_f64(w_bits), O.bf16_to_f64(h_bits))
    for l in range(L):
        for j in range(d_i):
            exact = sum(Fraction(int(w[l, j, i])) * Fraction(h[l, i]) for i in range(D))
            assert q[l, j] == float(exact)


def check_lowrank_reduces_to_full_rank(O=O):
    """With integer factors, W_2 . (W_1 . h) equals (W_2 W_1) . h exactly: the factorised
    encoder is the full-rank one whose W_q is the product of its factors."""
    rng = np.random.default_rng(21)
    L, d_i, r, D = 3, 6, 10, 16
    w1 = rng.integers(-4, 5, (L, r, D)).astype(np.float64)
    w2 = rng.integers(-4, 5, (L, d_i, r)).astype(np.float64)
    h = rng.integers(-8, 9, (L, D)).astype(np.float64) / 4.0
    wq = np.stack([(w2[l].astype(np.int64) @ w1[l].astype(np.int64)).astype(np.float64)
                   for l in range(L)])
    got = O.query_projection_lowrank(w1, w2, h)
    assert np.array_equal(got, O.query_projection(wq, h))
    # and against a brute-force triple loop in exact rationals
    for l in range(L):
        for j in range(d_i):
            acc = Fraction(0)
            for k in range(r):
                u = sum(Fraction(w1[l, k, i]) * Fraction(h[l, i]) for i in range(D))
                acc += Fraction(w2[l, j, k]) * u
            assert got[l, j] == float(acc)


def check_lowrank_unit_rows(O=O):
    """Unit-row factors pick components: W_1 row k = e_{a(k)}, W_2 row j = e_{b(j)} give
    q_l[j] = h_l[a(b(j))] in every layer, with the layer's own permutations."""
    rng = np.random.default_rng(22)
    L, d_i, r, D = 3, 8, 12, 30
    w1 = np.zeros((L, r, D)); w2 = np.zeros((L, d_i, r))
    a = [rng.permutation(D)[:r] for _ in range(L)]
    b = [rng.permutation(r)[:d_i] for _ in range(L)]
    for l in range(L):
        w1[l, np.arange(r), a[l]] = 1.0
        w2[l, np.arange(d_i), b[l]] = 1.0
    h = rng.standard_normal((L, D))
    q = O.query_projection_lowrank(w1, w2, h)
    for l in range(L):
        assert np.array_equal(q[l], h[l][a[l][b[l]]])
    # the whole pass: a block whose key is a unit vector e_j scores q_l[j] / sqrt(d_i) + bias
    k = np.eye(d_i)
    ids, z = O.index_pass_lowrank(f64_to_bf16_bits(w1), f64_to_bf16_bits(w2),
                                  f64_to_bf16_bits(np.round(h * 4) / 4), f64_to_bf16_bits(k), 0.0)
    hq = O.query_projection_lowrank(w1, w2, np.round(h * 4) / 4)
    assert np.allclose(z, hq / math.sqrt(d_i), rtol=0, atol=1e-15)
    assert list(ids) == list(np.flatnonzero((hq > 0).any(axis=0)))


def check_logits_closed_form(O=O):
    # d_i = 64 -> sqrt(d_i) = 8 exactly; q = (2, 0, ...), K_idx[c] = (c - 3, 0, ...)
    d_i, n = 64, 9
    q = np.zeros((3, d_i))
    q[:, 0] = [2.0, -1.0, 0.5]
    k = np.zeros((n, d_i))
    k[:, 0] = np.arange(n) - 3.0
    bias = -0.25
    z = O.block_logits(q, k, bias)
    for l in range(3):
        for c in range(n):
            assert z[l, c] == q[l, 0] * (c - 3.0) / 8.0 + bias
    # d_i = 128: q . k = 128 gives z = sqrt(128) + bias
    q2 = np.zeros((1, 128)); q2[0, :] = 1.0
    k2 = np.ones((1, 128))
    assert abs(O.block_logits(q2, k2, -2.0)[0, 0] - (math.sqrt(128.0) - 2.0)) < 1e-12


def check_threshold_strict(O=O):
    d_i = 64
    q = np.zeros((3, d_i)); q[:, 0] = 4.0
    k = np.zeros((3, d_i)); k[:, 0] = [4.0, 4.0 + 2.0 ** -20, 4.0 - 2.0 ** -20]
    z = O.block_logits(q, k, -2.0)          # z = 4k/8 - 2 -> exactly 0, +tiny, -tiny
    assert z[0, 0] == 0.0 and z[0, 1] > 0 and z[0, 2] < 0
    assert list(O.kept_blocks(z)) == [1]


def check_union_bruteforce(O=O):
    rng = np.random.default_rng(3)
    for trial in range(20):
        L, n = 3, int(rng.integers(0, 200))
        z = rng.standard_normal((L, n)) - 1.0
        z[rng.random((L, n)) < 0.05] = 0.0
        expect = []
        for c in range(n):
            if any(z[l, c] > 0 for l in range(L)):
                expect.append(c)
        got = list(O.kept_blocks(z))
        assert got == expect
        assert got == sorted(set(got))


def check_selection_rate(O=O):
    """Kept fraction vs 1 - prod_l (1 - Phi(bias / sigma_l)), sigma_l = |q_l| / sqrt(d_i).

    With orthogonal q_l and K_idx ~ N(0, I), the three logits of a block are independent
    normals N(bias, sigma_l^2), so the union rate has that closed form.
    """
    rng = np.random.default_rng(4)
    d_i, n = 128, 400_000
    qs = np.linalg.qr(rng.standard_normal((d_i, 3)))[0].T      # orthonormal rows
    norms = np.array([1.0, 1.3, 0.8]) * math.sqrt(d_i)
    q = qs * norms[:, None]
    k = rng.standard_normal((n, d_i))
    for bias in (-1.5, -2.0, -2.5):
        rate = len(O.kept_blocks(O.block_logits(q, k, bias))) / n
        sig = norms / math.sqrt(d_i)
        per = [0.5 * math.erfc(-(bias / s) / math.sqrt(2.0)) for s in sig]
        expect = 1.0 - np.prod([1.0 - p for p in per])
        sd = math.sqrt(expect * (1 - expect) / n)
        assert abs(rate - expect) < 5 * sd, (bias, rate, expect, sd)


def check_single_token(O=O):
    rng = np.random.default_rng(5)
    q = rng.standard_normal((4, 32)); K = rng.standard_normal((1, 32)); V = rng.standard_normal((1, 32))
    out = O.softmax_attention(q, K, V, 0.3)
    assert np.array_equal(out, np.repeat(V, 4, axis=0))


def check_two_token_closed_form(O=O):
    # scores a, b far from 0: weights are sigmoid(a - b), sigmoid(b - a)
    d = 8
    q = np.zeros((2, d)); q[0, 0] = 1.0; q[1, 0] = -1.0
    K = np.zeros((2, d)); K[0, 0] = 1000.0; K[1, 0] = 998.5
    V = np.zeros((2, d)); V[0, 1] = 1.0; V[1, 2] = 1.0
    out = O.softmax_attention(q, K, V, 1.0)
    w = 1.0 / (1.0 + math.exp(-1.5))
    assert abs(out[0, 1] - w) < 1e-15 and abs(out[0, 2] - (1 - w)) < 1e-15
    assert abs(out[1, 1] - (1 - w)) < 1e-15 and abs(out[1, 2] - w) < 1e-15


def check_matches_sdpa(O=O):
    rng = np.random.default_rng(6)
    H, T, d = 8, 300, 64
    q = rng.standard_normal((H, d)); K = rng.standard_normal((T, d)); V = rng.standard_normal((T, d))
    scale = 1.0 / math.sqrt(d)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None, :], torch.from_numpy(K)[None, None].expand(1, H, T, d),
        torch.from_numpy(V)[None, None].expand(1, H, T, d), scale=scale)[0, :, 0].numpy()
    out = O.softmax_attention(q, K, V, scale)
    assert np.max(np.abs(out - ref)) < 1e-12


def check_chunked_attention_matches_whole(O=O):
    """The chunked form over bf16 bits equals the whole-array form, for chunk sizes that
    do and do not divide T, and for a chunk larger than T."""
    rng = np.random.default_rng(11)
    H, T, d = 4, 1000, 32
    K_bits = f64_to_bf16_bits(np.round(rng.standard_normal((T, d)) * 8) / 8)
    V_bits = f64_to_bf16_bits(np.round(rng.standard_normal((T, d)) * 8) / 8)
    q = rng.standard_normal((H, d))
    whole = O.softmax_attention(q, O.bf16_to_f64(K_bits), O.bf16_to_f64(V_bits), 0.25)
    for chunk in (1, 7, 128, 1000, 4096):
        got = O.softmax_attention_bits(q, K_bits, V_bits, 0.25, chunk=chunk)
        assert np.max(np.abs(got - whole)) < 1e-12, chunk
    # one token: exactly that token's V for every head
    one = O.softmax_attention_bits(q, K_bits[:1], V_bits[:1], 0.25, chunk=1)
    assert np.array_equal(one, np.repeat(O.bf16_to_f64(V_bits[:1]), H, axis=0))


def check_uniform_when_q_zero(O=O):
    rng = np.random.default_rng(7)
    K = rng.standard_normal((50, 16)); V = rng.standard_normal((50, 16))
    out = O.softmax_attention(np.zeros((3, 16)), K, V, 0.7)
    assert np.max(np.abs(out - V.mean(axis=0))) < 1e-14


def _loop_case(O, bias, window, n_ctx0=384, passes=2, d=512):
    """Tiny LSA loop whose V rows are one-hot position codes and whose queries are 0.

    With q = 0 every attended token gets weight 1/|T|, so each output row is the
    indicator of the attended set divided by its size.
    """
    rng = np.random.default_rng(8)
    L, d_i, D = 3, 128, 64
    total = n_ctx0 + 64 * passes
    assert total <= d
    w_q = f64_to_bf16_bits(rng.integers(-4, 5, (L, d_i, D)) / 8.0)
    k_idx = f64_to_bf16_bits(rng.integers(-4, 5, (total // 64, d_i)) / 4.0)
    K = f64_to_bf16_bits(np.zeros((total, d)))
    V = f64_to_bf16_bits(np.eye(total, d))
    h = {p: f64_to_bf16_bits(rng.integers(-4, 5, (L, D)) / 4.0) for p in range(passes)}
    qz = f64_to_bf16_bits(np.zeros((2, d)))
    res = O.decode_sequence(w_q, k_idx, K, V, bias, n_ctx0, window, 1.0 / math.sqrt(d),
                            lambda p: h[p], lambda p, s: qz, passes)
    return res, n_ctx0, window, total


def check_attended_set(O=O):
    for bias, window in ((0.0, 128), (1e4, 128), (-1e4, 128), (0.3, 64), (0.0, 1024)):
        res, n_ctx0, W, total = _loop_case(O, bias, window)
        for p, (ids, z, outs) in enumerate(res):
            n_ctx = n_ctx0 + 64 * p
            n_cand = max(0, (n_ctx - W) // 64)
            assert z.shape == (3, n_cand)
            if bias == 1e4:
                assert list(ids) == list(range(n_cand))
            if bias == -1e4:
                assert len(ids) == 0
            for s in (0, 1, 31, 63):
                row = outs[s][0]
                members = np.flatnonzero(row > 0)
                expect = set()
                for c in ids:
                    expect.update(range(64 * c, 64 * c + 64))
                expect.update(range(max(0, n_ctx - W), n_ctx + s + 1))
                assert set(members.tolist()) == expect
                size = min(W, n_ctx) + s + 1 + 64 * len(ids)
                assert len(members) == size
                assert np.max(np.abs(row[members] - 1.0 / size)) < 1e-15


def _sdpa_over(q, K, V, scale):
    H, d = q.shape
    T = K.shape[0]
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None, :], torch.from_numpy(K)[None, None].expand(1, H, T, d),
        torch.from_numpy(V)[None, None].expand(1, H, T, d), scale=scale)[0, :, 0].numpy()


def check_special_cases_reduce_to_dense(O=O):
    """bias=+1e4 (all kept) or W >= context: full attention; bias=-1e4: sliding window."""
    rng = np.random.default_rng(9)
    d, H, n_ctx, s = 32, 4, 640, 5
    total = n_ctx + 64
    Kf = rng.standard_normal((total, d)); Vf = rng.standard_normal((total, d))
    K = f64_to_bf16_bits(torch.tensor(Kf).to(torch.bfloat16).double().numpy())
    V = f64_to_bf16_bits(torch.tensor(Vf).to(torch.bfloat16).double().numpy())
    q = f64_to_bf16_bits(torch.tensor(rng.standard_normal((H, d))).to(torch.bfloat16).double().numpy())
    scale = 1.0 / math.sqrt(d)
    qf, Kd, Vd = O.bf16_to_f64(q), O.bf16_to_f64(K), O.bf16_to_f64(V)
    all_ids = np.arange((n_ctx - 128) // 64)
    full = _sdpa_over(qf, Kd[:n_ctx + s + 1], Vd[:n_ctx + s + 1], scale)
    got = O.step_output(q, K, V, all_ids, n_ctx, 128, s, scale)
    assert np.max(np.abs(got - full)) < 1e-12
    got = O.step_output(q, K, V, [], n_ctx, 4096, s, scale)
    assert np.max(np.abs(got - full)) < 1e-12
    win = _sdpa_over(qf, Kd[n_ctx - 128:n_ctx + s + 1], Vd[n_ctx - 128:n_ctx + s + 1], scale)
    got = O.step_output(q, K, V, [], n_ctx, 128, s, scale)
    assert np.max(np.abs(got - win)) < 1e-12


def check_per_layer_keys(O=O):
    """Per-layer key tables: layer l scores against its own table (closed form), and
    identical tables reduce to the shared-key case."""
    d_i, n = 64, 7                     # sqrt(d_i) = 8 exactly
    q = np.zeros((3, d_i))
    q[:, 0] = [2.0, -1.0, 0.5]
    k = np.zeros((3, n, d_i))
    for l in range(3):
        k[l, :, 0] = (np.arange(n) - 3.0) * (l + 1)      # table l = (l + 1) x base
    bias = -0.125
    z = O.block_logits(q, k, bias)
    for l in range(3):
        for c in range(n):
            assert z[l, c] == q[l, 0] * (c - 3.0) * (l + 1) / 8.0 + bias
    rng = np.random.default_rng(5)
    qr = rng.standard_normal((3, 128))
    kr = rng.standard_normal((11, 128))
    same = O.block_logits(qr, np.stack([kr, kr, kr]), -2.0)
    assert np.allclose(same, O.block_logits(qr, kr, -2.0), rtol=1e-13, atol=1e-13)


def check_top_p_closed_forms(O=O):
    """Top-p on probabilities with known sums: exact boundary, ties by id, p = 1."""
    pr = np.array([0.1, 0.4, 0.2, 0.3])          # sorted: 0.4 (1), 0.3 (3), 0.2 (2), 0.1 (0)
    assert list(O.top_p_set(pr, 0.6)) == [1, 3]  # 0.4 + 0.3 = 0.7 >= 0.6
    assert list(O.top_p_set(pr, 0.4)) == [1]     # reaches p exactly with one entry
    assert list(O.top_p_set(pr, 0.71)) == [1, 2, 3]
    assert list(O.top_p_set(pr, 1.0)) == [0, 1, 2, 3]
    ties = np.full(8, 0.125)                     # equal probabilities: lower ids first
    assert list(O.top_p_set(ties, 0.6)) == [0, 1, 2, 3, 4]
    # softmax: uniform logits, and a closed form for two values
    assert np.allclose(O.softmax_f64(np.zeros(5)), 0.2, rtol=0, atol=1e-15)
    two = O.softmax_f64(np.array([math.log(3.0), 0.0]))
    assert abs(two[0] - 0.75) < 1e-15 and abs(two[1] - 0.25) < 1e-15


def check_top_p_bruteforce(O=O):
    """Smallest subset reaching p, by exhaustive search over subsets on tiny rows."""
    import itertools
    rng = np.random.default_rng(8)
    for trial in range(30):
        n = int(rng.integers(1, 9))
        pr = O.softmax_f64(rng.standard_normal(n) * 2.0)
        p = float(rng.uniform(0.05, 0.95))
        best = None
        for k in range(1, n + 1):
            for sub in itertools.combinations(range(n), k):
                if pr[list(sub)].sum() >= p:
                    best = k
                    break
            if best is not None:
                break
        got = O.top_p_set(pr, p)
        assert len(got) == best
        assert pr[got].sum() >= p
        # it takes the largest probabilities
        assert pr[got].min() >= np.sort(pr)[::-1][best - 1] - 1e-15


def check_vote(O=O):
    """Votes: a block is a label when at least 3 layers keep it."""
    n = 6
    logits = np.full((5, n), -50.0)
    keep = {0: [0, 1], 1: [1, 2], 2: [1], 3: [2, 3], 4: [3, 5]}
    for l, ids in keep.items():
        logits[l, ids] = 10.0                    # one or two equal dominant entries
    labels, sets = O.denoise_labels(logits, p=0.6, min_votes=3)
    for l, ids in keep.items():
        assert list(sets[l]) == ids              # two equal halves: both needed for 0.6
    # votes: block 1 -> 3, blocks 2 and 3 -> 2, blocks 0 and 5 -> 1
    assert list(labels) == [1]


PINS = [check_bf16_decode, check_projection_unit_rows, check_projection_bruteforce,
        check_lowrank_reduces_to_full_rank, check_lowrank_unit_rows,
        check_logits_closed_form, check_per_layer_keys, check_threshold_strict, check_union_bruteforce,
        check_selection_rate, check_single_token, check_two_token_closed_form,
        check_matches_sdpa, check_chunked_attention_matches_whole, check_uniform_when_q_zero, check_attended_set,
        check_special_cases_reduce_to_dense, check_top_p_closed_forms, check_top_p_bruteforce,
        check_vote]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


def test_candidate_count_grows_one_block_per_pass():
    for n_ctx0, W in ((16384, 1024), (1 << 20, 8192), (640, 4096)):
        counts = [O.n_candidates(n_ctx0 + 64 * p, W) for p in range(5)]
        base = max(0, (n_ctx0 - W) // 64)
        assert counts[0] == base
        if n_ctx0 > W:
            assert counts == [base + p for p in range(5)]


# ----------------------------------------------------------------- planted mistakes
class _Mutant:
    """A copy of the oracle module namespace with one function replaced."""

    def __init__(self, **repl):
        for k in dir(O):
            setattr(self, k, getattr(O, k))
        for k, v in repl.items():
            setattr(self, k, v)
        # decode_sequence/step_output/index_pass resolve helpers through the module;
        # rebuild them so they use the mutant helpers.
        me = self

        def index_pass(w_q_bits, h_bits, k_idx_bits, bias):
            q = me.query_projection(me.bf16_to_f64(w_q_bits), me.bf16_to_f64(h_bits))
            z = me.block_logits(q, me.bf16_to_f64(k_idx_bits), float(bias))
            return me.kept_blocks(z), z

        def index_pass_lowrank(w1_bits, w2_bits, h_bits, k_idx_bits, bias):
            q = me.query_projection_lowrank(me.bf16_to_f64(w1_bits), me.bf16_to_f64(w2_bits),
                                            me.bf16_to_f64(h_bits))
            z = me.block_logits(q, me.bf16_to_f64(k_idx_bits), float(bias))
            return me.kept_blocks(z), z

        def step_output(q_bits, K_bits, V_bits, ids, n_ctx, window, s, scale, heads=None, block=64):
            pos = me.attended_positions(ids, n_ctx, window, s, block)
            q = me.bf16_to_f64(q_bits)
            return me.softmax_attention(q, me.bf16_to_f64(K_bits[pos]), me.bf16_to_f64(V_bits[pos]), scale)

        def decode_sequence(w_q_bits, k_idx_bits, K_bits, V_bits, bias, n_ctx0, window, scale,
                            h_of_pass, q_of_step, passes, steps=64, block=64):
            out = []
            for p in range(passes):
                n_ctx = n_ctx0 + steps * p
                nc = me.n_candidates(n_ctx, window, block)
                ids, z = index_pass(w_q_bits, h_of_pass(p), k_idx_bits[:nc], bias)
                out.append((ids, z, [step_output(q_of_step(p, s), K_bits, V_bits, ids, n_ctx,
                                                 window, s, scale) for s in range(steps)]))
            return out

        self.index_pass = repl.get("index_pass", index_pass)
        self.index_pass_lowrank = repl.get("index_pass_lowrank", index_pass_lowrank)
        self.step_output = repl.get("step_output", step_output)
        self.decode_sequence = repl.get("decode_sequence", decode_sequence)


def _fails_some_pin(mutant):
    for pin in PINS:
        try:
            pin(mutant)
        except AssertionError:
            return True
        except Exception:
            return True
    return False


def _top_p_variant(pr, p, side="left", high_id=False, extra=0):
    n = len(pr)
    ids = np.arange(n)
    order = np.lexsort((-ids if high_id else ids, -pr))
    cum = np.cumsum(pr[order])
    k = min(int(np.searchsorted(cum, p, side=side)) + extra, n - 1)
    return np.sort(order[:k + 1])


MUTANTS = {
    "logit_no_bias": dict(block_logits=lambda q, k, b: (q @ k.T) / math.sqrt(k.shape[1])),
    "logit_no_scale": dict(block_logits=lambda q, k, b: (q @ k.T) + b),
    "logit_sqrt_of_wrong_dim": dict(block_logits=lambda q, k, b: (q @ k.T) / math.sqrt(q.shape[0]) + b),
    "per_layer_keys_shifted": dict(block_logits=lambda q, k, b: O.block_logits(
        q, k if k.ndim == 2 else np.roll(k, 1, axis=0), b)),
    "per_layer_keys_first_table_only": dict(block_logits=lambda q, k, b: O.block_logits(
        q, k if k.ndim == 2 else k[0], b)),
    "lowrank_skips_up_projection": dict(query_projection_lowrank=lambda w1, w2, h: np.stack(
        [(w1[l] @ h[l])[:w2.shape[1]] for l in range(w1.shape[0])])),
    "lowrank_down_projection_of_next_layer": dict(query_projection_lowrank=lambda w1, w2, h: np.stack(
        [w2[l] @ (w1[(l + 1) % w1.shape[0]] @ h[l]) for l in range(w1.shape[0])])),
    "lowrank_latent_rounded_to_bf16": dict(query_projection_lowrank=lambda w1, w2, h: np.stack(
        [w2[l] @ torch.from_numpy(w1[l] @ h[l]).to(torch.bfloat16).double().numpy()
         for l in range(w1.shape[0])])),
    "threshold_ge": dict(kept_blocks=lambda z: np.flatnonzero((z >= 0).any(axis=0))),
    "and_instead_of_or": dict(kept_blocks=lambda z: np.flatnonzero((z > 0).all(axis=0))),
    "only_first_layer": dict(kept_blocks=lambda z: np.flatnonzero(z[0] > 0)),
    "projection_transposed_layers": dict(query_projection=lambda w, h: np.stack(
        [w[l] @ h[(l + 1) % w.shape[0]] for l in range(w.shape[0])])),
    "window_excludes_current": dict(attended_positions=lambda ids, n, W, s, block=64: np.unique(
        np.concatenate([np.arange(c * block, c * block + block) for c in ids] +
                       [np.arange(max(0, n - W), n + s)]).astype(np.int64))),
    "window_not_growing": dict(attended_positions=lambda ids, n, W, s, block=64: np.unique(
        np.concatenate([np.arange(c * block, c * block + block) for c in ids] +
                       [np.arange(max(0, n - W), n + 1)]).astype(np.int64))),
    "softmax_no_max_shift_wrong": dict(softmax_attention=lambda q, K, V, sc: (
        np.exp(sc * (q @ K.T)) @ V) / np.exp(sc * (q @ K.T)).sum(axis=1, keepdims=True) * 1.0001),
    "softmax_unscaled": dict(softmax_attention=lambda q, K, V, sc: O.softmax_attention(q, K, V, 1.0)),
    "candidates_include_window": dict(n_candidates=lambda n, W, block=64: n // block),
    "top_p_strict_gt": dict(top_p_set=lambda pr, p: _top_p_variant(pr, p, side="right")),
    "top_p_ties_by_high_id": dict(top_p_set=lambda pr, p: _top_p_variant(pr, p, high_id=True)),
    "top_p_one_extra": dict(top_p_set=lambda pr, p: _top_p_variant(pr, p, extra=1)),
    "vote_ge_2": dict(denoise_labels=lambda lg, p=0.6, min_votes=3: O.denoise_labels(lg, p, 2)),
    "chunked_attention_drops_ragged_tail": dict(
        softmax_attention_bits=lambda q, Kb, Vb, sc, chunk=65536: O.softmax_attention_bits(
            q, Kb[:max(chunk, len(Kb) // chunk * chunk)], Vb[:max(chunk, len(Kb) // chunk * chunk)],
            sc, chunk)),
    "bf16_truncated_wrong_shift": dict(bf16_to_f64=lambda b: (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(15)).view(np.float32).astype(np.float64)),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    assert _fails_some_pin(_Mutant(**MUTANTS[name])), name
