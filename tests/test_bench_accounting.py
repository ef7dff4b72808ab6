"""The byte counts behind the bench's roofline figures, against closed forms written from
the step definitions: a decode step streams K and V (d bf16 each) of every attended token,
T = 64 |S| + W + s + 1, and reads q and writes the output (H x d bf16 each); an indexer
pass reads W_q, h, one K_idx row per candidate block (per table) and writes the ids; a
gather moves K and V of 64 tokens per kept block. Worked numbers are the 1M-token
workload at bias -2 with 1,079 kept blocks of 16,256 candidates."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402
import lsa_inputs as LI  # noqa: E402


def test_decode_step_bytes_1m():
    c = LI.by_name("1m_b20")
    ctx = [1_048_576]
    for s in (0, 31, 63):
        T = 64 * 1079 + 8192 + s + 1
        want = T * 512 * 2 * 2 + 2 * 64 * 512 * 2
        assert bench.attn_bytes_per_step(c, ctx, [1079], s) == want
    # the mean over the 64 steps of a pass, as the bench's roofline line reports it
    mean = sum(bench.attn_bytes_per_step(c, ctx, [1079], s) for s in range(64)) / 64
    assert mean == 158_401_536


def test_decode_step_bytes_window_longer_than_context():
    """A sequence shorter than the window attends to all of its tokens."""
    c = LI.by_name("tiny_16k")
    T = 64 * 3 + 500 + 5 + 1
    assert bench.attn_bytes_per_step(c, [500], [3], 5) == T * c.d * 2 * 2 + 2 * c.H * c.d * 2


def test_indexer_bytes_1m():
    c = LI.by_name("1m_b20")
    want = (3 * 128 * 4096 * 2        # W_q
            + 1 * 3 * 4096 * 2        # h
            + 16_256 * 128 * 2        # one shared K_idx row per candidate
            + 4 * 1079)               # ids
    assert want == 7_336_156
    assert bench.index_bytes(c, [16_256], [1079]) == want


def test_indexer_bytes_per_layer_tables():
    c = LI.by_name("1m_b20_lk")
    assert c.kidx_per_layer
    want = 3 * 128 * 4096 * 2 + 3 * 4096 * 2 + 3 * 16_256 * 128 * 2 + 4 * 1000
    assert bench.index_bytes(c, [16_256], [1000]) == want


def test_launches_per_pass():
    """Pass set-up, the indexer and the gather, then one fused launch per decode step."""
    assert bench.LAUNCHES_PER_PASS_HEAD + 64 * bench.LAUNCHES_PER_DECODE_STEP == 67
