"""The C-ABI library: it loads without a GPU, exports every declared entry point, and its
host-side argument checks answer before any device work (no compute calls here)."""
import ctypes as C
import os
import re

import pytest

from lookahead_sparse_kv_lsa_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lsa.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(lsa_[a-z_0-9]+)\s*\(",
                       text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from lookahead_sparse_kv_lsa_b200 import build
    build.build()          # incremental: a no-op when the library is current
    return _lib.lib()


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("lsa_index", "lsa_gather", "lsa_decode_attn", "lsa_step", "lsa_status_str"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    # the ctypes signatures cover exactly the declared functions
    assert sorted(_lib.SIGNATURES) == declared_functions()


def test_state_struct_matches(lib):
    assert lib.lsa_state_size() == C.sizeof(_lib.LsaState)


def test_status_strings(lib):
    assert lib.lsa_status_str(0) == b"ok"
    assert lib.lsa_status_str(1) == b"invalid argument"
    assert lib.lsa_status_str(99) == b"unknown status"
    assert lib.lsa_version() >= 100


def test_workspace_sizes(lib):
    # (n_sm + B) slots of H*(d + 4) floats, rounded to 256 bytes, + one 256-byte line of
    # grid-barrier counters
    body = 149 * 64 * 516 * 4
    assert lib.lsa_decode_attn_workspace_size(1, 64, 512, 148) == (body + 255) // 256 * 256 + 256
    assert lib.lsa_decode_attn_workspace_size(0, 64, 512, 148) == 0
    assert lib.lsa_index_workspace_size(1, 3, 128, 16256) > 3 * 128 * 4
    assert lib.lsa_index_workspace_size(1, 3, 64, 100) == 0


def test_index_workspace_layout(lib):
    """The grid-barrier counter's 256-byte line comes first, then q fp32 [L][B][128] and
    the keep words u32 [B][ceil(max_cand/32)], each rounded up to 256 bytes: a workspace
    sized for one shape serves every shape that is no larger."""
    def expect(B, L, mc):
        r = lambda x: (x + 255) // 256 * 256
        return 256 + r(L * B * 128 * 4) + r(B * max(1, (mc + 31) // 32) * 4)
    for B, L, mc in ((1, 3, 16256), (64, 3, 4032), (300, 4, 90), (1, 1, 0), (7, 2, 33)):
        assert lib.lsa_index_workspace_size(B, L, 128, mc) == expect(B, L, mc)
    sizes = [lib.lsa_index_workspace_size(B, L, 128, mc)
             for B in (1, 2, 9) for L in (1, 3, 4) for mc in (0, 31, 32, 1000)]
    big = lib.lsa_index_workspace_size(9, 4, 128, 1000)
    assert max(sizes) == big


def test_invalid_arguments_rejected_before_device_work(lib):
    # null pointers
    assert lib.lsa_decode_attn(None, None, 1, None, 1, None, None, 1, 8, 128, 0.1, None, None, 0,
                               None, None) == _lib.LSA_ERR_INVALID_ARG
    fake = C.c_void_p(16)
    # unsupported head dimension / head count / scale
    for (H, d, sc) in ((8, 96, 0.1), (65, 128, 0.1), (8, 128, -1.0), (8, 128, float("nan"))):
        assert lib.lsa_decode_attn(fake, fake, 1, fake, 1, fake, fake, 1, H, d, sc, fake, fake,
                                   1 << 30, fake, None) == _lib.LSA_ERR_INVALID_ARG
    # indexer: d_i must be 128, D a multiple of 256, L in 1..4
    for (L, D, d_i) in ((3, 1000, 128), (3, 1024, 64), (0, 1024, 128), (5, 1024, 128)):
        assert lib.lsa_index(fake, fake, fake, fake, fake, fake, 1, L, D, d_i, 10, fake, fake, 4,
                             None, None, fake, 1 << 20, fake, None) == _lib.LSA_ERR_INVALID_ARG
    # gather: block table too narrow for cap + resident pages
    assert lib.lsa_gather(fake, 10, fake, fake, fake, 8, fake, fake, 4, 1, 128, fake, 100, 0, 10,
                          fake, 11, fake, fake, None) == _lib.LSA_ERR_INVALID_ARG
    assert lib.lsa_state_check(None) == _lib.LSA_ERR_INVALID_ARG
    st = _lib.LsaState()
    assert lib.lsa_state_check(C.byref(st)) == _lib.LSA_ERR_INVALID_ARG
    assert lib.lsa_step(None, 0, None, None, None, None, None, None) == _lib.LSA_ERR_INVALID_ARG
    # label denoising: layers 1..63, blocks 1..45056, 0 < top_p <= 1, ids when cap > 0
    ok = dict(W=4, L=21, N=1000, p=0.6, cap=8, ids=fake, logits=fake)
    for bad in (dict(L=0), dict(L=64), dict(N=0), dict(N=45057), dict(p=0.0), dict(p=1.5),
                dict(p=float("nan")), dict(cap=-1), dict(ids=None), dict(W=0), dict(logits=None)):
        a = dict(ok, **bad)
        assert lib.lsa_denoise_labels(a["logits"], a["W"], a["L"], a["N"], a["p"], 3, fake, None,
                                      None, a["ids"], a["cap"], fake, fake,
                                      None) == _lib.LSA_ERR_INVALID_ARG, bad
    # the bounded-wait self-test: a flag and an error word, 1 ns .. 10 s
    assert lib.lsa_wait_selftest(None, 1, 1000, fake, None) == _lib.LSA_ERR_INVALID_ARG
    assert lib.lsa_wait_selftest(fake, 1, 0, fake, None) == _lib.LSA_ERR_INVALID_ARG
    assert lib.lsa_wait_selftest(fake, 1, 10**10 + 1, fake, None) == _lib.LSA_ERR_INVALID_ARG
