"""lsa_decode_attn_noalloc: decode attention for callers that cannot allocate device
memory (a host framework that owns all allocations, a loop that must not enter the CUDA
allocator, a plugin handed only its inputs and outputs). It keeps its split partials in
a fixed device array inside the library instead of a caller workspace.

Checked through the C ABI against lsa_decode_attn (which takes a caller workspace) and
against the oracle, on two calls in a row with different shapes, so the shared array is
reused between calls. The first call of a process is checked too, in a fresh child
process, on a non-default stream with nothing synchronised before it: that call sets the
array up, and the set-up must be ordered before the kernel on the caller's stream.
This file is collected last on purpose."""
import ctypes as C
import math
import os
import subprocess
import sys
import zlib

import numpy as np
import pytest
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
for p in (ROOT, HERE):
    if p not in sys.path:
        sys.path.insert(0, p)

import lookahead_sparse_kv_lsa_b200 as lsa  # noqa: E402
from lookahead_sparse_kv_lsa_b200 import _lib  # noqa: E402
from gpu_util import ATTN_MAX_ABS, ATTN_REL_L2, paged_oracle_out  # noqa: E402

pytestmark = pytest.mark.gpu


def _case(name, B, H, d, entries, tails):
    """Random pool and distinct pages per sequence (host tensors)."""
    g = torch.Generator().manual_seed(zlib.crc32(name.encode()) & 0xFFFF)
    n_pages = sum(entries) + 2
    pool = torch.randn((n_pages, 2, 64, d), generator=g).to(torch.bfloat16)
    perm = torch.randperm(n_pages, generator=g)
    bt = torch.full((B, max(entries)), -1, dtype=torch.int32)
    k = 0
    for b in range(B):
        for e in range(entries[b]):
            bt[b, e] = int(perm[k])
            k += 1
    q = torch.randn((B, H, d), generator=g).to(torch.bfloat16)
    return dict(q=q, pool=pool, bt=bt, entries=list(entries), tails=list(tails), B=B, H=H, d=d)


def _to_dev(c, dev):
    return dict(q=c["q"].to(dev), pool=c["pool"].to(dev), bt=c["bt"].to(dev),
                ne=torch.tensor(c["entries"], dtype=torch.int32, device=dev),
                tl=torch.tensor(c["tails"], dtype=torch.int32, device=dev))


def _noalloc(c, g, out, err, stream):
    return _lib.lib().lsa_decode_attn_noalloc(
        g["q"].data_ptr(), g["pool"].data_ptr(), g["pool"].shape[0], g["bt"].data_ptr(),
        g["bt"].shape[1], g["ne"].data_ptr(), g["tl"].data_ptr(), c["B"], c["H"], c["d"],
        1.0 / math.sqrt(c["d"]), out.data_ptr(), err.data_ptr(), stream.cuda_stream)


def _with_workspace(c, g):
    out = torch.empty((c["B"], c["H"], c["d"]), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(lsa.decode_attn_workspace_size(c["B"], c["H"], c["d"]), dtype=torch.uint8,
                     device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    lsa.lsa_decode_attn(g["q"], g["pool"], g["bt"], g["ne"], g["tl"], 1.0 / math.sqrt(c["d"]),
                        out, ws, err)
    torch.cuda.synchronize()
    return out, int(err.item())


def _close(got, ref):
    g = got.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(g))
    assert np.abs(g - ref).max() <= ATTN_MAX_ABS
    assert np.linalg.norm(g - ref) / np.linalg.norm(ref) <= ATTN_REL_L2


CASES = [("noalloc_a", 2, 64, 512, [300, 77], [33, 5]),
         ("noalloc_b", 3, 8, 128, [1, 40, 9], [1, 64, 20])]


def _check_cases(first_on_fresh_stream: bool):
    """Two no-alloc calls in a row (different shapes), each compared with the oracle and
    with lsa_decode_attn. When first_on_fresh_stream, the first call is issued on a new
    non-default stream that only waits (on the device) for the input copies."""
    dev = torch.device("cuda")
    for i, spec in enumerate(CASES):
        c = _case(*spec)
        g = _to_dev(c, dev)
        out = torch.full((c["B"], c["H"], c["d"]), float("nan"), dtype=torch.bfloat16, device=dev)
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        if first_on_fresh_stream and i == 0:
            s = torch.cuda.Stream()
            s.wait_stream(torch.cuda.current_stream())
            assert _noalloc(c, g, out, err, s) == _lib.LSA_OK
            torch.cuda.current_stream().wait_stream(s)
        else:
            assert _noalloc(c, g, out, err, torch.cuda.current_stream()) == _lib.LSA_OK
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        scale = 1.0 / math.sqrt(c["d"])
        ref = paged_oracle_out(c["pool"], c["bt"], c["q"], c["entries"], c["tails"], scale)
        _close(out, ref)
        ws_out, ws_err = _with_workspace(c, g)
        assert ws_err == 0
        _close(out, ws_out.float().cpu().numpy().astype(np.float64))


def test_noalloc_matches_workspace_entry_point_and_oracle_twice(cuda_ok):
    _check_cases(first_on_fresh_stream=False)


def test_noalloc_first_call_of_a_process_on_a_fresh_stream(cuda_ok):
    """A child process makes its very first no-alloc call on a new non-default stream."""
    r = subprocess.run([sys.executable, os.path.abspath(__file__), "--first-call-child"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "first-call ok" in r.stdout


def test_noalloc_rejects_sizes_beyond_its_array(cuda_ok):
    # 2,000 sequences x 64 heads x 512 need far more than LSA_NOALLOC_SCRATCH_BYTES; the
    # pointers are never dereferenced (the call returns before anything is enqueued)
    p = C.c_void_p(16)
    st = _lib.lib().lsa_decode_attn_noalloc(p, p, 1, p, 1, p, p, 2000, 64, 512, 0.1, p, p, None)
    assert st == _lib.LSA_ERR_CAPACITY
    # a malformed call is reported as such even when it is also too large
    st = _lib.lib().lsa_decode_attn_noalloc(p, p, 1, p, 1, p, p, 2000, 65, 512, 0.1, p, p, None)
    assert st == _lib.LSA_ERR_INVALID_ARG
    st = _lib.lib().lsa_decode_attn_noalloc(p, p, 1, p, 1, p, p, 2000, 64, 500, 0.1, p, p, None)
    assert st == _lib.LSA_ERR_INVALID_ARG


if __name__ == "__main__" and "--first-call-child" in sys.argv:
    torch.cuda.init()
    _check_cases(first_on_fresh_stream=True)
    print("first-call ok")
