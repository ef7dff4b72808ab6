"""lsa_decode_attn_noalloc: decode attention for callers that cannot allocate device
memory (a host framework that owns all allocations, a loop that must not enter the CUDA
allocator, a plugin handed only its inputs and outputs). It keeps its split partials in
a fixed device array inside the library instead of a caller workspace.

Checked through the C ABI against lsa_decode_attn (which takes a caller workspace) on two
calls in a row with different shapes, so the shared array is reused between calls.
This file is collected last on purpose."""
import ctypes as C
import math
import zlib

import numpy as np
import pytest
import torch

import lookahead_sparse_kv_lsa_b200 as lsa
from lookahead_sparse_kv_lsa_b200 import _lib
from gpu_util import ATTN_MAX_ABS, ATTN_REL_L2

pytestmark = pytest.mark.gpu


def _case(name, B, H, d, entries, tails):
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
    dev = torch.device("cuda")
    return dict(q=q.to(dev), pool=pool.to(dev), bt=bt.to(dev),
                ne=torch.tensor(entries, dtype=torch.int32, device=dev),
                tl=torch.tensor(tails, dtype=torch.int32, device=dev), B=B, H=H, d=d)


def _noalloc(c, out, err):
    return _lib.lib().lsa_decode_attn_noalloc(
        c["q"].data_ptr(), c["pool"].data_ptr(), c["pool"].shape[0], c["bt"].data_ptr(),
        c["bt"].shape[1], c["ne"].data_ptr(), c["tl"].data_ptr(), c["B"], c["H"], c["d"],
        1.0 / math.sqrt(c["d"]), out.data_ptr(), err.data_ptr(),
        torch.cuda.current_stream().cuda_stream)


def _with_workspace(c):
    out = torch.empty((c["B"], c["H"], c["d"]), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(lsa.decode_attn_workspace_size(c["B"], c["H"], c["d"]), dtype=torch.uint8,
                     device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    lsa.lsa_decode_attn(c["q"], c["pool"], c["bt"], c["ne"], c["tl"], 1.0 / math.sqrt(c["d"]),
                        out, ws, err)
    return out, int(err.item())


def test_noalloc_matches_workspace_entry_point_twice(cuda_ok):
    cases = [_case("noalloc_a", 2, 64, 512, [300, 77], [33, 5]),
             _case("noalloc_b", 3, 8, 128, [1, 40, 9], [1, 64, 20])]
    for c in cases:                    # two calls in a row share the library's array
        ref, err_ref = _with_workspace(c)
        out = torch.full_like(ref, float("nan"))
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        assert _noalloc(c, out, err) == _lib.LSA_OK
        torch.cuda.synchronize()
        assert err_ref == 0 and int(err.item()) == 0
        g = out.float().cpu().numpy()
        r = ref.float().cpu().numpy()
        assert np.all(np.isfinite(g))
        assert np.abs(g - r).max() <= ATTN_MAX_ABS
        assert np.linalg.norm(g - r) / np.linalg.norm(r) <= ATTN_REL_L2


def test_noalloc_rejects_sizes_beyond_its_array(cuda_ok):
    # 2,000 sequences x 64 heads x 512 need far more than LSA_NOALLOC_SCRATCH_BYTES
    p = C.c_void_p(16)
    st = _lib.lib().lsa_decode_attn_noalloc(p, p, 1, p, 1, p, p, 2000, 64, 512, 0.1, p, p, None)
    assert st == _lib.LSA_ERR_CAPACITY
