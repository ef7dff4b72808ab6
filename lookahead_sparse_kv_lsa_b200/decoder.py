"""Device buffers and the lsa_state of one batch of LSA decode sequences.

PyTorch only allocates memory here; the decode loop itself is the library's lsa_step
(index + gather at every 64th step, append + attention at every step).
"""
from __future__ import annotations

from typing import Optional

import torch

from . import _lib
from ._lib import LsaState, BLOCK


class LsaDecoder:
    """Owns the HBM pool, block tables, per-pass buffers and workspaces of a batch.

    w_q      bf16 [L][d_i][D]            (device)
    k_idx    bf16 [rows][d_i] or [L][rows][d_i] per layer (device); kidx_off int64 [B]
             row of block 0
    bias     f32 [B]
    host_pool bf16 [blocks][2][64][d]    pinned host cold pool; host_blk_off int64 [B+1]
    nb0      context blocks per sequence when pass 0 starts
    W        window tokens; H heads; cap max kept blocks per sequence and pass;
    max_cand bound on candidate counts over the run; sel_pages HBM pages for kept blocks
    """

    def __init__(self, w_q, k_idx, kidx_off, bias, host_pool, host_blk_off, nb0, W: int,
                 H: int, cap: int, max_cand: int, scale: float, sel_pages: Optional[int] = None,
                 device=None, delta_gather: bool = False):
        dev = torch.device(device) if device is not None else w_q.device
        self.device = dev
        L, d_i, D = w_q.shape
        B = len(nb0)
        d = host_pool.shape[-1]
        wb1 = W // BLOCK + 1
        self.B, self.L, self.D, self.d_i, self.H, self.d, self.W = B, L, D, d_i, H, d, W
        self.cap, self.max_cand = cap, max_cand
        if sel_pages is None:
            sel_pages = B * cap
        self.n_pages = B * wb1 + max(1, sel_pages)
        i32 = dict(dtype=torch.int32, device=dev)
        self.w_q, self.k_idx, self.bias = w_q, k_idx, bias
        self.kidx_off = torch.as_tensor(kidx_off, dtype=torch.int64).to(dev)
        self.host_pool = host_pool
        self.host_blk_off = torch.as_tensor(host_blk_off, dtype=torch.int64).to(dev)
        self.nb0 = torch.as_tensor(nb0, dtype=torch.int32).to(dev)
        # zero-filled pool: a tail page's unused slots must hold finite values
        self.hbm_pool = torch.zeros((self.n_pages, 2, BLOCK, d), dtype=torch.bfloat16, device=dev)
        self.n_cand = torch.zeros(B, **i32)
        self.sel_ids = torch.zeros((B, max(1, cap)), **i32)
        self.sel_cnt = torch.zeros(B, **i32)
        self.res_pages = torch.zeros((B, wb1), **i32)
        self.n_res = torch.zeros(B, **i32)
        self.bt_stride = cap + wb1
        self.block_table = torch.zeros((B, self.bt_stride), **i32)
        self.n_entries = torch.zeros(B, **i32)
        self.tail_len = torch.zeros(B, **i32)
        idx_bytes = _lib.lib().lsa_index_workspace_size(B, L, d_i, max_cand)
        n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
        attn_bytes = _lib.lib().lsa_decode_attn_workspace_size(B, H, d, n_sm)
        self.index_ws = torch.zeros(idx_bytes, dtype=torch.uint8, device=dev)
        self.attn_ws = torch.zeros(attn_bytes, dtype=torch.uint8, device=dev)
        self.err = torch.zeros(1, **i32)
        s = LsaState()
        s.B, s.L, s.D, s.d_i, s.H, s.d, s.W = B, L, D, d_i, H, d, W
        s.cap, s.max_cand, s.scale = cap, max_cand, float(scale)
        s.w_q, s.k_idx, s.kidx_off, s.bias = (w_q.data_ptr(), k_idx.data_ptr(),
                                              self.kidx_off.data_ptr(), bias.data_ptr())
        s.host_pool, s.host_blocks = host_pool.data_ptr(), host_pool.shape[0]
        s.host_blk_off, s.nb0 = self.host_blk_off.data_ptr(), self.nb0.data_ptr()
        s.hbm_pool, s.n_pages = self.hbm_pool.data_ptr(), self.n_pages
        s.n_cand, s.sel_ids, s.sel_cnt = (self.n_cand.data_ptr(), self.sel_ids.data_ptr(),
                                          self.sel_cnt.data_ptr())
        s.res_pages, s.n_res = self.res_pages.data_ptr(), self.n_res.data_ptr()
        s.block_table, s.bt_stride = self.block_table.data_ptr(), self.bt_stride
        s.n_entries, s.tail_len = self.n_entries.data_ptr(), self.tail_len.data_ptr()
        s.index_ws, s.index_ws_bytes = self.index_ws.data_ptr(), idx_bytes
        s.attn_ws, s.attn_ws_bytes = self.attn_ws.data_ptr(), attn_bytes
        s.err = self.err.data_ptr()
        s.kidx_layer_stride = k_idx.shape[1] if k_idx.dim() == 3 else 0
        self.delta_gather = delta_gather
        if delta_gather:     # resident-page reuse across passes
            self.kept_ids = torch.zeros((B, max(1, cap)), **i32)
            self.kept_pages = torch.zeros((B, max(1, cap)), **i32)
            self.kept_cnt = torch.zeros(B, **i32)
            self.copied = torch.zeros(1, **i32)
            gbytes = _lib.lib().lsa_gather_delta_workspace_size(
                B, cap, self.n_pages - B * wb1, n_sm)
            self.gather_ws = torch.zeros(gbytes, dtype=torch.uint8, device=dev)
            s.kept_ids, s.kept_pages = self.kept_ids.data_ptr(), self.kept_pages.data_ptr()
            s.kept_cnt = self.kept_cnt.data_ptr()
            s.gather_ws, s.gather_ws_bytes = self.gather_ws.data_ptr(), gbytes
        self.state = s
        _lib.check("lsa_state_check", _lib.lib().lsa_state_check(s))

    def load_window(self, pass_idx: int = 0, stream=None) -> None:
        from . import lsa_load_window
        lsa_load_window(self.state, pass_idx, stream)

    def step(self, step: int, h, q, k_new, v_new, out, stream=None) -> None:
        from . import lsa_step
        lsa_step(self.state, step, h, q, k_new, v_new, out, stream)

    # -- the pieces of one step, as lsa_step composes them ------------------------
    def pass_setup(self, pass_idx: int, stream=None) -> None:
        from . import lsa_pass_setup
        lsa_pass_setup(self.state, pass_idx, stream)

    def index(self, h, stream=None) -> None:
        from . import lsa_index
        lsa_index(h, self.w_q, self.bias, self.k_idx, self.kidx_off, self.n_cand, self.max_cand,
                  self.sel_ids if self.cap > 0 else self.sel_ids[:, :0], self.sel_cnt,
                  self.index_ws, self.err, stream=stream)

    def gather(self, stream=None) -> None:
        from . import lsa_gather, lsa_gather_delta
        base = self.B * (self.W // BLOCK + 1)
        if self.delta_gather:
            lsa_gather_delta(self.host_pool, self.host_blk_off, self.sel_ids, self.sel_cnt,
                             self.res_pages, self.n_res, self.hbm_pool, base, self.n_pages - base,
                             self.block_table, self.n_entries, self.kept_ids, self.kept_pages,
                             self.kept_cnt, self.gather_ws, self.err, self.copied, stream)
            return
        lsa_gather(self.host_pool, self.host_blk_off, self.sel_ids, self.sel_cnt, self.res_pages,
                   self.n_res, self.hbm_pool, base, self.n_pages - base, self.block_table,
                   self.n_entries, self.err, stream)

    def append(self, step: int, k_new, v_new, stream=None) -> None:
        from . import lsa_append
        lsa_append(self.state, step, k_new, v_new, stream)

    def decode_step(self, step: int, q, k_new, v_new, out, stream=None) -> None:
        from . import lsa_decode_step
        lsa_decode_step(self.state, step, q, k_new, v_new, out, stream)

    def attend(self, q, out, stream=None) -> None:
        from . import lsa_decode_attn
        lsa_decode_attn(q, self.hbm_pool, self.block_table, self.n_entries, self.tail_len,
                        self.state.scale, out, self.attn_ws, self.err, stream)

    def read_err(self) -> int:
        return int(self.err.item())
