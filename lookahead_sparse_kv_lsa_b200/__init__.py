"""Lookahead Sparse Attention (LSA) decode hot path for B200 (sm_100a).

Thin Python binding over the C ABI of include/lsa.h: every function below only checks
and marshals torch tensors (device memory, streams) into the library's entry points.
All computation happens in the library's CUDA kernels.
"""
from __future__ import annotations

import ctypes as C
from typing import Optional

import torch

from . import _lib
from ._lib import LsaError, LsaState, BLOCK, TAU

__all__ = ["lsa_index", "lsa_index_lowrank", "index_lowrank_workspace_size", "lsa_gather", "lsa_gather_delta", "lsa_decode_attn", "lsa_step",
           "lsa_load_window", "gather_delta_workspace_size", "lsa_denoise_labels",
           "DENOISE_MAX_BLOCKS", "lsa_wait_selftest",
           "lsa_pass_setup", "lsa_append", "lsa_decode_step",
           "index_workspace_size", "decode_attn_workspace_size", "LsaDecoder", "LsaError",
           "LsaState", "BLOCK", "TAU", "library_path"]


def library_path() -> str:
    return _lib.LIB_PATH


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dev(t: torch.Tensor, dtype, name: str, numel: Optional[int] = None) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if numel is not None and t.numel() < numel:
        raise ValueError("%s holds %d elements, needs %d" % (name, t.numel(), numel))
    return t.data_ptr()


def _opt(t, dtype, name, numel=None) -> Optional[int]:
    return None if t is None else _dev(t, dtype, name, numel)


def index_workspace_size(B: int, L: int, d_i: int, max_cand: int) -> int:
    return int(_lib.lib().lsa_index_workspace_size(B, L, d_i, max_cand))


def decode_attn_workspace_size(B: int, H: int, d: int, n_sm: Optional[int] = None) -> int:
    if n_sm is None:
        n_sm = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    return int(_lib.lib().lsa_decode_attn_workspace_size(B, H, d, n_sm))


def lsa_index(h, w_q, bias, k_idx, kidx_off, n_cand, max_cand: int, sel_ids, sel_cnt, ws, err,
              logits=None, layer_mask=None, stream=None) -> None:
    """One indexer pass; see lsa_index / lsa_index_ex in include/lsa.h. h [L][B][D],
    w_q [L][d_i][D]; k_idx [rows][d_i] (shared by the layers) or [L][rows][d_i] (one
    table per layer)."""
    L, B, D = h.shape
    d_i = w_q.shape[1]
    cap = sel_ids.shape[1] if sel_ids.dim() == 2 else 0
    if k_idx.dim() == 3:
        if k_idx.shape[0] != L:
            raise ValueError("per-layer k_idx must have L = %d tables" % L)
        layer_stride = k_idx.shape[1]
    else:
        layer_stride = 0
    st = _lib.lib().lsa_index_ex(
        _dev(h, torch.bfloat16, "h"), _dev(w_q, torch.bfloat16, "w_q", L * d_i * D),
        _dev(bias, torch.float32, "bias", B), _dev(k_idx, torch.bfloat16, "k_idx"), layer_stride,
        _dev(kidx_off, torch.int64, "kidx_off", B), _dev(n_cand, torch.int32, "n_cand", B),
        B, L, D, d_i, max_cand,
        _dev(sel_ids, torch.int32, "sel_ids"), _dev(sel_cnt, torch.int32, "sel_cnt", B), cap,
        _opt(logits, torch.float32, "logits", L * B * max_cand),
        _opt(layer_mask, torch.int32, "layer_mask", (L + 1) * B * ((max_cand + 31) // 32)),
        _dev(ws, torch.uint8, "ws"), ws.numel(), _dev(err, torch.int32, "err", 1), _stream(stream))
    _lib.check("lsa_index", st)


def index_lowrank_workspace_size(B: int, L: int, d_i: int, r: int, max_cand: int) -> int:
    return int(_lib.lib().lsa_index_lowrank_workspace_size(B, L, d_i, r, max_cand))


def lsa_index_lowrank(h, w_1, w_2, bias, k_idx, kidx_off, n_cand, max_cand: int, sel_ids,
                      sel_cnt, ws, err, logits=None, layer_mask=None, stream=None) -> None:
    """One indexer pass with factorised query encoders q = W_2 (W_1 h); see
    lsa_index_lowrank in include/lsa.h. w_1 [L][r][D], w_2 [L][d_i][r]."""
    L, B, D = h.shape
    r = w_1.shape[1]
    d_i = w_2.shape[1]
    cap = sel_ids.shape[1] if sel_ids.dim() == 2 else 0
    layer_stride = k_idx.shape[1] if k_idx.dim() == 3 else 0
    st = _lib.lib().lsa_index_lowrank(
        _dev(h, torch.bfloat16, "h"), _dev(w_1, torch.bfloat16, "w_1", L * r * D),
        _dev(w_2, torch.bfloat16, "w_2", L * d_i * r), r,
        _dev(bias, torch.float32, "bias", B), _dev(k_idx, torch.bfloat16, "k_idx"), layer_stride,
        _dev(kidx_off, torch.int64, "kidx_off", B), _dev(n_cand, torch.int32, "n_cand", B),
        B, L, D, d_i, max_cand,
        _dev(sel_ids, torch.int32, "sel_ids"), _dev(sel_cnt, torch.int32, "sel_cnt", B), cap,
        _opt(logits, torch.float32, "logits", L * B * max_cand),
        _opt(layer_mask, torch.int32, "layer_mask", (L + 1) * B * ((max_cand + 31) // 32)),
        _dev(ws, torch.uint8, "ws"), ws.numel(), _dev(err, torch.int32, "err", 1), _stream(stream))
    _lib.check("lsa_index_lowrank", st)


def lsa_gather(host_pool, host_blk_off, sel_ids, sel_cnt, res_pages, n_res, hbm_pool,
               sel_page_base: int, sel_page_count: int, block_table, n_entries, err,
               stream=None) -> None:
    """Copy kept blocks host pool -> HBM pool and build block tables (lsa_gather in lsa.h)."""
    if host_pool.is_cuda or not host_pool.is_pinned() or host_pool.dtype != torch.bfloat16:
        raise ValueError("host_pool must be a pinned host bf16 tensor")
    B = sel_cnt.shape[0]
    d = hbm_pool.shape[-1]
    st = _lib.lib().lsa_gather(
        host_pool.data_ptr(), host_pool.shape[0], _dev(host_blk_off, torch.int64, "host_blk_off", B),
        _dev(sel_ids, torch.int32, "sel_ids"), _dev(sel_cnt, torch.int32, "sel_cnt", B),
        sel_ids.shape[1], _dev(res_pages, torch.int32, "res_pages"),
        _dev(n_res, torch.int32, "n_res", B), res_pages.shape[1], B, d,
        _dev(hbm_pool, torch.bfloat16, "hbm_pool"), hbm_pool.shape[0], sel_page_base,
        sel_page_count, _dev(block_table, torch.int32, "block_table"), block_table.shape[1],
        _dev(n_entries, torch.int32, "n_entries", B), _dev(err, torch.int32, "err", 1),
        _stream(stream))
    _lib.check("lsa_gather", st)


def gather_delta_workspace_size(B: int, cap: int, sel_page_count: int,
                                n_sm: Optional[int] = None) -> int:
    if n_sm is None:
        n_sm = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    return int(_lib.lib().lsa_gather_delta_workspace_size(B, cap, sel_page_count, n_sm))


def lsa_gather_delta(host_pool, host_blk_off, sel_ids, sel_cnt, res_pages, n_res, hbm_pool,
                     sel_page_base: int, sel_page_count: int, block_table, n_entries, kept_ids,
                     kept_pages, kept_cnt, ws, err, copied=None, stream=None) -> None:
    """lsa_gather with resident-page reuse across passes (lsa_gather_delta in lsa.h)."""
    if host_pool.is_cuda or not host_pool.is_pinned() or host_pool.dtype != torch.bfloat16:
        raise ValueError("host_pool must be a pinned host bf16 tensor")
    B = sel_cnt.shape[0]
    d = hbm_pool.shape[-1]
    cap = sel_ids.shape[1]
    st = _lib.lib().lsa_gather_delta(
        host_pool.data_ptr(), host_pool.shape[0], _dev(host_blk_off, torch.int64, "host_blk_off", B),
        _dev(sel_ids, torch.int32, "sel_ids"), _dev(sel_cnt, torch.int32, "sel_cnt", B), cap,
        _dev(res_pages, torch.int32, "res_pages"), _dev(n_res, torch.int32, "n_res", B),
        res_pages.shape[1], B, d, _dev(hbm_pool, torch.bfloat16, "hbm_pool"), hbm_pool.shape[0],
        sel_page_base, sel_page_count, _dev(block_table, torch.int32, "block_table"),
        block_table.shape[1], _dev(n_entries, torch.int32, "n_entries", B),
        _dev(kept_ids, torch.int32, "kept_ids", B * cap), _dev(kept_pages, torch.int32, "kept_pages", B * cap),
        _dev(kept_cnt, torch.int32, "kept_cnt", B), _dev(ws, torch.uint8, "ws"), ws.numel(),
        _opt(copied, torch.int32, "copied", 1), _dev(err, torch.int32, "err", 1), _stream(stream))
    _lib.check("lsa_gather_delta", st)


DENOISE_MAX_BLOCKS = 45056


def lsa_denoise_labels(logits, set_mask, label_cnt, err, top_p: float = 0.6,
                       min_votes: int = 3, set_cnt=None, label_mask=None, label_ids=None,
                       stream=None) -> None:
    """Label denoising (lsa_denoise_labels in lsa.h). logits: f32 [W][L][N] on the device;
    set_mask: u32 words [W][L][ceil(N/32)] (an int32 tensor); label_cnt: i32 [W];
    label_ids: i32 [W][cap] or None."""
    W, L, N = logits.shape
    NW = (N + 31) // 32
    cap = 0 if label_ids is None else label_ids.shape[1]
    st = _lib.lib().lsa_denoise_labels(
        _dev(logits, torch.float32, "logits"), W, L, N, float(top_p), int(min_votes),
        _dev(set_mask, torch.int32, "set_mask", W * L * NW),
        _opt(set_cnt, torch.int32, "set_cnt", W * L),
        _opt(label_mask, torch.int32, "label_mask", W * NW),
        _opt(label_ids, torch.int32, "label_ids", W * cap), cap,
        _dev(label_cnt, torch.int32, "label_cnt", W), _dev(err, torch.int32, "err", 1),
        _stream(stream))
    _lib.check("lsa_denoise_labels", st)


def lsa_wait_selftest(flag, target: int, limit_ns: int, err, stream=None) -> None:
    """The library's bounded device wait on its own (lsa_wait_selftest in lsa.h): polls the
    device u32 `flag` (an int32 tensor) until it reaches `target`, or ORs the timeout bit
    into `err` after `limit_ns`."""
    st = _lib.lib().lsa_wait_selftest(_dev(flag, torch.int32, "flag", 1), int(target) & 0xffffffff,
                                      int(limit_ns), _dev(err, torch.int32, "err", 1),
                                      _stream(stream))
    _lib.check("lsa_wait_selftest", st)


def lsa_decode_attn(q, hbm_pool, block_table, n_entries, tail_len, scale: float, out, ws, err,
                    stream=None) -> None:
    """One block-sparse MQA decode step (lsa_decode_attn in lsa.h). q, out: [B][H][d] bf16."""
    B, H, d = q.shape
    st = _lib.lib().lsa_decode_attn(
        _dev(q, torch.bfloat16, "q"), _dev(hbm_pool, torch.bfloat16, "hbm_pool"),
        hbm_pool.shape[0], _dev(block_table, torch.int32, "block_table"), block_table.shape[1],
        _dev(n_entries, torch.int32, "n_entries", B), _dev(tail_len, torch.int32, "tail_len", B),
        B, H, d, float(scale), _dev(out, torch.bfloat16, "out", B * H * d),
        _dev(ws, torch.uint8, "ws"), ws.numel(), _dev(err, torch.int32, "err", 1),
        _stream(stream))
    _lib.check("lsa_decode_attn", st)


def lsa_load_window(state: LsaState, pass_idx: int, stream=None) -> None:
    _lib.check("lsa_load_window", _lib.lib().lsa_load_window(C.byref(state), pass_idx,
                                                               _stream(stream)))


def lsa_pass_setup(state: LsaState, pass_idx: int, stream=None) -> None:
    """Pass start bookkeeping of the step driver (lsa_pass_setup in lsa.h)."""
    _lib.check("lsa_pass_setup", _lib.lib().lsa_pass_setup(C.byref(state), pass_idx,
                                                             _stream(stream)))


def lsa_append(state: LsaState, step: int, k_new, v_new, stream=None) -> None:
    """Append the step's token to the tail pages (lsa_append in lsa.h)."""
    st = _lib.lib().lsa_append(C.byref(state), step, _dev(k_new, torch.bfloat16, "k_new"),
                               _dev(v_new, torch.bfloat16, "v_new"), _stream(stream))
    _lib.check("lsa_append", st)


def lsa_decode_step(state: LsaState, step: int, q, k_new, v_new, out, stream=None) -> None:
    """Decode attention with the token append fused in (lsa_decode_step in lsa.h)."""
    st = _lib.lib().lsa_decode_step(C.byref(state), step, _dev(q, torch.bfloat16, "q"),
                                    _dev(k_new, torch.bfloat16, "k_new"),
                                    _dev(v_new, torch.bfloat16, "v_new"),
                                    _dev(out, torch.bfloat16, "out"), _stream(stream))
    _lib.check("lsa_decode_step", st)


def lsa_step(state: LsaState, step: int, h, q, k_new, v_new, out, stream=None) -> None:
    """One decode step of the LSA loop (lsa_step in lsa.h)."""
    hp = None if h is None else _dev(h, torch.bfloat16, "h")
    st = _lib.lib().lsa_step(C.byref(state), step, hp, _dev(q, torch.bfloat16, "q"),
                             _dev(k_new, torch.bfloat16, "k_new"),
                             _dev(v_new, torch.bfloat16, "v_new"),
                             _dev(out, torch.bfloat16, "out"), _stream(stream))
    _lib.check("lsa_step", st)


from .decoder import LsaDecoder  # noqa: E402
