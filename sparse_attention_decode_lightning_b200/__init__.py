"""Thin Python binding of libdsa (DSA decode on B200, sm_100a).

Argument marshalling only: every function below forwards torch tensors'
device pointers to the C ABI declared in include/dsa.h, under the same name,
and raises DSAError on a non-zero status.  No step of the computation runs in
Python, and there is no fallback: if libdsa.so is missing, loading fails.
"""
import ctypes
import os
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdsa.so")

PAGE_SIZE = 64
TIER_PAGE = 16       # tokens per slot of the two-tier (HiSparse) cache
HEADS = 128          # MLA heads, DeepSeek-V3.2
HEADS_GLM = 64       # MLA heads, GLM-5.2
DIM = 576
DIM_V = 512
IDX_HEADS = 64       # indexer heads, DeepSeek-V3.2
IDX_HEADS_GLM = 32   # indexer heads, GLM-5.2
IDX_DIM = 128
MAX_TOPK = 2048
MAX_Q_PER_SEQ = 8

STATUS = {0: "DSA_OK", 1: "DSA_ERR_INVALID_ARG", 2: "DSA_ERR_UNSUPPORTED", 3: "DSA_ERR_CUDA",
          4: "DSA_ERR_DEVICE_BOUNDS", 5: "DSA_ERR_TIMEOUT", 6: "DSA_ERR_WORKSPACE"}

# name -> (restype, argtypes) of every exported entry point
_P, _I, _I64, _SZ, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
_PP = ctypes.POINTER(ctypes.c_void_p)
SIGNATURES = {
    "dsa_status_string": (ctypes.c_char_p, [_I]),
    "dsa_version": (_I, []),
    "dsa_workspace_bytes": (_SZ, [_I, _I, _I, _I]),
    "dsa_choose_splits": (_I, [_I, _I, _I]),
    "dsa_mla_group_plan": (_I, [_I, _I, _P, _P, _P]),
    "dsa_indexer_scores": (_I, [_P, _P, _P, _I64, _P, _P, _P, _I, _I, _I, _I, _I, _P, _I, _P, _SZ,
                                _P]),
    "dsa_topk_select": (_I, [_P, _I, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _SZ, _P]),
    "dsa_indexer_topk": (_I, [_P, _P, _P, _I64, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _SZ,
                              _P]),
    "dsa_indexer_topk_fused": (_I, [_P, _P, _P, _I64, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P,
                                    _P, _SZ, _P]),
    "dsa_sparse_mla_decode": (_I, [_P, _P, _I, _I, _P, _I, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P,
                                   _P, _P, _SZ, _P]),
    "dsa_sparse_mla_decode_noalloc": (_I, [_P, _P, _I, _I, _P, _I, _P, _P, _P, _I, _I, _I, _I, _F,
                                           _I, _P, _P, _P]),
    "dsa_sparse_mla_decode_window": (_I, [_P, _P, _I, _I, _P, _I, _P, _I, _P, _P, _P, _P, _I, _I,
                                          _I, _I, _I, _F, _I, _P, _P, _P, _SZ, _P]),
    "dsa_sparse_mla_decode_fp8": (_I, [_P, _P, _F, _I, _I, _P, _I, _P, _P, _P, _I, _I, _I, _I, _F,
                                       _I, _P, _P, _P, _SZ, _P]),
    "dsa_lse_combine": (_I, [_P, _P, _I, _I, _I, _P, _P, _P]),
    "dsa_decode_step": (_I, [_I, _I, _I, _PP, _PP, _PP, _I64, _P, _P, _P, _I, _I, _I, _I, _I, _I,
                             _PP, _PP, _I, _I, _PP, _I, _F, _I, _PP, _PP, _P, _P, _SZ, _P]),
    "dsa_tier_state_bytes": (_SZ, [_I, _I, _I]),
    "dsa_tier_init": (_I, [_P, _SZ, _I, _I, _I]),
    "dsa_tier_plan": (_I, [_P, _P, _I, _I, _P, _P, _P, _I, _P, _P]),
    "dsa_tier_fetch": (_I, [_P, _I64, _P, _I64, _P, _I, _P, _P, _P]),
    "dsa_tier_dev_state_bytes": (_SZ, [_I, _I, _I]),
    "dsa_tier_dev_init": (_I, [_P, _SZ, _I, _I, _I, _P, _P]),
    "dsa_tier_swap_in": (_I, [_P, _SZ, _I, _I, _I, _P, _I, _I, _P, _P, _P, _P, _P, _P]),
    "dsa_tier_dev_stats": (_I, [_P, _P, _P]),
    "dsa_tier_dev_copies": (_P, [_P, _I, _I, _I]),
    "dsa_check_error": (_I, [_P, _P]),
    "dsa_noalloc_check_error": (_I, [_P]),
    "dsa_selftest_bounded_wait": (_I, [_I, _P, _SZ, _P]),
}

_lib = None


class DSAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


def lib() -> ctypes.CDLL:
    """Load libdsa.so (built in-tree by build.py); fails loudly if it is absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m sparse_attention_decode_lightning_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libdsa takes device tensors")
    if not t.is_contiguous():
        raise ValueError("libdsa takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _host_ptr(t: torch.Tensor):
    if t.is_cuda:
        raise ValueError("this argument is host memory")
    if not t.is_contiguous():
        raise ValueError("libdsa takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(status: int, where: str):
    if status != 0:
        raise DSAError(status, where)


def _ptr_array(ts: Sequence[Optional[torch.Tensor]]):
    arr = (ctypes.c_void_p * len(ts))()
    for i, t in enumerate(ts):
        arr[i] = None if t is None else _ptr(t).value
    return arr


def dsa_version() -> int:
    return lib().dsa_version()


def dsa_status_string(s: int) -> str:
    return lib().dsa_status_string(s).decode()


def dsa_choose_splits(Q: int, topk: int, num_splits: int = 0) -> int:
    return lib().dsa_choose_splits(Q, topk, num_splits)


def dsa_mla_group_plan(units: int, topk: int):
    """(head_units, tail_units, tail_splits) of an IndexShare group's grouped
    attention, or None for invalid sizes."""
    h, t, ts = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    if not lib().dsa_mla_group_plan(units, topk, ctypes.byref(h), ctypes.byref(t), ctypes.byref(ts)):
        return None
    return h.value, t.value, ts.value


def dsa_workspace_bytes(Q: int, max_len: int, topk: int, num_splits: int = 0) -> int:
    return lib().dsa_workspace_bytes(Q, max_len, topk, num_splits)


def workspace(Q: int, max_len: int, topk: int, num_splits: int = 0, device="cuda") -> torch.Tensor:
    """A zeroed device workspace of dsa_workspace_bytes(...) bytes."""
    n = dsa_workspace_bytes(Q, max_len, topk, num_splits)
    if n == 0:
        raise DSAError(1, "dsa_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def dsa_indexer_scores(q_idx, w, k_idx, seq_offsets, q_offsets, q_vis, B, max_len, scores, ws,
                       first_only=False, stream=None):
    _check(lib().dsa_indexer_scores(
        _ptr(q_idx), _ptr(w), _ptr(k_idx), k_idx.shape[0], _ptr(seq_offsets), _ptr(q_offsets),
        _ptr(q_vis), B, q_idx.shape[0], q_idx.shape[1], max_len, int(first_only), _ptr(scores),
        scores.shape[1], _ptr(ws), ws.numel(), _stream(stream)), "dsa_indexer_scores")


def dsa_topk_select(scores, q_offsets, q_vis, B, max_len, topk, out_idx, ws, out_scores=None,
                    first_only=False, stream=None):
    _check(lib().dsa_topk_select(
        _ptr(scores), scores.shape[1], _ptr(q_offsets), _ptr(q_vis), B, scores.shape[0], max_len,
        topk, int(first_only), _ptr(out_idx), _ptr(out_scores), _ptr(ws), ws.numel(),
        _stream(stream)), "dsa_topk_select")


def dsa_indexer_topk(q_idx, w, k_idx, seq_offsets, q_offsets, q_vis, B, max_len, topk, out_idx,
                     ws, out_scores=None, first_only=False, stream=None):
    _check(lib().dsa_indexer_topk(
        _ptr(q_idx), _ptr(w), _ptr(k_idx), k_idx.shape[0], _ptr(seq_offsets), _ptr(q_offsets),
        _ptr(q_vis), B, q_idx.shape[0], q_idx.shape[1], max_len, topk, int(first_only),
        _ptr(out_idx), _ptr(out_scores), _ptr(ws), ws.numel(), _stream(stream)), "dsa_indexer_topk")


def dsa_indexer_topk_fused(q_idx, w, k_idx, seq_offsets, q_offsets, q_vis, B, max_len, topk,
                           out_idx, ws, out_scores=None, first_only=False, stream=None):
    _check(lib().dsa_indexer_topk_fused(
        _ptr(q_idx), _ptr(w), _ptr(k_idx), k_idx.shape[0], _ptr(seq_offsets), _ptr(q_offsets),
        _ptr(q_vis), B, q_idx.shape[0], q_idx.shape[1], max_len, topk, int(first_only),
        _ptr(out_idx), _ptr(out_scores), _ptr(ws), ws.numel(), _stream(stream)),
        "dsa_indexer_topk_fused")


def dsa_sparse_mla_decode(q, kv_pool, page_table, q_offsets, q_vis, idx, B, scale, out, lse, ws,
                          num_splits=0, stream=None):
    _check(lib().dsa_sparse_mla_decode(
        _ptr(q), _ptr(kv_pool), kv_pool.shape[0], kv_pool.shape[1], _ptr(page_table),
        page_table.shape[1],
        _ptr(q_offsets), _ptr(q_vis), _ptr(idx), B, q.shape[0], q.shape[1], idx.shape[1],
        float(scale), num_splits, _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)),
        "dsa_sparse_mla_decode")


def dsa_sparse_mla_decode_noalloc(q, kv_pool, page_table, q_offsets, q_vis, idx, B, scale, out,
                                  lse, num_splits=0, stream=None):
    """dsa_sparse_mla_decode without a workspace (split-K partials in the
    library's own fixed device array; see include/dsa.h)."""
    _check(lib().dsa_sparse_mla_decode_noalloc(
        _ptr(q), _ptr(kv_pool), kv_pool.shape[0], kv_pool.shape[1], _ptr(page_table),
        page_table.shape[1],
        _ptr(q_offsets), _ptr(q_vis), _ptr(idx), B, q.shape[0], q.shape[1], idx.shape[1],
        float(scale), num_splits, _ptr(out), _ptr(lse), _stream(stream)),
        "dsa_sparse_mla_decode_noalloc")


def dsa_sparse_mla_decode_window(q, kv_pool, page_table, win_page_table, q_offsets, q_vis,
                                 win_vis, idx, B, window, scale, out, lse, ws, num_splits=0,
                                 stream=None):
    """Sparse MLA over the selected compressed entries plus a sliding window of
    raw tokens (DeepSeek-V4 CSA); see include/dsa.h."""
    _check(lib().dsa_sparse_mla_decode_window(
        _ptr(q), _ptr(kv_pool), kv_pool.shape[0], kv_pool.shape[1], _ptr(page_table),
        page_table.shape[1], _ptr(win_page_table), win_page_table.shape[1], _ptr(q_offsets),
        _ptr(q_vis), _ptr(win_vis), _ptr(idx), B, q.shape[0], q.shape[1], idx.shape[1], window,
        float(scale), num_splits, _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)),
        "dsa_sparse_mla_decode_window")


def dsa_sparse_mla_decode_fp8(q, kv_pool, kv_scale, page_table, q_offsets, q_vis, idx, B, scale,
                              out, lse, ws, num_splits=0, stream=None):
    """Sparse MLA over an e4m3 latent cache (uint8 [pages,page_size,576]) with one
    per-tensor scale; see include/dsa.h."""
    _check(lib().dsa_sparse_mla_decode_fp8(
        _ptr(q), _ptr(kv_pool), float(kv_scale), kv_pool.shape[0], kv_pool.shape[1],
        _ptr(page_table), page_table.shape[1], _ptr(q_offsets), _ptr(q_vis), _ptr(idx), B,
        q.shape[0], q.shape[1], idx.shape[1], float(scale), num_splits, _ptr(out), _ptr(lse),
        _ptr(ws), ws.numel(), _stream(stream)), "dsa_sparse_mla_decode_fp8")


def dsa_lse_combine(o_parts, lse_parts, out, lse, stream=None):
    Q, S, H = lse_parts.shape[0], lse_parts.shape[1], lse_parts.shape[2]
    _check(lib().dsa_lse_combine(_ptr(o_parts), _ptr(lse_parts), Q, S, H, _ptr(out), _ptr(lse),
                                 _stream(stream)), "dsa_lse_combine")


def dsa_decode_step(q_idx_layers, w_layers, k_idx_layers, seq_offsets, q_offsets, q_vis, B,
                    max_len, topk, q_layers, pool_layers, page_table_layers, scale, out_layers,
                    lse_layers, idx_out, ws, index_share=1, mtp_index_share=False, num_splits=0,
                    stream=None):
    """Per-layer lists; entries of the indexer lists for non-indexer layers may be None."""
    n = len(q_layers)
    lead = next(t for t in k_idx_layers if t is not None)
    lead_q = next(t for t in q_idx_layers if t is not None)
    _check(lib().dsa_decode_step(
        n, index_share, int(mtp_index_share), _ptr_array(q_idx_layers), _ptr_array(w_layers),
        _ptr_array(k_idx_layers), lead.shape[0], _ptr(seq_offsets), _ptr(q_offsets), _ptr(q_vis),
        B, q_layers[0].shape[0], q_layers[0].shape[1], lead_q.shape[1], max_len, topk,
        _ptr_array(q_layers), _ptr_array(pool_layers),
        pool_layers[0].shape[0], pool_layers[0].shape[1], _ptr_array(page_table_layers),
        page_table_layers[0].shape[1],
        float(scale), num_splits, _ptr_array(out_layers), _ptr_array(lse_layers), _ptr(idx_out),
        _ptr(ws), ws.numel(), _stream(stream)), "dsa_decode_step")


def dsa_tier_state_bytes(B: int, dev_slots: int, max_pages: int) -> int:
    return lib().dsa_tier_state_bytes(B, dev_slots, max_pages)


def tier_state(B: int, dev_slots: int, max_pages: int) -> torch.Tensor:
    """Host memory for a two-tier cache's state, initialised (every slot empty)."""
    n = dsa_tier_state_bytes(B, dev_slots, max_pages)
    if n == 0:
        raise DSAError(1, "dsa_tier_state_bytes")
    st = torch.empty((n + 7) // 8, dtype=torch.int64)      # 8-byte aligned host bytes
    dsa_tier_init(st, B, dev_slots, max_pages)
    return st


def dsa_tier_init(state: torch.Tensor, B: int, dev_slots: int, max_pages: int):
    _check(lib().dsa_tier_init(_host_ptr(state), state.numel() * state.element_size(), B,
                               dev_slots, max_pages), "dsa_tier_init")


def dsa_tier_plan(state, idx, q_offsets, copies, page_table=None):
    """Host tensors: idx int32 [Q,topk], q_offsets int32 [B+1], copies int32
    [cap,3] (out), page_table None or int32 [B,max_pages] (out).  Returns
    (n_copies, (hits, misses, evictions))."""
    n = ctypes.c_int(0)
    stats = (ctypes.c_int64 * 3)()
    _check(lib().dsa_tier_plan(_host_ptr(state), _host_ptr(idx), idx.shape[0], idx.shape[1],
                               _host_ptr(q_offsets),
                               None if page_table is None else _host_ptr(page_table),
                               _host_ptr(copies), copies.shape[0], ctypes.byref(n), stats),
           "dsa_tier_plan")
    return n.value, (stats[0], stats[1], stats[2])


def dsa_tier_fetch(host_cache, dev_pool, copies, n, ws, page_table=None, stream=None):
    """host_cache: pinned host tensor [host_pages,16,576] bf16; dev_pool: device
    tensor [dev_pages,16,576] bf16; copies: device int32 [>=n,3]; page_table:
    None or the device int32 [B,max_pages] table to patch."""
    if not host_cache.is_pinned():
        raise ValueError("host_cache must be pinned host memory")
    _check(lib().dsa_tier_fetch(_host_ptr(host_cache), host_cache.shape[0], _ptr(dev_pool),
                                dev_pool.shape[0], _ptr(copies), n, _ptr(page_table), _ptr(ws),
                                _stream(stream)), "dsa_tier_fetch")


def tier_dev_state(B: int, dev_slots: int, max_pages: int, page_table, stream=None) -> torch.Tensor:
    """Device memory for the on-device planner's state, initialised; page_table
    (device int32 [B,max_pages]) is set to all -1."""
    n = lib().dsa_tier_dev_state_bytes(B, dev_slots, max_pages)
    if n == 0:
        raise DSAError(2, "dsa_tier_dev_state_bytes")
    st = torch.empty(n, dtype=torch.uint8, device=page_table.device)
    _check(lib().dsa_tier_dev_init(_ptr(st), n, B, dev_slots, max_pages, _ptr(page_table),
                                   _stream(stream)), "dsa_tier_dev_init")
    return st


def dsa_tier_swap_in(dev_state, B, dev_slots, max_pages, idx, q_offsets, page_table, host_cache,
                     dev_pool, ws, stream=None):
    """Plan on the device and fetch: idx device int32 [Q,topk], q_offsets device
    int32 [B+1], page_table device int32 [B,max_pages] (updated), host_cache
    pinned host bf16 [B*max_pages,16,576], dev_pool device bf16 [B*dev_slots,16,576]."""
    if not host_cache.is_pinned():
        raise ValueError("host_cache must be pinned host memory")
    _check(lib().dsa_tier_swap_in(_ptr(dev_state), dev_state.numel(), B, dev_slots, max_pages,
                                  _ptr(idx), idx.shape[0], idx.shape[1], _ptr(q_offsets),
                                  _ptr(page_table), _host_ptr(host_cache), _ptr(dev_pool), _ptr(ws),
                                  _stream(stream)), "dsa_tier_swap_in")


def dsa_tier_dev_stats(dev_state, stream=None):
    """(n_copies, hits, misses, evictions) of the last device step, and the step count."""
    out = (ctypes.c_int64 * 5)()
    _check(lib().dsa_tier_dev_stats(_ptr(dev_state), out, _stream(stream)), "dsa_tier_dev_stats")
    return tuple(out[:4]), out[4]


def dsa_tier_dev_copies(dev_state, B, dev_slots, max_pages, n):
    """The device planner's copy list (int32 [n,3]) as a tensor view of dev_state."""
    p = lib().dsa_tier_dev_copies(_ptr(dev_state), B, dev_slots, max_pages)
    off = p - dev_state.data_ptr()
    return dev_state[off:off + 12 * n].view(torch.int32).view(n, 3)


def dsa_check_error(ws, stream=None):
    _check(lib().dsa_check_error(_ptr(ws), _stream(stream)), "dsa_check_error")


def dsa_selftest_bounded_wait(limit_us, ws, stream=None):
    """Makes the library's bounded device-side waits run out (see include/dsa.h)."""
    _check(lib().dsa_selftest_bounded_wait(int(limit_us), _ptr(ws), ws.numel(), _stream(stream)),
           "dsa_selftest_bounded_wait")


def dsa_noalloc_check_error(stream=None):
    """Reads and clears dsa_sparse_mla_decode_noalloc's error word (synchronises)."""
    _check(lib().dsa_noalloc_check_error(_stream(stream)), "dsa_noalloc_check_error")
