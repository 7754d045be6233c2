"""The allocation-free sparse MLA entry point (for callers that cannot give
the library device memory: their allocator owns all of HBM, or they may not
call cudaMalloc because it synchronises the device) must match the regular
entry point and the oracle, refuse exactly the requests its fixed array cannot
hold, and report range violations through its own error word.  Collected last
so that a run stopping at the first failure has already run every other test;
it also passes alone in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

import sparse_attention_decode_lightning_b200 as dsa
from synth import get_workload, make_inputs
from tests._helpers import np_bits
from tests._parity import check_attention, oracle_attention_for_idx

pytestmark = pytest.mark.gpu
DEV = "cuda"
DSA_OK, DSA_ERR_UNSUPPORTED, DSA_ERR_DEVICE_BOUNDS = 0, 2, 4


def _call_noalloc(inp, layer, idx, out, lse, num_splits, page_table=None):
    L = dsa.lib()
    pt = inp.page_table if page_table is None else page_table
    return L.dsa_sparse_mla_decode_noalloc(
        ctypes.c_void_p(inp.layers[layer]["q"].data_ptr()),
        ctypes.c_void_p(inp.layers[layer]["pool"].data_ptr()), inp.num_pages, 64,
        ctypes.c_void_p(pt.data_ptr()), inp.max_pages,
        ctypes.c_void_p(inp.q_offsets.data_ptr()), ctypes.c_void_p(inp.q_vis.data_ptr()),
        ctypes.c_void_p(idx.data_ptr()), inp.B, inp.Q, inp.layers[layer]["q"].shape[1], idx.shape[1],
        ctypes.c_float(inp.scale),
        num_splits, ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _check_word():
    return dsa.lib().dsa_noalloc_check_error(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _random_idx(inp, seed, short=37):
    """Distinct visible positions per query, some rows padded with -1."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    vis = inp.q_vis.cpu()
    idx = torch.full((inp.Q, 2048), -1, dtype=torch.int32)
    for q in range(inp.Q):
        n = max(1, min(int(vis[q]), 2048 - short * q))
        idx[q, :n] = torch.randperm(int(vis[q]), generator=g)[:n].to(torch.int32)
    return idx.to(DEV)


def _reference(inp, layer, idx, num_splits):
    heads = inp.layers[layer]["q"].shape[1]
    out = torch.empty(inp.Q, heads, 512, device=DEV)
    lse = torch.empty(inp.Q, heads, device=DEV)
    ws = dsa.workspace(inp.Q, 1, 2048, num_splits)
    dsa.dsa_sparse_mla_decode(inp.layers[layer]["q"], inp.layers[layer]["pool"], inp.page_table,
                              inp.q_offsets, inp.q_vis, idx, inp.B, inp.scale, out, lse, ws,
                              num_splits=num_splits)
    dsa.dsa_check_error(ws)
    return out, lse


def _noalloc(inp, layer, idx, num_splits):
    heads = inp.layers[layer]["q"].shape[1]
    out = torch.full((inp.Q, heads, 512), float("nan"), device=DEV)
    lse = torch.full((inp.Q, heads), float("nan"), device=DEV)
    st = _call_noalloc(inp, layer, idx, out, lse, num_splits)
    assert st == DSA_OK, dsa.dsa_status_string(st)
    assert _check_word() == DSA_OK
    return out, lse


@pytest.mark.parametrize("num_splits", [0, 1, 4])
def test_noalloc_matches_workspace_entry_point_twice(num_splits):
    inp = make_inputs(get_workload("indexshare4_b64_ctx16k_128k", B=3, L_range=(3000, 9000)),
                      seed=21, device=DEV)
    for call in range(2):                       # two calls in a row share the static array
        layer = call
        idx = _random_idx(inp, 3 + call)
        out_ref, lse_ref = _reference(inp, layer, idx, num_splits)
        out, lse = _noalloc(inp, layer, idx, num_splits)
        torch.cuda.synchronize()
        for q in range(inp.Q):
            check_attention(out[q].cpu().numpy().astype(np.float64), lse[q].cpu().numpy().astype(np.float64),
                            out_ref[q].cpu().numpy().astype(np.float64),
                            lse_ref[q].cpu().numpy().astype(np.float64))


@pytest.mark.parametrize("name,num_splits", [("indexshare4_b64_ctx16k_128k", 1),
                                             ("indexshare4_b64_ctx16k_128k", 3),
                                             ("glm52_indexshare4_b64_ctx16k_128k", 1),
                                             ("glm52_indexshare4_b64_ctx16k_128k", 4)])
def test_noalloc_matches_oracle(name, num_splits):
    """128 heads (DeepSeek-V3.2) and 64 (GLM-5.2), one split and several."""
    inp = make_inputs(get_workload(name, B=2, L_range=(2500, 7000)), seed=33, device=DEV)
    idx = _random_idx(inp, 9, short=300)
    out, lse = _noalloc(inp, 0, idx, num_splits)
    torch.cuda.synchronize()
    pool, pt, qb = np_bits(inp.layers[0]["pool"]), np_bits(inp.page_table), np_bits(inp.layers[0]["q"])
    for q in range(inp.Q):
        ix = idx[q].cpu().numpy()
        o_ref, l_ref = oracle_attention_for_idx(pool, pt[q], qb[q], ix, inp.scale)
        check_attention(out[q].cpu().numpy().astype(np.float64), lse[q].cpu().numpy().astype(np.float64),
                        o_ref, l_ref)


# The fixed array (16 MiB less the 256-byte error word) holds Q x splits
# partials of heads x (512 + 1) floats: 63 at 128 heads, 127 at 64 heads.
@pytest.mark.parametrize("name,heads,Q,S,ok", [("decode_b32_ctx128k", 128, 21, 3, True),
                                               ("decode_b32_ctx128k", 128, 32, 2, False),
                                               ("glm52_decode_b32_ctx128k", 64, 63, 2, True),
                                               ("glm52_decode_b32_ctx128k", 64, 64, 2, False)])
def test_noalloc_limit_at_its_exact_edge(name, heads, Q, S, ok):
    inp = make_inputs(get_workload(name, B=Q, L=300), seed=5, device=DEV)
    assert inp.layers[0]["q"].shape[1] == heads
    idx = _random_idx(inp, 11, short=0)
    out = torch.full((inp.Q, heads, 512), float("nan"), device=DEV)
    lse = torch.full((inp.Q, heads), float("nan"), device=DEV)
    st = _call_noalloc(inp, 0, idx, out, lse, S)
    if not ok:
        assert st == DSA_ERR_UNSUPPORTED
        assert bool(torch.isnan(out).all())          # nothing was enqueued
        return
    assert st == DSA_OK
    assert _check_word() == DSA_OK
    out_ref, lse_ref = _reference(inp, 0, idx, S)
    torch.cuda.synchronize()
    for q in range(0, inp.Q, 7):
        check_attention(out[q].cpu().numpy().astype(np.float64), lse[q].cpu().numpy().astype(np.float64),
                        out_ref[q].cpu().numpy().astype(np.float64),
                        lse_ref[q].cpu().numpy().astype(np.float64))


def test_noalloc_reports_out_of_range_pages_through_its_error_word():
    """A page id beyond the pool (planted on the host) is skipped and reported
    by dsa_noalloc_check_error, which then clears the word."""
    inp = make_inputs(get_workload("decode_b32_ctx128k", B=2, L=3000), seed=8, device=DEV)
    idx = _random_idx(inp, 13, short=0)
    bad = inp.page_table.clone()
    bad[1, 5] = inp.num_pages + 7              # tokens 320..383 of sequence 1
    out = torch.empty(inp.Q, 128, 512, device=DEV)
    lse = torch.empty(inp.Q, 128, device=DEV)
    assert _call_noalloc(inp, 0, idx, out, lse, 2, page_table=bad) == DSA_OK
    assert _check_word() == DSA_ERR_DEVICE_BOUNDS
    assert _check_word() == DSA_OK             # read and cleared
    assert bool(torch.isfinite(out).all())
    _noalloc(inp, 0, idx, 2)                   # a clean call leaves the word clear
