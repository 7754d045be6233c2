"""The allocation-free sparse MLA entry point (for callers that cannot give
the library device memory: their allocator owns all of HBM, or they may not
call cudaMalloc because it synchronises the device) must match the regular
entry point.  Collected last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

import sparse_attention_decode_lightning_b200 as dsa
from synth import get_workload, make_inputs
from tests._parity import check_attention

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _call_noalloc(inp, layer, idx, out, lse, num_splits):
    L = dsa.lib()
    st = L.dsa_sparse_mla_decode_noalloc(
        ctypes.c_void_p(inp.layers[layer]["q"].data_ptr()),
        ctypes.c_void_p(inp.layers[layer]["pool"].data_ptr()), inp.num_pages, 64,
        ctypes.c_void_p(inp.page_table.data_ptr()), inp.max_pages,
        ctypes.c_void_p(inp.q_offsets.data_ptr()), ctypes.c_void_p(inp.q_vis.data_ptr()),
        ctypes.c_void_p(idx.data_ptr()), inp.B, inp.Q, inp.layers[layer]["q"].shape[1], idx.shape[1],
        ctypes.c_float(inp.scale),
        num_splits, ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, dsa.dsa_status_string(st)


@pytest.mark.parametrize("num_splits", [0, 1, 4])
def test_noalloc_matches_workspace_entry_point_twice(num_splits):
    inp = make_inputs(get_workload("indexshare4_b64_ctx16k_128k", B=3, L_range=(3000, 9000)),
                      seed=21, device=DEV)
    g = torch.Generator(device="cpu").manual_seed(3)
    vis = inp.q_vis.cpu()
    for call in range(2):                       # two calls in a row share the static array
        layer = call
        idx = torch.full((inp.Q, 2048), -1, dtype=torch.int32)
        for q in range(inp.Q):
            n = min(int(vis[q]), 2048 - 37 * q)
            idx[q, :n] = torch.randperm(int(vis[q]), generator=g)[:n].to(torch.int32)
        idx = idx.to(DEV)
        out_ref = torch.empty(inp.Q, 128, 512, device=DEV)
        lse_ref = torch.empty(inp.Q, 128, device=DEV)
        ws = dsa.workspace(inp.Q, 1, 2048, num_splits)
        dsa.dsa_sparse_mla_decode(inp.layers[layer]["q"], inp.layers[layer]["pool"], inp.page_table,
                                  inp.q_offsets, inp.q_vis, idx, inp.B, inp.scale, out_ref, lse_ref,
                                  ws, num_splits=num_splits)
        dsa.dsa_check_error(ws)
        out = torch.full((inp.Q, 128, 512), float("nan"), device=DEV)
        lse = torch.full((inp.Q, 128), float("nan"), device=DEV)
        _call_noalloc(inp, layer, idx, out, lse, num_splits)
        torch.cuda.synchronize()
        for q in range(inp.Q):
            check_attention(out[q].cpu().numpy().astype(np.float64), lse[q].cpu().numpy().astype(np.float64),
                            out_ref[q].cpu().numpy().astype(np.float64),
                            lse_ref[q].cpu().numpy().astype(np.float64))


def test_noalloc_rejects_requests_beyond_its_array():
    inp = make_inputs(get_workload("decode_b32_ctx128k", B=32, L=300), seed=5, device=DEV)
    idx = torch.zeros(inp.Q, 2048, dtype=torch.int32, device=DEV)
    out = torch.empty(inp.Q, 128, 512, device=DEV)
    lse = torch.empty(inp.Q, 128, device=DEV)
    L = dsa.lib()
    st = L.dsa_sparse_mla_decode_noalloc(
        ctypes.c_void_p(inp.layers[0]["q"].data_ptr()), ctypes.c_void_p(inp.layers[0]["pool"].data_ptr()),
        inp.num_pages, 64, ctypes.c_void_p(inp.page_table.data_ptr()), inp.max_pages,
        ctypes.c_void_p(inp.q_offsets.data_ptr()), ctypes.c_void_p(inp.q_vis.data_ptr()),
        ctypes.c_void_p(idx.data_ptr()), inp.B, inp.Q, 128, 2048, ctypes.c_float(inp.scale), 2,
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()), None)
    assert st == 2          # 32 queries x 2 splits > 63 partials: DSA_ERR_UNSUPPORTED
