"""Sparse MLA over an FP8 (e4m3) latent cache with one per-tensor scale (the
deploy page's fp8_e4m3 KV cache, "GLM-5.2 推理部署").  Parity with the oracle,
which decodes the codes exactly and multiplies by the scale; and, with scale
1, bitwise equality with the bf16 call on the exactly widened cache.  Over an
FP8 cache the kernel widens the latent dims on chip to fp16 (exact) and takes
the query's latent dims as fp16, which is exact for every bf16 element that is
zero or an fp16 normal; the equality case uses such queries.  A query element
beyond fp16's range is flagged as out of range."""
import numpy as np
import pytest
import torch

import oracle as O
import sparse_attention_decode_lightning_b200 as dsa
from synth import get_workload, make_inputs
from tests._helpers import np_bits
from tests._parity import check_attention

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _fp8_case(name, seed, heads):
    inp = make_inputs(get_workload(name, B=3, L=1500), seed=seed, device=DEV)
    pool = inp.layers[0]["pool"]
    codes = (pool.float() * 2).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    g = torch.Generator().manual_seed(seed)
    idx = torch.full((inp.Q, 2048), -1, dtype=torch.int32)
    for q in range(inp.Q):
        n = [1500, 600, 1][q]
        idx[q, :n] = torch.randperm(1500, generator=g)[:n].to(torch.int32)
    return inp, codes.contiguous(), idx.to(DEV)


@pytest.mark.parametrize("name,S,kv_scale", [("decode_b32_ctx128k", 1, 1.0), ("decode_b32_ctx128k", 3, 0.37),
                                             ("glm52_decode_b32_ctx128k", 1, 0.37),
                                             ("glm52_decode_b32_ctx128k", 16, 2.5)])
def test_fp8_cache_matches_oracle(name, S, kv_scale):
    inp, codes, idx = _fp8_case(name, 5, None)
    H = inp.heads
    out = torch.empty(inp.Q, H, 512, device=DEV)
    lse = torch.empty(inp.Q, H, device=DEV)
    ws = dsa.workspace(inp.Q, 1, 2048, S)
    dsa.dsa_sparse_mla_decode_fp8(inp.layers[0]["q"], codes, kv_scale, inp.page_table, inp.q_offsets,
                                  inp.q_vis, idx, inp.B, inp.scale, out, lse, ws, num_splits=S)
    dsa.dsa_check_error(ws)
    cb, pt, qb, ix = codes.cpu().numpy(), np_bits(inp.page_table), np_bits(inp.layers[0]["q"]), idx.cpu().numpy()
    for q in range(inp.Q):
        sel = ix[q][ix[q] >= 0]
        rows = O.latent_rows_e4m3(cb, pt[q], sel, kv_scale)
        o_ref, l_ref = O.sparse_mla(O.bf16_decode(qb[q]), rows, inp.scale)
        check_attention(out[q].cpu().numpy(), lse[q].cpu().numpy(), o_ref, l_ref)


@pytest.mark.parametrize("name", ["decode_b32_ctx128k", "glm52_decode_b32_ctx128k"])
def test_fp8_cache_equals_bf16_call_on_widened_cache(name):
    inp, codes, idx = _fp8_case(name, 9, None)
    widened = codes.view(torch.float8_e4m3fn).to(torch.bfloat16).contiguous()
    q = inp.layers[0]["q"].clone()
    q[q.abs() < 2.0 ** -14] = 0               # fp16 subnormals would be rounded
    assert (q != 0).float().mean() > 0.99
    res = []
    for fp8 in (True, False):
        out = torch.empty(inp.Q, inp.heads, 512, device=DEV)
        lse = torch.empty(inp.Q, inp.heads, device=DEV)
        ws = dsa.workspace(inp.Q, 1, 2048, 2)
        if fp8:
            dsa.dsa_sparse_mla_decode_fp8(q, codes, 1.0, inp.page_table, inp.q_offsets,
                                          inp.q_vis, idx, inp.B, inp.scale, out, lse, ws, num_splits=2)
        else:
            dsa.dsa_sparse_mla_decode(q, widened, inp.page_table, inp.q_offsets,
                                      inp.q_vis, idx, inp.B, inp.scale, out, lse, ws, num_splits=2)
        dsa.dsa_check_error(ws)
        res.append((out, lse))
    assert torch.equal(res[0][0], res[1][0]) and torch.equal(res[0][1], res[1][1])


@pytest.mark.parametrize("name", ["decode_b32_ctx128k", "glm52_decode_b32_ctx128k"])
def test_fp8_cache_flags_query_beyond_f16_range(name):
    inp, codes, idx = _fp8_case(name, 11, None)
    q = inp.layers[0]["q"].clone()
    ws = dsa.workspace(inp.Q, 1, 2048, 1)
    out = torch.empty(inp.Q, inp.heads, 512, device=DEV)
    lse = torch.empty(inp.Q, inp.heads, device=DEV)
    q[1, 3, 100] = 65280.0                    # fp16 holds it: no flag
    dsa.dsa_sparse_mla_decode_fp8(q, codes, 1.0, inp.page_table, inp.q_offsets, inp.q_vis, idx,
                                  inp.B, inp.scale, out, lse, ws, num_splits=1)
    dsa.dsa_check_error(ws)
    q[1, 3, 300] = -65536.0                   # the next bf16 value: beyond fp16
    dsa.dsa_sparse_mla_decode_fp8(q, codes, 1.0, inp.page_table, inp.q_offsets, inp.q_vis, idx,
                                  inp.B, inp.scale, out, lse, ws, num_splits=1)
    with pytest.raises(dsa.DSAError) as e:
        dsa.dsa_check_error(ws)
    assert e.value.status == 4
    dsa.dsa_check_error(ws)                   # the flag was cleared
