"""Full-size parity at every workload's own sizes and launch configuration
(the one bench.py times): properties that hold at any size are checked for
every query on the device; sampled queries are checked against the oracle one
by one (top-k under the swap rule, attention on the GPU's indices)."""
import numpy as np
import pytest
import torch

import oracle as O
import sparse_attention_decode_lightning_b200 as dsa
from synth import get_workload, make_inputs
from tests._helpers import np_bits
from tests._parity import check_attention, check_topk_row
from tests._gpu import run_decode_step

pytestmark = pytest.mark.gpu
DEV = "cuda"

FULL = ["decode_b32_ctx128k", "indexshare4_b64_ctx16k_128k", "mtp_verify_b16_t8_ctx128k",
        "mtp_verify_reuse_b16_t8_ctx128k", "decode_b4_ctx1m_split16", "glm52_decode_b32_ctx128k",
        "glm52_indexshare4_b64_ctx16k_128k", "glm52_decode_b4_ctx1m_split16"]


def _check_index_properties(idx: torch.Tensor, vis: torch.Tensor, topk: int):
    """Every row: min(topk, vis) distinct visible positions, then -1 padding."""
    n = torch.clamp(vis.long(), max=topk)
    valid = idx >= 0
    assert torch.equal(valid.sum(1), n)
    ar = torch.arange(topk, device=idx.device)[None]
    # the library writes the selected positions first, padding last
    assert torch.equal(valid, ar < n[:, None])
    assert bool((idx < vis[:, None]).all())
    s, _ = torch.sort(torch.where(valid, idx, torch.full_like(idx, -2)), dim=1)
    dup = (s[:, 1:] == s[:, :-1]) & (s[:, 1:] >= 0)
    assert not bool(dup.any())


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled_against_oracle(name):
    w = get_workload(name)
    inp = make_inputs(w, seed=0, device=DEV)
    outs, lses, idx = run_decode_step(inp)
    T, G = inp.T, inp.index_share
    for g in range(idx.shape[0]):
        _check_index_properties(idx[g], inp.q_vis, inp.topk)
    for l in range(inp.n_layers):
        assert bool(torch.isfinite(outs[l]).all()) and bool(torch.isfinite(lses[l]).all())
    so = inp.seq_offsets.cpu().numpy()
    vis = inp.q_vis.cpu().numpy()
    samples = sorted({0, inp.Q - 1, inp.Q // 2 + (1 if T > 1 else 0)})
    for q in samples:
        b = q // T
        src = b * T if inp.mtp_index_share else q
        ind = inp.indexer[0]
        keys = np_bits(ind["k_idx"][int(so[b]):int(so[b]) + int(vis[src])])
        sc = O.indexer_scores(np_bits(ind["q_idx"][src]), np_bits(ind["w"][src]), keys)
        check_topk_row(idx[0, q].cpu().numpy(), sc, inp.topk)
        ix = idx[0, q]
        sel = ix[ix >= 0].long()
        for l in range(inp.n_layers):
            pt = inp.page_table[b].long()
            rows = inp.layers[l]["pool"][pt[sel // 64], sel % 64]          # [n,576] bf16
            rows = O.bf16_decode(np_bits(rows))
            qf = O.bf16_decode(np_bits(inp.layers[l]["q"][q]))
            o_ref, l_ref = O.sparse_mla(qf, rows, inp.scale)
            check_attention(outs[l][q].cpu().numpy(), lses[l][q].cpu().numpy(), o_ref, l_ref)
    del inp, outs, lses, idx
    torch.cuda.empty_cache()
