"""Sparse MLA with a sliding window: DeepSeek-V4's CSA ("大语言模型结构总览",
section 2.3: KV compressed 4x along the sequence, top-1024 / top-512
compressed entries chosen by DSA, plus a 128-token window of raw tokens).
Both caches live in one paged pool under two page tables; the oracle attends,
in one softmax, to the selected compressed rows followed by the window rows."""
import math

import numpy as np
import pytest
import torch

import oracle as O
import sparse_attention_decode_lightning_b200 as dsa
from tests._helpers import np_bits
from tests._parity import check_attention

pytestmark = pytest.mark.gpu
DEV = "cuda"
PG = 64


def _case(seed, B, L_raw, heads=128, ratio=4):
    """Compressed cache (L_raw / ratio entries) and raw cache in one permuted pool."""
    g = torch.Generator().manual_seed(seed)
    Lc = [l // ratio for l in L_raw]
    pc = [(n + PG - 1) // PG for n in Lc]
    pr = [(n + PG - 1) // PG for n in L_raw]
    total = sum(pc) + sum(pr)
    perm = torch.randperm(total, generator=g)
    ct = torch.full((B, max(pc)), -1, dtype=torch.int32)
    rt = torch.full((B, max(pr)), -1, dtype=torch.int32)
    k = 0
    for b in range(B):
        ct[b, :pc[b]] = perm[k:k + pc[b]]
        k += pc[b]
        rt[b, :pr[b]] = perm[k:k + pr[b]]
        k += pr[b]
    pool = torch.randn(total, PG, 576, generator=g).to(torch.bfloat16)
    q = torch.randn(B, heads, 576, generator=g).to(torch.bfloat16)
    return Lc, pool, ct, rt, q


def _oracle(pool_b, ct_b, rt_b, q_b, sel, wv, window, scale):
    # the window rule (the last `window` raw tokens, none below 0) is the
    # oracle's own, pinned in test_oracle_pins.py
    return O.csa_window_attention(O.bf16_decode(q_b), pool_b, ct_b, rt_b, sel, wv, window, scale)


@pytest.mark.parametrize("topk,window,S,heads", [(512, 128, 1, 128), (1024, 128, 4, 128),
                                                 (512, 128, 3, 64), (300, 200, 2, 128)])
def test_window_attention_matches_oracle(topk, window, S, heads):
    B = 3
    L_raw = [6000, 4100, 90]                  # the last sequence is shorter than the window
    Lc, pool, ct, rt, q = _case(7 + topk, B, L_raw, heads)
    rng = np.random.default_rng(topk)
    idx = np.full((B, topk), -1, dtype=np.int32)
    for b in range(B):
        n = min(topk, Lc[b])
        idx[b, :n] = rng.choice(Lc[b], n, replace=False)
    scale = 1 / math.sqrt(192)
    out = torch.empty(B, heads, 512, device=DEV)
    lse = torch.empty(B, heads, device=DEV)
    ws = dsa.workspace(B, 1, topk + window, S)
    qo = torch.arange(B + 1, dtype=torch.int32, device=DEV)
    dsa.dsa_sparse_mla_decode_window(q.to(DEV), pool.to(DEV), ct.to(DEV), rt.to(DEV), qo,
                                     torch.tensor(Lc, dtype=torch.int32, device=DEV),
                                     torch.tensor(L_raw, dtype=torch.int32, device=DEV),
                                     torch.from_numpy(idx).to(DEV), B, window, scale, out, lse, ws,
                                     num_splits=S)
    dsa.dsa_check_error(ws)
    pb, qb = np_bits(pool), np_bits(q)
    for b in range(B):
        sel = idx[b][idx[b] >= 0]
        o_ref, l_ref = _oracle(pb, ct[b].numpy(), rt[b].numpy(), qb[b], sel, L_raw[b], window, scale)
        check_attention(out[b].cpu().numpy(), lse[b].cpu().numpy(), o_ref, l_ref)


def test_window_zero_is_the_plain_call():
    B = 2
    Lc, pool, ct, rt, q = _case(3, B, [3000, 2400])
    rng = np.random.default_rng(1)
    idx = torch.from_numpy(np.stack([rng.choice(Lc[b], 512, replace=False) for b in range(B)])
                           .astype(np.int32)).to(DEV)
    qo = torch.arange(B + 1, dtype=torch.int32, device=DEV)
    vis = torch.tensor(Lc, dtype=torch.int32, device=DEV)
    outs = []
    for window in (0, None):
        out = torch.empty(B, 128, 512, device=DEV)
        lse = torch.empty(B, 128, device=DEV)
        ws = dsa.workspace(B, 1, 512, 2)
        if window is None:
            dsa.dsa_sparse_mla_decode(q.to(DEV), pool.to(DEV), ct.to(DEV), qo, vis, idx, B, 0.07,
                                      out, lse, ws, num_splits=2)
        else:
            dsa.dsa_sparse_mla_decode_window(q.to(DEV), pool.to(DEV), ct.to(DEV), rt.to(DEV), qo, vis,
                                             vis, idx, B, 0, 0.07, out, lse, ws, num_splits=2)
        dsa.dsa_check_error(ws)
        outs.append((out, lse))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


def test_csa_step_indexer_on_compressed_keys_then_window():
    """The whole CSA decode: the lightning indexer scores the compressed keys,
    the selector keeps top-512, attention adds the raw window."""
    B, topk, window = 2, 512, 128
    L_raw = [20000, 9000]
    Lc, pool, ct, rt, q = _case(11, B, L_raw)
    g = torch.Generator().manual_seed(2)
    keys = torch.randn(sum(Lc), 128, generator=g).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    qi = torch.randn(B, 64, 128, generator=g).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    w = torch.randn(B, 64, generator=g) / 8
    so = torch.tensor([0, Lc[0], Lc[0] + Lc[1]], dtype=torch.int64, device=DEV)
    qo = torch.arange(B + 1, dtype=torch.int32, device=DEV)
    vis = torch.tensor(Lc, dtype=torch.int32, device=DEV)
    idx = torch.empty(B, topk, dtype=torch.int32, device=DEV)
    ws = dsa.workspace(B, max(Lc), topk + window, 0)
    dsa.dsa_indexer_topk(qi.to(DEV), w.to(DEV), keys.to(DEV), so, qo, vis, B, max(Lc), topk, idx, ws)
    out = torch.empty(B, 128, 512, device=DEV)
    lse = torch.empty(B, 128, device=DEV)
    scale = 1 / math.sqrt(192)
    dsa.dsa_sparse_mla_decode_window(q.to(DEV), pool.to(DEV), ct.to(DEV), rt.to(DEV), qo, vis,
                                     torch.tensor(L_raw, dtype=torch.int32, device=DEV), idx, B,
                                     window, scale, out, lse, ws)
    dsa.dsa_check_error(ws)
    from tests._parity import check_topk_row
    kb, qb_i, wb = keys.numpy(), qi.numpy(), w.numpy()
    pb, qb = np_bits(pool), np_bits(q)
    ix = idx.cpu().numpy()
    for b in range(B):
        k0 = 0 if b == 0 else Lc[0]
        sc = O.indexer_scores(qb_i[b], wb[b], kb[k0:k0 + Lc[b]])
        check_topk_row(ix[b], sc, topk)
        o_ref, l_ref = _oracle(pb, ct[b].numpy(), rt[b].numpy(), qb[b], ix[b][ix[b] >= 0], L_raw[b],
                               window, scale)
        check_attention(out[b].cpu().numpy(), lse[b].cpu().numpy(), o_ref, l_ref)
