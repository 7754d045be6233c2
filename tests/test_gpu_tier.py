"""Two-tier (HiSparse) latent cache on the GPU: the host plan, the fetch kernel
from pinned host memory, then sparse MLA over the 16-token device buffer.
Attention through the tier must equal the oracle's attention over the full
cache; fetched slots must hold their host pages bit for bit.

Source: "GLM-5.2 推理部署", section "HiSparse 的通信路径：GPU↔CPU KV swap"."""
import ctypes
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
PT = dsa.TIER_PAGE


def _local_rows(rng, hot, L, topk):
    pages = rng.choice(hot, topk)
    pos = pages * PT + rng.integers(0, PT, topk)
    pos = np.minimum(pos, L - 1)
    pos = np.unique(pos)                       # distinct positions, like a top-k row
    row = np.full(topk, -1, dtype=np.int32)
    row[:len(pos)] = pos
    return row


@pytest.mark.parametrize("heads,qk", [(64, 256), (128, 192)])
def test_tiered_attention_matches_full_cache(heads, qk):
    rng = np.random.default_rng(heads)
    B, L, D, topk = 2, 6000, 96, 2048
    P = (L + PT - 1) // PT
    g = torch.Generator().manual_seed(5)
    host = torch.randn(B * P, PT, 576, generator=g).to(torch.bfloat16).pin_memory()
    pool = torch.full((B * D, PT, 576), float("nan"), dtype=torch.bfloat16, device=DEV)
    q = torch.randn(B, heads, 576, generator=g).to(torch.bfloat16).to(DEV)
    q_off = torch.arange(B + 1, dtype=torch.int32)
    vis = torch.full((B,), L, dtype=torch.int32, device=DEV)
    scale = 1 / math.sqrt(qk)
    st = dsa.tier_state(B, D, P)
    pt = torch.empty(B, P, dtype=torch.int32)
    cp = torch.empty(B * D, 3, dtype=torch.int32)
    pt_dev = torch.full((B, P), -1, dtype=torch.int32, device=DEV)   # patched by every fetch
    ws = dsa.workspace(B, 1, topk, 1)
    out = torch.empty(B, heads, 512, device=DEV)
    lse = torch.empty(B, heads, device=DEV)
    hot = [list(rng.choice(P, 70, replace=False)) for _ in range(B)]
    host_np = np_bits(host).reshape(B, P * PT, 576)
    q_np = np_bits(q)
    total_miss = total_ev = 0
    for step in range(6):
        for b in range(B):
            for _ in range(12):                  # the hot set drifts: misses and evictions
                hot[b][int(rng.integers(70))] = int(rng.integers(P))
        idx = torch.from_numpy(np.stack([_local_rows(rng, np.array(hot[b]), L, topk)
                                         for b in range(B)]))
        n, (hits, misses, ev) = dsa.dsa_tier_plan(st, idx, q_off, cp, page_table=pt)
        total_miss += misses
        total_ev += ev
        copies = cp[:n].to(DEV)
        dsa.dsa_tier_fetch(host, pool, copies, n, ws, page_table=pt_dev)
        dsa.dsa_sparse_mla_decode(q, pool, pt_dev, q_off.to(DEV), vis, idx.to(DEV), B, scale,
                                  out, lse, ws, num_splits=1)
        dsa.dsa_check_error(ws)
        # the patched device table equals the plan's full table
        assert torch.equal(pt_dev.cpu(), pt)
        # resident slots hold their host pages exactly
        ptn = pt.numpy()
        pool_np = np_bits(pool)
        for b in range(B):
            res = np.flatnonzero(ptn[b] >= 0)
            assert np.array_equal(pool_np[ptn[b, res]], np_bits(host)[b * P + res])
        # attention through the tier equals attention over the full cache
        for b in range(B):
            ix = idx[b].numpy()
            sel = ix[ix >= 0]
            rows = O.bf16_decode(host_np[b][sel])
            o_ref, l_ref = O.sparse_mla(O.bf16_decode(q_np[b]), rows, scale)
            check_attention(out[b].cpu().numpy(), lse[b].cpu().numpy(), o_ref, l_ref)
    assert total_ev > 0 and total_miss > total_ev     # the buffer filled and turned over


def test_fetch_refuses_memory_it_cannot_read():
    L = dsa.lib()
    pool = torch.empty(4, PT, 576, dtype=torch.bfloat16, device=DEV)
    copies = torch.zeros(1, 3, dtype=torch.int32, device=DEV)
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    pageable = torch.empty(4, PT, 576, dtype=torch.bfloat16)
    dev_src = torch.empty(4, PT, 576, dtype=torch.bfloat16, device=DEV)
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for src in (pageable, dev_src):
        st = L.dsa_tier_fetch(ctypes.c_void_p(src.data_ptr()), 4, ctypes.c_void_p(pool.data_ptr()),
                              4, ctypes.c_void_p(copies.data_ptr()), 1, None,
                              ctypes.c_void_p(ws.data_ptr()), s)
        assert st == 1
    # a pinned cache shorter than the extent claimed for it is refused too
    pinned = torch.empty(2, PT, 576, dtype=torch.bfloat16).pin_memory()
    torch.cuda.synchronize()
    st = L.dsa_tier_fetch(ctypes.c_void_p(pinned.data_ptr()), 1 << 20, ctypes.c_void_p(pool.data_ptr()),
                          4, ctypes.c_void_p(copies.data_ptr()), 1, None,
                          ctypes.c_void_p(ws.data_ptr()), s)
    assert st == 1


def test_fetch_skips_and_flags_copies_outside_the_caches():
    host = torch.randn(3, PT, 576).to(torch.bfloat16).pin_memory()
    pool = torch.zeros(2, PT, 576, dtype=torch.bfloat16, device=DEV)
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    copies = torch.tensor([[2, 1, -1], [3, 0, -1], [0, 2, -1]], dtype=torch.int32, device=DEV)
    dsa.dsa_tier_fetch(host, pool, copies, 3, ws)
    with pytest.raises(dsa.DSAError) as e:
        dsa.dsa_check_error(ws)
    assert e.value.status == 4
    assert torch.equal(pool[1].cpu(), host[2]) and bool((pool[0] == 0).all())


# ------------------------------------------------------------------ device planner
def _trace(rng, B, P, steps, hot, churn, rows_per_seq, topk):
    hot_sets = [list(rng.choice(P, hot, replace=False)) for _ in range(B)]
    out = []
    for _ in range(steps):
        rows = []
        for b in range(B):
            for _ in range(churn):
                hot_sets[b][int(rng.integers(hot))] = int(rng.integers(P))
            for _ in range(rows_per_seq):
                rows.append(_local_rows(rng, np.array(hot_sets[b]), P * PT, topk))
        out.append(np.stack(rows))
    return out


@pytest.mark.parametrize("B,D,P,hot,churn,rows", [(3, 64, 400, 50, 6, 2), (2, 1024, 4000, 700, 60, 1)])
def test_device_planner_matches_oracle(B, D, P, hot, churn, rows):
    rng = np.random.default_rng(D)
    topk = 256 if D == 64 else 2048
    host = torch.randn(B * P, PT, 576).to(torch.bfloat16).pin_memory()
    pool = torch.full((B * D, PT, 576), float("nan"), dtype=torch.bfloat16, device=DEV)
    pt = torch.empty(B, P, dtype=torch.int32, device=DEV)
    st = dsa.tier_dev_state(B, D, P, pt)
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    q_off_h = torch.arange(B + 1, dtype=torch.int32) * rows
    q_off = q_off_h.to(DEV)
    tier = O.TierOracle(B, D, P)
    host_bits = np_bits(host)
    for step, idx_np in enumerate(_trace(rng, B, P, 12, hot, churn, rows, topk)):
        idx = torch.from_numpy(idx_np).to(DEV)
        dsa.dsa_tier_swap_in(st, B, D, P, idx, q_off, pt, host, pool, ws)
        (n, hits, misses, ev), steps = dsa.dsa_tier_dev_stats(st)
        dsa.dsa_check_error(ws)
        per_seq = [[list(r) for r in idx_np[b * rows:(b + 1) * rows]] for b in range(B)]
        table, copies, h_o, m_o, e_o = tier.step(per_seq)
        assert steps == step + 1
        assert (n, hits, misses, ev) == (len(copies), h_o, m_o, e_o)
        assert pt.cpu().tolist() == table
        got = sorted(tuple(x) for x in dsa.dsa_tier_dev_copies(st, B, D, P, n).cpu().tolist())
        assert got == sorted(copies)
        ptn = pt.cpu().numpy()
        pool_bits = np_bits(pool)
        for b in range(B):
            res = np.flatnonzero(ptn[b] >= 0)
            assert np.array_equal(pool_bits[ptn[b, res]], host_bits[b * P + res])


def test_device_planner_refuses_a_step_beyond_its_slots():
    B, D, P = 2, 8, 100
    host = torch.randn(B * P, PT, 576).to(torch.bfloat16).pin_memory()
    pool = torch.zeros(B * D, PT, 576, dtype=torch.bfloat16, device=DEV)
    pt = torch.empty(B, P, dtype=torch.int32, device=DEV)
    st = dsa.tier_dev_state(B, D, P, pt)
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    q_off = torch.arange(B + 1, dtype=torch.int32, device=DEV)
    ok = torch.full((B, 16), -1, dtype=torch.int32)
    ok[:, :3] = torch.tensor([0, 16, 32])
    dsa.dsa_tier_swap_in(st, B, D, P, ok.to(DEV), q_off, pt, host, pool, ws)
    dsa.dsa_check_error(ws)
    before = pt.clone()
    bad = ok.clone()
    bad[0] = torch.arange(16, dtype=torch.int32) * 16          # 16 distinct pages for 8 slots
    dsa.dsa_tier_swap_in(st, B, D, P, bad.to(DEV), q_off, pt, host, pool, ws)
    with pytest.raises(dsa.DSAError) as e:
        dsa.dsa_check_error(ws)
    assert e.value.status == 2
    assert torch.equal(pt[0], before[0])                         # sequence 0 was left as it was


def test_device_tier_step_in_a_cuda_graph():
    """Swap-in (plan + fetch) and sparse MLA captured once and replayed for
    several steps with new index rows written in place: the device path needs
    no host round trip, so the replays must follow the oracle step by step."""
    rng = np.random.default_rng(21)
    B, D, P, topk, heads = 2, 96, 400, 512, 64
    host = torch.randn(B * P, PT, 576).to(torch.bfloat16).pin_memory()
    pool = torch.zeros(B * D, PT, 576, dtype=torch.bfloat16, device=DEV)
    pt = torch.empty(B, P, dtype=torch.int32, device=DEV)
    q = torch.randn(B, heads, 576).to(torch.bfloat16).to(DEV)
    q_off = torch.arange(B + 1, dtype=torch.int32, device=DEV)
    vis = torch.full((B,), P * PT, dtype=torch.int32, device=DEV)
    idx = torch.full((B, topk), -1, dtype=torch.int32, device=DEV)
    out = torch.empty(B, heads, 512, device=DEV)
    lse = torch.empty(B, heads, device=DEV)
    ws = dsa.workspace(B, 1, topk, 1)
    scale = 1 / math.sqrt(256)
    side = torch.cuda.Stream()
    st = dsa.tier_dev_state(B, D, P, pt, stream=side)
    trace = _trace(rng, B, P, 6, 60, 8, 1, topk)

    def step():
        dsa.dsa_tier_swap_in(st, B, D, P, idx, q_off, pt, host, pool, ws, stream=side)
        dsa.dsa_sparse_mla_decode(q, pool, pt, q_off, vis, idx, B, scale, out, lse, ws,
                                  num_splits=1, stream=side)

    # first step eagerly (sets kernel attributes), then capture the step once
    tier = O.TierOracle(B, D, P)
    idx.copy_(torch.from_numpy(trace[0]))
    torch.cuda.synchronize()
    step()
    side.synchronize()
    tier.step([[list(trace[0][b])] for b in range(B)])
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        step()
    host_bits, q_np = np_bits(host).reshape(B, P * PT, 576), np_bits(q)
    for idx_np in trace[1:]:
        idx.copy_(torch.from_numpy(idx_np))
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        dsa.dsa_check_error(ws)
        table, *_ = tier.step([[list(idx_np[b])] for b in range(B)])
        assert pt.cpu().tolist() == table
        for b in range(B):
            sel = idx_np[b][idx_np[b] >= 0]
            o_ref, l_ref = O.sparse_mla(O.bf16_decode(q_np[b]), O.bf16_decode(host_bits[b][sel]), scale)
            check_attention(out[b].cpu().numpy(), lse[b].cpu().numpy(), o_ref, l_ref)
