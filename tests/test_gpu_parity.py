"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle on
the same seeded inputs, at sizes the oracle finishes in seconds that still
span several tiles and ragged tails."""
import math

import numpy as np
import pytest
import torch

import oracle as O
import sparse_attention_decode_lightning_b200 as dsa
from synth import get_workload, make_inputs
from tests._helpers import np_bits, oracle_inputs
from tests._parity import check_attention, check_topk_row, oracle_attention_for_idx
from tests._gpu import run_decode_step

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _e4m3(x: torch.Tensor) -> torch.Tensor:
    return x.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)


# ------------------------------------------------------------------ indexer
def _indexer_case(counts, first_only, hi, seed=0):
    """Scores of sequences of lengths `lens` with counts[b] queries each (an MTP
    verify sequence's position t sees all but its last counts[b]-1-t keys)."""
    torch.manual_seed(seed)
    lens = [1000, 300, 129, 4096 + 77]
    B = len(lens)
    Q = int(sum(counts))
    seq_off = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int64, device=DEV)
    q_off = torch.tensor([0] + list(np.cumsum(counts)), dtype=torch.int32, device=DEV)
    pos = [(b, t) for b in range(B) for t in range(counts[b])]
    vis = torch.tensor([lens[b] - (counts[b] - 1 - t) for b, t in pos], dtype=torch.int32, device=DEV)
    k = _e4m3(torch.randn(int(sum(lens)), 128, device=DEV))
    qi = _e4m3(torch.randn(Q, hi, 128, device=DEV))
    w = torch.randn(Q, hi, device=DEV) / 8
    ld = max(lens) + 60
    ld += (-ld) % 4
    scores = torch.full((Q, ld), float("nan"), device=DEV)
    ws = torch.zeros(1 << 16, dtype=torch.uint8, device=DEV)
    dsa.dsa_indexer_scores(qi, w, k, seq_off, q_off, vis, B, max(lens), scores, ws,
                           first_only=first_only)
    dsa.dsa_check_error(ws)
    sc = scores.cpu().numpy()
    kb, qb, wb = np_bits(k), np_bits(qi), w.cpu().numpy()
    so = seq_off.cpu().numpy()
    vv = vis.cpu().numpy()
    for q, (b, t) in enumerate(pos):
        if first_only and t > 0:
            assert np.isnan(sc[q]).all()
            continue
        keys = kb[so[b]:so[b] + vv[q]]
        ref = O.indexer_scores(qb[q], wb[q], keys)
        # fp32 summation bound for the hi-head reduction (products are exact)
        d = O.e4m3_decode(keys) @ O.e4m3_decode(qb[q]).T
        mag = np.abs(np.maximum(d, 0) * wb[q].astype(np.float64)).sum(1)
        tol = hi * 2.0 ** -24 * mag + 1e-30
        got = sc[q, :vv[q]].astype(np.float64)
        bad = np.abs(got - ref) > tol
        assert not bad.any(), (q, np.flatnonzero(bad)[:5], got[bad][:5], ref[bad][:5])
        assert np.isnan(sc[q, vv[q]:]).all()


# indexer heads: 64 (DeepSeek-V3.2) and 32 (GLM-5.2)
@pytest.mark.parametrize("T,first_only,hi", [(1, False, 64), (8, False, 64), (8, True, 64),
                                             (1, False, 32), (8, False, 32), (8, True, 32)])
def test_indexer_scores_match_oracle(T, first_only, hi):
    _indexer_case([T] * 4, first_only, hi)


# several queries a sequence with odd counts: a pair's second query is absent
@pytest.mark.parametrize("hi", [64, 32])
def test_indexer_scores_ragged_queries_per_sequence(hi):
    _indexer_case([3, 8, 1, 5], False, hi, seed=1)


# ------------------------------------------------------------------ selector
def _topk_case(name, rng):
    if name == "normal":
        return rng.standard_normal(5000).astype(np.float32)
    if name == "int_ties":
        return rng.integers(-3, 4, 6000).astype(np.float32)
    if name == "all_equal":
        return np.full(3000, 1.5, dtype=np.float32)
    if name == "signed_zero":
        x = np.where(rng.random(4000) < 0.5, 0.0, -0.0).astype(np.float32)
        x[rng.choice(4000, 100, replace=False)] = -1.0
        return x
    if name == "narrow_band":
        return (10.0 + rng.random(40000) * 1e-3).astype(np.float32)
    if name == "long":
        return (rng.standard_normal(200000) * 7).astype(np.float32)
    if name == "very_long":       # slices longer than the on-chip copy: tails re-read
        return (rng.standard_normal(400000) * 7).astype(np.float32)
    if name == "long_int_ties":   # threshold bin too large for the candidate lists
        return rng.integers(-3, 4, 400000).astype(np.float32)
    raise KeyError(name)


@pytest.mark.parametrize("case", ["normal", "int_ties", "all_equal", "signed_zero", "narrow_band",
                                  "long", "very_long", "long_int_ties"])
def test_topk_select_exact_on_fixed_scores(case):
    rng = np.random.default_rng(7)
    x = _topk_case(case, rng)
    L = x.shape[0]
    rows = [x, x[: 2048], x[: 2049], x[: 1], x[: 2047]]
    Q = len(rows)
    ld = L + (-L) % 4
    s = np.zeros((Q, ld), dtype=np.float32)
    vis = np.zeros(Q, dtype=np.int32)
    for i, r in enumerate(rows):
        s[i, : r.shape[0]] = r
        vis[i] = r.shape[0]
    scores = torch.from_numpy(s).to(DEV)
    q_off = torch.arange(Q + 1, dtype=torch.int32, device=DEV)
    out = torch.empty(Q, 2048, dtype=torch.int32, device=DEV)
    osc = torch.empty(Q, 2048, dtype=torch.float32, device=DEV)
    ws = dsa.workspace(Q, ld, 2048, 1)
    dsa.dsa_topk_select(scores, q_off, torch.from_numpy(vis).to(DEV), Q, L, 2048, out, ws,
                        out_scores=osc)
    dsa.dsa_check_error(ws)
    out = out.cpu().numpy()
    osc = osc.cpu().numpy()
    for i, r in enumerate(rows):
        ref = O.topk_select(r.astype(np.float64), 2048)
        n = min(2048, r.shape[0])
        assert set(out[i][out[i] >= 0].tolist()) == set(ref[:n].tolist())   # exact
        assert (out[i][n:] == -1).all()
        sel = out[i][:n]
        assert np.array_equal(osc[i][:n], r[sel])
        assert np.isneginf(osc[i][n:]).all()


# ------------------------------------------------------------------ sparse MLA
@pytest.mark.parametrize("S,name", [(1, "decode_b32_ctx128k"), (3, "decode_b32_ctx128k"),
                                    (16, "decode_b32_ctx128k"), (1, "glm52_decode_b32_ctx128k"),
                                    (3, "glm52_decode_b32_ctx128k")])
def test_sparse_mla_matches_oracle(S, name):
    w = get_workload(name, B=3, L=1500, topk=2048)
    inp = make_inputs(w, seed=11, device=DEV)
    Q = inp.Q
    g = torch.Generator(device="cpu").manual_seed(5)
    idx = torch.full((Q, 2048), -1, dtype=torch.int32)
    for q in range(Q):
        n = [1500, 700, 1][q]
        idx[q, :n] = torch.randperm(1500, generator=g)[:n].to(torch.int32)
    idx = idx.to(DEV)
    out = torch.empty(Q, inp.heads, 512, device=DEV)
    lse = torch.empty(Q, inp.heads, device=DEV)
    ws = dsa.workspace(Q, 1, 2048, S)
    dsa.dsa_sparse_mla_decode(inp.layers[0]["q"], inp.layers[0]["pool"], inp.page_table,
                              inp.q_offsets, inp.q_vis, idx, inp.B, inp.scale, out, lse, ws,
                              num_splits=S)
    dsa.dsa_check_error(ws)
    pool, pt, qb = np_bits(inp.layers[0]["pool"]), np_bits(inp.page_table), np_bits(inp.layers[0]["q"])
    ix = idx.cpu().numpy()
    for q in range(Q):
        o_ref, l_ref = oracle_attention_for_idx(pool, pt[q], qb[q], ix[q], inp.scale)
        check_attention(out[q].cpu().numpy(), lse[q].cpu().numpy(), o_ref, l_ref)


@pytest.mark.parametrize("heads,idx_heads,qk", [(128, 64, 192), (64, 32, 256)])
def test_sparse_mla_all_padding_gives_zero_and_neg_inf(heads, idx_heads, qk):
    inp = make_inputs(get_workload("decode_b1_ctx8k", L=256, heads=heads, idx_heads=idx_heads,
                                   qk_head_dim=qk), seed=2, device=DEV)
    idx = torch.full((1, 2048), -1, dtype=torch.int32, device=DEV)
    out = torch.full((1, heads, 512), 7.0, device=DEV)
    lse = torch.zeros(1, heads, device=DEV)
    for S in (1, 4):
        ws = dsa.workspace(1, 1, 2048, S)
        dsa.dsa_sparse_mla_decode(inp.layers[0]["q"], inp.layers[0]["pool"], inp.page_table,
                                  inp.q_offsets, inp.q_vis, idx, 1, inp.scale, out, lse, ws,
                                  num_splits=S)
        dsa.dsa_check_error(ws)
        assert (out == 0).all() and torch.isneginf(lse).all()


@pytest.mark.parametrize("H", [128, 64])
def test_lse_combine_matches_oracle(H):
    rng = np.random.default_rng(3)
    Q, S = 3, 5
    o = rng.standard_normal((Q, S, H, 512)).astype(np.float32)
    l = (rng.standard_normal((Q, S, H)) * 4).astype(np.float32)
    l[0, 2] = -np.inf
    l[1, :, :7] = -np.inf
    out = torch.empty(Q, H, 512, device=DEV)
    lse = torch.empty(Q, H, device=DEV)
    dsa.dsa_lse_combine(torch.from_numpy(o).to(DEV), torch.from_numpy(l).to(DEV), out, lse)
    torch.cuda.synchronize()
    for q in range(Q):
        o_ref, l_ref = O.lse_combine(o[q].astype(np.float64), l[q].astype(np.float64))
        assert np.allclose(out[q].cpu().numpy(), o_ref, rtol=1e-5, atol=1e-5)
        fin = np.isfinite(l_ref)
        assert np.allclose(lse[q].cpu().numpy()[fin], l_ref[fin], atol=1e-5)
        assert np.isneginf(lse[q].cpu().numpy()[~fin]).all()


# ------------------------------------------------------------------ whole step
SMALL = {
    "decode_b1_ctx8k": dict(),
    "decode_b32_ctx128k": dict(B=4, L=9000),
    "indexshare4_b64_ctx16k_128k": dict(B=5, L_range=(1500, 7000)),
    "mtp_verify_b16_t8_ctx128k": dict(B=2, L=5000),
    "mtp_verify_reuse_b16_t8_ctx128k": dict(B=2, L=5000),
    "decode_b4_ctx1m_split16": dict(B=2, L=40000),
    "glm52_decode_b32_ctx128k": dict(B=4, L=9000),
    "glm52_indexshare4_b64_ctx16k_128k": dict(B=5, L_range=(1500, 7000)),
    "glm52_decode_b4_ctx1m_split16": dict(B=2, L=40000),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_decode_step_matches_oracle(name):
    w = get_workload(name, **SMALL[name])
    inp = make_inputs(w, seed=0, device=DEV)
    outs, lses, idx = run_decode_step(inp)
    host = oracle_inputs(inp)
    ix = idx.cpu().numpy()
    T, G = inp.T, inp.index_share
    swaps = 0
    for g in range(ix.shape[0]):
        ind = host["indexer"][g]
        for q in range(inp.Q):
            b = q // T
            src = b * T if inp.mtp_index_share else q
            k0, vis = int(host["seq_offsets"][b]), int(host["q_vis"][src])
            sc = O.indexer_scores(ind["q_idx"][src], ind["w"][src], ind["k_idx"][k0:k0 + vis])
            swaps += check_topk_row(ix[g, q], sc, inp.topk)
            if inp.mtp_index_share:
                assert np.array_equal(ix[g, q], ix[g, src])
    for l in range(inp.n_layers):
        lay = host["layers"][l]
        for q in range(inp.Q):
            b = q // T
            o_ref, l_ref = oracle_attention_for_idx(lay["pool"], host["page_table"][b], lay["q"][q],
                                                    ix[l // G, q], inp.scale)
            check_attention(outs[l][q].cpu().numpy(), lses[l][q].cpu().numpy(), o_ref, l_ref)


def test_indexshare_layers_use_the_leader_indices():
    inp = make_inputs(get_workload("indexshare4_b64_ctx16k_128k", B=3, L_range=(3000, 5000)),
                      seed=4, device=DEV)
    outs, lses, idx = run_decode_step(inp)
    assert idx.shape[0] == 1
    # the shared layers' outputs equal direct sparse-MLA calls on the leader's indices
    for l in range(1, 4):
        out = torch.empty_like(outs[l])
        lse = torch.empty_like(lses[l])
        ws = dsa.workspace(inp.Q, 1, inp.topk, 0)
        dsa.dsa_sparse_mla_decode(inp.layers[l]["q"], inp.layers[l]["pool"], inp.page_table,
                                  inp.q_offsets, inp.q_vis, idx[0], inp.B, inp.scale, out, lse, ws)
        dsa.dsa_check_error(ws)
        assert torch.equal(out, outs[l]) and torch.equal(lse, lses[l])


@pytest.mark.parametrize("B", [20, 25])
def test_indexshare_tail_split_matches_oracle(B):
    """Four layers x B queries leave a last wave of at most half the SM pairs,
    which runs as split units merged by LSE (B = 25: the split tail starts in
    layer 2 and ends in layer 3)."""
    inp = make_inputs(get_workload("indexshare4_b64_ctx16k_128k", B=B, L_range=(2500, 6000)),
                      seed=12, device=DEV)
    pairs = 74
    units = inp.n_layers * inp.Q
    assert units >= pairs and units % pairs <= pairs // 2
    outs, lses, idx = run_decode_step(inp, num_splits=1)    # one split: the grouped launch
    host = oracle_inputs(inp)
    ix = idx.cpu().numpy()
    for l in range(inp.n_layers):
        lay = host["layers"][l]
        for q in range(inp.Q):
            o_ref, l_ref = oracle_attention_for_idx(lay["pool"], host["page_table"][q], lay["q"][q],
                                                    ix[0, q], inp.scale)
            check_attention(outs[l][q].cpu().numpy(), lses[l][q].cpu().numpy(), o_ref, l_ref)


@pytest.mark.parametrize("n_layers,G", [(6, 4), (9, 8)])
def test_index_groups_of_uneven_and_long_length_match_oracle(n_layers, G):
    """Six layers in groups of four (a full group, then two layers) and nine
    in groups of eight (a group longer than one grouped launch of four
    layers, then one layer alone): every layer attends over its group
    leader's indices."""
    inp = make_inputs(get_workload("indexshare4_b64_ctx16k_128k", B=3, L_range=(2500, 5000),
                                   n_layers=n_layers, index_share=G), seed=17, device=DEV)
    outs, lses, idx = run_decode_step(inp, num_splits=1)
    host = oracle_inputs(inp)
    ix = idx.cpu().numpy()
    assert ix.shape[0] == (n_layers + G - 1) // G
    for g in range(ix.shape[0]):
        ind = host["indexer"][g]
        for q in range(inp.Q):
            k0, vis = int(host["seq_offsets"][q]), int(host["q_vis"][q])
            sc = O.indexer_scores(ind["q_idx"][q], ind["w"][q], ind["k_idx"][k0:k0 + vis])
            check_topk_row(ix[g, q], sc, inp.topk)
    for l in range(n_layers):
        lay = host["layers"][l]
        for q in range(inp.Q):
            o_ref, l_ref = oracle_attention_for_idx(lay["pool"], host["page_table"][q], lay["q"][q],
                                                    ix[l // G, q], inp.scale)
            check_attention(outs[l][q].cpu().numpy(), lses[l][q].cpu().numpy(), o_ref, l_ref)


def test_device_bounds_are_flagged_not_faulted():
    inp = make_inputs(get_workload("decode_b32_ctx128k", B=2, L=3000), seed=9, device=DEV)
    bad_pt = inp.page_table.clone()
    bad_pt[0, 3] = inp.num_pages + 5          # page id out of range
    idx = torch.arange(2048, dtype=torch.int32, device=DEV).repeat(inp.Q, 1)
    out = torch.empty(inp.Q, 128, 512, device=DEV)
    lse = torch.empty(inp.Q, 128, device=DEV)
    ws = dsa.workspace(inp.Q, 1, 2048, 2)
    dsa.dsa_sparse_mla_decode(inp.layers[0]["q"], inp.layers[0]["pool"], bad_pt, inp.q_offsets,
                              inp.q_vis, idx, inp.B, inp.scale, out, lse, ws, num_splits=2)
    with pytest.raises(dsa.DSAError) as e:
        dsa.dsa_check_error(ws)
    assert e.value.status == 4
    assert torch.isfinite(out).all()
    dsa.dsa_check_error(ws)                   # the flag was cleared
    # an index beyond the visible length is flagged too
    idx2 = idx.clone()
    idx2[1, 5] = 2999 + 10
    dsa.dsa_sparse_mla_decode(inp.layers[0]["q"], inp.layers[0]["pool"], inp.page_table,
                              inp.q_offsets, inp.q_vis, idx2, inp.B, inp.scale, out, lse, ws,
                              num_splits=2)
    with pytest.raises(dsa.DSAError):
        dsa.dsa_check_error(ws)
