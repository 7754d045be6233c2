"""The fused indexer -> selector path (dsa_indexer_topk_fused): the indexer
emits per-query histograms of the selector's first radix digit and the
selector starts from them.  Its index sets must equal, exactly and ties
included, the oracle's selection (oracle.topk_select: a full sort by score
desc, position asc) over the fp32 scores the same indexer writes
(dsa_indexer_scores), over ordinary, all-equal,
tied and narrow-band score rows, single and multi-query sequences."""
import numpy as np
import pytest
import torch

import sparse_attention_decode_lightning_b200 as dsa
from oracle import topk_select

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _e4m3(x):
    return x.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)


def _inputs(case, lens, T, seed, hi=64):
    g = torch.Generator(device=DEV).manual_seed(seed)
    B = len(lens)
    Q = B * T
    keys = torch.randn(sum(lens), 128, generator=g, device=DEV)
    qi = torch.randn(Q, hi, 128, generator=g, device=DEV)
    w = torch.randn(Q, hi, generator=g, device=DEV) / 8
    if case == "all_zero":            # every score is +-0: one bin holds the whole row
        qi.zero_()
    elif case == "tied_keys":         # every key row repeated 16 times: exact ties
        keys = keys[torch.arange(sum(lens), device=DEV) // 16]
    elif case == "narrow":            # a dominant constant head: scores in a narrow band
        keys[:, 0] = 4.0
        qi[:, :, 0] = 4.0
        qi[:, :, 1:] *= 0.01
    return _e4m3(keys.contiguous()), _e4m3(qi), w


def _expected(scores_row, vis, topk):
    """The oracle's selection (stable sort by score desc, position asc; -0 ==
    +0) over the fp32 scores the GPU indexer wrote, as a set."""
    sel = topk_select(scores_row[:vis].astype(np.float32), topk)
    return set(sel[sel >= 0].tolist())


@pytest.mark.parametrize("case", ["normal", "all_zero", "tied_keys", "narrow"])
@pytest.mark.parametrize("T,first_only", [(1, False), (8, False), (8, True)])
def test_fused_selection_is_exact(case, T, first_only):
    lens = [150000, 9000, 1500] if T == 1 else [40000, 2100]
    topk = 2048
    k, qi, w = _inputs(case, lens, T, seed=len(case) + T)
    B, Q = len(lens), len(lens) * T
    seq_off = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int64, device=DEV)
    q_off = torch.arange(B + 1, dtype=torch.int32, device=DEV) * T
    vis = torch.tensor([lens[b] - (T - 1 - t) for b in range(B) for t in range(T)],
                       dtype=torch.int32, device=DEV)
    L = max(lens)
    idx = torch.empty(Q, topk, dtype=torch.int32, device=DEV)
    ws = dsa.workspace(Q, L, topk, 1)
    for rep in range(2):                            # the histograms are reset between calls
        dsa.dsa_indexer_topk_fused(qi, w, k, seq_off, q_off, vis, B, L, topk, idx, ws, first_only=first_only)
        dsa.dsa_check_error(ws)
    ld = ((L + 63) // 64) * 64
    scores = torch.full((Q, ld), float("nan"), device=DEV)
    ws2 = dsa.workspace(Q, L, topk, 1)
    dsa.dsa_indexer_scores(qi, w, k, seq_off, q_off, vis, B, L, scores, ws2, first_only=first_only)
    dsa.dsa_check_error(ws2)
    sc, ix, vv = scores.cpu().numpy(), idx.cpu().numpy(), vis.cpu().numpy()
    for q in range(Q):
        b, t = divmod(q, T)
        src = b * T if first_only else q
        want = _expected(sc[src], int(vv[src]), topk)
        row = ix[q]
        got = set(row[row >= 0].tolist())
        assert len(got) == int((row >= 0).sum()), "duplicate positions"
        assert got == want, (case, q, len(got ^ want))
        assert (row[len(want):] == -1).all() if len(want) < topk else True


def _check_rows(scores, idx, vis, topk):
    sc, ix, vv = scores.cpu().numpy(), idx.cpu().numpy(), vis.cpu().numpy()
    for q in range(ix.shape[0]):
        want = _expected(sc[q], int(vv[q]), topk)
        row = ix[q]
        got = set(row[row >= 0].tolist())
        assert len(got) == int((row >= 0).sum()), ("duplicate positions", q)
        assert got == want, (q, len(got ^ want))


@pytest.mark.parametrize("dirty,hi", [(False, 64), (True, 64), (False, 32)])
def test_fused_selection_many_rows(dirty, hi):
    """64 single-query sequences of 16K to 128K keys: enough rows that the
    selector's CTAs of one row finish in varied orders.  Every call of several
    back to back is checked.  With dirty=True the workspace is filled with
    non-zero bytes (all but its error word) before the first call: the call
    must not depend on a previous call having left its histograms zeroed.
    hi = 32 runs the GLM-5.2 indexer head count."""
    rng = np.random.default_rng(11)
    lens = rng.integers(16384, 131073, size=64).tolist()
    topk = 2048
    k, qi, w = _inputs("normal", lens, 1, seed=5, hi=hi)
    B = Q = len(lens)
    seq_off = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int64, device=DEV)
    q_off = torch.arange(B + 1, dtype=torch.int32, device=DEV)
    vis = torch.tensor(lens, dtype=torch.int32, device=DEV)
    L = max(lens)
    ld = ((L + 63) // 64) * 64
    scores = torch.full((Q, ld), float("nan"), device=DEV)
    ws2 = dsa.workspace(Q, L, topk, 1)
    dsa.dsa_indexer_scores(qi, w, k, seq_off, q_off, vis, B, L, scores, ws2)
    dsa.dsa_check_error(ws2)
    ws = dsa.workspace(Q, L, topk, 1)
    if dirty:
        ws.fill_(0xA5)
        ws[:256].zero_()
    for rep in range(4):
        idx = torch.full((Q, topk), -7, dtype=torch.int32, device=DEV)
        dsa.dsa_indexer_topk_fused(qi, w, k, seq_off, q_off, vis, B, L, topk, idx, ws)
        dsa.dsa_check_error(ws)
        _check_rows(scores, idx, vis, topk)


def test_fused_out_scores_match_the_selected_positions():
    """out_scores: the score of each selected position as the indexer wrote
    it, and -inf in the padding of a row with fewer visible keys than topk."""
    lens = [150000, 9000, 1500]
    topk = 2048
    k, qi, w = _inputs("normal", lens, 1, seed=23)
    B = Q = len(lens)
    seq_off = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int64, device=DEV)
    q_off = torch.arange(B + 1, dtype=torch.int32, device=DEV)
    vis = torch.tensor(lens, dtype=torch.int32, device=DEV)
    L = max(lens)
    ld = ((L + 63) // 64) * 64
    scores = torch.full((Q, ld), float("nan"), device=DEV)
    ws2 = dsa.workspace(Q, L, topk, 1)
    dsa.dsa_indexer_scores(qi, w, k, seq_off, q_off, vis, B, L, scores, ws2)
    dsa.dsa_check_error(ws2)
    idx = torch.empty(Q, topk, dtype=torch.int32, device=DEV)
    osc = torch.full((Q, topk), float("nan"), device=DEV)
    ws = dsa.workspace(Q, L, topk, 1)
    dsa.dsa_indexer_topk_fused(qi, w, k, seq_off, q_off, vis, B, L, topk, idx, ws, out_scores=osc)
    dsa.dsa_check_error(ws)
    _check_rows(scores, idx, vis, topk)
    sc, ix, os_ = scores.cpu().numpy(), idx.cpu().numpy(), osc.cpu().numpy()
    for q in range(Q):
        sel = ix[q] >= 0
        assert np.array_equal(os_[q][sel], sc[q][ix[q][sel]]), q
        assert np.all(np.isneginf(os_[q][~sel])), q
