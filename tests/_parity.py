"""Parity criteria between the CUDA library and the fp64 oracle.

* top-k index sets: equal, except that a position may be swapped for another
  when both oracle scores lie within 1e-6 (relative) of the oracle's k-th
  score; padding (-1) exactly where the visible length is below k;
* attention output: max |O - O*| / rms(O*) <= 1e-2 and
  mean |O - O*| / rms(O*) <= 5e-3, with O* the oracle on the indices the GPU
  chose; log-sum-exp within 1e-3 absolute (and -inf exactly where O* has no
  token).
"""
import numpy as np
import torch

import oracle as O
from tests._helpers import np_bits

TOPK_REL = 1e-6
O_MAX_REL = 1e-2
O_MEAN_REL = 5e-3
LSE_ABS = 1e-3


def check_topk_row(gpu_row: np.ndarray, scores: np.ndarray, topk: int, rel: float = TOPK_REL):
    """gpu_row: int32[topk] from the library; scores: oracle fp64 scores of the visible keys."""
    vis = scores.shape[0]
    n = min(topk, vis)
    sel = gpu_row[gpu_row >= 0]
    assert sel.shape[0] == n, (sel.shape[0], n)
    assert (gpu_row[n:] == -1).all() if n < topk else True
    assert np.unique(sel).shape[0] == n, "duplicate positions"
    assert sel.min(initial=0) >= 0 and sel.max(initial=0) < vis
    ref = O.topk_select(scores, topk)[:n]
    if n == vis:
        assert set(sel.tolist()) == set(range(vis))
        return 0
    ik = scores[ref[n - 1]]
    diff = set(sel.tolist()) ^ set(ref.tolist())
    for s in diff:
        assert abs(scores[s] - ik) <= rel * abs(ik), (s, scores[s], ik)
    return len(diff)


def check_attention(o: np.ndarray, lse: np.ndarray, o_ref: np.ndarray, lse_ref: np.ndarray):
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse), fin), "empty-set heads differ"
    if not fin.any():
        assert np.all(o == 0)
        return
    r = float(np.sqrt(np.mean(np.square(o_ref[fin]))))
    err = np.abs(o[fin] - o_ref[fin])
    assert err.max() / r <= O_MAX_REL, ("max", err.max() / r)
    assert err.mean() / r <= O_MEAN_REL, ("mean", err.mean() / r)
    assert np.abs(lse[fin] - lse_ref[fin]).max() <= LSE_ABS, np.abs(lse[fin] - lse_ref[fin]).max()
    assert np.all(o[~fin] == 0)


def oracle_attention_for_idx(pool_bits, page_row, q_bits, idx_row, scale, num_splits=1, vis=None):
    pos = idx_row[idx_row >= 0].astype(np.int64)
    rows = O.latent_rows(pool_bits, page_row, pos)
    qf = O.bf16_decode(q_bits)
    if num_splits > 1:
        return O.sparse_mla_split(qf, rows, pos, int(vis), num_splits, scale)
    return O.sparse_mla(qf, rows, scale)
