"""Two-tier (HiSparse) latent cache: the oracle's LRU bookkeeping pinned to a
library LRU and to invariants, then the library's host planner compared with
the oracle step by step (no GPU: the plan is host code).

Source: "GLM-5.2 推理部署", section "HiSparse 的通信路径：GPU↔CPU KV swap"
(top-K miss detection, LRU eviction, page-table update and H2D fetch; slots
of 16 tokens)."""
import functools

import numpy as np
import pytest
import torch

import oracle as O
import oracle.hisparse as OH
import sparse_attention_decode_lightning_b200 as dsa

PT = O.TIER_PAGE_TOKENS


def _single_page_trace_faults(trace, frames):
    """Faults of the oracle on a one-sequence trace that selects one page per step."""
    tier = O.TierOracle(1, frames, max(trace) + 1)
    faults = 0
    for p in trace:
        _, copies, hits, misses, _ = tier.step([[[p * PT + 3]]])
        faults += misses
    return faults


def _lru_cache_faults(trace, frames):
    """The same trace through Python's own LRU cache (functools.lru_cache)."""
    @functools.lru_cache(maxsize=frames)
    def page(p):
        return p
    for p in trace:
        page(p)
    return page.cache_info().misses


def test_one_page_per_step_is_textbook_lru():
    # the classic reference string of operating-systems textbooks: LRU with 3
    # frames takes 12 faults (FIFO 15, optimal 9)
    classic = [7, 0, 1, 2, 0, 3, 0, 4, 2, 3, 0, 3, 2, 1, 2, 0, 1, 7, 0, 1]
    assert _single_page_trace_faults(classic, 3) == _lru_cache_faults(classic, 3) == 12
    rng = np.random.default_rng(7)
    for frames in (1, 2, 5, 16):
        trace = [int(x) for x in rng.integers(0, 40, 300)]
        assert _single_page_trace_faults(trace, frames) == _lru_cache_faults(trace, frames)


def _local_trace(rng, B, max_pages, steps, hot, churn, rows_per_seq=1, topk=64):
    """Index rows with locality: each sequence keeps a hot set of pages that
    changes by `churn` pages a step; positions are drawn inside the hot pages."""
    hot_sets = [list(rng.choice(max_pages, hot, replace=False)) for _ in range(B)]
    out = []
    for _ in range(steps):
        step = []
        for b in range(B):
            for _ in range(churn):
                hot_sets[b][int(rng.integers(hot))] = int(rng.integers(max_pages))
            rows = []
            for _ in range(rows_per_seq):
                pages = rng.choice(hot_sets[b], topk)
                pos = pages * PT + rng.integers(0, PT, topk)
                row = [int(x) for x in pos]
                pad = int(rng.integers(0, 4))          # a few -1 entries at the end
                if pad:
                    row[-pad:] = [-1] * pad
                rows.append(row)
            step.append(rows)
        out.append(step)
    return out


def test_oracle_invariants_on_local_traces():
    rng = np.random.default_rng(3)
    B, D, P = 3, 24, 200
    tier = O.TierOracle(B, D, P)
    prev_res = [set() for _ in range(B)]
    last_step_of = [dict() for _ in range(B)]
    for t, step in enumerate(_local_trace(rng, B, P, 40, hot=18, churn=3, rows_per_seq=2)):
        table, copies, hits, misses, ev = tier.step(step)
        for b in range(B):
            need = {pos // PT for row in step[b] for pos in row if pos >= 0}
            res = {p for p in range(P) if table[b][p] >= 0}
            assert need <= res                          # every selected page is resident
            assert len(res) <= D                        # the buffer never overflows
            slots = [table[b][p] for p in res]
            assert len(set(slots)) == len(slots)        # one page per slot
            assert all(b * D <= s < (b + 1) * D for s in slots)
            evicted = prev_res[b] - res
            assert not (evicted & need)                 # nothing selected now was evicted
            # every evicted page was used no later than every kept page not selected now
            kept_idle = (prev_res[b] & res) - need
            if evicted and kept_idle:
                assert max(last_step_of[b][p] for p in evicted) <= min(last_step_of[b][p] for p in kept_idle)
            for p in need:
                last_step_of[b][p] = t
            prev_res[b] = res
        assert misses == len(copies)
        assert hits + misses == sum(len({pos // PT for row in step[b] for pos in row if pos >= 0})
                                    for b in range(B))


def test_oracle_refuses_overflow():
    tier = O.TierOracle(1, 2, 10)
    with pytest.raises(O.TierOverflow):
        tier.step([[[0, 16, 32]]])


def test_planted_mru_is_caught(monkeypatch):
    # an oracle that evicts the most recently used slot must fail the library-LRU pin
    real_sorted = sorted

    def mru_sorted(seq, key=None, reverse=False):
        if key is not None:
            return real_sorted(seq, key=key, reverse=not reverse)
        return real_sorted(seq, reverse=reverse)

    monkeypatch.setattr(OH, "sorted", mru_sorted, raising=False)
    with pytest.raises(AssertionError):
        test_one_page_per_step_is_textbook_lru()


# ------------------------------------------------------------------ library planner
def _run_library(B, D, P, trace, topk):
    st = dsa.tier_state(B, D, P)
    qo = torch.tensor([sum(len(s) for s in trace[0][:b]) for b in range(B + 1)], dtype=torch.int32)
    pt = torch.empty(B, P, dtype=torch.int32)
    cp = torch.empty(B * D, 3, dtype=torch.int32)
    for step in trace:
        rows = [r for b in range(B) for r in step[b]]
        idx = torch.tensor(rows, dtype=torch.int32)
        n, stats = dsa.dsa_tier_plan(st, idx, qo, cp, page_table=pt)
        yield pt.clone(), cp[:n].clone(), stats


@pytest.mark.parametrize("B,D,P,hot,churn,rows", [(1, 8, 50, 6, 1, 1), (3, 24, 200, 18, 3, 2),
                                                  (2, 64, 1000, 60, 10, 8)])
def test_library_plan_equals_oracle(B, D, P, hot, churn, rows):
    rng = np.random.default_rng(B * 100 + D)
    trace = _local_trace(rng, B, P, 30, hot=hot, churn=churn, rows_per_seq=rows)
    tier = O.TierOracle(B, D, P)
    for step, (pt, cp, stats) in zip(trace, _run_library(B, D, P, trace, 64)):
        table, copies, hits, misses, ev = tier.step(step)
        assert pt.tolist() == table
        assert [tuple(x) for x in cp.tolist()] == copies
        assert stats == (hits, misses, ev)


def test_library_refusals_leave_state_unchanged():
    B, D, P = 1, 3, 20
    st = dsa.tier_state(B, D, P)
    qo = torch.tensor([0, 1], dtype=torch.int32)
    pt = torch.empty(B, P, dtype=torch.int32)
    cp = torch.empty(8, 3, dtype=torch.int32)
    ok = torch.tensor([[0, 16, -1, -1]], dtype=torch.int32)
    assert dsa.dsa_tier_plan(st, ok, qo, cp, page_table=pt)[0] == 2
    snap = st.clone()
    for bad, code in (([[0, 16, 32, 48]], 2),        # four pages for three slots
                      ([[0, 16, 20 * 16, -1]], 4)):  # a position beyond max_pages
        with pytest.raises(dsa.DSAError) as e:
            dsa.dsa_tier_plan(st, torch.tensor(bad, dtype=torch.int32), qo, cp, page_table=pt)
        assert e.value.status == code
        assert torch.equal(st, snap)
    # copy list too short
    with pytest.raises(dsa.DSAError) as e:
        dsa.dsa_tier_plan(st, torch.tensor([[32, 48, -1, -1]], dtype=torch.int32), qo, cp[:1],
                          page_table=pt)
    assert e.value.status == 6 and torch.equal(st, snap)
    # the same step then runs and matches the oracle
    tier = O.TierOracle(B, D, P)
    tier.step([[[0, 16, -1, -1]]])
    table, copies, *_ = tier.step([[[32, 48, -1, -1]]])
    n, _ = dsa.dsa_tier_plan(st, torch.tensor([[32, 48, -1, -1]], dtype=torch.int32), qo, cp,
                             page_table=pt)
    assert pt.tolist() == table and [tuple(x) for x in cp[:n].tolist()] == copies


def test_tier_state_sizes():
    assert dsa.dsa_tier_state_bytes(0, 4, 4) == 0
    assert dsa.dsa_tier_state_bytes(1, 0, 4) == 0
    assert dsa.dsa_tier_state_bytes(4, 6144, 65536) >= 4 * (6144 * 12 + 65536 * 12)
