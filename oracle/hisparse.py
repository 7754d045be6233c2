"""Plain CPU oracle of the two-tier (HiSparse) latent cache's bookkeeping.

TEST INFRASTRUCTURE ONLY: imported by the tests, never by the library.

Source: "GLM-5.2 推理部署" (inference deployment), section "HiSparse 的通信路径：
GPU↔CPU KV swap".  The full KV cache lives in pinned host memory; HBM holds a
buffer of hot slots, each one KV page of 16 tokens.  After the indexer has
chosen a step's top-K positions:
  1. top-K miss detection: the chosen positions are compared with the device
     buffer and the pages not in it are found;
  2. LRU eviction: victims are taken from the device buffer, least recently
     used first;
  3. H2D fetch: the page table is updated and the missing entries are pulled
     from host memory.

Readings where the page is silent (the library takes the same ones):
  * each sequence owns `dev_slots` slots; a slot holds one page of 16 tokens;
  * "used" is counted per step: every page a step selects is used at that step
    (the K positions of a step form a set, with no order among them);
  * among the slots not selected at this step, the one with the oldest last use
    is evicted first; slots never used are older than any used one; equal ages
    go to the lower slot index;
  * a step's misses are placed in ascending page order into the victims in
    eviction order;
  * a step that selects more distinct pages of a sequence than it has slots
    cannot be served and is refused.

Written with Python dicts and lists, one step at a time, in the page's order.
"""
from typing import Dict, List, Sequence, Tuple

PAGE_TOKENS = 16


class TierOverflow(Exception):
    """A step selected more distinct pages of a sequence than its slots."""


class TierOracle:
    def __init__(self, B: int, dev_slots: int, max_pages: int):
        self.B, self.D, self.P = B, dev_slots, max_pages
        self.slot_of: List[Dict[int, int]] = [dict() for _ in range(B)]      # page -> slot
        self.page_in: List[List[int]] = [[-1] * dev_slots for _ in range(B)]  # slot -> page
        self.last_use: List[List[int]] = [[-1] * dev_slots for _ in range(B)]
        self.step_no = 0

    def step(self, rows_per_seq: Sequence[Sequence[Sequence[int]]]):
        """rows_per_seq[b]: the index rows of sequence b's queries at this step.

        Returns (page_table [B][P] of device pool pages or -1, copies [(host
        page fetched, device page it goes to, host page evicted from that
        slot or -1)], hits, misses, evictions)."""
        t = self.step_no
        # 1. miss detection
        needed, missing = [], []
        for b in range(self.B):
            pages = sorted({pos // PAGE_TOKENS for row in rows_per_seq[b] for pos in row if pos >= 0})
            if len(pages) > self.D:
                raise TierOverflow(b)
            needed.append(pages)
            missing.append([p for p in pages if p not in self.slot_of[b]])
        hits = sum(len(needed[b]) - len(missing[b]) for b in range(self.B))
        # hits are used at this step
        for b in range(self.B):
            for p in needed[b]:
                if p in self.slot_of[b]:
                    self.last_use[b][self.slot_of[b][p]] = t
        # 2. LRU eviction and 3. fetch plan
        copies, evictions = [], 0
        for b in range(self.B):
            if not missing[b]:
                continue
            chosen_now = set(needed[b])
            free_or_old = [s for s in range(self.D) if self.page_in[b][s] not in chosen_now]
            victims = sorted(free_or_old, key=lambda s: (self.last_use[b][s], s))[:len(missing[b])]
            for p, s in zip(missing[b], victims):
                old = self.page_in[b][s]
                if old >= 0:
                    del self.slot_of[b][old]
                    evictions += 1
                self.page_in[b][s] = p
                self.slot_of[b][p] = s
                self.last_use[b][s] = t
                copies.append((b * self.P + p, b * self.D + s, b * self.P + old if old >= 0 else -1))
        self.step_no += 1
        table = [[-1] * self.P for _ in range(self.B)]
        for b in range(self.B):
            for p, s in self.slot_of[b].items():
                table[b][p] = b * self.D + s
        return table, copies, hits, sum(len(m) for m in missing), evictions
