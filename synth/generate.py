"""Seeded generator of DSA decode inputs.

Value recipe (the same for every workload):
  * indexer queries q_idx [Q,64,128] and indexer keys K [sum L,128]: N(0,1)
    samples clamped to +-448 and rounded to FP8 e4m3 (round to nearest even),
    scale 1, stored as raw e4m3 bytes;
  * indexer head weights w [Q,64]: N(0,1)/8 in fp32;
  * MLA queries q [Q,128,576] and latent cache rows [.,576]: N(0,1) rounded to
    bf16 (round to nearest even), stored as bf16;
  * paged latent pool [num_pages,64,576] with a page table [B,max_pages]; pages
    either identity-ordered or randomly permuted (seeded), unused table slots -1;
  * ragged context lengths: integers uniform in [lo, hi].

Every tensor draws from its own torch.Generator, seeded from (seed, tensor
name) via numpy's SeedSequence, on the requested device.  The same seed gives
the same bytes on the same device type; CPU and CUDA streams differ, so a run
always hands one set of bytes to both the oracle and the library.
"""
from dataclasses import dataclass, field
from typing import List, Dict, Optional
import math
import zlib

import numpy as np
import torch

from .workloads import Workload

PAGE = 64          # latent-cache page size (tokens)
D = 576            # latent row: 512 latent + 64 rope
DV = 512           # value dims
DI = 128           # indexer head dim
# head counts come from the workload (128 / 64 DeepSeek-V3.2, 64 / 32 GLM-5.2)
FP8_MAX = 448.0


def _gen(seed: int, name: str, device) -> torch.Generator:
    ss = np.random.SeedSequence([int(seed), zlib.crc32(name.encode())])
    s = int(ss.generate_state(1, dtype=np.uint64)[0] & ((1 << 63) - 1))
    g = torch.Generator(device=device)
    g.manual_seed(s)
    return g


def _randn_e4m3(shape, g, device, chunk_rows: int = 1 << 20) -> torch.Tensor:
    """N(0,1) -> clamp to the e4m3 range -> e4m3 bytes (uint8)."""
    out = torch.empty(shape, dtype=torch.uint8, device=device)
    flat = out.view(shape[0], -1)
    for r0 in range(0, shape[0], chunk_rows):
        r1 = min(shape[0], r0 + chunk_rows)
        x = torch.randn((r1 - r0, flat.shape[1]), generator=g, device=device, dtype=torch.float32)
        x.clamp_(-FP8_MAX, FP8_MAX)
        flat[r0:r1] = x.to(torch.float8_e4m3fn).view(torch.uint8)
    return out


def _randn_bf16(shape, g, device) -> torch.Tensor:
    x = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = x.view(-1)
    step = 1 << 28
    for i in range(0, flat.numel(), step):
        j = min(flat.numel(), i + step)
        flat[i:j] = torch.randn(j - i, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    return x


@dataclass
class DSAInputs:
    workload: Workload
    seed: int
    device: str
    B: int
    T: int
    Q: int
    topk: int
    scale: float
    num_splits: int
    heads: int                      # MLA heads
    idx_heads: int                  # indexer heads
    n_layers: int
    index_share: int
    mtp_index_share: bool
    seq_lens: np.ndarray            # int64 [B] keys cached per sequence (incl. appended)
    seq_offsets: torch.Tensor       # int64 [B+1]
    q_offsets: torch.Tensor         # int32 [B+1]
    q_vis: torch.Tensor             # int32 [Q] keys visible to each query
    total_keys: int
    max_len: int
    page_table: torch.Tensor        # int32 [B, max_pages]
    num_pages: int
    max_pages: int
    indexer: List[Dict[str, torch.Tensor]]   # per indexer group: q_idx, w, k_idx
    layers: List[Dict[str, torch.Tensor]]    # per layer: q, pool

    def indexer_group_of(self, layer: int) -> int:
        return layer // self.index_share

    def to_host(self) -> "DSAInputs":
        """A copy whose tensors live in host memory (for the oracle)."""
        def h(t):
            return t.cpu() if isinstance(t, torch.Tensor) else t
        return DSAInputs(
            **{**self.__dict__,
               "device": "cpu",
               "seq_offsets": h(self.seq_offsets), "q_offsets": h(self.q_offsets),
               "q_vis": h(self.q_vis), "page_table": h(self.page_table),
               "indexer": [{k: h(v) for k, v in d.items()} for d in self.indexer],
               "layers": [{k: h(v) for k, v in d.items()} for d in self.layers]})


def make_inputs(w: Workload, seed: int = 0, device="cpu", layers_to_make: Optional[int] = None) -> DSAInputs:
    """Draw every input tensor of workload `w` on `device`."""
    dev = torch.device(device)
    B, T = w.B, w.T
    Q = B * T
    # context lengths
    if w.L_range is not None:
        lo, hi = w.L_range
        g = _gen(seed, "lengths", "cpu")
        ctx = torch.randint(lo, hi + 1, (B,), generator=g, dtype=torch.int64).numpy()
    else:
        ctx = np.full(B, w.L, dtype=np.int64)
    seq_lens = ctx + w.appended
    seq_offsets = np.zeros(B + 1, dtype=np.int64)
    seq_offsets[1:] = np.cumsum(seq_lens)
    total_keys = int(seq_offsets[-1])
    # visible keys per query: decode sees its whole context; MTP position t
    # (at absolute position ctx + t) sees keys 0 .. ctx + t.
    q_vis = np.zeros(Q, dtype=np.int32)
    for b in range(B):
        for t in range(T):
            q_vis[b * T + t] = ctx[b] + t + 1 if w.appended else ctx[b]
    q_offsets = (np.arange(B + 1, dtype=np.int64) * T).astype(np.int32)
    # paged latent pool
    pages_per_seq = (seq_lens + PAGE - 1) // PAGE
    num_pages = int(pages_per_seq.sum())
    max_pages = int(pages_per_seq.max())
    if w.paged_permuted:
        g = _gen(seed, "page_perm", "cpu")
        perm = torch.randperm(num_pages, generator=g).numpy().astype(np.int64)
    else:
        perm = np.arange(num_pages, dtype=np.int64)
    page_table = np.full((B, max_pages), -1, dtype=np.int32)
    p0 = 0
    for b in range(B):
        n = int(pages_per_seq[b])
        page_table[b, :n] = perm[p0:p0 + n]
        p0 += n

    n_groups = (w.n_layers + w.index_share - 1) // w.index_share
    indexer = []
    for gi in range(n_groups):
        indexer.append({
            "q_idx": _randn_e4m3((Q, w.idx_heads, DI), _gen(seed, f"q_idx{gi}", dev), dev),
            "w": torch.randn((Q, w.idx_heads), generator=_gen(seed, f"w{gi}", dev), device=dev,
                             dtype=torch.float32) / 8.0,
            "k_idx": _randn_e4m3((total_keys, DI), _gen(seed, f"k_idx{gi}", dev), dev),
        })
    n_make = w.n_layers if layers_to_make is None else layers_to_make
    layers = []
    for li in range(n_make):
        layers.append({
            "q": _randn_bf16((Q, w.heads, D), _gen(seed, f"q{li}", dev), dev),
            "pool": _randn_bf16((num_pages, PAGE, D), _gen(seed, f"pool{li}", dev), dev),
        })
    return DSAInputs(
        workload=w, seed=seed, device=str(dev), B=B, T=T, Q=Q, topk=w.topk,
        scale=1.0 / math.sqrt(float(w.qk_head_dim)), num_splits=w.num_splits,
        heads=w.heads, idx_heads=w.idx_heads, n_layers=w.n_layers,
        index_share=w.index_share, mtp_index_share=w.mtp_index_share,
        seq_lens=seq_lens, seq_offsets=torch.from_numpy(seq_offsets).to(dev),
        q_offsets=torch.from_numpy(q_offsets).to(dev), q_vis=torch.from_numpy(q_vis).to(dev),
        total_keys=total_keys, max_len=int(seq_lens.max()),
        page_table=torch.from_numpy(page_table).to(dev), num_pages=num_pages,
        max_pages=max_pages, indexer=indexer, layers=layers)
