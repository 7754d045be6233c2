"""The DSA decode workloads, named by what they are and their sizes.

Shapes follow the DeepSeek-V3.2 DSA description (DeepSeek-V3.2 section of the
2026 architecture survey page: lightning indexer with 64 heads of dim 128 in
FP8, top-k = 2048 over prior tokens, MLA in MQA mode with a 512-d latent plus a
64-d RoPE part, 128 heads) and the GLM-5.2 IndexShare / MTP descriptions
(GLM-5.2 section of the same survey; MTP section of the GLM-5.2 inference
page).  The glm52_* workloads take GLM-5.2's shapes from the same survey's
GLM-5.2 section: 64 MLA heads with qk head dim 192 + 64 RoPE (softmax scale
1/sqrt(256)) over the same 512 + 64 latent, and a 32-head FP8 indexer.
"""
from dataclasses import dataclass, field
from typing import Optional, Tuple


@dataclass(frozen=True)
class Workload:
    name: str
    B: int                      # sequences
    T: int                      # query positions per sequence (1 decode, 8 MTP verify)
    L: int                      # context length (keys already cached before the step)
    L_range: Optional[Tuple[int, int]] = None   # ragged: per-sequence L ~ U[lo, hi]
    appended: int = 0           # MTP: query positions appended causally after the context
    n_layers: int = 1           # sparse layers in the step
    index_share: int = 1        # layers per indexer group (4 = IndexShare)
    mtp_index_share: bool = False  # position 0's top-k reused by positions 1..T-1
    num_splits: int = 0         # 0 = let the library choose; >0 = split-K partitions
    paged_permuted: bool = True  # pages of 64 randomly permuted in the pool
    topk: int = 2048
    heads: int = 128            # MLA heads (GLM-5.2: 64)
    idx_heads: int = 64         # indexer heads (GLM-5.2: 32)
    qk_head_dim: int = 192      # softmax scale 1/sqrt(qk_head_dim) (GLM-5.2: 192 + 64 = 256)
    note: str = ""

    @property
    def Q(self) -> int:
        return self.B * self.T


WORKLOADS = {
    w.name: w
    for w in [
        Workload("decode_b1_ctx8k", B=1, T=1, L=8192, paged_permuted=False,
                 note="tiny one-layer decode, contiguous cache (identity page table)"),
        Workload("decode_b32_ctx128k", B=32, T=1, L=131072,
                 note="batch-32 decode at 128K, pages of 64 permuted in the pool"),
        Workload("indexshare4_b64_ctx16k_128k", B=64, T=1, L=131072, L_range=(16384, 131072),
                 n_layers=4, index_share=4,
                 note="IndexShare: indexer on layer 1, layers 2-4 reuse its top-k"),
        Workload("mtp_verify_b16_t8_ctx128k", B=16, T=8, L=131072, appended=8,
                 note="MTP verify: 8 causal positions per sequence, per-position top-k"),
        Workload("mtp_verify_reuse_b16_t8_ctx128k", B=16, T=8, L=131072, appended=8,
                 mtp_index_share=True,
                 note="MTP verify with position 0's top-k reused by the drafts"),
        Workload("decode_b4_ctx1m_split16", B=4, T=1, L=1048576, num_splits=16,
                 note="1M-context decode, 16-way split-K plus LSE combine"),
        Workload("glm52_decode_b32_ctx128k", B=32, T=1, L=131072,
                 heads=64, idx_heads=32, qk_head_dim=256,
                 note="GLM-5.2 shapes: batch-32 decode at 128K"),
        Workload("glm52_indexshare4_b64_ctx16k_128k", B=64, T=1, L=131072,
                 L_range=(16384, 131072), n_layers=4, index_share=4,
                 heads=64, idx_heads=32, qk_head_dim=256,
                 note="GLM-5.2 shapes with its IndexShare: one indexer per 4 layers"),
        Workload("glm52_decode_b4_ctx1m_split16", B=4, T=1, L=1048576, num_splits=16,
                 heads=64, idx_heads=32, qk_head_dim=256,
                 note="GLM-5.2 shapes at its 1M context, 16-way split-K"),
    ]
}


def get_workload(name: str, **overrides) -> Workload:
    """Look up a workload; keyword overrides give scaled-down copies for tests."""
    w = WORKLOADS[name]
    if overrides:
        d = dict(w.__dict__)
        d.update(overrides)
        w = Workload(**d)
    return w
