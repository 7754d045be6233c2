"""Plain, slow, fp64 CPU oracle of DSA decode.

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the library.  Nothing here is blocked,
fused or reordered beyond the definitions it restates; numpy's matmul, sort and
exp serve as library primitives.

Sources (pages are cited by title and section):
  [ARCH]  "大语言模型结构总览" (LLM structure overview), section 2.2 DeepSeek-V3.2:
          DSA is a select-then-attend pipeline; a lightning indexer (64 heads,
          head dim 128, FP8, parameters separate from the backbone) gives every
          prior token a scalar score; a token selector keeps the k = 2048
          highest-scoring tokens per query; attention runs on MLA in MQA mode
          over those tokens only; paged and non-paged kernels exist.
  [ARCH-2.1] same page, section 2.1 DeepSeek-V3: MLA caches one latent per
          token, kv rank 512 plus a 64-d RoPE part; 128 attention heads.
  [ARCH-7.2] same page, section 7.2 GLM-5.2 and Figure 7-2: IndexShare, one
          indexer per 4 sparse layers whose top-k indices the next 3 layers
          reuse; causal top-2048.  GLM-5.2's shapes: 64 MLA heads over a
          kv rank of 512 with a 64-d RoPE part, a 32-head FP8 indexer of head
          dim 128.  Every function below takes its head counts from the
          arrays it is given, so both models' shapes go through the same code.
  [ARCH-2.3] same page, section 2.3 DeepSeek-V4: compressed sparse attention
          (CSA) keeps the top-k of a 4x compressed KV cache plus a 128-token
          sliding window of raw tokens.
  [GLM-INF] "GLM-5.2 推理部署" (inference deployment), MTP draft + verify flow:
          top-K = 2048 indices computed at draft step 1 and reused by later
          steps; verify appends the drafts and runs one prefill-style forward.

Readings where the pages are silent (each is listed in the design notes):
  * indexer score I(q,s) = sum_h w[q,h] * ReLU(q_idx[q,h,:] . K[s,:]), with
    e4m3 inputs at scale 1 and fp32 head weights;
  * ties in the selector go to the lower token index; with fewer visible
    tokens than k all of them are kept and the rest of the list is -1;
  * the attention value is the first 512 dims of the selected 576-d latent
    row; the softmax scale multiplies the full 576-d dot product, and the
    log-sum-exp is the natural log of sum_j exp(scale * q.c_j);
  * split-K: the context is cut into S contiguous equal ranges, each attends to
    the selected tokens inside it, and the partial results are merged exactly
    through their log-sum-exps; an empty range has LSE = -inf and weight 0;
  * CSA window: a query that sees win_vis raw tokens attends to the last
    `window` of them (fewer when win_vis < window), in the same softmax as its
    selected compressed entries; how entries are compressed is learned and
    outside this path, so the compressed rows are inputs.
"""
import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

PAGE = 64
H = 128
D = 576
DV = 512
HI = 64
DI = 128

__all__ = [
    "e4m3_table", "e4m3_decode", "bf16_decode",
    "indexer_scores", "topk_select", "latent_rows", "latent_rows_e4m3",
    "sparse_mla", "sparse_mla_split", "lse_combine",
    "csa_window_positions", "csa_window_attention",
    "query_step", "decode_step",
]


# --------------------------------------------------------------------------
# Input decoding (independent of any GPU-side conversion)
# --------------------------------------------------------------------------
def _e4m3_value(code: int) -> float:
    """OCP 8-bit floating point, E4M3 variant: 1 sign bit, 4 exponent bits with
    bias 7, 3 mantissa bits; exponent field 0 is subnormal (m/8 * 2^-6); no
    infinities; S.1111.111 is NaN; the largest finite magnitude is 448."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * (m / 8.0) * 2.0 ** -6
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


_E4M3 = np.array([_e4m3_value(c) for c in range(256)], dtype=np.float64)


def e4m3_table() -> np.ndarray:
    return _E4M3.copy()


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """e4m3 bytes -> float64 (exact)."""
    return _E4M3[np.asarray(codes, dtype=np.uint8)]


def bf16_decode(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16/int16) -> float64 (exact): a bf16 value is the
    upper half of an IEEE binary32 word."""
    u = np.asarray(bits).view(np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# Stage 1: lightning indexer  [ARCH]
# --------------------------------------------------------------------------
def indexer_scores(q_idx: np.ndarray, w: np.ndarray, keys: np.ndarray) -> np.ndarray:
    """Scores of every key for one query.

    q_idx: e4m3 bytes [HI,128] (one query's indexer heads: 64, or GLM-5.2's 32)
    w:     float [HI] head weights
    keys:  e4m3 bytes [n,128] (the query's visible indexer keys)
    returns float64 [n]: I[s] = sum_h w[h] * max(0, sum_d q[h,d] * K[s,d])
    """
    qf = e4m3_decode(q_idx)                      # [HI,128]
    kf = e4m3_decode(keys)                       # [n,128]
    dots = kf @ qf.T                             # [n,HI]  per-head q.k
    relu = np.maximum(dots, 0.0)
    return relu @ np.asarray(w, dtype=np.float64)


# --------------------------------------------------------------------------
# Stage 2: token selector  [ARCH], [ARCH-7.2]
# --------------------------------------------------------------------------
def topk_select(scores: np.ndarray, k: int) -> np.ndarray:
    """The k highest-scoring token positions (ties -> lower position).

    Full stable sort by (-score, position); keeps min(k, n) positions and pads
    the list with -1 up to k.  Returned in sort order (best first).
    """
    n = scores.shape[0]
    order = np.lexsort((np.arange(n), -np.asarray(scores, dtype=np.float64)))
    keep = order[: min(k, n)].astype(np.int64)
    out = np.full(k, -1, dtype=np.int64)
    out[: keep.shape[0]] = keep
    return out


# --------------------------------------------------------------------------
# Stage 3: sparse MLA in MQA (absorbed) mode  [ARCH], [ARCH-2.1]
# --------------------------------------------------------------------------
def latent_rows(pool: np.ndarray, page_table_row: np.ndarray, positions: np.ndarray) -> np.ndarray:
    """Gather 576-d latent rows for token positions of one sequence through its
    page table (page size 64) and decode them to float64 [n,576]."""
    positions = np.asarray(positions, dtype=np.int64)
    pages = np.asarray(page_table_row, dtype=np.int64)[positions // PAGE]
    return bf16_decode(pool[pages, positions % PAGE])


def latent_rows_e4m3(pool: np.ndarray, page_table_row: np.ndarray, positions: np.ndarray,
                     kv_scale: float, page_size: int = PAGE) -> np.ndarray:
    """Selected rows of an FP8 latent cache (the deploy page's fp8_e4m3 KV cache,
    "GLM-5.2 推理部署"): e4m3 codes [P,page_size,576] through the page table,
    decoded exactly and multiplied by the cache's one scale, as float64 [n,576]."""
    positions = np.asarray(positions, dtype=np.int64)
    pages = np.asarray(page_table_row, dtype=np.int64)[positions // page_size]
    codes = pool[pages, positions % page_size]
    return e4m3_decode(codes) * float(kv_scale)


def sparse_mla(q: np.ndarray, rows: np.ndarray, scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """Attention of H heads (128, or GLM-5.2's 64) over n selected latent
    rows (one shared row per token serves every head).

    q:    float64 [H,576]
    rows: float64 [n,576]
    returns O float64 [H,512] = softmax_j(scale * q.c_j) @ c_j[:512]
            LSE float64 [H]   = ln sum_j exp(scale * q.c_j)
    With n = 0: O = 0 and LSE = -inf.
    """
    nh = q.shape[0]
    if rows.shape[0] == 0:
        return np.zeros((nh, DV)), np.full(nh, -np.inf)
    s = scale * (q @ rows.T)                     # [H,n]
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    p = e / l
    o = p @ rows[:, :DV]
    lse = m[:, 0] + np.log(l[:, 0])
    return o, lse


def lse_combine(o_parts: np.ndarray, lse_parts: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Exact merge of partial attentions over disjoint token sets:
    LSE = ln sum_c exp(LSE_c);  O = sum_c exp(LSE_c - LSE) * O_c.
    Parts with LSE_c = -inf get weight 0; if all are empty, O = 0, LSE = -inf."""
    lse_parts = np.asarray(lse_parts, dtype=np.float64)   # [S,H]
    m = lse_parts.max(axis=0)                              # [H]
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    wts = np.where(np.isfinite(lse_parts), np.exp(lse_parts - m_safe[None, :]), 0.0)  # [S,H]
    tot = wts.sum(axis=0)
    lse = np.where(finite, m_safe + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    o = np.einsum("sh,shd->hd", wts, o_parts)
    o = np.where(finite[:, None], o / np.where(tot > 0, tot, 1.0)[:, None], 0.0)
    return o, lse


def sparse_mla_split(q: np.ndarray, rows: np.ndarray, positions: np.ndarray, context: int,
                     num_splits: int, scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """Split-K form: cut [0, context) into num_splits contiguous equal ranges
    [c*context/S, (c+1)*context/S), attend within each, merge by LSE."""
    positions = np.asarray(positions, dtype=np.int64)
    o_parts = np.zeros((num_splits, q.shape[0], DV))
    lse_parts = np.full((num_splits, q.shape[0]), -np.inf)
    for c in range(num_splits):
        lo = (c * context) // num_splits
        hi = ((c + 1) * context) // num_splits
        sel = (positions >= lo) & (positions < hi)
        o_parts[c], lse_parts[c] = sparse_mla(q, rows[sel], scale)
    return lse_combine(o_parts, lse_parts)


# --------------------------------------------------------------------------
# DeepSeek-V4 CSA: selected compressed entries plus a raw sliding window
# [ARCH-2.3] "大语言模型结构总览", section 2.3 DeepSeek-V4: the KV cache is
# compressed 4x along the sequence, DSA selects the top-1024 (Pro) or top-512
# (Flash) compressed entries, and a 128-token sliding window of uncompressed
# tokens is attended as well, for locality.
# --------------------------------------------------------------------------
def csa_window_positions(win_vis: int, window: int) -> np.ndarray:
    """The raw tokens of a query's sliding window: the `window` most recent of
    the win_vis visible raw positions, win_vis-window .. win_vis-1, with the
    positions below 0 (a window that starts before the first token) left out."""
    lo = max(0, int(win_vis) - int(window))
    return np.arange(lo, int(win_vis), dtype=np.int64)


def csa_window_attention(q: np.ndarray, pool: np.ndarray, page_row_c: np.ndarray,
                         page_row_raw: np.ndarray, selected: np.ndarray, win_vis: int,
                         window: int, scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """One query of CSA decode attention: a single softmax over the selected
    compressed entries (positions of the compressed cache, through page_row_c)
    together with the raw window rows (through page_row_raw), both caches in
    the same latent pool.  q float64 [H,576]; returns (O [H,512], LSE [H])."""
    rows_c = latent_rows(pool, page_row_c, np.asarray(selected, dtype=np.int64))
    rows_w = latent_rows(pool, page_row_raw, csa_window_positions(win_vis, window))
    return sparse_mla(q, np.concatenate([rows_c, rows_w]), scale)


# --------------------------------------------------------------------------
# One query through the whole step; the whole step  [ARCH], [ARCH-7.2], [GLM-INF]
# --------------------------------------------------------------------------
def query_step(q_idx, w, keys_seq, vis: int, topk: int) -> Tuple[np.ndarray, np.ndarray]:
    """Indexer + selector for one query: returns (scores[vis], idx[topk])."""
    sc = indexer_scores(q_idx, w, keys_seq[:vis])
    return sc, topk_select(sc, topk)


def decode_step(inp: Dict, queries: Optional[Sequence[int]] = None,
                layers: Optional[Sequence[int]] = None) -> Dict:
    """The DSA decode step over host numpy inputs.

    inp keys (numpy arrays): B, T, topk, scale, num_splits, index_share,
      mtp_index_share, n_layers, seq_offsets[B+1], q_vis[Q], page_table[B,P],
      indexer: list per group of {q_idx[Q,HI,128] u8, w[Q,HI] f32, k_idx[N,128] u8},
      layers: list per layer of {q[Q,H,576] u16 bits, pool[P,64,576] u16 bits},
      with (H, HI) = (128, 64) for DeepSeek-V3.2 and (64, 32) for GLM-5.2.
    Layer l takes its indices from the indexer of group l // index_share
    (IndexShare); with mtp_index_share the first position of each sequence
    supplies the indices of all its positions (IndexShare on MTP).
    Returns {"idx": {(g,q): idx}, "scores": {(g,q): scores},
             "out": {(l,q): O}, "lse": {(l,q): LSE}} for the requested queries.
    """
    B, T = inp["B"], inp["T"]
    Q = B * T
    queries = list(range(Q)) if queries is None else list(queries)
    layers = list(range(inp["n_layers"])) if layers is None else list(layers)
    G = inp["index_share"]
    res = {"idx": {}, "scores": {}, "out": {}, "lse": {}}

    def idx_for(g: int, q: int) -> np.ndarray:
        src = (q // T) * T if inp["mtp_index_share"] else q
        if (g, src) not in res["idx"]:
            b = src // T
            ind = inp["indexer"][g]
            k0 = int(inp["seq_offsets"][b])
            keys = ind["k_idx"][k0:int(inp["seq_offsets"][b + 1])]
            sc, idx = query_step(ind["q_idx"][src], ind["w"][src], keys,
                                 int(inp["q_vis"][src]), inp["topk"])
            res["idx"][(g, src)] = idx
            res["scores"][(g, src)] = sc
        return res["idx"][(g, src)]

    for l in layers:
        g = l // G
        lay = inp["layers"][l]
        for q in queries:
            b = q // T
            idx = idx_for(g, q)
            res["idx"][(g, q)] = idx
            pos = idx[idx >= 0]
            rows = latent_rows(lay["pool"], inp["page_table"][b], pos)
            qf = bf16_decode(lay["q"][q])
            if inp["num_splits"] and inp["num_splits"] > 1:
                o, lse = sparse_mla_split(qf, rows, pos, int(inp["q_vis"][q]),
                                          inp["num_splits"], inp["scale"])
            else:
                o, lse = sparse_mla(qf, rows, inp["scale"])
            res["out"][(l, q)] = o
            res["lse"][(l, q)] = lse
    return res
