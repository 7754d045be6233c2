"""Driving the library's decode step from a DSAInputs (device tensors)."""
import torch

import sparse_attention_decode_lightning_b200 as dsa

DEV = "cuda"


def run_decode_step(inp, num_splits=None, ws=None):
    n, G, Q = inp.n_layers, inp.index_share, inp.Q
    qi = [inp.indexer[l // G]["q_idx"] if l % G == 0 else None for l in range(n)]
    wl = [inp.indexer[l // G]["w"] if l % G == 0 else None for l in range(n)]
    kl = [inp.indexer[l // G]["k_idx"] if l % G == 0 else None for l in range(n)]
    outs = [torch.empty(Q, inp.heads, 512, dtype=torch.float32, device=DEV) for _ in range(n)]
    lses = [torch.empty(Q, inp.heads, dtype=torch.float32, device=DEV) for _ in range(n)]
    ng = (n + G - 1) // G
    idx = torch.empty(ng, Q, inp.topk, dtype=torch.int32, device=DEV)
    S = inp.num_splits if num_splits is None else num_splits
    if ws is None:
        ws = dsa.workspace(Q, inp.max_len, inp.topk, S)
    dsa.dsa_decode_step(qi, wl, kl, inp.seq_offsets, inp.q_offsets, inp.q_vis, inp.B, inp.max_len,
                        inp.topk, [L["q"] for L in inp.layers], [L["pool"] for L in inp.layers],
                        [inp.page_table] * n, inp.scale, outs, lses, idx, ws, index_share=G,
                        mtp_index_share=inp.mtp_index_share, num_splits=S)
    dsa.dsa_check_error(ws)
    return outs, lses, idx
