"""Glue between the seeded generator (torch tensors) and the numpy oracle."""
import numpy as np
import torch


def np_bits(t: torch.Tensor) -> np.ndarray:
    """Raw bytes of a tensor as a numpy array (bf16 -> uint16 bit patterns)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.uint8:
        return t.numpy()
    return t.numpy()


def oracle_inputs(inp) -> dict:
    """The oracle's view of a DSAInputs (host numpy arrays)."""
    return {
        "B": inp.B, "T": inp.T, "topk": inp.topk, "scale": inp.scale,
        "num_splits": inp.num_splits, "index_share": inp.index_share,
        "mtp_index_share": inp.mtp_index_share, "n_layers": inp.n_layers,
        "seq_offsets": np_bits(inp.seq_offsets), "q_vis": np_bits(inp.q_vis),
        "page_table": np_bits(inp.page_table),
        "indexer": [{k: np_bits(v) for k, v in d.items()} for d in inp.indexer],
        "layers": [{k: np_bits(v) for k, v in d.items()} for d in inp.layers],
    }


def rms(x: np.ndarray) -> float:
    return float(np.sqrt(np.mean(np.square(x, dtype=np.float64))))
