"""Device-side failure detection without a GPU fault: a bounded wait that
nothing completes runs out after its limit, raises the timeout flag, and the
kernel returns; the host reads DSA_ERR_TIMEOUT from the error word and the
context stays usable for the next call.  The waiting kernel holds no copy in
flight, no tensor memory and no peer CTA."""
import time

import pytest
import torch

import sparse_attention_decode_lightning_b200 as dsa
from synth import get_workload, make_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"
DSA_ERR_TIMEOUT = 5


def test_expired_bounded_wait_is_reported_and_the_context_survives():
    ws = torch.zeros(1 << 12, dtype=torch.uint8, device=DEV)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    dsa.dsa_selftest_bounded_wait(2000, ws)            # two waits of 2 ms each
    with pytest.raises(dsa.DSAError) as e:
        dsa.dsa_check_error(ws)
    elapsed = time.perf_counter() - t0
    assert e.value.status == DSA_ERR_TIMEOUT
    assert elapsed >= 0.004                            # both waits ran their limit
    dsa.dsa_check_error(ws)                            # the flag was cleared

    # the context still runs the library's kernels
    inp = make_inputs(get_workload("decode_b1_ctx8k"), seed=1, device=DEV)
    idx = torch.arange(2048, dtype=torch.int32, device=DEV)[None] * 3
    out = torch.empty(1, 128, 512, device=DEV)
    lse = torch.empty(1, 128, device=DEV)
    ws2 = dsa.workspace(1, 1, 2048, 0)
    dsa.dsa_sparse_mla_decode(inp.layers[0]["q"], inp.layers[0]["pool"], inp.page_table, inp.q_offsets,
                              inp.q_vis, idx, inp.B, inp.scale, out, lse, ws2)
    dsa.dsa_check_error(ws2)
    assert bool(torch.isfinite(out).all()) and bool(torch.isfinite(lse).all())


def test_selftest_refuses_limits_beyond_the_library_limit():
    ws = torch.zeros(1 << 12, dtype=torch.uint8, device=DEV)
    for bad in (0, 2000001):
        with pytest.raises(dsa.DSAError):
            dsa.dsa_selftest_bounded_wait(bad, ws)
