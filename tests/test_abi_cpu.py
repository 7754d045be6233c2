"""The C-ABI library loads without a GPU, exports every declared symbol, and
rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

import sparse_attention_decode_lightning_b200 as dsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    from sparse_attention_decode_lightning_b200.build import build
    build()


def declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = declared()
    assert len(names) >= 9
    out = subprocess.run(["nm", "-D", "--defined-only", dsa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(l.split()[-1] for l in out.splitlines() if l.strip())
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    # the binding wraps exactly the declared entry points
    assert set(dsa.SIGNATURES) == set(names)


def test_library_loads_and_reports_version_and_status_names():
    L = dsa.lib()
    assert L.dsa_version() == 300
    for code, name in dsa.STATUS.items():
        assert dsa.dsa_status_string(code) == name
    assert dsa.dsa_status_string(99) == "DSA_ERR_UNKNOWN"


def test_split_choice():
    f = dsa.dsa_choose_splits
    assert f(0, 2048, 0) == 0 and f(1, 0, 0) == 0 and f(1, 2048, 33) == 0
    assert f(32, 2048, 5) == 5 and f(4, 2048, 16) == 16
    assert f(1, 8, 16) == 8                      # never more parts than tokens
    # the library's choice: 32 queries on 74 SM pairs -> 2 parts (64 units, 86%)
    assert f(32, 2048, 0) == 2
    assert f(128, 2048, 0) == 1 and f(74, 2048, 0) == 1
    for q in (1, 3, 16, 40, 500):
        s = f(q, 2048, 0)
        assert 1 <= s <= 16 and 2048 // s >= 64


def test_mla_group_plan():
    plan = dsa.dsa_mla_group_plan
    assert plan(0, 2048) is None and plan(10, 0) is None and plan(10, 4096) is None
    # fewer units than SM pairs: one wave, nothing split
    assert plan(64, 2048) == (64, 0, 1)
    assert plan(74, 2048) == (74, 0, 1)
    # IndexShare, 4 layers x 64 queries: three full waves, the last 34 units in 2 splits
    assert plan(256, 2048) == (222, 34, 2)
    assert plan(80, 2048) == (74, 6, 12)
    assert plan(100, 2048) == (74, 26, 2)
    assert plan(111, 2048) == (74, 37, 2)
    # a last wave more than half full runs whole
    assert plan(112, 2048) == (112, 0, 1)
    assert plan(128, 2048) == (128, 0, 1)
    # splits capped at DSA_MAX_SPLITS (32) and at one split per 64 selected tokens
    assert plan(150, 2048) == (148, 2, 32)
    assert plan(150, 256) == (148, 2, 4)
    assert plan(75, 64) == (75, 0, 1)
    for units in range(1, 600):
        head, tail, ts = plan(units, 2048)
        assert head + tail == units and head % 74 == 0 or tail == 0
        assert tail * ts <= 74


def test_workspace_bytes_arithmetic():
    f = dsa.dsa_workspace_bytes
    assert f(0, 10, 2048, 0) == 0
    assert f(1, 0, 2048, 0) == 0
    assert f(1, 10, 4096, 0) == 0
    assert f(1, 10, 2048, 33) == 0
    small = f(1, 8192, 2048, 1)
    # error flag + fp32 score row + one partial output and its LSE row
    assert small >= 256 + 8192 * 4 + 128 * 512 * 4 + 128 * 4
    assert f(32, 131072, 2048, 1) >= 32 * 131072 * 4
    # per key, nothing beyond the fp32 score and the fused selector's candidate
    # room (1/16 of a row of u64 keys)
    assert f(32, 131072, 2048, 1) < 32 * 131072 * 4 + (64 << 20)
    # every documented region fits: error word, scores [Q, ld], one split's
    # partials, and the fused selector's u32 histograms [Q, 4096], counters
    # [Q, 4] and candidate lists [Q, cap], cap = max_len/16 clamped to 4096-65536
    for Q, L in ((1, 8192), (32, 131072), (4, 1 << 20), (3, 1000)):
        cap = min(max(L // 16, 4096), 65536)
        ld = (L + 63) // 64 * 64
        base = 256 + Q * ld * 4 + Q * 128 * 512 * 4 + Q * 128 * 4
        assert f(Q, L, 2048, 1) >= base + Q * 4096 * 4 + Q * 16 + Q * cap * 8, (Q, L)
    assert f(4, 1 << 20, 2048, 16) > f(4, 1 << 20, 2048, 1)
    assert f(4, 1 << 20, 2048, 16) - f(4, 1 << 20, 2048, 1) >= 4 * 15 * 128 * 512 * 4


def test_host_checks_reject_bad_arguments_without_a_device():
    L = dsa.lib()
    P = ctypes.c_void_p
    fake = P(1 << 20)          # never dereferenced: checks fail first
    null = P(0)
    # null pointers
    assert L.dsa_indexer_topk(null, fake, fake, 100, fake, fake, fake, 1, 1, 64, 100, 2048, 0, fake,
                              null, fake, 1 << 30, null) == 1
    # top-k above the supported maximum
    assert L.dsa_indexer_topk(fake, fake, fake, 100, fake, fake, fake, 1, 1, 64, 100, 4096, 0, fake,
                              null, fake, 1 << 30, null) == 2
    # more queries than sequences allow
    assert L.dsa_indexer_topk(fake, fake, fake, 100, fake, fake, fake, 1, 9, 64, 100, 2048, 0, fake,
                              null, fake, 1 << 30, null) == 2
    # misaligned pointer
    assert L.dsa_indexer_topk(P((1 << 20) + 4), fake, fake, 100, fake, fake, fake, 1, 1, 64, 100,
                              2048, 0, fake, null, fake, 1 << 30, null) == 1
    # indexer head counts other than 64 (DeepSeek-V3.2) and 32 (GLM-5.2)
    for hi, want in ((48, 2), (128, 2), (0, 2)):
        assert L.dsa_indexer_topk(fake, fake, fake, 100, fake, fake, fake, 1, 1, hi, 100, 2048, 0,
                                  fake, null, fake, 1 << 30, null) == want
    # workspace too small
    assert L.dsa_indexer_topk(fake, fake, fake, 100, fake, fake, fake, 1, 1, 64, 100, 2048, 0, fake,
                              null, fake, 16, null) == 6
    # the fused form checks the same way
    for fn in (L.dsa_indexer_topk, L.dsa_indexer_topk_fused):
        assert fn(null, fake, fake, 100, fake, fake, fake, 1, 1, 64, 100, 2048, 0, fake,
                  null, fake, 1 << 30, null) == 1
        assert fn(fake, fake, fake, 100, fake, fake, fake, 1, 1, 48, 100, 2048, 0, fake,
                  null, fake, 1 << 30, null) == 2
        assert fn(fake, fake, fake, 100, fake, fake, fake, 1, 1, 64, 100, 2048, 0, fake,
                  null, fake, 16, null) == 6
    # sparse MLA: bad scale, bad split count, null page table
    assert L.dsa_sparse_mla_decode(fake, fake, 10, 64, fake, 4, fake, fake, fake, 1, 1, 128, 2048,
                                   ctypes.c_float(0.0), 0, fake, fake, fake, 1 << 30, null) == 1
    assert L.dsa_sparse_mla_decode(fake, fake, 10, 64, fake, 4, fake, fake, fake, 1, 1, 128, 2048,
                                   ctypes.c_float(0.07), 33, fake, fake, fake, 1 << 30, null) == 2
    assert L.dsa_sparse_mla_decode(fake, fake, 10, 64, null, 4, fake, fake, fake, 1, 1, 128, 2048,
                                   ctypes.c_float(0.07), 0, fake, fake, fake, 1 << 30, null) == 1
    # MLA head counts other than 128 (DeepSeek-V3.2) and 64 (GLM-5.2)
    for h in (32, 96, 256):
        assert L.dsa_sparse_mla_decode(fake, fake, 10, 64, fake, 4, fake, fake, fake, 1, 1, h, 2048,
                                       ctypes.c_float(0.07), 0, fake, fake, fake, 1 << 30,
                                       null) == 2
        assert L.dsa_lse_combine(fake, fake, 1, 2, h, fake, fake, null) == 2
    # window mode: window without its tables, and more rows than the selector's maximum
    assert L.dsa_sparse_mla_decode_window(fake, fake, 10, 64, fake, 4, null, 4, fake, fake, fake,
                                          fake, 1, 1, 128, 512, 128, ctypes.c_float(0.07), 0,
                                          fake, fake, fake, 1 << 30, null) == 1
    assert L.dsa_sparse_mla_decode_window(fake, fake, 10, 64, fake, 4, fake, 4, fake, fake, fake,
                                          fake, 1, 1, 128, 2048, 128, ctypes.c_float(0.07), 0,
                                          fake, fake, fake, 1 << 30, null) == 2
    # decode step: no layers, zero share group
    PP = ctypes.POINTER(ctypes.c_void_p)
    arr = (ctypes.c_void_p * 1)(1 << 20)
    assert L.dsa_decode_step(0, 1, 0, arr, arr, arr, 100, fake, fake, fake, 1, 1, 128, 64, 100,
                             2048, arr, arr, 10, 64, arr, 4, ctypes.c_float(0.07), 0, arr, arr, fake,
                             fake, 1 << 30, null) == 1
    assert L.dsa_decode_step(1, 0, 0, arr, arr, arr, 100, fake, fake, fake, 1, 1, 128, 64, 100,
                             2048, arr, arr, 10, 64, arr, 4, ctypes.c_float(0.07), 0, arr, arr, fake,
                             fake, 1 << 30, null) == 1
    # check_error without a workspace
    assert L.dsa_check_error(null, null) == 1


def test_binding_refuses_host_tensors():
    import torch
    with pytest.raises(ValueError):
        dsa._ptr(torch.zeros(4))
