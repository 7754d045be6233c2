"""Pins of the fp64 CPU oracle against what the pages and the mathematics fix.

Each pin is chosen so that a plausible slip in the oracle (a dropped ReLU, a
missing softmax scale, a wrong tie order, a transposed operand, a lost split)
fails at least one of them; test_planted_mistakes_are_caught plants such slips
in a copy of the oracle and checks that.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from synth import get_workload, make_inputs
from tests._helpers import np_bits, oracle_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def _e4m3_bytes(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.clip(x, -448, 448).astype(np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


# ---------------------------------------------------------------- decoders
def test_e4m3_all_codes_match_torch():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.e4m3_table()
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()


def test_e4m3_ocp_spec_values():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "e4m3_ocp_values.txt"))
            if l.strip() and not l.startswith("#")]
    assert len(rows) >= 10
    for code, val in rows:
        got = O.e4m3_decode(np.array([int(code, 16)], dtype=np.uint8))[0]
        want = float(val)
        if math.isnan(want):
            assert math.isnan(got)
        else:
            assert got == want and math.copysign(1, got) == math.copysign(1, want)


def test_bf16_decode_matches_torch():
    x = RNG.standard_normal(4096) * 10.0 ** RNG.integers(-30, 30, 4096)
    bits = _bf16_bits(x)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.bf16_decode(bits), ref)


# Model shapes: DeepSeek-V3.2 (128 MLA heads, 64 indexer heads, qk head dim
# 192) and GLM-5.2 (64 MLA heads, 32 indexer heads, qk head dim 256; "大语言
# 模型结构总览" section 7.2).
IDX_HEADS = [64, 32]
MLA_SHAPES = [(128, 1 / math.sqrt(192)), (64, 1 / math.sqrt(256))]


# ---------------------------------------------------------------- indexer
@pytest.mark.parametrize("hi", IDX_HEADS)
def test_indexer_brute_force_loops(hi):
    q = _e4m3_bytes(RNG.standard_normal((hi, 128)))
    k = _e4m3_bytes(RNG.standard_normal((5, 128)))
    w = (RNG.standard_normal(hi) / 8).astype(np.float32)
    got = O.indexer_scores(q, w, k)
    tab = O.e4m3_table()
    for s in range(5):
        acc = 0.0
        for h in range(hi):
            d = sum(float(tab[q[h, i]]) * float(tab[k[s, i]]) for i in range(128))
            acc += float(w[h]) * (d if d > 0 else 0.0)
        assert abs(got[s] - acc) <= 1e-12 * max(1.0, abs(acc))


@pytest.mark.parametrize("hi", IDX_HEADS)
def test_indexer_one_hot_keys_closed_form(hi):
    # K[s] = e_s (a single 1.0 at dim s): q_h . K[s] = q_h[s], so
    # I[s] = sum_h w_h * max(0, q_h[s]).
    q = _e4m3_bytes(RNG.standard_normal((hi, 128)))
    w = (RNG.standard_normal(hi) / 8).astype(np.float32)
    keys = np.zeros((128, 128), dtype=np.uint8)
    keys[np.arange(128), np.arange(128)] = 0x38          # e4m3 1.0
    qf = O.e4m3_decode(q)
    want = np.maximum(qf, 0).T @ w.astype(np.float64)
    assert np.allclose(O.indexer_scores(q, w, keys), want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("hi", IDX_HEADS)
def test_indexer_relu_sign_identity(hi):
    # I(q,K) - I(q,-K) = sum_h w_h (q_h . K): catches a dropped or mirrored ReLU.
    q = _e4m3_bytes(RNG.standard_normal((hi, 128)))
    k = _e4m3_bytes(RNG.standard_normal((33, 128)))
    w = (RNG.standard_normal(hi) / 8).astype(np.float32)
    k_neg = k ^ 0x80
    lhs = O.indexer_scores(q, w, k) - O.indexer_scores(q, w, k_neg)
    qw = O.e4m3_decode(q).T @ w.astype(np.float64)              # [128]
    rhs = O.e4m3_decode(k) @ qw
    assert np.allclose(lhs, rhs, rtol=1e-12, atol=1e-9)
    # and the scores are not already linear in K (the ReLU is active)
    assert not np.allclose(O.indexer_scores(q, w, k), 0.5 * rhs, atol=1e-3)


# ---------------------------------------------------------------- selector
def _brute_topk_set(scores, k):
    n = len(scores)
    order = sorted(range(n), key=lambda s: (-scores[s], s))   # Python's own sort
    return set(order[: min(k, n)])


@pytest.mark.parametrize("n", [1, 7, 16, 64])
def test_topk_equals_full_sort_with_ties(n):
    for trial in range(5):
        sc = RNG.integers(-3, 4, n).astype(np.float64)        # many exact ties
        if trial == 0:
            sc[:] = 2.0                                       # all tied
        if trial == 1:
            sc = RNG.standard_normal(n)
        for k in sorted({1, 4, max(1, n - 1), n, n + 5}):
            idx = O.topk_select(sc, k)
            assert idx.shape == (k,)
            sel = [int(i) for i in idx if i >= 0]
            assert len(sel) == min(k, n) and len(set(sel)) == len(sel)
            assert (idx[len(sel):] == -1).all()
            assert set(sel) == _brute_topk_set(list(sc), k)
            # every kept position beats every dropped one under (score, lower index)
            drop = set(range(n)) - set(sel)
            for a, b in itertools.product(sel, drop):
                assert sc[a] > sc[b] or (sc[a] == sc[b] and a < b)


def test_topk_negative_zero_equals_zero():
    sc = np.array([0.0, -0.0, 0.0, -0.0, -1.0])
    assert list(O.topk_select(sc, 2)) == [0, 1]


# ---------------------------------------------------------------- sparse MLA
def _rows(n, dtype_bits=True):
    return O.bf16_decode(_bf16_bits(RNG.standard_normal((n, 576))))


@pytest.mark.parametrize("nh,scale", MLA_SHAPES)
def test_mla_k_ge_L_equals_library_dense_attention(nh, scale):
    # with k >= L the selector keeps every token, so DSA is dense MLA; compare
    # with torch's scaled_dot_product_attention in float64 (value = first 512).
    rows = _rows(37)
    q = O.bf16_decode(_bf16_bits(RNG.standard_normal((nh, 576))))
    sc = RNG.standard_normal(37)
    idx = O.topk_select(sc, 2048)
    sel = idx[idx >= 0]
    assert sorted(sel.tolist()) == list(range(37))
    o, lse = O.sparse_mla(q, rows[sel], scale)
    tq = torch.from_numpy(q)[None]
    tk = torch.from_numpy(rows)[None]
    tv = torch.from_numpy(rows[:, :512])[None]
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=scale)[0].numpy()
    ref_lse = torch.logsumexp(scale * (tq[0] @ tk[0].T), dim=1).numpy()
    assert np.allclose(o, ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(lse, ref_lse, rtol=1e-13, atol=1e-12)


@pytest.mark.parametrize("nh,scale", MLA_SHAPES)
def test_mla_softmax_weights_sum_to_one(nh, scale):
    # value dims all equal to 1 -> O = sum_j p_j = 1 for every head and dim
    rows = _rows(50)
    rows[:, :512] = 1.0
    q = O.bf16_decode(_bf16_bits(RNG.standard_normal((nh, 576)) * 3))
    o, _ = O.sparse_mla(q, rows, scale)
    assert o.shape == (nh, 512)
    assert np.allclose(o, 1.0, rtol=0, atol=1e-12)


@pytest.mark.parametrize("nh,scale", MLA_SHAPES)
def test_mla_closed_forms(nh, scale):
    q = O.bf16_decode(_bf16_bits(RNG.standard_normal((nh, 576))))
    r = _rows(1)
    # one row: O = its latent, LSE = its score
    o, lse = O.sparse_mla(q, r, scale)
    assert np.allclose(o, np.broadcast_to(r[0, :512], (nh, 512)), atol=1e-12)
    assert np.allclose(lse, scale * (q @ r[0]), atol=1e-12)
    # n identical rows: O = the row, LSE = s + ln n
    o, lse = O.sparse_mla(q, np.repeat(r, 9, axis=0), scale)
    assert np.allclose(o, np.broadcast_to(r[0, :512], (nh, 512)), atol=1e-12)
    assert np.allclose(lse, scale * (q @ r[0]) + math.log(9), atol=1e-12)
    # two rows: O = sigmoid(s1 - s2) c1 + sigmoid(s2 - s1) c2
    r2 = _rows(2)
    o, _ = O.sparse_mla(q, r2, scale)
    s1, s2 = scale * (q @ r2[0]), scale * (q @ r2[1])
    a = 1 / (1 + np.exp(s2 - s1))
    want = a[:, None] * r2[0, :512] + (1 - a)[:, None] * r2[1, :512]
    assert np.allclose(o, want, atol=1e-12)
    # no rows: O = 0, LSE = -inf
    o, lse = O.sparse_mla(q, r2[:0], scale)
    assert (o == 0).all() and np.isneginf(lse).all()


def test_fp8_rows_decode_then_scale():
    # one e4m3 row: O = kv_scale * decoded row, LSE = scale * q . (kv_scale * row)
    codes = _e4m3_bytes(RNG.standard_normal((1, 576)) * 3).reshape(1, 1, 576)
    kv = 0.37
    rows = O.latent_rows_e4m3(codes, np.array([0]), np.array([0]), kv, page_size=1)
    dec = torch.from_numpy(codes.reshape(576).copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(rows[0], dec * kv)
    q = O.bf16_decode(_bf16_bits(RNG.standard_normal((128, 576))))
    o, lse = O.sparse_mla(q, rows, 1 / math.sqrt(192))
    assert np.allclose(o, np.broadcast_to(kv * dec[:512], (128, 512)), atol=1e-12)
    assert np.allclose(lse, (q @ (kv * dec)) / math.sqrt(192), atol=1e-12)
    # paging: page p, slot s of a page_size-16 cache is pool[table[p], s]
    pool = _e4m3_bytes(RNG.standard_normal((5, 16, 576))).reshape(5, 16, 576)
    table = np.array([3, 0, 4])
    pos = np.array([0, 17, 40, 15])
    got = O.latent_rows_e4m3(pool, table, pos, 1.0, page_size=16)
    want = O.e4m3_decode(np.stack([pool[3, 0], pool[0, 1], pool[4, 8], pool[3, 15]]))
    assert np.array_equal(got, want)


def test_lse_combine_equals_unsplit_and_ignores_empty_parts():
    scale = 1 / math.sqrt(192)
    q = O.bf16_decode(_bf16_bits(RNG.standard_normal((128, 576))))
    rows = _rows(300)
    pos = np.sort(RNG.choice(5000, 300, replace=False))
    o_full, lse_full = O.sparse_mla(q, rows, scale)
    for S in (1, 2, 16, 64):        # 64 chunks over 300 picks leaves empty chunks
        o, lse = O.sparse_mla_split(q, rows, pos, 5000, S, scale)
        assert np.allclose(o, o_full, rtol=1e-12, atol=1e-12)
        assert np.allclose(lse, lse_full, rtol=1e-12, atol=1e-12)
    o, lse = O.lse_combine(np.zeros((3, 128, 512)), np.full((3, 128), -np.inf))
    assert (o == 0).all() and np.isneginf(lse).all()


# ---------------------------------------------------------------- whole step
def _small(name, **kw):
    return make_inputs(get_workload(name, **kw), seed=3)


def test_permutation_of_key_order_leaves_outputs_unchanged():
    # Relabel the token positions of one sequence by a permutation pi: the
    # indexer key and the latent row of token s move to position pi(s).  The
    # selected set must map through pi and attention must not change.
    inp = _small("decode_b1_ctx8k", L=700, topk=64)
    a = oracle_inputs(inp)
    base = O.decode_step(a)
    L = 700
    pi = RNG.permutation(L)
    b = dict(a)
    keys = a["indexer"][0]["k_idx"]
    new_keys = keys.copy()
    new_keys[pi] = keys[:L]
    b["indexer"] = [dict(a["indexer"][0], k_idx=new_keys)]
    pool = a["layers"][0]["pool"]
    flat = pool.reshape(-1, 576)                   # identity page table: row = position
    new_flat = flat.copy()
    new_flat[pi] = flat[:L]
    b["layers"] = [{"q": a["layers"][0]["q"], "pool": new_flat.reshape(pool.shape)}]
    other = O.decode_step(b)
    i0 = base["idx"][(0, 0)]
    i1 = other["idx"][(0, 0)]
    assert set(pi[i0[i0 >= 0]].tolist()) == set(i1[i1 >= 0].tolist())
    assert np.allclose(base["out"][(0, 0)], other["out"][(0, 0)], rtol=1e-12, atol=1e-13)
    assert np.allclose(base["lse"][(0, 0)], other["lse"][(0, 0)], rtol=1e-13, atol=1e-13)


def test_paging_is_transparent():
    # the same rows stored under a different page permutation give the same result
    inp = _small("decode_b32_ctx128k", B=2, L=700, topk=64)
    a = oracle_inputs(inp)
    base = O.decode_step(a)
    P = a["layers"][0]["pool"]
    perm = RNG.permutation(P.shape[0])
    inv = np.argsort(perm)
    b = dict(a)
    b["layers"] = [{"q": a["layers"][0]["q"], "pool": P[perm]}]
    pt = a["page_table"].copy()
    ok = pt >= 0
    pt[ok] = inv[pt[ok]]
    b["page_table"] = pt
    other = O.decode_step(b)
    for key in base["out"]:
        assert np.array_equal(base["out"][key], other["out"][key])
        assert np.array_equal(base["lse"][key], other["lse"][key])


def test_permutation_of_selected_order_leaves_attention_unchanged():
    scale = 1 / math.sqrt(192)
    q = O.bf16_decode(_bf16_bits(RNG.standard_normal((128, 576))))
    rows = _rows(200)
    o1, l1 = O.sparse_mla(q, rows, scale)
    p = RNG.permutation(200)
    o2, l2 = O.sparse_mla(q, rows[p], scale)
    assert np.allclose(o1, o2, rtol=1e-12, atol=1e-13) and np.allclose(l1, l2, rtol=1e-13)


def test_indexshare_layers_equal_direct_calls_with_shared_indices():
    inp = _small("indexshare4_b64_ctx16k_128k", B=3, L_range=(300, 900), topk=128)
    a = oracle_inputs(inp)
    res = O.decode_step(a)
    assert len(a["indexer"]) == 1
    for l in range(4):
        for q in range(3):
            idx = res["idx"][(0, q)]
            pos = idx[idx >= 0]
            rows = O.latent_rows(a["layers"][l]["pool"], a["page_table"][q], pos)
            o, lse = O.sparse_mla(O.bf16_decode(a["layers"][l]["q"][q]), rows, a["scale"])
            assert np.array_equal(o, res["out"][(l, q)]) and np.array_equal(lse, res["lse"][(l, q)])


def test_mtp_reuse_takes_position_zero_indices_and_causal_visibility():
    inp = _small("mtp_verify_reuse_b16_t8_ctx128k", B=2, L=500, topk=64)
    a = oracle_inputs(inp)
    vis = a["q_vis"]
    assert list(vis[:8]) == [501 + t for t in range(8)]
    res = O.decode_step(a)
    for b in range(2):
        for t in range(8):
            assert np.array_equal(res["idx"][(0, b * 8 + t)], res["idx"][(0, b * 8)])
    a["mtp_index_share"] = False
    res2 = O.decode_step(a)
    # per-position top-k: position t may select up to key 500 + t
    for t in range(8):
        idx = res2["idx"][(0, t)]
        assert idx.max() <= 500 + t


def test_page_ratios_stated_for_128k():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "dsa_page_ratios.txt"))
            if l.strip() and not l.startswith("#")]
    q = _e4m3_bytes(RNG.standard_normal((64, 128)))
    w = (RNG.standard_normal(64) / 8).astype(np.float32)
    L = int(rows[0][1])
    k = int(rows[0][2])
    keys = _e4m3_bytes(RNG.standard_normal((L, 128)))
    idx = O.topk_select(O.indexer_scores(q, w, keys), k)
    kept = int((idx >= 0).sum())
    vals = {"keys_seen_fraction": kept / L, "dense_over_sparse": L / kept}
    for name, _, _, stated, tol in rows:
        assert abs(vals[name] - float(stated)) <= float(tol), (name, vals[name])


# ---------------------------------------------------------------- CSA window
PAGE_T = 64          # tokens per latent-cache page of the oracle


def _csa_case(seed, n_pages=8, one_row=False):
    rng = np.random.default_rng(seed)
    vals = rng.standard_normal((n_pages, PAGE_T, 576))
    if one_row:
        vals[:] = rng.standard_normal(576)
    pool = _bf16_bits(vals)
    perm = rng.permutation(n_pages)
    return rng, pool, perm[:2], perm[2:]          # compressed pages, raw pages


def test_csa_window_zero_is_sparse_mla():
    rng, pool, pc, pr = _csa_case(1)
    q = O.bf16_decode(_bf16_bits(rng.standard_normal((64, 576))))
    sel = rng.choice(2 * PAGE_T, 37, replace=False)
    o, l = O.csa_window_attention(q, pool, pc, pr, sel, 150, 0, 0.07)
    o2, l2 = O.sparse_mla(q, O.latent_rows(pool, pc, sel), 0.07)
    assert np.array_equal(o, o2) and np.array_equal(l, l2)


@pytest.mark.parametrize("win_vis,window", [(200, 128), (5, 128), (0, 16)])
def test_csa_identical_rows_closed_form(win_vis, window):
    """Every row the same latent c: O = c[:512] and LSE = scale q.c + ln(n), with
    n = the selected entries plus the window tokens at or after position 0."""
    rng, pool, pc, pr = _csa_case(2, one_row=True)
    c = O.bf16_decode(pool[0, 0])
    q = O.bf16_decode(_bf16_bits(rng.standard_normal((128, 576))))
    sel = rng.choice(2 * PAGE_T, 9, replace=False)
    o, l = O.csa_window_attention(q, pool, pc, pr, sel, win_vis, window, 0.05)
    n = 9 + min(window, win_vis)
    assert np.allclose(o, np.broadcast_to(c[:512], o.shape), rtol=0, atol=1e-12)
    assert np.allclose(l, 0.05 * (q @ c) + math.log(n), rtol=0, atol=1e-12)


def test_csa_window_before_token_zero_keeps_only_nonnegative_tokens():
    rng, pool, pc, pr = _csa_case(3)
    q = O.bf16_decode(_bf16_bits(rng.standard_normal((128, 576))))
    sel = rng.choice(2 * PAGE_T, 20, replace=False)
    o, l = O.csa_window_attention(q, pool, pc, pr, sel, 5, 128, 0.06)
    o2, l2 = O.csa_window_attention(q, pool, pc, pr, sel, 5, 5, 0.06)
    assert np.array_equal(o, o2) and np.array_equal(l, l2)
    assert np.array_equal(O.csa_window_positions(5, 128), np.arange(5))


@pytest.mark.parametrize("win_vis", [1, 64, 300])
def test_csa_one_token_window_is_the_latest_raw_token(win_vis):
    """No selected entry and a window of 1: the attention is the latent of raw
    token win_vis-1 (a softmax over one row), LSE = scale q.c."""
    rng, pool, pc, pr = _csa_case(4)
    q = O.bf16_decode(_bf16_bits(rng.standard_normal((64, 576))))
    o, l = O.csa_window_attention(q, pool, pc, pr, np.zeros(0, np.int64), win_vis, 1, 0.08)
    t = win_vis - 1
    c = O.bf16_decode(pool[pr[t // PAGE_T], t % PAGE_T])
    assert np.allclose(o, np.broadcast_to(c[:512], o.shape), rtol=0, atol=1e-12)
    assert np.allclose(l, 0.08 * (q @ c), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- planted slips
def test_planted_mistakes_are_caught(monkeypatch):
    """Each slip planted in the oracle must make a pin fail."""
    real_scores = O.indexer_scores
    real_mla = O.sparse_mla
    real_topk = O.topk_select

    def no_relu(q, w, k):
        return (O.e4m3_decode(k) @ O.e4m3_decode(q).T) @ np.asarray(w, np.float64)

    def ties_high(sc, k):
        n = len(sc)
        order = np.lexsort((-np.arange(n), -np.asarray(sc)))
        out = np.full(k, -1)
        out[:min(k, n)] = order[:min(k, n)]
        return out

    def no_scale(q, rows, scale):
        return real_mla(q, rows, 1.0)

    def value_from_rope_end(q, rows, scale):
        o, l = real_mla(q, rows, scale)
        return real_mla(q, np.concatenate([rows[:, 64:], rows[:, :64]], 1), scale)[0], l

    import oracle.dsa_oracle as OD
    real_window = OD.csa_window_positions

    def window_shifted(win_vis, window):
        return real_window(win_vis, window) - 1

    monkeypatch.setattr(OD, "csa_window_positions", window_shifted)
    try:
        test_csa_one_token_window_is_the_latest_raw_token(64)
        window_caught = False
    except (AssertionError, IndexError):
        window_caught = True
    monkeypatch.setattr(OD, "csa_window_positions", real_window)

    caught = [("window", window_caught)]
    for name, fn, attr, pins in [
        ("relu", no_relu, "indexer_scores", [lambda: test_indexer_relu_sign_identity(32),
                                             lambda: test_indexer_one_hot_keys_closed_form(64)]),
        ("ties", ties_high, "topk_select", [lambda: test_topk_equals_full_sort_with_ties(7)]),
        ("scale", no_scale, "sparse_mla", [lambda: test_mla_k_ge_L_equals_library_dense_attention(
            *MLA_SHAPES[1])]),
        ("value", value_from_rope_end, "sparse_mla", [lambda: test_mla_closed_forms(*MLA_SHAPES[0])]),
    ]:
        monkeypatch.setattr(O, attr, fn)
        failed = False
        for pin in pins:
            try:
                pin()
            except AssertionError:
                failed = True
        caught.append((name, failed))
        monkeypatch.setattr(O, attr, {"indexer_scores": real_scores, "sparse_mla": real_mla,
                                      "topk_select": real_topk}[attr])
    assert all(f for _, f in caught), caught
