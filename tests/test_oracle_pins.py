"""Pins of the fp64 oracle against what the sources and the mathematics fix:
hand-typed values from the model card, textbook special cases, library
routines (torch float64 scaled_dot_product_attention), brute force on tiny
inputs and invariants.  Every pin runs on both statements of the oracle:
the numpy one (oracle/tokenbutler.py) and the C++ one (oracle/tokenbutler.cpp
through oracle/native.py).  CPU only."""
import itertools
import math
import os

import numpy as np
import pytest
import torch

from oracle import native as _native
from oracle import tokenbutler as _numpy_oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(params=["numpy", "cpp"])
def O(request):
    """The oracle under test."""
    return _numpy_oracle if request.param == "numpy" else _native


def _rows(name, tag=None):
    out = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].split()
            if not line:
                continue
            if tag is None:
                out.append(line)
            elif line[0] == tag:
                out.append(line[1:])
    return out


# ----------------------------------------------------------------- layers / slots
def test_slot_map_matches_model_card_table(O):
    rows = _rows("slot_map_G4.txt")
    assert len(rows) == 32
    for layer, prod, slot in rows:
        assert O.producer_of(int(layer), 4) == int(prod)
        assert O.consumer_slot(int(layer), 4) == int(slot)


def test_each_producer_serves_itself_and_next_G_minus_1_layers_with_distinct_slots(O):
    for G in (1, 2, 3, 4, 8):
        for p in range(0, 64, G):
            layers = range(p, p + G)
            assert all(O.producer_of(l, G) == p for l in layers)
            assert sorted(O.consumer_slot(l, G) for l in layers) == list(range(G))


def test_importance_query_layout_picks_slot_and_position(O):
    # Q_imp is (B*H) x G x L x d' (model card, Method).  B=1, Hq=2, G=2, 3 positions, d'=2.
    q = np.arange(1 * 2 * 2 * 3 * 2, dtype=np.float64).reshape(2, 2, 3, 2)
    # layer 2 reads slot (2-1) mod 2 = 1; head 1 is row 1
    qh = O.importance_queries(q, layer=2, G=2, B=1, Hq=2, position=2)
    assert qh.shape == (1, 2, 2)
    # q[1, 1, 2, :] = flat index ((1*2+1)*3+2)*2 + {0,1} = 22, 23
    assert qh[0, 1].tolist() == [22.0, 23.0]
    assert qh[0, 0].tolist() == [10.0, 11.0]   # ((0*2+1)*3+2)*2 = 10


def test_gqa_head_map(O):
    assert [O.kv_head_of(h, 32, 8) for h in range(8)] == [0, 0, 0, 0, 1, 1, 1, 1]
    assert O.kv_head_of(31, 32, 8) == 7
    assert [O.kv_head_of(h, 4, 2) for h in range(4)] == [0, 0, 1, 1]


# ----------------------------------------------------------------- budget
def test_policy_and_budget_golden(O):
    for name, pct in _rows("budget.txt", "policy"):
        assert O.keep_pct_from_policy(name) == int(pct)
    for L, pct, k in _rows("budget.txt", "budget"):
        assert O.token_budget(int(L), int(pct)) == int(k)
    with pytest.raises(ValueError):
        O.keep_pct_from_policy("topk_50")


def test_budget_floor_and_limits(O):
    assert O.token_budget(131072, 30) == 39321      # floor(39321.6)
    assert O.token_budget(7, 50) == 3
    assert O.token_budget(0, 50) == 0
    assert O.token_budget(1000, 100) == 1000
    assert O.token_budget(1000, 0) == 0


# ----------------------------------------------------------------- K_imp and scores
def test_project_keys_special_cases(O):
    rng = np.random.default_rng(1)
    K = rng.standard_normal((5, 7, 8))
    W = np.zeros((8, 3))
    W[0, 0] = W[1, 1] = W[2, 2] = 1.0          # [I; 0] keeps the first d' coordinates
    assert np.array_equal(O.project_keys(K, W), K[..., :3])
    W = np.zeros((8, 3))
    W[5, 1] = 2.5                              # one entry: column 1 = 2.5 * K[..., 5]
    out = O.project_keys(K, W)
    assert np.array_equal(out[..., 1], 2.5 * K[..., 5])
    assert np.all(out[..., [0, 2]] == 0)


def test_project_keys_is_linear_and_matches_loops_on_tiny(O):
    rng = np.random.default_rng(2)
    K = rng.standard_normal((4, 6))
    W = rng.standard_normal((6, 3))
    ref = [[sum(K[t, d] * W[d, j] for d in range(6)) for j in range(3)] for t in range(4)]
    assert np.allclose(O.project_keys(K, W), ref, rtol=0, atol=1e-12)
    K2 = rng.standard_normal((4, 6))
    assert np.allclose(O.project_keys(K + K2, W), O.project_keys(K, W) + O.project_keys(K2, W), atol=1e-12)


def test_scores_basis_query_reads_one_coordinate(O):
    rng = np.random.default_rng(3)
    Kimp = rng.standard_normal((9, 4))
    for j in range(4):
        e = np.zeros(4)
        e[j] = 1.0
        assert np.array_equal(O.importance_scores(e, Kimp), Kimp[:, j])
    q = rng.standard_normal(4)
    assert np.allclose(O.importance_scores(2 * q, Kimp), 2 * O.importance_scores(q, Kimp), atol=1e-12)


# ----------------------------------------------------------------- selection
def test_select_hand_example(O):
    s = np.array([9, 1, 5, 5, 2, 7, 5, 0, 3, 4], dtype=np.float64)
    # L=10, sink 1, window 2: candidates are tokens 1..7.
    # 50 %: k = 5 -> scores 7(t5), 5(t2), 5(t3), 5(t6), 2(t4)
    assert O.select_tokens(s, 10, 50, 1, 2).tolist() == [0, 2, 3, 4, 5, 6, 8, 9]
    # 30 %: k = 3 -> 7(t5), then the tie at 5 goes to the lower indices t2, t3
    assert O.select_tokens(s, 10, 30, 1, 2).tolist() == [0, 2, 3, 5, 8, 9]
    # the window and sink are kept even with a zero budget
    assert O.select_tokens(s, 10, 0, 1, 2).tolist() == [0, 8, 9]


def _brute_force_top(s, cand, k):
    """Among all k-subsets of the candidates with the largest score sum, the
    lexicographically smallest (ties -> lower indices)."""
    best, best_sum = None, -math.inf
    for sub in itertools.combinations(cand, k):   # combinations come in lexicographic order
        tot = sum(s[i] for i in sub)
        if tot > best_sum:
            best, best_sum = sub, tot
    return set(best)


@pytest.mark.parametrize("seed", range(12))
def test_select_matches_brute_force_on_tiny_rows(O, seed):
    rng = np.random.default_rng(seed)
    L = int(rng.integers(1, 13))
    s = rng.integers(-3, 4, size=L).astype(np.float64)   # small integers: many exact ties, exact sums
    sink, window = int(rng.integers(0, 3)), int(rng.integers(0, 3))
    for pct in (0, 10, 30, 50, 70, 100):
        sel = O.select_tokens(s, L, pct, sink, window)
        cand = [t for t in range(L) if sink <= t < L - window]
        k = min(O.token_budget(L, pct), len(cand))
        forced = {t for t in range(L) if t < sink or t >= L - window}
        expect = forced | (_brute_force_top(s, cand, k) if k else set())
        assert set(sel.tolist()) == expect
        assert sel.tolist() == sorted(expect)


@pytest.mark.parametrize("L,pct,sink,window", [(4096, 50, 16, 64), (4096, 30, 16, 64), (1000, 10, 4, 16),
                                                (80, 50, 16, 64), (70, 50, 16, 64), (1, 50, 16, 64),
                                                (0, 50, 4, 4), (333, 100, 0, 0), (333, 50, 0, 0)])
def test_select_invariants(O, L, pct, sink, window):
    rng = np.random.default_rng(L + pct)
    s = np.round(rng.standard_normal(L) * 4) / 4          # quantised: exact ties
    sel = O.select_tokens(s, L, pct, sink, window)
    assert np.all(np.diff(sel) > 0) and (sel.size == 0 or (sel[0] >= 0 and sel[-1] < L))
    cand = [t for t in range(L) if sink <= t < L - window]
    k = min(O.token_budget(L, pct), len(cand))
    assert sel.size == min(L, min(sink, L) + min(window, L) + k) if L >= sink + window else sel.size == L
    chosen = set(sel.tolist())
    assert set(range(min(sink, L))) <= chosen and set(range(max(L - window, 0), L)) <= chosen
    top = [t for t in cand if t in chosen]
    rest = [t for t in cand if t not in chosen]
    assert len(top) == k
    if top and rest:
        assert min(s[t] for t in top) >= max(s[t] for t in rest)
        thr = min(s[t] for t in top)
        tied_in = [t for t in top if s[t] == thr]
        tied_out = [t for t in rest if s[t] == thr]
        if tied_out:
            assert max(tied_in) < min(tied_out)


def test_select_negative_zero_equals_positive_zero(O):
    s = np.array([0.0, -0.0, 0.0, -0.0, -1.0])
    assert O.select_tokens(s, 5, 40, 0, 0).tolist() == [0, 1]
    s = np.array([-0.0, 0.0, -0.0, 0.0, -1.0])
    assert O.select_tokens(s, 5, 40, 0, 0).tolist() == [0, 1]


def test_select_invariant_under_softmax_and_positive_affine_maps(O):
    rng = np.random.default_rng(7)
    s = rng.standard_normal(4096) * 3
    base = O.select_tokens(s, 4096, 30, 16, 64)
    p = np.exp(s - s.max())
    p /= p.sum()
    assert np.array_equal(O.select_tokens(p, 4096, 30, 16, 64), base)
    assert np.array_equal(O.select_tokens(2.5 * s + 7, 4096, 30, 16, 64), base)
    assert not np.array_equal(O.select_tokens(-s, 4096, 30, 16, 64), base)


# ----------------------------------------------------------------- attention
def _sdpa64(q, K, V):
    """torch float64 scaled_dot_product_attention of one query row."""
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None, None], torch.from_numpy(K)[None, None], torch.from_numpy(V)[None, None])
    return out[0, 0, 0].numpy()


def test_attend_equals_library_attention_on_all_tokens(O):
    rng = np.random.default_rng(4)
    q, K, V = rng.standard_normal(64), rng.standard_normal((300, 64)), rng.standard_normal((300, 64))
    o, lse = O.attend(q, K, V, np.arange(300), 1 / 8)
    assert np.allclose(o, _sdpa64(q, K, V), rtol=0, atol=1e-12)
    assert math.isclose(lse, float(np.log(np.exp(K @ q / 8).sum())), rel_tol=1e-12)


def test_attend_textbook_loops_on_tiny(O):
    rng = np.random.default_rng(5)
    q, K, V = rng.standard_normal(3), rng.standard_normal((5, 3)), rng.standard_normal((5, 3))
    idx = [0, 2, 3]
    w = [math.exp(sum(q[d] * K[t, d] for d in range(3)) * 0.5) for t in idx]
    ref = [sum(w[i] * V[t, d] for i, t in enumerate(idx)) / sum(w) for d in range(3)]
    o, lse = O.attend(q, K, V, np.array(idx), 0.5)
    assert np.allclose(o, ref, atol=1e-12)
    assert math.isclose(lse, math.log(sum(w)), rel_tol=1e-12)


def test_attend_special_cases(O):
    rng = np.random.default_rng(6)
    q, K, V = rng.standard_normal(16), rng.standard_normal((50, 16)), rng.standard_normal((50, 16))
    o, _ = O.attend(q, K, V, np.array([17]), 0.25)          # one token: its value row
    assert np.allclose(o, V[17], atol=1e-14)
    Ks = np.repeat(K[:1], 50, axis=0)                        # equal keys: the plain mean
    o, lse = O.attend(q, Ks, V, np.array([1, 5, 9]), 0.25)
    assert np.allclose(o, V[[1, 5, 9]].mean(axis=0), atol=1e-13)
    assert math.isclose(lse, 0.25 * float(Ks[0] @ q) + math.log(3), rel_tol=1e-12)
    o, lse = O.attend(q, K, V, np.array([], dtype=np.int64), 0.25)
    assert np.all(o == 0) and lse == -math.inf


def test_attend_order_free_and_lse_merge(O):
    rng = np.random.default_rng(8)
    q, K, V = rng.standard_normal(32), rng.standard_normal((200, 32)), rng.standard_normal((200, 32))
    a, b = np.arange(0, 200, 3), np.arange(1, 200, 3)
    o_ab, lse_ab = O.attend(q, K, V, np.concatenate([a, b]), 0.2)
    o_ba, _ = O.attend(q, K, V, np.concatenate([b[::-1], a]), 0.2)
    assert np.allclose(o_ab, o_ba, atol=1e-13)
    oa, la = O.attend(q, K, V, a, 0.2)
    ob, lb = O.attend(q, K, V, b, 0.2)
    m = max(la, lb)
    lse = m + math.log(math.exp(la - m) + math.exp(lb - m))
    assert math.isclose(lse, lse_ab, rel_tol=1e-12)
    assert np.allclose((math.exp(la - lse) * oa + math.exp(lb - lse) * ob), o_ab, atol=1e-12)


# ----------------------------------------------------------------- one decode layer
def _layer_inputs(rng, B, Hq, Hkv, L, D, dimp, G):
    q = rng.standard_normal((B, Hq, D))
    K = rng.standard_normal((B, Hkv, L, D))
    V = rng.standard_normal((B, Hkv, L, D))
    W = rng.standard_normal((D, dimp)) / math.sqrt(D)
    qi = rng.standard_normal((B * Hq, G, 1, dimp))
    return q, K, V, W, qi


def test_full_budget_equals_dense_gqa_attention_from_library(O):
    rng = np.random.default_rng(9)
    B, Hq, Hkv, L, D = 2, 8, 2, 96, 32
    q, K, V, W, qi = _layer_inputs(rng, B, Hq, Hkv, L, D, 8, 4)
    sel, out, lse, _ = O.decode_layer(q, K, V, W, qi, layer=5, G=4, L=L, keep_pct=100, sink=4, window=8,
                                      dense=False)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[:, :, None], torch.from_numpy(K), torch.from_numpy(V), enable_gqa=True)[:, :, 0]
    for b in range(B):
        for h in range(Hq):
            assert sel[b, h].tolist() == list(range(L))
            assert np.allclose(out[b, h], ref[b, h].numpy(), atol=1e-12)
    # a dense layer gives the same result without scoring
    _, out_d, _, sc = O.decode_layer(q, K, V, W, qi, layer=0, G=4, L=L, keep_pct=30, sink=4, window=8,
                                     dense=True)
    assert all(v is None for v in sc.values())
    assert all(np.allclose(out_d[k], out[k], atol=1e-12) for k in out)


def test_sparse_layer_uses_consumer_slot_and_own_kv_head(O):
    rng = np.random.default_rng(10)
    B, Hq, Hkv, L, D, dimp, G = 1, 4, 2, 64, 16, 4, 4
    q, K, V, W, qi = _layer_inputs(rng, B, Hq, Hkv, L, D, dimp, G)
    layer = 6                                    # slot (6-1) mod 4 = 1
    sel, out, _, sc = O.decode_layer(q, K, V, W, qi, layer, G, L, 50, 2, 4, dense=False)
    for h in range(Hq):
        g = h // 2
        s = (K[0, g] @ W) @ qi[h, 1, 0]
        assert np.allclose(sc[0, h], s, atol=1e-12)
        assert not np.allclose(sc[0, h], (K[0, g] @ W) @ qi[h, 0, 0])
        assert sel[0, h].size == 2 + 4 + 32


def test_ragged_lengths_per_sequence(O):
    rng = np.random.default_rng(11)
    q, K, V, W, qi = _layer_inputs(rng, 3, 4, 2, 50, 16, 4, 1)
    lens = [50, 17, 1]
    sel, out, _, _ = O.decode_layer(q, K, V, W, qi, 0, 1, lens, 50, 2, 4, dense=False)
    for b, Lb in enumerate(lens):
        for h in range(4):
            assert sel[b, h].size == min(Lb, 6 + (Lb * 50) // 100) if Lb >= 6 else sel[b, h].size == Lb
            assert sel[b, h].max() == Lb - 1


def test_planted_tokens_are_selected_tiny_f32(O):
    from query_aware_sparse_decode_b200 import synth as S
    wl = S.TINY_F32
    W = S.w_k(wl, 0)
    qi = S.q_imp(wl, 0)
    qhat = O.importance_queries(S.widen(qi, wl.dtype), 0, wl.G, wl.B, wl.Hq)
    delta = S.plant_delta(S.widen(W, wl.dtype), qhat, wl.Hkv)
    K = S.widen(S.kv_cache_host(wl, 0, S.K_CACHE, 0, wl.L, delta), wl.dtype).reshape(1, 2, wl.L, wl.D)
    V = S.widen(S.kv_cache_host(wl, 0, S.V_CACHE, 0, wl.L), wl.dtype).reshape(1, 2, wl.L, wl.D)
    q = S.widen(S.query(wl, 0), wl.dtype)
    sel, _, _, sc = O.decode_layer(q, K, V, S.widen(W, wl.dtype), S.widen(qi, wl.dtype), 0, wl.G, wl.L,
                                   wl.keep_pct, wl.sink, wl.window, dense=False)
    planted = S.plant_list8(wl, 0)
    assert planted.size == 8
    for h in range(wl.Hq):
        assert sel[0, h].size == 256 + 4 + 16
        assert set(planted.tolist()) <= set(sel[0, h].tolist())
        # planted scores sit far above the typical score of the head
        s = sc[0, h]
        assert np.mean(s[planted]) > np.mean(s) + 2 * np.std(s)


# ----------------------------------------------------------------- prefill rows
def test_prefill_rows_are_causal_and_match_brute_force(O):
    rng = np.random.default_rng(12)
    Hq, Hkv, dimp, row0, nrows = 2, 1, 3, 5, 6
    Kimp = np.round(rng.standard_normal((Hkv, row0 + nrows, dimp)) * 2) / 2
    qh = np.round(rng.standard_normal((Hq, nrows, dimp)) * 2) / 2
    res = O.prefill_select(qh, Kimp, row0, 50, 1, 2)
    for h in range(Hq):
        for r in range(nrows):
            p = row0 + r
            s = Kimp[0, :p + 1] @ qh[h, r]
            cand = [t for t in range(p + 1) if 1 <= t < p + 1 - 2]
            k = min((50 * (p + 1)) // 100, len(cand))
            expect = {0} | set(range(max(p + 1 - 2, 0), p + 1)) | _brute_force_top(s, cand, k)
            assert res[h, p].tolist() == sorted(expect)
            assert res[h, p].max() == p


# ----------------------------------------------------------------- soft voting
def test_softvote_votes_sum_to_heads_and_equal_keys_vote_uniformly(O):
    rng = np.random.default_rng(13)
    q, K = rng.standard_normal((8, 16)), rng.standard_normal((2, 40, 16))
    v = O.softvote_scores(q, K, 40)
    assert math.isclose(v.sum(), 8.0, rel_tol=1e-12)
    Ku = np.repeat(K[:, :1], 40, axis=1)
    assert np.allclose(O.softvote_scores(q, Ku, 40), 8.0 / 40, atol=1e-14)


def test_softvote_two_tokens_closed_form_and_single_head_reduction(O):
    D = 16
    q = np.zeros((1, D))
    q[0, 0] = 1.0
    K = np.zeros((1, 2, D))
    K[0, 0, 0], K[0, 1, 0] = 2.0, -2.0
    # logits +-2/sqrt(16) = +-0.5: p0 = 1 / (1 + e^-1)
    v = O.softvote_scores(q, K, 2)
    assert math.isclose(v[0], 1 / (1 + math.exp(-1.0)), rel_tol=1e-12)
    rng = np.random.default_rng(14)
    q1, K1 = rng.standard_normal((1, 32)), rng.standard_normal((1, 500, 32))
    v1 = O.softvote_scores(q1, K1, 500)
    assert np.array_equal(O.select_tokens(v1, 500, 30, 4, 8), O.select_tokens(K1[0] @ q1[0], 500, 30, 4, 8))


def test_softvote_layer_shares_one_set_over_heads(O):
    rng = np.random.default_rng(15)
    q, K, V = rng.standard_normal((1, 4, 16)), rng.standard_normal((1, 2, 64, 16)), rng.standard_normal((1, 2, 64, 16))
    sel, out, _, votes = O.softvote_layer(q, K, V, 64, 30, 2, 4)
    assert sel[0].size == 2 + 4 + 19
    for h in range(4):
        o, _ = O.attend(q[0, h], K[0, h // 2], V[0, h // 2], sel[0], 0.25)
        assert np.allclose(out[0, h], o, atol=1e-14)


# --------------------------------------------------------------------------- per-group option
def test_group_scores_one_head_is_the_head_and_sum_is_the_summed_query(O):
    rng = np.random.default_rng(11)
    K_imp = rng.standard_normal((40, 6))
    q1 = rng.standard_normal((1, 6))
    assert np.array_equal(O.group_scores(q1, K_imp), O.importance_scores(q1[0], K_imp))
    q4 = rng.standard_normal((4, 6))
    # textbook loops over the summed query (the scores are linear in q)
    qsum = [sum(q4[h, j] for h in range(4)) for j in range(6)]
    want = np.array([sum(qsum[j] * K_imp[t, j] for j in range(6)) for t in range(40)])
    assert np.allclose(O.group_scores(q4, K_imp), want, rtol=1e-13, atol=1e-13)


def test_group_selection_shares_one_set_per_group_and_equals_per_head_for_equal_queries(O):
    rng = np.random.default_rng(12)
    B, Hq, Hkv, D, dimp, L, G = 1, 8, 2, 16, 4, 300, 1
    q = rng.standard_normal((B, Hq, D))
    K = rng.standard_normal((B, Hkv, L, D))
    V = rng.standard_normal((B, Hkv, L, D))
    W = rng.standard_normal((D, dimp))
    qi = rng.standard_normal((B * Hq, G, 1, dimp))
    sel, out, _, sc = O.decode_layer(q, K, V, W, qi, 1, G, L, 30, 4, 16, dense=False, group=True)
    gs = Hq // Hkv
    for h in range(Hq):
        lead = (h // gs) * gs
        assert np.array_equal(sel[0, h], sel[0, lead])            # one set per group
        assert np.array_equal(sc[0, h], sc[0, lead])
        ref, _ = O.attend(q[0, h], K[0, h // gs], V[0, h // gs], sel[0, h], 1 / math.sqrt(D))
        assert np.allclose(out[0, h], ref)
    # every head of a group with the same importance query: the group sum is a
    # positive multiple of each head's scores, so the sets are the per-head sets
    qi_same = np.repeat(qi.reshape(B, Hkv, gs, G, 1, dimp)[:, :, :1], gs, axis=2).reshape(B * Hq, G, 1, dimp)
    sel_g, _, _, _ = O.decode_layer(q, K, V, W, qi_same, 1, G, L, 30, 4, 16, dense=False, group=True)
    sel_h, _, _, _ = O.decode_layer(q, K, V, W, qi_same, 1, G, L, 30, 4, 16, dense=False)
    for h in range(Hq):
        assert np.array_equal(sel_g[0, h], sel_h[0, h])


# --------------------------------------------------------------------------- amortised selection (R18)
def test_reuse_decision_rules(O):
    q = np.array([1.0, 0.0, 0.0])
    near = np.array([1.0, 0.1, 0.0])            # cos 0.995
    far = np.array([0.0, 1.0, 0.0])             # cos 0
    args = dict(interval=4, tau=0.9, keep_pct=30, sink=4, window=16)
    assert O.reuse_decision(q, near, 200, 198, **args)
    assert not O.reuse_decision(q, far, 200, 198, **args)
    assert not O.reuse_decision(q, near, 200, 195, **args)          # older than the interval
    assert not O.reuse_decision(q, near, 200, 0, **args)            # empty cache
    assert not O.reuse_decision(q, near, 15, 14, **args)            # no top-k at this length
    assert not O.reuse_decision(np.zeros(3), near, 200, 198, **args)
    assert O.reuse_decision(q, q, 200, 200, **args)                 # same step, same query
    assert not O.reuse_decision(q, near, 200, 198, **dict(args, keep_pct=100))  # 100 %: all candidates


def test_reused_set_keeps_cached_topk_window_and_sink_with_neighbours(O):
    sink, window = 2, 4
    len0, L = 40, 42
    topk = np.array([5, 9, 20, 33])               # 33 = len0 - window - 3, still a candidate then
    cached = np.concatenate([np.arange(sink), topk, np.arange(len0 - window, len0)])
    got = O.reused_set(cached, len0, L, sink, window, radius=0)
    want = np.concatenate([np.arange(sink), topk, np.arange(L - window, L)])
    assert np.array_equal(got, want)
    # cached window tokens (36..39) are not top-k: only 38, 39 stay, as window of L = 42
    got2 = O.reused_set(cached, len0, L, sink, window, radius=2)
    want2 = sorted(set(range(sink)) | {3, 4, 5, 6, 7, 8, 9, 10, 11, 18, 19, 20, 21, 22, 31, 32, 33, 34, 35}
                   | set(range(L - window, L)))
    assert np.array_equal(got2, np.array(want2))
    assert got2.min() >= 0 and got2.max() < L


# ------------------------------------------------------------ bf16 K_imp storage
def test_round_to_bf16_closed_forms(O):
    """Nearest bfloat16 with ties to the even significand (8 significant
    bits: spacing 2^-7 on [1, 2)), rounded once from the exact value."""
    r = O.round_to_bf16
    cases = [
        (1.0 + 2.0 ** -8, 1.0),                          # tie between 1 and 1 + 2^-7: even is 1
        (1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -6),          # tie between 1 + 2^-7 (odd) and 1 + 2^-6 (even)
        (1.0 + 2.0 ** -8 + 2.0 ** -40, 1.0 + 2.0 ** -7),  # just above the tie: one rounding, not two
        (-(1.0 + 2.0 ** -8), -1.0),                      # sign-symmetric
        (255.5, 256.0),                                  # 255.5 is a tie on [128, 256): 255 odd -> 256
        (254.5, 254.0),                                  # tie: 254 even
        (3.0 * 2.0 ** 100, 3.0 * 2.0 ** 100),            # representable values are kept
        (1.3 * 2.0 ** -130, 10 * 2.0 ** -133),           # subnormal: quantum 2^-133
    ]
    for x, want in cases:
        assert r(np.array(x)) == want, x
    z = r(np.array([0.0, -0.0]))
    assert z[0] == 0 and not np.signbit(z[0]) and np.signbit(z[1])


def test_round_to_bf16_equals_library_cast_on_fp32_values(O):
    """On values an fp32 holds exactly, rounding once equals the library's
    round-to-nearest-even fp32 -> bf16 conversion."""
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.standard_normal(200000) * 10.0 ** rng.integers(-30, 30, 200000),
                        np.float32(1.0) + np.arange(-4096, 4096) * np.float32(2.0 ** -23)]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.round_to_bf16(x.astype(np.float64)), want)


def test_bf16_storage_rounds_the_sum_not_the_terms(O):
    """K = [1, 2^-8], W_K = [[1], [1]]: the exact K_imp 1 + 2^-8 is a tie and
    stores as 1.0; rounding each term (or none) would give 1 + 2^-8."""
    K = np.array([[1.0, 2.0 ** -8]])
    W = np.array([[1.0], [1.0]])
    assert O.project_keys(K, W)[0, 0] == 1.0 + 2.0 ** -8
    assert O.project_keys(K, W, "bf16")[0, 0] == 1.0
    K2 = np.array([[1.0, 2.0 ** -8 + 2.0 ** -30]])
    assert O.project_keys(K2, W, "bf16")[0, 0] == 1.0 + 2.0 ** -7


def test_bf16_storage_decides_the_selection_in_decode_layer(O):
    """Two candidates whose exact scores differ by less than half a bf16 step
    tie after storage, and the tie goes to the lower index (R8): the stored
    precision must reach the selection."""
    B, Hq, Hkv, D, dimp, G = 1, 1, 1, 2, 1, 1
    W = np.array([[1.0], [0.0]])
    K = np.zeros((B, Hkv, 2, D))
    K[0, 0, 0, 0] = 1.0
    K[0, 0, 1, 0] = 1.0 + 2.0 ** -9
    V = np.arange(B * Hkv * 2 * D, dtype=np.float64).reshape(B, Hkv, 2, D)
    q = np.ones((B, Hq, D))
    qimp = np.ones((B * Hq, G, 1, dimp))
    args = (q, K, V, W, qimp, 1, G, 2, 50, 0, 0)
    sel64, *_ = O.decode_layer(*args, dense=False)
    sel16, out16, _, sc16 = O.decode_layer(*args, dense=False, kimp_storage="bf16")
    assert sel64[0, 0].tolist() == [1]
    assert sel16[0, 0].tolist() == [0] and sc16[0, 0].tolist() == [1.0, 1.0]
    assert np.array_equal(out16[0, 0], V[0, 0, 0])


# ------------------------------------------------------------ sequence sharding (R19)
def test_merge_partials_equals_attention_over_the_union(O):
    """Splitting a set into disjoint parts and merging the parts' outputs by
    their log-sum-exp is attention over the whole set (softmax identity)."""
    rng = np.random.default_rng(19)
    q, K, V = rng.standard_normal(64), rng.standard_normal((300, 64)), rng.standard_normal((300, 64))
    idx = np.sort(rng.choice(300, 120, replace=False))
    parts = [idx[idx < 90], idx[(idx >= 90) & (idx < 90)], idx[(idx >= 90) & (idx < 250)], idx[idx >= 250]]
    assert parts[1].size == 0
    res = [O.attend(q, K, V, p, 0.125) for p in parts]
    o, lse = O.merge_partials([r[0] for r in res], [r[1] for r in res])
    o_all, lse_all = O.attend(q, K, V, idx, 0.125)
    assert np.allclose(o, o_all, rtol=0, atol=1e-12) and math.isclose(lse, lse_all, rel_tol=1e-13)
    # the merge is symmetric in its parts
    o2, lse2 = O.merge_partials([r[0] for r in res[::-1]], [r[1] for r in res[::-1]])
    assert np.allclose(o2, o, atol=1e-14) and math.isclose(lse2, lse, rel_tol=1e-15)


def test_merge_partials_special_cases(O):
    o = np.arange(4.0)
    got, lse = O.merge_partials([o], [1.5])                       # one part: itself
    assert np.array_equal(got, o) and lse == 1.5
    got, lse = O.merge_partials([np.zeros(4), o], [-math.inf, 0.0])  # an empty part carries no weight
    assert np.array_equal(got, o) and lse == 0.0
    got, lse = O.merge_partials([np.zeros(4), np.zeros(4)], [-math.inf, -math.inf])
    assert np.array_equal(got, np.zeros(4)) and lse == -math.inf    # every part empty: as an empty set
    # two equal-mass parts average: lse = l + log 2
    got, lse = O.merge_partials([np.ones(4), 3 * np.ones(4)], [0.7, 0.7])
    assert np.allclose(got, 2.0) and math.isclose(lse, 0.7 + math.log(2.0))


@pytest.mark.parametrize("group", [False, True])
def test_sharded_decode_equals_unsharded(O, group):
    rng = np.random.default_rng(23)
    B, Hq, Hkv, L, D, dimp, G = 2, 4, 2, 700, 32, 8, 1
    q, K, V, W, qimp = _layer_inputs(rng, B, Hq, Hkv, L, D, dimp, G)
    lens = [700, 455]
    args = (q, K, V, W, qimp, 1, G, lens, 30, 8, 32)
    sel, out, lse, _ = O.decode_layer(*args, dense=False, group=group)
    bounds = [(0, 200), (200, 420), (420, 700)]
    sel_s, out_s, lse_s, parts = O.decode_layer_sharded(*args, bounds, group=group)
    for key in sel:
        assert np.array_equal(sel_s[key], sel[key])
        assert np.allclose(out_s[key], out[key], atol=1e-12) and math.isclose(lse_s[key], lse[key], rel_tol=1e-12)
        pieces = parts[key]
        assert np.array_equal(np.concatenate(pieces), sel[key])      # disjoint, in rank order, covering the set
        for (t0, t1), p in zip(bounds, pieces):
            assert p.size == 0 or (p.min() >= t0 and p.max() < t1)
    # sequence 1 ends inside rank 2's range; rank 2 still holds its window
    assert parts[1, 0][2].size > 0
