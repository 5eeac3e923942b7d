"""Plain fp64 CPU oracle of the TokenButler decode-step hot path.

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or run
this module.  It shares no code with the CUDA path: it is numpy in float64,
step by step in the order and notation of the sources, with no blocking,
fusion or reordering.

Sources (cited by page title and section):
  [MC]  "Meta-Llama-3.1-8B-Instruct-Butler" model card: section "Method"
        (producer layers, Q_imp, W_K, K_imp, consumer slot, top-x selection
        with sink prefix and local window, full KV cache kept) and section
        "Memory requirements" (fixed_<N>pc policy, default 50 %, layer 0 dense,
        min_sparse_index = sink length, sliding_window).
  [AB]  "TokenButler: Token Importance is Predictable", abstract (fixed budget,
        per-token selection, full KV cache preserved).
  [TS]  TokenSelect README, "Dynamic Token-Level KV Cache Selection" and
        "Per-head Soft Voting Mechanism".

Readings where the sources leave a step open (each marked "Reading" below):
  R1  W_K is one D x d' matrix per layer, shared by all KV heads.
  R2  query head h reads KV head h // (Hq / Hkv).
  R3  importance scores carry no scale (a scale cannot change a top-k).
  R4  consumer layer l reads producer G * floor(l / G), slot (l - 1) mod G
      (non-negative mod); layer 0's slot is never used (layer 0 is dense).
  R5  budget k = floor(P * L / 100), L counting the current token.
  R6  the top-k candidates exclude the sink and the window, so the selected
      set has exactly min(L, s + w + k) tokens.
  R7  k is clamped to the candidate count; a 100 % budget selects every token.
  R8  ties in score go to the lower token index; -0.0 equals +0.0.
  R9  attention uses the real query q, full head dim, scale 1/sqrt(D), over
      the untouched K/V.
  R13 prefill row p uses its causal prefix [0, p] with L -> p + 1.
  R14 soft voting: softmax over all t < L per head, scale 1/sqrt(D), votes
      summed over all query heads, one set shared by all heads.
  An empty selected set gives a zero output and lse = -inf.

  R18 amortised selection (TokenButler abstract: prediction interval with
      neighbour fetching; TokenSelect README, "Selection Cache"): a row reuses
      its cached top-k when it takes a real top-k now, the cache holds a top-k
      chosen at length len0 > 0 with len - len0 <= interval, and the cosine of
      the current and cached importance queries is >= tau; the reused set is
      the cached top-k widened by `radius` tokens each side, kept inside the
      current candidates, plus the current sink and window (reuse_decision,
      reused_set).  The pages fix none of these numbers.

Option beyond the sources (not a reading of them): per-KV-group selection,
where the importance scores of a group's query heads are summed and the
group selects once with the same budget, sink, window and tie rules; every
head of the group then attends over that set (group_scores, decode_layer
with group=True).

  R19 sequence-sharded decode (beyond the sources, which run one device):
      rank r holds the contiguous tokens [t0_r, t1_r), ranks in token order;
      the selection is the unsharded one (global budget from the global
      length, ties at the threshold to the lower index, hence to the lower
      rank), and the output merges the ranks' attention over their parts of
      the set by log-sum-exp (merge_partials, decode_layer_sharded).

Option beyond the sources: a bf16 K_imp cache (round_to_bf16,
project_keys with storage="bf16"): K_imp is rounded once, from its exact
value, to the nearest bfloat16 (ties to even) and scored as stored.

Parity pins (tests/test_oracle_pins.py) cover every function here; the
readings R4, R6, R13, R14 and R18 are consistent with the sources but not
fixed by them (parity unpinned against the pages for those readings), and
R19 and the two options go beyond the sources (pinned by identities:
equality with the unsharded step, the softmax split, single rounding).
"""
from __future__ import annotations

import math

import numpy as np


# ------------------------------------------------------------------ layers
def producer_of(layer: int, G: int) -> int:
    """[MC] Method: producers sit at layers 0, G, 2G, ...; each predicts for
    itself and the next G - 1 layers.  Reading R4."""
    return G * (layer // G)


def consumer_slot(layer: int, G: int) -> int:
    """[MC] Method: a consumer at layer l uses slot (l - 1) mod G of its
    producer's importance queries.  Reading R4: non-negative mod."""
    return (layer - 1) % G


def importance_queries(q_imp_producer: np.ndarray, layer: int, G: int, B: int, Hq: int,
                       position: int = 0) -> np.ndarray:
    """[MC] Method: Q_imp has shape (B*H) x G x L x d'.  Returns the consumer's
    query per (b, h): q_hat[b, h] = Q_imp[b*Hq + h, slot, position, :]."""
    slot = consumer_slot(layer, G)
    q = np.asarray(q_imp_producer, dtype=np.float64)
    return q[:, slot, position, :].reshape(B, Hq, q.shape[-1])


def kv_head_of(h: int, Hq: int, Hkv: int) -> int:
    """Reading R2: contiguous groups of Hq / Hkv query heads share a KV head."""
    return h // (Hq // Hkv)


def keep_pct_from_policy(policy: str) -> int:
    """[MC] Memory requirements: "fixed_<N>pc" sparsifies N % of the tokens,
    i.e. retains 100 - N %."""
    if not (policy.startswith("fixed_") and policy.endswith("pc")):
        raise ValueError(f"unsupported policy {policy!r}")
    n = int(policy[len("fixed_"):-len("pc")])
    if not 0 <= n <= 100:
        raise ValueError(f"sparsity {n} % out of range")
    return 100 - n


# ------------------------------------------------------------------ a1: K_imp
def project_keys(K: np.ndarray, W_K: np.ndarray, storage: str = "f64") -> np.ndarray:
    """[MC] Method: K_imp = K . W_K on the post-RoPE cached keys (fp64, no
    rounding).  K: [..., D], W_K: [D, d'] (Reading R1).  storage="bf16": the
    bf16 K_imp cache option, each exact value rounded once to bfloat16."""
    kimp = np.asarray(K, dtype=np.float64) @ np.asarray(W_K, dtype=np.float64)
    return round_to_bf16(kimp) if storage == "bf16" else kimp


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Nearest bfloat16 value (8 significant bits, fp32's exponent range),
    ties to the even significand, returned as float64.  For finite |x| below
    the largest bfloat16; below 2^-126 the quantum is fixed at 2^-133
    (subnormal bfloat16)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                      # x = m * 2^e, 0.5 <= |m| < 1
    e = np.maximum(e, -125)                 # subnormal range: fixed quantum 2^-133
    q = np.ldexp(1.0, e - 8)                # one unit in the 8th significant bit
    return np.rint(x / q) * q               # np.rint rounds half to even; x / q is exact


# ------------------------------------------------------------------ a3: scores
def importance_scores(q_hat: np.ndarray, K_imp: np.ndarray) -> np.ndarray:
    """[MC] Method: score every cached token with the consumer's importance
    query: s[t] = q_hat . K_imp[t] (Reading R3: no scale).  q_hat: [d'],
    K_imp: [L, d']."""
    return np.asarray(K_imp, dtype=np.float64) @ np.asarray(q_hat, dtype=np.float64)


# ------------------------------------------------------------------ a4/a5: select
def token_budget(L: int, keep_pct: int) -> int:
    """Reading R5: k = floor(P * L / 100)."""
    return (keep_pct * L) // 100


def select_tokens(scores: np.ndarray, L: int, keep_pct: int, sink: int, window: int) -> np.ndarray:
    """[MC] Method + Memory requirements: the top-x tokens under a fixed
    budget, plus the sink prefix (min_sparse_index) and the recent window
    (sliding_window).  Returns the selected token indices, ascending.

    Candidates are [sink, L - window) (Reading R6); the budget is clamped to
    their number (R7); order is (score descending, index ascending) (R8)."""
    s = np.asarray(scores, dtype=np.float64)[:L]
    sink_set = np.arange(0, min(sink, L), dtype=np.int64)
    window_set = np.arange(max(L - window, 0), L, dtype=np.int64)
    cand = np.arange(sink, L - window, dtype=np.int64) if L - window > sink else np.zeros(0, np.int64)
    k = min(token_budget(L, keep_pct), cand.size)
    order = np.lexsort((cand, -s[cand]))  # primary key last: score desc, then index asc
    top = cand[order[:k]]
    return np.union1d(np.union1d(sink_set, window_set), top).astype(np.int64)


# ------------------------------------------------------------------ a6: attention
def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, idx: np.ndarray, scale: float):
    """[AB] + [MC] Method: exact attention over the selected tokens of the full
    KV cache: o = sum_{t in Sel} softmax_t(scale * q . K[t]) V[t].  Returns
    (o, lse) with lse = log sum_{t in Sel} exp(scale * q . K[t]) (natural log).
    Reading R9: scale = 1/sqrt(D)."""
    q = np.asarray(q, dtype=np.float64)
    idx = np.asarray(idx, dtype=np.int64)
    if idx.size == 0:
        return np.zeros(q.shape[-1], np.float64), -math.inf
    Ks = np.asarray(K, dtype=np.float64)[idx]
    Vs = np.asarray(V, dtype=np.float64)[idx]
    logits = scale * (Ks @ q)
    m = logits.max()
    w = np.exp(logits - m)
    z = w.sum()
    return (w @ Vs) / z, m + math.log(z)


# ------------------------------------------------------------------ group option
def group_scores(q_hat_heads: np.ndarray, K_imp: np.ndarray) -> np.ndarray:
    """Per-KV-group option: the group's per-head importance scores summed,
    s_g[t] = sum_h q_hat_h . K_imp[t] (fp64).  q_hat_heads: [GS][d']; K_imp:
    [L][d']."""
    q = np.asarray(q_hat_heads, dtype=np.float64)
    total = np.zeros(np.asarray(K_imp).shape[0], np.float64)
    for h in range(q.shape[0]):
        total += importance_scores(q[h], K_imp)
    return total


# ------------------------------------------------------------------ amortised selection
def reuse_decision(q_now, q_cached, L: int, len0: int, interval: int, tau: float, keep_pct: int, sink: int,
                   window: int) -> bool:
    """Reading R18: whether a row reuses its cached selection this step."""
    cand = L - window - sink if L - window > sink else 0
    k = min(token_budget(L, keep_pct), cand)
    if not (0 < k < cand):
        return False
    if len0 <= 0 or L < len0 or L - len0 > interval:
        return False
    a = np.asarray(q_now, dtype=np.float64)
    c = np.asarray(q_cached, dtype=np.float64)
    na, nc = math.sqrt(float(a @ a)), math.sqrt(float(c @ c))
    if na == 0.0 or nc == 0.0:
        return False
    return float(a @ c) / (na * nc) >= tau


def reused_set(cached: np.ndarray, len0: int, L: int, sink: int, window: int, radius: int) -> np.ndarray:
    """Reading R18: the set a reusing row attends to at length L."""
    cached = np.asarray(cached, dtype=np.int64)
    topk = cached[(cached >= sink) & (cached < len0 - window)]
    widened = set(topk.tolist())
    for d in range(1, radius + 1):
        widened.update((topk - d).tolist())
        widened.update((topk + d).tolist())
    keep = {t for t in widened if sink <= t < L - window}
    keep.update(range(0, min(sink, L)))
    keep.update(range(max(L - window, 0), L))
    return np.array(sorted(keep), dtype=np.int64)


# ------------------------------------------------------------------ one decode layer
def decode_layer(q, K, V, W_K, q_imp_producer, layer, G, L, keep_pct, sink, window, dense: bool,
                 K_imp=None, heads=None, batches=None, group: bool = False, kimp_storage: str = "f64"):
    """One consumer layer's decode step, [MC] Method in order:
    K_imp = K W_K; consumer slot (l - 1) mod G; score every cached token;
    top-k + sink + window per query head; attention over the selected tokens.
    A dense layer (layer 0, [MC] Memory requirements) attends to every token.

    q: [B][Hq][D]; K, V: [B][Hkv][>=L][D]; W_K: [D][d'];
    q_imp_producer: [(B*Hq)][G][1][d']; L: int or per-sequence list.
    Returns dicts keyed by (b, h): selected indices, output [D], lse; and the
    fp64 scores per (b, h) (None for dense layers).  With group=True (the
    per-KV-group option) the scores and the set are the head's group's.
    kimp_storage="bf16": scores are taken on the bf16-rounded K_imp."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, D = q.shape
    Hkv = K.shape[1]
    lens = [L] * B if np.isscalar(L) else list(L)
    scale = 1.0 / math.sqrt(D)
    heads = range(Hq) if heads is None else heads
    batches = range(B) if batches is None else batches
    sel, out, lse, scores = {}, {}, {}, {}
    q_hat = None if dense else importance_queries(q_imp_producer, layer, G, B, Hq)
    for b in batches:
        Lb = lens[b]
        kimp_b = {}
        for h in heads:
            g = kv_head_of(h, Hq, Hkv)
            if dense:
                idx = np.arange(Lb, dtype=np.int64)
                scores[b, h] = None
            else:
                if g not in kimp_b:
                    kimp_b[g] = (project_keys(K[b, g, :Lb], W_K, kimp_storage) if K_imp is None
                                 else np.asarray(K_imp[b, g, :Lb], dtype=np.float64))
                if group:
                    gs = Hq // Hkv
                    s = group_scores(q_hat[b, g * gs:(g + 1) * gs], kimp_b[g])
                else:
                    s = importance_scores(q_hat[b, h], kimp_b[g])
                scores[b, h] = s
                idx = select_tokens(s, Lb, keep_pct, sink, window)
            sel[b, h] = idx
            out[b, h], lse[b, h] = attend(q[b, h], K[b, g, :Lb], V[b, g, :Lb], idx, scale)
    return sel, out, lse, scores


# ------------------------------------------------------------------ sequence sharding (R19)
def merge_partials(outs, lses):
    """Attention over a set split into disjoint parts, from each part's
    normalised output o_r and log-sum-exp lse_r: weights exp(lse_r - lse)
    with lse = log sum_r exp(lse_r).  Parts with lse_r = -inf (empty) carry
    no weight; when every part is empty the result is a zero output and
    lse = -inf (as for an empty set)."""
    lses = np.asarray(lses, dtype=np.float64)
    outs = np.asarray(outs, dtype=np.float64)
    if np.all(np.isneginf(lses)):
        return np.zeros(outs.shape[1:]), -math.inf
    m = lses[~np.isneginf(lses)].max()
    w = np.where(np.isneginf(lses), 0.0, np.exp(lses - m))
    total = w.sum()
    return (w[:, None] * outs).sum(axis=0) / total, m + math.log(total)


def decode_layer_sharded(q, K, V, W_K, q_imp_producer, layer, G, L, keep_pct, sink, window, bounds,
                         group: bool = False, kimp_storage: str = "f64", heads=None, batches=None):
    """Reading R19: the decode step of one layer with the tokens split over
    ranks, bounds = [(t0_r, t1_r)] contiguous and in order.  The selected set
    is the unsharded step's; rank r attends over its part of it and the parts
    are merged (merge_partials).  Returns (sel, out, lse, parts) with parts
    {(b, h): [indices of rank r]}.  `heads`, `batches`: as for decode_layer."""
    sel, _, _, _ = decode_layer(q, K, V, W_K, q_imp_producer, layer, G, L, keep_pct, sink, window, dense=False,
                                group=group, kimp_storage=kimp_storage, heads=heads, batches=batches)
    q = np.asarray(q, dtype=np.float64)
    B, Hq, D = q.shape
    Hkv = K.shape[1]
    lens = [L] * B if np.isscalar(L) else list(L)
    scale = 1.0 / math.sqrt(D)
    out, lse, parts = {}, {}, {}
    for (b, h), idx in sel.items():
        g = kv_head_of(h, Hq, Hkv)
        pieces, outs, lses = [], [], []
        for t0, t1 in bounds:
            mine = idx[(idx >= t0) & (idx < t1)]
            o_r, l_r = attend(q[b, h], K[b, g, :lens[b]], V[b, g, :lens[b]], mine, scale)
            pieces.append(mine)
            outs.append(o_r)
            lses.append(l_r)
        out[b, h], lse[b, h] = merge_partials(outs, lses)
        parts[b, h] = pieces
    return sel, out, lse, parts


# ------------------------------------------------------------------ a7: prefill rows
def prefill_select(q_hat_rows: np.ndarray, K_imp: np.ndarray, row0: int, keep_pct: int, sink: int,
                   window: int) -> dict:
    """Per-row selection of a prefill query chunk (Reading R13): row p of head
    h scores its causal prefix s_p[t] = q_hat[h, p - row0] . K_imp[g(h), t],
    t <= p, and selects with L -> p + 1.  q_hat_rows: [Hq][nrows][d'];
    K_imp: [Hkv][>= row0 + nrows][d'].  Returns {(h, p): indices}."""
    Hq, nrows, _ = q_hat_rows.shape
    Hkv = K_imp.shape[0]
    out = {}
    for h in range(Hq):
        g = kv_head_of(h, Hq, Hkv)
        for r in range(nrows):
            p = row0 + r
            s = importance_scores(q_hat_rows[h, r], K_imp[g, :p + 1])
            out[h, p] = select_tokens(s, p + 1, keep_pct, sink, window)
    return out


# ------------------------------------------------------------------ a8: soft voting
def softvote_scores(q: np.ndarray, K: np.ndarray, L: int) -> np.ndarray:
    """[TS] Per-head Soft Voting: per-head criticality a[h, t] = q_h . K[g(h), t]
    / sqrt(D), normalised by a softmax over the tokens, summed over all heads
    (Reading R14).  q: [Hq][D]; K: [Hkv][>=L][D].  Returns votes [L]."""
    q = np.asarray(q, dtype=np.float64)
    Hq, D = q.shape
    Hkv = K.shape[0]
    votes = np.zeros(L, np.float64)
    for h in range(Hq):
        a = (np.asarray(K[kv_head_of(h, Hq, Hkv), :L], dtype=np.float64) @ q[h]) / math.sqrt(D)
        p = np.exp(a - a.max())
        votes += p / p.sum()
    return votes


def softvote_layer(q, K, V, L, keep_pct, sink, window, batches=None):
    """[TS] soft-voting variant of one decode layer: one shared selection per
    sequence from the summed per-head softmaxes, then exact attention per
    head over that set.  q: [B][Hq][D]; K, V: [B][Hkv][>=L][D]."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, D = q.shape
    Hkv = K.shape[1]
    lens = [L] * B if np.isscalar(L) else list(L)
    batches = range(B) if batches is None else batches
    sel, out, lse, votes = {}, {}, {}, {}
    for b in batches:
        votes[b] = softvote_scores(q[b], K[b], lens[b])
        sel[b] = select_tokens(votes[b], lens[b], keep_pct, sink, window)
        for h in range(Hq):
            g = kv_head_of(h, Hq, Hkv)
            out[b, h], lse[b, h] = attend(q[b, h], K[b, g, :lens[b]], V[b, g, :lens[b]], sel[b],
                                          1.0 / math.sqrt(D))
    return sel, out, lse, votes
