"""Pins for the float64 CPU oracle: it is checked against what the pages and the
mathematics fix -- hand-worked values (tests/golden/), closed forms, brute force on tiny
inputs, invariants, and special cases that reduce to a library routine (torch's float64
scaled_dot_product_attention on CPU).  None of these retypes the oracle's own formula.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _arr(x):
    """JSON nested lists (with "-inf" strings) -> float64 array."""
    return np.array(json.loads(json.dumps(x).replace('"-inf"', "-1e999")), dtype=np.float64)


# ----------------------------------------------------------------------------- scores
@pytest.mark.parametrize("relu", ["none", "post_sum", "per_head"])
def test_scores_hand_worked(relu):
    g = _load("index_score_worked.json")
    sc = O.index_scores(np.array(g["q_idx"], float), np.array(g["k_idx"], float),
                        np.array(g["w"], float), g["scale"], relu=relu)
    exp = _arr(g["scores"][relu])
    assert sc.shape == exp.shape
    assert np.array_equal(sc, exp)


def test_topk_hand_worked():
    g = _load("index_score_worked.json")
    args = (np.array(g["q_idx"], float), np.array(g["k_idx"], float), np.array(g["w"], float),
            g["scale"])
    for key, (relu, K) in {"none_K2": ("none", 2), "none_K3": ("none", 3),
                           "post_sum_K1": ("post_sum", 1), "per_head_K2": ("per_head", 2)}.items():
        sc = O.index_scores(*args, relu=relu)
        got = O.topk_indices(sc, K)
        assert got.dtype == np.int32
        assert np.array_equal(got, np.array(g["topk"][key])), key


def test_scores_all_ones_closed_form():
    # all-ones q_I, k_I: every head dot is DI, so score = scale * DI * sum_h w[s,h]
    B, S, HI, DI = 2, 5, 3, 7
    w = np.arange(B * S * HI, dtype=float).reshape(B, S, HI) % 4 + 1
    sc = O.index_scores(np.ones((B, S, HI, DI)), np.ones((B, S, DI)), w, 0.25)
    for b in range(B):
        for s in range(S):
            expect = 0.25 * DI * w[b, s].sum()
            assert np.all(sc[b, s, : s + 1] == expect)
            assert np.all(np.isneginf(sc[b, s, s + 1:]))


def test_scores_one_hot_orientation():
    # q_I[s,h] = e_{a(h)}, k_I[t] = c_t * e_j.  score = scale * c_t * sum_{h: a(h)=j} w[s,h].
    # A transposed operand (k indexed by s, or q by t) or a dropped head term fails this.
    S, T, HI, DI = 3, 6, 4, 5
    a = [0, 2, 2, 4]
    q = np.zeros((1, S, HI, DI))
    for h in range(HI):
        q[0, :, h, a[h]] = 1.0
    c = np.array([3.0, -1.0, 2.0, 5.0, -4.0, 1.0])
    j = 2
    k = np.zeros((1, T, DI))
    k[0, :, j] = c
    w = np.array([[[1.0, 2.0, 3.0, 4.0], [4.0, 3.0, 2.0, 1.0], [1.0, 1.0, 1.0, 1.0]]])
    sc = O.index_scores(q, k, w, 0.5)  # q_off = 3
    for s in range(S):
        for t in range(T):
            if t > s + 3:
                assert sc[0, s, t] == -np.inf
            else:
                assert sc[0, s, t] == 0.5 * c[t] * (w[0, s, 1] + w[0, s, 2])


def test_scores_invariants():
    rng = np.random.default_rng(1)
    B, S, T, HI, DI = 2, 6, 9, 4, 8
    q = rng.integers(-2, 3, (B, S, HI, DI)).astype(float)
    k = rng.integers(-2, 3, (B, T, DI)).astype(float)
    w = rng.integers(1, 5, (B, S, HI)).astype(float)
    base = O.index_scores(q, k, w, 2.0 ** -4)
    # permuting the heads (q and w together) changes nothing
    perm = [2, 0, 3, 1]
    assert np.array_equal(base, O.index_scores(q[:, :, perm], k, w[:, :, perm], 2.0 ** -4))
    # scores are linear in w and in scale
    assert np.array_equal(2 * base, O.index_scores(q, k, 2 * w, 2.0 ** -4))
    assert np.array_equal(base, O.index_scores(q, k, 2 * w, 2.0 ** -5))
    # causal boundary with q_off = T - S = 3
    s_pos = np.arange(S)[:, None] + 3
    assert np.array_equal(np.isneginf(base[0]), np.arange(T)[None, :] > s_pos)
    # batches are independent
    assert np.array_equal(base[1:], O.index_scores(q[1:], k[1:], w[1:], 2.0 ** -4))


def test_scores_relu_modes_relationship():
    rng = np.random.default_rng(2)
    q = rng.integers(-2, 3, (1, 4, 3, 4)).astype(float)
    k = rng.integers(-2, 3, (1, 4, 4)).astype(float)
    w = rng.integers(1, 5, (1, 4, 3)).astype(float)
    none = O.index_scores(q, k, w, 1.0)
    post = O.index_scores(q, k, w, 1.0, relu="post_sum")
    per = O.index_scores(q, k, w, 1.0, relu="per_head")
    fin = np.isfinite(none)
    assert np.array_equal(post[fin], np.maximum(none[fin], 0))
    # with non-negative weights, the per-head form is >= the post-sum form
    assert np.all(per[fin] >= post[fin])
    with pytest.raises(ValueError):
        O.index_scores(q, k, w, 1.0, relu="bogus")


# ----------------------------------------------------------------------------- top-k
def _brute_force_topk(row, K):
    """The unique K-subset whose every member beats every non-member in the order
    (higher score, then lower index), found by enumerating all subsets."""
    n = len(row)
    kk = min(K, n)
    beats = lambda a, b: (row[a] > row[b]) or (row[a] == row[b] and a < b)  # noqa: E731
    found = []
    for sub in itertools.combinations(range(n), kk):
        rest = set(range(n)) - set(sub)
        if all(beats(a, b) for a in sub for b in rest):
            found.append(sub)
    assert len(found) == 1
    return list(found[0]) + [-1] * (K - kk)


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(3)
    for trial in range(60):
        T = int(rng.integers(1, 9))
        S = int(rng.integers(1, T + 1))
        K = int(rng.integers(1, 5))
        sc = rng.integers(-2, 3, (1, S, T)).astype(float) * 0.5  # many ties
        q_off = T - S
        for s in range(S):
            sc[0, s, s + q_off + 1:] = -np.inf
        got = O.topk_indices(sc, K)
        for s in range(S):
            n = s + q_off + 1
            assert got[0, s].tolist() == _brute_force_topk(sc[0, s, :n].tolist(), K), (trial, s)


def test_topk_special_cases():
    # all-equal row: the tie-break keeps the K lowest indices
    sc = np.zeros((1, 1, 10))
    assert O.topk_indices(sc, 4)[0, 0].tolist() == [0, 1, 2, 3]
    # -0.0 and +0.0 tie
    row = np.array([[[0.0, -0.0, 0.0]]])
    assert O.topk_indices(row, 1)[0, 0].tolist() == [0]
    row = np.array([[[-0.0, 0.0, 0.0]]])
    assert O.topk_indices(row, 1)[0, 0].tolist() == [0]
    # fewer valid keys than K: all valid keys, then -1
    sc = np.array([[[1.0, 2.0, -np.inf, -np.inf]]])
    assert O.topk_indices(sc, 3, q_off=1)[0, 0].tolist() == [0, 1, -1]
    # descending scores still come out in ascending index order
    sc = np.array([[[5.0, 4.0, 3.0, 9.0, 1.0]]])
    assert O.topk_indices(sc, 3)[0, 0].tolist() == [0, 1, 3]


# ----------------------------------------------------------------------------- attention
def test_attention_two_keys_hand_worked():
    g = _load("attention_two_keys.json")
    q, k, v = (np.array(g[n]) for n in ("q", "k", "v"))
    idx = np.array(g["idx"], dtype=np.int32)
    out = O.sparse_attention(q, k, v, idx, sm_scale=g["sm_scale"])
    assert np.allclose(out, np.array(g["out"]), rtol=0, atol=1e-13)
    outg = O.sparse_attention(q, k, v, idx, sm_scale=1.0, gate=np.array(g["gate_ln3"]),
                              gate_mode="sigmoid")
    assert np.allclose(outg, np.array(g["out_sigmoid_gate_ln3"]), rtol=0, atol=1e-13)
    outs = O.sparse_attention(q, k, v, idx, sm_scale=1.0, gate=np.zeros((1, 1, 1)),
                              gate_mode="silu")
    assert np.array_equal(outs, np.array(g["out_silu_gate_0"]))


def test_attention_sinks_hand_worked():
    g = _load("attention_sink.json")
    q, k, v = (np.array(g[n]) for n in ("q", "k", "v"))
    sk, sv = np.array(g["sink_k"]), np.array(g["sink_v"])
    out = O.sparse_attention(q, k, v, np.array(g["idx"], dtype=np.int32), sm_scale=1.0,
                             sink_k=sk, sink_v=sv)
    assert np.allclose(out, np.array(g["out"]), rtol=0, atol=1e-12)
    out0 = O.sparse_attention(q, k, v, np.array(g["idx_none"], dtype=np.int32), sm_scale=1.0,
                              sink_k=sk, sink_v=sv)
    assert np.allclose(out0, np.array(g["out_sinks_only"]), rtol=0, atol=1e-12)


def test_attention_sinks_library_special_cases():
    # (1) with no selected key the result is plain SDPA of the query over the sink entries;
    # (2) a sink that copies a selected key equals SDPA with that key listed twice;
    # (3) sinks far below every logit change nothing; (4) the order of the sinks does not matter
    rng = np.random.default_rng(5)
    B, S, T, H, D, DV, NS = 1, 5, 9, 3, 8, 6, 4
    q, k = rng.standard_normal((B, S, H, D)), rng.standard_normal((B, T, H, D))
    v = rng.standard_normal((B, T, H, DV))
    sk, sv = rng.standard_normal((NS, H, D)), rng.standard_normal((NS, H, DV))
    # (1)
    none = -np.ones((B, S, 2), dtype=np.int32)
    got = O.sparse_attention(q, k, v, none, sink_k=sk, sink_v=sv)
    ref = _sdpa_f64(q, np.ascontiguousarray(np.broadcast_to(sk[None], (B, NS, H, D))),
                    np.ascontiguousarray(np.broadcast_to(sv[None], (B, NS, H, DV))),
                    causal=False)
    assert np.allclose(got, ref, rtol=0, atol=1e-12)
    # (2) every query selects keys 0 and 3 (3 only where causal: q_off = 4); the one sink
    # is a copy of key 3, always visible
    idx = np.stack([np.zeros((B, S), np.int32), np.full((B, S), 3, np.int32)], axis=-1)
    got = O.sparse_attention(q, k, v, idx, sink_k=k[0, 3:4], sink_v=v[0, 3:4])
    for s in range(S):
        keys = [0, 3, 3] if s + (T - S) >= 3 else [0, 3]
        ref = _sdpa_f64(q[:, s:s + 1], k[:, keys], v[:, keys], causal=False)
        assert np.allclose(got[:, s:s + 1], ref, rtol=0, atol=1e-12)
    # (3) positive queries and sink keys of -1e3: logits below the others by > 1e3 (keys
    # 0..4 are visible to every query, q_off = 4, so no row is left to the sinks alone)
    sel = rng.integers(0, T - S + 1, (B, S, 4)).astype(np.int32)
    qq = np.abs(q) + 1.0
    got = O.sparse_attention(qq, k, v, sel, sink_k=np.full((NS, H, D), -1e3),
                             sink_v=np.full((NS, H, DV), 1e6))
    assert np.array_equal(got, O.sparse_attention(qq, k, v, sel))
    # (4)
    perm = rng.permutation(NS)
    a = O.sparse_attention(q, k, v, sel, sink_k=sk, sink_v=sv)
    b = O.sparse_attention(q, k, v, sel, sink_k=sk[perm], sink_v=sv[perm])
    assert np.allclose(a, b, rtol=0, atol=1e-13)


def _sdpa_f64(q, k, v, causal=True, mask=None, scale=None):
    """torch's CPU float64 SDPA, [B,S,H,D] layout in and out."""
    tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(x)).transpose(1, 2) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, attn_mask=None if mask is None else torch.from_numpy(mask),
        is_causal=causal and mask is None, scale=scale)
    return o.transpose(1, 2).numpy()


def test_full_selection_reduces_to_causal_attention():
    # K >= causal length: every causal key is selected, so DSA == plain causal attention
    rng = np.random.default_rng(4)
    B, S, H, Dqk, Dv = 2, 12, 3, 8, 6
    q, k = rng.standard_normal((2, B, S, H, Dqk))
    v = rng.standard_normal((B, S, H, Dv))
    qi = rng.integers(-2, 3, (B, S, 2, 4)).astype(float)
    ki = rng.integers(-2, 3, (B, S, 4)).astype(float)
    w = rng.integers(1, 5, (B, S, 2)).astype(float)
    _, idx, out = O.dsa_forward(qi, ki, w, 0.25, S, q, k, v)
    # row s keeps every causal key 0..s, then -1 padding
    expect_idx = np.where(np.arange(S)[None, :] <= np.arange(S)[:, None], np.arange(S)[None, :], -1)
    assert np.array_equal(idx, np.broadcast_to(expect_idx, idx.shape))
    ref = _sdpa_f64(q, k, v, causal=True)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_attention_closed_forms():
    rng = np.random.default_rng(5)
    B, S, T, H, Dqk, Dv, K = 1, 5, 9, 2, 6, 4, 3
    q = rng.standard_normal((B, S, H, Dqk))
    k = rng.standard_normal((B, T, H, Dqk))
    idx = np.stack([np.sort(rng.choice(s + 5, size=K, replace=False)) for s in range(S)])[None]
    idx = idx.astype(np.int32)
    # V constant per head -> output equals that constant
    v = np.broadcast_to(np.array([1.5, -2.0, 0.25, 3.0]), (B, T, H, Dv)).copy()
    out = O.sparse_attention(q, k, v, idx)
    assert np.allclose(out, v[:, :S], rtol=0, atol=1e-14)
    # a single selected key -> output is exactly that key's v row
    v = rng.standard_normal((B, T, H, Dv))
    one = np.full((B, S, K), -1, np.int32)
    one[0, :, 0] = [1, 0, 3, 2, 4]
    out = O.sparse_attention(q, k, v, one)
    for s in range(S):
        assert np.array_equal(out[0, s], v[0, one[0, s, 0]])


def test_attention_masking_invariants():
    rng = np.random.default_rng(6)
    B, S, T, H, Dqk, Dv, K = 1, 6, 10, 2, 4, 3, 3
    q = rng.standard_normal((B, S, H, Dqk))
    k = rng.standard_normal((B, T, H, Dqk))
    v = rng.standard_normal((B, T, H, Dv))
    idx = np.stack([np.sort(rng.choice(s + 5, size=K, replace=False)) for s in range(S)])[None]
    idx = idx.astype(np.int32)
    base = O.sparse_attention(q, k, v, idx)
    # poisoning every unselected key leaves each row bitwise unchanged
    for s in range(S):
        k2, v2 = k.copy(), v.copy()
        unsel = np.setdiff1d(np.arange(T), idx[0, s])
        k2[0, unsel] = 50.0
        v2[0, unsel] = 1e4
        assert np.array_equal(O.sparse_attention(q, k2, v2, idx)[0, s], base[0, s])
    # a selected index in the future of the query is masked by the causal mask
    fut = idx.copy()
    fut[0, 0, 0] = 9  # query 0 sits at position 4, so key 9 is in its future
    dropped = idx.copy()
    dropped[0, 0, 0] = -1
    ref = O.sparse_attention(q, k, v, dropped)
    assert np.array_equal(O.sparse_attention(q, k, v, fut), ref)
    # -1 and out-of-range entries are skipped; an empty row gives zeros
    empty = np.full((B, S, K), -1, np.int32)
    empty[0, 1] = [T + 3, -1, -7]
    assert np.array_equal(O.sparse_attention(q, k, v, empty), np.zeros((B, S, H, Dv)))


def test_gate_closed_forms():
    rng = np.random.default_rng(7)
    o = rng.standard_normal((2, 3, 4, 5))
    # gate logits at 0 scale the output by exactly 0.5
    assert np.array_equal(O.apply_gate(o, np.zeros((2, 3, 4)), "sigmoid"), o * 0.5)
    # gate off is the identity
    assert np.array_equal(O.apply_gate(o, None, "off"), o)
    # sigmoid(ln 3) = 3/4, sigmoid(-ln 3) = 1/4; silu(ln 3) = (3/4) ln 3
    g = np.full((2, 3, 4), math.log(3.0))
    assert np.allclose(O.apply_gate(o, g, "sigmoid"), 0.75 * o, rtol=1e-15, atol=0)
    assert np.allclose(O.apply_gate(o, -g, "sigmoid"), 0.25 * o, rtol=1e-15, atol=0)
    assert np.allclose(O.apply_gate(o, g, "silu"), 0.75 * math.log(3.0) * o, rtol=1e-15, atol=0)
    # one scalar per (token, head): the gate never mixes heads or dims
    g = rng.standard_normal((2, 3, 4))
    got = O.apply_gate(o, g, "sigmoid")
    assert np.allclose(got[1, 2, 3], o[1, 2, 3] / (1 + math.exp(-g[1, 2, 3])), rtol=1e-15)
    with pytest.raises(ValueError):
        O.apply_gate(o, g, "tanh")


# ----------------------------------------------------------------------------- SWA
def test_window_attention_library_special_cases():
    rng = np.random.default_rng(8)
    B, S, H, HKV, Dqk, Dv = 1, 20, 4, 2, 8, 6
    q = rng.standard_normal((B, S, H, Dqk))
    k = rng.standard_normal((B, S, HKV, Dqk))
    v = rng.standard_normal((B, S, HKV, Dv))
    kr = np.repeat(k, H // HKV, axis=2)
    vr = np.repeat(v, H // HKV, axis=2)
    # a window at least as long as the sequence is plain causal attention
    full = O.window_attention(q, k, v, window=S)
    assert np.allclose(full, _sdpa_f64(q, kr, vr, causal=True), rtol=1e-12, atol=1e-12)
    # a band of W keys equals SDPA with the explicit band mask
    W = 5
    i = np.arange(S)[:, None]
    j = np.arange(S)[None, :]
    band = (j <= i) & (j > i - W)
    got = O.window_attention(q, k, v, window=W)
    assert np.allclose(got, _sdpa_f64(q, kr, vr, mask=band), rtol=1e-12, atol=1e-12)
    # window 1: each query sees only itself
    one = O.window_attention(q, k, v, window=1)
    for h in range(H):
        assert np.array_equal(one[0, :, h], v[0, :, h // (H // HKV)])


def test_window_equals_sparse_with_band_indices():
    # the SWA band is a particular index set: DSA attention over it gives the same result
    rng = np.random.default_rng(9)
    B, S, H, Dqk, Dv, W = 1, 12, 2, 4, 4, 4
    q, k = rng.standard_normal((2, B, S, H, Dqk))
    v = rng.standard_normal((B, S, H, Dv))
    idx = np.full((B, S, W), -1, np.int32)
    for s in range(S):
        band = np.arange(max(0, s - W + 1), s + 1)
        idx[0, s, : band.size] = band
    assert np.allclose(O.window_attention(q, k, v, W), O.sparse_attention(q, k, v, idx),
                       rtol=1e-13, atol=1e-13)
    # the same with attention sinks in both (H == HKV, so the KV-head map is the identity)
    sk, sv = rng.standard_normal((3, H, Dqk)), rng.standard_normal((3, H, Dv))
    assert np.allclose(O.window_attention(q, k, v, W, sink_k=sk, sink_v=sv),
                       O.sparse_attention(q, k, v, idx, sink_k=sk, sink_v=sv),
                       rtol=1e-13, atol=1e-13)


def test_window_sinks_with_grouped_heads():
    # GQA: query head h sees the sinks of KV head h // G.  (1) Expanding K, V and the sinks
    # to one head per query head gives the same result; (2) with window 1 (each query sees
    # only its own key) the result is SDPA of the query over {its key, its head's sinks}.
    rng = np.random.default_rng(13)
    B, S, H, HKV, D, Dv, W, NS = 1, 7, 4, 2, 8, 5, 3, 2
    G = H // HKV
    q = rng.standard_normal((B, S, H, D))
    k, v = rng.standard_normal((B, S, HKV, D)), rng.standard_normal((B, S, HKV, Dv))
    sk, sv = rng.standard_normal((NS, HKV, D)), rng.standard_normal((NS, HKV, Dv))
    got = O.window_attention(q, k, v, W, sink_k=sk, sink_v=sv)
    rep = lambda x, ax: np.repeat(x, G, axis=ax)  # noqa: E731
    ref = O.window_attention(q, rep(k, 2), rep(v, 2), W, sink_k=rep(sk, 1), sink_v=rep(sv, 1))
    assert np.allclose(got, ref, rtol=0, atol=1e-13)
    one = O.window_attention(q, k, v, 1, sink_k=sk, sink_v=sv)
    for s in range(S):
        for h in range(H):
            kh = h // G
            keys = np.concatenate([k[0, s:s + 1, kh], sk[:, kh]])[None, :, None]
            vals = np.concatenate([v[0, s:s + 1, kh], sv[:, kh]])[None, :, None]
            r = _sdpa_f64(q[:, s:s + 1, h:h + 1], keys, vals, causal=False)
            assert np.allclose(one[0, s, h], r[0, 0, 0], rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- decode
def test_decode_row_equals_last_prefill_row():
    # decode: one new query at position T-1 against the whole cache == last prefill row
    rng = np.random.default_rng(10)
    B, T, HI, DI, H, Dqk, Dv, K = 2, 16, 2, 4, 2, 6, 4, 5
    qi = rng.integers(-2, 3, (B, T, HI, DI)).astype(float)
    ki = rng.integers(-2, 3, (B, T, DI)).astype(float)
    w = rng.integers(1, 5, (B, T, HI)).astype(float)
    q, k = rng.standard_normal((2, B, T, H, Dqk))
    v = rng.standard_normal((B, T, H, Dv))
    g = rng.standard_normal((B, T, H))
    sc_p, idx_p, out_p = O.dsa_forward(qi, ki, w, 0.125, K, q, k, v, gate=g, gate_mode="sigmoid")
    sc_d, idx_d, out_d = O.dsa_forward(qi[:, -1:], ki, w[:, -1:], 0.125, K, q[:, -1:], k, v,
                                       gate=g[:, -1:], gate_mode="sigmoid")
    assert np.array_equal(sc_d[:, 0], sc_p[:, -1])
    assert np.array_equal(idx_d[:, 0], idx_p[:, -1])
    assert np.allclose(out_d[:, 0], out_p[:, -1], rtol=1e-14, atol=1e-14)


def test_hadamard_rotation_pins():
    # H is symmetric and H H = d I: rotating twice is the identity; rotation preserves dot
    # products (the scores do not change); the first basis vector maps to the all-equal
    # vector 1/sqrt(d); a hand-written 4x4 case
    rng = np.random.default_rng(9)
    for d in (4, 64, 128):
        x = rng.standard_normal((3, 5, d))
        assert np.allclose(O.hadamard_rotate(O.hadamard_rotate(x)), x, rtol=0, atol=1e-12)
        y = rng.standard_normal((7, d))
        assert np.allclose(O.hadamard_rotate(x[0]) @ O.hadamard_rotate(y).T, x[0] @ y.T,
                           rtol=0, atol=1e-10)
        e0 = np.zeros(d)
        e0[0] = 1.0
        assert np.allclose(O.hadamard_rotate(e0), np.full(d, d ** -0.5), rtol=0, atol=1e-15)
    x4 = np.array([1.0, 2.0, 3.0, 4.0])
    # rows of H_4: (1,1,1,1), (1,-1,1,-1), (1,1,-1,-1), (1,-1,-1,1); x @ H / 2
    assert np.allclose(O.hadamard_rotate(x4), np.array([10.0, -2.0, -4.0, 0.0]) / 2.0,
                       rtol=0, atol=1e-15)
    # the indexer scores are unchanged when both q_I and k_I are rotated
    cfg_q = rng.integers(-2, 3, (1, 6, 4, 64)).astype(np.float64)
    cfg_k = rng.integers(-2, 3, (1, 9, 64)).astype(np.float64)
    w = rng.integers(1, 5, (1, 6, 4)).astype(np.float64)
    a = O.index_scores(cfg_q, cfg_k, w, 0.25)
    b = O.index_scores(O.hadamard_rotate(cfg_q), O.hadamard_rotate(cfg_k), w, 0.25)
    fin = np.isfinite(a)
    assert np.array_equal(np.isfinite(b), fin)
    assert np.allclose(a[fin], b[fin], rtol=0, atol=1e-9)



# ------------------------------------------------------------ latent (MQA-form) attention
def test_latent_attention_hand_worked():
    """Two selected rows of a 2-dim latent cache, dv = 1, sm_scale 1.  With q = (ln 3, 0) the
    logits are 0 and ln 3, so the weights are 1/4 and 3/4; the values are the rows' first
    dims, 0 and 1: output 3/4.  q = 0 weighs the two rows equally: 1/2.  Row 2 (a large
    value) is not selected and must not count."""
    kv = np.array([[[0.0, 0.0], [1.0, 5.0], [7.0, -3.0]]])  # [B=1, T=3, 2]
    q = np.array([[[[math.log(3.0), 0.0], [0.0, 0.0]]]])  # [B=1, S=1, H=2, 2]
    idx = np.array([[[0, 1]]])
    out = O.sparse_attention_latent(q, kv, idx, dv=1, sm_scale=1.0)
    assert out.shape == (1, 1, 2, 1)
    np.testing.assert_allclose(out[0, 0, :, 0], [0.75, 0.5], rtol=0, atol=1e-15)


def test_latent_attention_equals_the_per_head_form():
    """Setting every head's key row to the shared latent row and its value row to the latent
    row's first dv dims turns the per-head sparse attention (pinned against SDPA) into the
    latent form: both give the same output, with and without sinks and the gate.  The index
    lists hold -1, out-of-range and future entries."""
    rng = np.random.default_rng(11)
    B, S, T, H, D, dv, K = 2, 6, 9, 3, 8, 5, 4
    q = rng.standard_normal((B, S, H, D))
    kv = rng.standard_normal((B, T, D))
    idx = rng.integers(-1, T + 2, size=(B, S, K))
    g = rng.standard_normal((B, S, H))
    k = np.repeat(kv[:, :, None, :], H, axis=2)
    v = np.ascontiguousarray(k[..., :dv])
    for sinks in (None, rng.standard_normal((3, D))):
        for gm in ("off", "sigmoid"):
            gate = g if gm != "off" else None
            a = O.sparse_attention_latent(q, kv, idx, dv, gate=gate, gate_mode=gm, sink_kv=sinks)
            sk = sv = None
            if sinks is not None:
                sk = np.repeat(sinks[:, None, :], H, axis=1)
                sv = np.ascontiguousarray(sk[..., :dv])
            b = O.sparse_attention(q, k, v, idx, gate=gate, gate_mode=gm, sink_k=sk, sink_v=sv)
            np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)


def test_latent_attention_closed_forms():
    """One selected row gives every head that row's first dv dims; q = 0 gives every head
    the mean of the selected rows' values; rows that are unselected or in the future never
    count (poisoned with 1e4); permuting the heads of q permutes the output."""
    rng = np.random.default_rng(12)
    B, S, T, H, D, dv = 1, 4, 10, 5, 6, 4
    kv = rng.standard_normal((B, T, D))
    q = rng.standard_normal((B, S, H, D))
    q_off = T - S
    # a single selected key per query, plus a future key that the causal mask must drop
    idx = np.array([[[3, T - 1], [5, -1], [0, 2 * T], [7, -1]]])
    poisoned = kv.copy()
    poisoned[0, 8] = 1e4  # selected only by the first query, at t = 9 > 0 + q_off: future
    out = O.sparse_attention_latent(q, poisoned, idx, dv)
    for s, t in enumerate([3, 5, 0, 7]):
        np.testing.assert_allclose(out[0, s], np.broadcast_to(poisoned[0, t, :dv], (H, dv)),
                                   rtol=0, atol=1e-12)
    # q = 0: uniform weights over the selected causal rows
    sel = np.array([[[1, 4, 6, -1]] * S])
    out0 = O.sparse_attention_latent(np.zeros_like(q), kv, sel, dv)
    mean = kv[0, [1, 4, 6], :dv].mean(axis=0)
    for s in range(S):
        np.testing.assert_allclose(out0[0, s], np.broadcast_to(mean, (H, dv)), rtol=0,
                                   atol=1e-12)
    # head permutation
    perm = rng.permutation(H)
    sel3 = rng.integers(0, q_off + 1, size=(B, S, 3))
    a = O.sparse_attention_latent(q[:, :, perm], kv, sel3, dv)
    b = O.sparse_attention_latent(q, kv, sel3, dv)[:, :, perm]
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_latent_decode_row_equals_last_prefill_row():
    """A decode call (one query at position T-1) equals the last query row of the prefill call
    over the same cache and the same index list, sinks and gate included."""
    rng = np.random.default_rng(13)
    B, S, T, H, D, dv, K = 2, 7, 7, 4, 8, 6, 5
    q = rng.standard_normal((B, S, H, D))
    kv = rng.standard_normal((B, T, D))
    idx = np.stack([np.stack([np.sort(rng.choice(s + 1, size=min(K, s + 1), replace=False))
                              .tolist() + [-1] * (K - min(K, s + 1)) for s in range(S)])
                    for _ in range(B)])
    g = rng.standard_normal((B, S, H))
    sink = rng.standard_normal((2, D))
    full = O.sparse_attention_latent(q, kv, idx, dv, gate=g, gate_mode="sigmoid", sink_kv=sink)
    last = O.sparse_attention_latent(q[:, -1:], kv, idx[:, -1:], dv, gate=g[:, -1:],
                                     gate_mode="sigmoid", sink_kv=sink)
    np.testing.assert_allclose(last[:, 0], full[:, -1], rtol=0, atol=1e-13)
