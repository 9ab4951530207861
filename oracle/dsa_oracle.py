"""Plain, slow, float64 CPU oracle for the DeepSeek-style sparse attention (DSA) hot path.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or link this
module: only the test suite, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it.  It shares no code with the CUDA
library (``sparse_attention_15_b200``) and imports nothing from it.

Every function is written straight from the definition it cites, in float64, with
numpy matmuls / sorts as the only library steps.  Sources (web pages, by title):

* [AXK2]  "Transformers 中的 AXK2 架构解析：SK Telecom A.X-K2 稀疏注意力 MoE 大模型集成指南",
  sections "注意力前向的骨架：MLA + 显式稀疏掩码" and
  "SK Telecom 三大改进 / 1. Sparse Gated Attention（SGA）", and
  "AXK2Config：核心配置与默认值" (index_topk clamp).
* [SPARK] Spark-X2.5-1.7B-Base headwise attention output gate walkthrough, sections
  "在 Spark-X2.5-1.7B-Base 中如何开启？" and "前向流程：从 gate_score 计算到相乘".
* [DSV2]  DeepSeek-V2 attention parameter guide ("参数详解"), items 4-6
  (qk_nope_head_dim, qk_rope_head_dim, v_head_dim).
* [PANGU] openPangu-2.0 technical-report reading, §3.2 (SWA, window 512, DSA-SWA-SWA),
  §3.3 (Lightning Indexer, fixed K), §3.5 Table 1 (cost model).

Readings where the pages are silent (each also listed in the design notes):

* top-k tie-break: higher score first, then lower key index; -0.0 equals +0.0.
* top-k output order: ascending key index; rows with fewer valid keys than K are padded
  with -1 after the valid keys.
* ReLU placement in the indexer: the printed formula has none (``relu="none"``, the
  graded mode); the prose's "weighted sum, then ReLU" is ``relu="post_sum"``; the
  per-head form ``relu="per_head"`` (ReLU of each head's dot product before weighting)
  is offered as an option.
* attention scale defaults to 1/sqrt(qk_nope + qk_rope), the SDPA default.
* gate rounding: multiply in float, round once (the A.X-K2 order).
* an attention row with no selectable key outputs zeros.
* SWA window W covers keys s+q_off-W < t <= s+q_off (W keys including the query itself).
* latent (MQA-form) attention: every head attends over the same cached latent row, keys
  = the whole row, values = its first dv dims (the absorbed MLA form flash-mla consumes).

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py`` against
closed forms, hand-worked values (``tests/golden/``), brute force and library special
cases (torch's float64 scaled_dot_product_attention on CPU).
"""
from __future__ import annotations

import numpy as np

RELU_MODES = ("none", "post_sum", "per_head")
GATE_MODES = ("off", "sigmoid", "silu")


def _f64(x):
    """Convert a numpy array or a CPU torch tensor (any float dtype, incl. bf16) to float64."""
    if hasattr(x, "detach"):  # torch tensor: go through float32, which holds bf16 exactly
        x = x.detach().cpu()
        if x.dtype.is_floating_point:
            x = x.float()
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


def index_scores(q_idx, k_idx, w, scale, relu="none", q_off=None):
    """Lightning-indexer scores, with the causal mask applied.

    [AXK2] SGA section: index_score[b,s,t] = sum_h weight[b,s,h] * softmax_scale *
    (q[b,s,h,:] . k[b,t,:]); causality comes from adding the causal mask while scoring.
    [PANGU] §3.3: the indexer scores each query against the historical keys.

    q_idx [B,S,HI,DI], k_idx [B,T,DI], w [B,S,HI]; ``q_off`` is the position of query 0
    (defaults to T-S, i.e. the queries are the last S of the T positions).
    Returns float64 [B,S,T] with -inf where t > s + q_off.
    """
    if relu not in RELU_MODES:
        raise ValueError(f"relu mode {relu!r} not in {RELU_MODES}")
    q = _f64(q_idx)
    k = _f64(k_idx)
    wt = _f64(w)
    B, S, HI, DI = q.shape
    T = k.shape[1]
    if q_off is None:
        q_off = T - S
    # per-head dot products d[b,s,h,t] = q[b,s,h,:] . k[b,t,:]   (a plain matmul)
    dots = np.matmul(q, np.swapaxes(k, 1, 2)[:, None])
    if relu == "per_head":
        dots = np.maximum(dots, 0.0)
    # weighted sum over heads, each head term carrying the softmax_scale factor
    score = np.matmul((wt * float(scale))[:, :, None, :], dots)[:, :, 0, :]
    if relu == "post_sum":
        score = np.maximum(score, 0.0)
    s_pos = np.arange(S)[:, None] + q_off
    t_pos = np.arange(T)[None, :]
    score = np.where((t_pos <= s_pos)[None], score, -np.inf)
    return score


def topk_indices(scores, K, q_off=None):
    """Per-query top-k over the causal keys.

    [AXK2] SGA section: the indexer returns int32 token indices of shape [B, S, topk];
    "AXK2Config" section: topk = min(index_topk, number of keys).
    [PANGU] §3.3: a fixed K (e.g. 2048) of historical keys is selected per query.

    Each row keeps the min(K, n) valid keys (t <= s + q_off, n of them) that come first
    in the order (higher score, then lower index); they are emitted in ascending index
    order and the rest of the row is -1.  Returns int32 [B,S,K].
    """
    sc = _f64(scores)
    B, S, T = sc.shape
    if q_off is None:
        q_off = T - S
    out = np.full((B, S, K), -1, dtype=np.int32)
    for b in range(B):
        for s in range(S):
            n = min(T, s + q_off + 1)
            if n <= 0:
                continue
            t = np.arange(n)
            v = sc[b, s, :n] + 0.0  # + 0.0 turns -0.0 into +0.0
            order = np.lexsort((t, -v))  # primary: score descending, then index ascending
            keep = np.sort(order[: min(K, n)])
            out[b, s, : keep.size] = keep
    return out


def _gate_factor(g, gate_mode):
    """[SPARK] forward step 3: gate = sigmoid(g) or silu(g), evaluated in float."""
    g = _f64(g)
    if gate_mode == "sigmoid":
        return 1.0 / (1.0 + np.exp(-g))
    if gate_mode == "silu":
        return g / (1.0 + np.exp(-g))
    raise ValueError(f"gate mode {gate_mode!r} not in {GATE_MODES}")


def apply_gate(o, g, gate_mode="sigmoid"):
    """Headwise output gate: o[b,s,h,:] * act(g[b,s,h]).

    [SPARK] "前向流程" steps 2-3: one scalar gate per (token, head), broadcast over the
    head dimension; act is sigmoid (or silu), computed in float.  [AXK2] SGA/output-gate
    section: the attention output is multiplied by the sigmoid gate before o_proj.
    ``gate_mode="off"`` returns ``o`` unchanged (the gate is an optional switch, [SPARK]).
    """
    o = _f64(o)
    if gate_mode == "off" or g is None:
        return o
    return o * _gate_factor(g, gate_mode)[..., None]


def sparse_attention(q, k, v, idx, sm_scale=None, gate=None, gate_mode="off", q_off=None,
                     sink_k=None, sink_v=None):
    """Attention over the indexer-selected keys, by dense masked softmax.

    [AXK2] "注意力前向的骨架": the selected positions become an additive sparse mask that
    is folded, together with the causal mask, into attention_mask; every other position
    is -inf, and the attention runs with that mask (eager/SDPA).  [AXK2] notes that the
    cache holds the expanded per-head K/V (expand_kv output); [DSV2] items 4-6 give the
    head widths qk_nope + qk_rope for q/k and v_head_dim for v.

    q [B,S,H,Dqk], k [B,T,H,Dqk], v [B,T,H,Dv], idx [B,S,K] (entries outside [0,T) or
    equal to -1 are ignored).  Returns float64 [B,S,H,Dv].

    Optional attention sinks, [PANGU] §3.4 (PAS): a layer's learnable key-value pairs
    act at inference as a fixed set of virtual KV entries that every query sees.  sink_k
    [NS,H,Dqk] and sink_v [NS,H,Dv] (the per-head form, like the expanded cache) join the
    softmax of every query, unmasked, beside its selected keys.
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    idx = np.asarray(idx)
    sinks = sink_k is not None
    if sinks:
        sk = _f64(sink_k).transpose(1, 0, 2)  # [H,NS,Dqk]
        sv = _f64(sink_v).transpose(1, 0, 2)  # [H,NS,Dv]
    B, S, H, Dqk = q.shape
    T = k.shape[1]
    if q_off is None:
        q_off = T - S
    if sm_scale is None or sm_scale <= 0:
        sm_scale = 1.0 / np.sqrt(Dqk)
    out = np.zeros((B, S, H, v.shape[-1]), dtype=np.float64)
    for b in range(B):
        kt = k[b].transpose(1, 0, 2)  # [H,T,Dqk]
        vt = v[b].transpose(1, 0, 2)  # [H,T,Dv]
        for s in range(S):
            allowed = np.zeros(T, dtype=bool)
            sel = idx[b, s]
            sel = sel[(sel >= 0) & (sel < T)]
            allowed[sel] = True
            allowed[np.arange(T) > s + q_off] = False  # the causal mask
            if not allowed.any() and not sinks:
                continue
            logits = sm_scale * np.matmul(kt, q[b, s][:, :, None])[:, :, 0]  # [H,T]
            logits[:, ~allowed] = -np.inf
            vals = vt
            if sinks:  # the sink entries, always visible
                sl = sm_scale * np.matmul(sk, q[b, s][:, :, None])[:, :, 0]  # [H,NS]
                logits = np.concatenate([logits, sl], axis=1)
                vals = np.concatenate([vt, sv], axis=1)
            m = logits.max(axis=1, keepdims=True)
            p = np.exp(logits - m)
            p /= p.sum(axis=1, keepdims=True)
            out[b, s] = np.matmul(p[:, None, :], vals)[:, 0, :]
    if gate_mode != "off":
        out = apply_gate(out, gate, gate_mode)
    return out


def sparse_attention_latent(q, kv, idx, dv, sm_scale=None, gate=None, gate_mode="off",
                            q_off=None, sink_kv=None):
    """Attention over the indexer-selected rows of a latent cache shared by all heads.

    [AXK2] "注意力前向的骨架" step 2: kv_a_proj_with_mqa compresses K/V into a kv_lora_rank
    latent plus a RoPE key slice shared by all heads; [AXK2] "注意力后端选择": the selected
    positions are meant for flash-mla, which attends over that cache.  Reading taken: with
    the up-projections absorbed into the queries and the output, head h's logit for key t is
    sm_scale * q[h,:] . kv[t,:] and its output is the softmax-weighted sum of kv[t, :dv]
    (the latent part of the row).  The mask is the one of sparse_attention: selected and
    causal.  [PANGU] §3.4: for MLA the PAS pairs are latent KV rows, so the optional sinks
    are sink_kv [NS,Dqk], visible to every query.

    q [B,S,H,Dqk], kv [B,T,Dqk], idx [B,S,K].  Returns float64 [B,S,H,dv].
    """
    q = _f64(q)
    kv = _f64(kv)
    idx = np.asarray(idx)
    B, S, H, Dqk = q.shape
    T = kv.shape[1]
    if q_off is None:
        q_off = T - S
    if sm_scale is None or sm_scale <= 0:
        sm_scale = 1.0 / np.sqrt(Dqk)
    sinks = sink_kv is not None
    if sinks:
        skv = _f64(sink_kv)  # [NS,Dqk]
    out = np.zeros((B, S, H, dv), dtype=np.float64)
    for b in range(B):
        for s in range(S):
            allowed = np.zeros(T, dtype=bool)
            sel = idx[b, s]
            sel = sel[(sel >= 0) & (sel < T)]
            allowed[sel] = True
            allowed[np.arange(T) > s + q_off] = False  # the causal mask
            if not allowed.any() and not sinks:
                continue
            logits = sm_scale * (q[b, s] @ kv[b].T)  # [H,T]: every head reads the same rows
            logits[:, ~allowed] = -np.inf
            vals = kv[b, :, :dv]
            if sinks:  # the latent sink rows, always visible
                logits = np.concatenate([logits, sm_scale * (q[b, s] @ skv.T)], axis=1)
                vals = np.concatenate([vals, skv[:, :dv]])
            m = logits.max(axis=1, keepdims=True)
            p = np.exp(logits - m)
            p /= p.sum(axis=1, keepdims=True)
            out[b, s] = p @ vals
    if gate_mode != "off":
        out = apply_gate(out, gate, gate_mode)
    return out


def window_attention(q, k, v, window, sm_scale=None, gate=None, gate_mode="off", q_off=None,
                     sink_k=None, sink_v=None):
    """Sliding-window causal attention with grouped KV heads (the SWA layers).

    [PANGU] §3.2: SWA layers interleave with DSA layers in a DSA-SWA-SWA pattern, with
    a fixed 512-token window.  [SPARK] "为什么 Spark-X2.5 要加这一层门控？": sliding layers
    with window 512, GQA with several query heads per KV head, headwise gate on top.

    q [B,S,H,Dqk], k [B,T,HKV,Dqk], v [B,T,HKV,Dv]; query head h reads KV head
    h // (H // HKV).  Query s sees keys s+q_off-window < t <= s+q_off.
    Optional attention sinks ([PANGU] §3.4, every layer): sink_k [NS,HKV,Dqk], sink_v
    [NS,HKV,Dv], seen by every query (head h through KV head h // (H // HKV)).
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    B, S, H, Dqk = q.shape
    T, HKV = k.shape[1], k.shape[2]
    if H % HKV:
        raise ValueError("query heads must be a multiple of KV heads")
    G = H // HKV
    if q_off is None:
        q_off = T - S
    if sm_scale is None or sm_scale <= 0:
        sm_scale = 1.0 / np.sqrt(Dqk)
    sinks = sink_k is not None
    if sinks:
        sk, sv = _f64(sink_k), _f64(sink_v)
    out = np.zeros((B, S, H, v.shape[-1]), dtype=np.float64)
    t_all = np.arange(T)
    for b in range(B):
        for s in range(S):
            pos = s + q_off
            allowed = (t_all <= pos) & (t_all > pos - window)
            if not allowed.any() and not sinks:
                continue
            for h in range(H):
                kh = h // G
                logits = sm_scale * (k[b, :, kh, :] @ q[b, s, h, :])
                logits[~allowed] = -np.inf
                vals = v[b, :, kh, :]
                if sinks:  # the sink entries, always visible
                    logits = np.concatenate([logits, sm_scale * (sk[:, kh, :] @ q[b, s, h, :])])
                    vals = np.concatenate([vals, sv[:, kh, :]])
                p = np.exp(logits - logits.max())
                p /= p.sum()
                out[b, s, h] = p @ vals
    if gate_mode != "off":
        out = apply_gate(out, gate, gate_mode)
    return out


def hadamard_rotate(x):
    """The indexer's rotation of its inputs before FP8 quantisation.

    [AXK2] SGA notes: the upstream indexer applies a Hadamard transform (rotate_activation)
    before its FP8 scoring kernel, and since the transform is orthogonal (Hq . Hk = q . k)
    the scores are unchanged.  Here: x [..., d] -> x @ H / sqrt(d) with H the d x d Sylvester
    Hadamard matrix (natural order, H = H^T), d a power of two.  Returns float64.
    """
    from scipy.linalg import hadamard

    x = _f64(x)
    d = x.shape[-1]
    return x @ hadamard(d).astype(np.float64) / np.sqrt(d)


def dsa_forward(q_idx, k_idx, w, scale, K, q, k, v, sm_scale=None, gate=None,
                gate_mode="off", relu="none", q_off=None, sink_k=None, sink_v=None):
    """The whole DSA step: indexer scores -> top-k -> sparse attention -> gate.

    [AXK2] "注意力前向的骨架" steps 4-5 and the SGA section; [PANGU] §3.3 (and §3.4 for
    the optional sinks).
    Returns (scores float64 [B,S,T], idx int32 [B,S,min(K,T)], out float64 [B,S,H,Dv]).
    """
    T = _f64(k_idx).shape[1] if not hasattr(k_idx, "shape") else k_idx.shape[1]
    scores = index_scores(q_idx, k_idx, w, scale, relu=relu, q_off=q_off)
    idx = topk_indices(scores, min(K, T), q_off=q_off)
    out = sparse_attention(q, k, v, idx, sm_scale=sm_scale, gate=gate,
                           gate_mode=gate_mode, q_off=q_off, sink_k=sink_k, sink_v=sink_v)
    return scores, idx, out
