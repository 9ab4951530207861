"""Helpers for the GPU parity tests: tolerances, sampled-row oracle evaluation and
size-independent property checks.  The expected values always come from the CPU oracle
(or, for whole score matrices, from exact integer arithmetic in torch float32)."""
from __future__ import annotations

import numpy as np
import torch

from oracle import dsa_oracle as O

# bf16 outputs vs the float64 oracle: max-abs <= 2e-2 and max-rel <= 1e-2, the relative
# error taken as |a - r| / max(|r|, 2^-4).  float32 outputs: 1e-4 on both.
TOL = {torch.bfloat16: (2e-2, 1e-2), torch.float32: (1e-4, 1e-4)}


def to_np(t):
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.detach().cpu().numpy()


def assert_attn_close(got, ref, dtype, what=""):
    """Element-wise tolerance check of an attention output against the oracle."""
    a = to_np(got).astype(np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert a.shape == r.shape, (a.shape, r.shape)
    assert np.isfinite(a).all(), f"{what}: non-finite output"
    err = np.abs(a - r)
    rel = err / np.maximum(np.abs(r), 2.0 ** -4)
    atol, rtol = TOL[dtype]
    assert err.max() <= atol, f"{what}: max-abs {err.max():.3e} > {atol}"
    assert rel.max() <= rtol, f"{what}: max-rel {rel.max():.3e} > {rtol}"
    return float(err.max()), float(rel.max())


def oracle_score_rows(q_idx, k_idx, w, scale, rows, q_off, relu="none", b=0):
    """Oracle scores [len(rows), T] of batch row b, for the given query rows."""
    out = []
    for s in rows:
        sc = O.index_scores(q_idx[b:b + 1, s:s + 1], k_idx[b:b + 1], w[b:b + 1, s:s + 1], scale,
                            relu=relu, q_off=int(s) + q_off)
        out.append(sc[0, 0])
    return np.stack(out)


def oracle_attn_rows(q, k, v, idx_rows, rows, q_off, sm_scale=None, gate=None,
                     gate_mode="off", b=0):
    """Oracle attention outputs [len(rows), H, Dv] of batch row b for the given queries,
    each over its own selected keys.  The selected K/V rows are copied to the host and the
    problem restated on them: query s at position s+q_off sees the selected keys (all
    causal), so the dense masked softmax over the compacted keys is the same computation."""
    out = []
    for i, s in enumerate(rows):
        sel = np.asarray(idx_rows[i])
        sel = sel[(sel >= 0) & (sel <= int(s) + q_off)]
        if sel.size == 0:
            out.append(np.zeros((q.shape[2], v.shape[-1])))
            continue
        ti = torch.from_numpy(sel.astype(np.int64)).to(k.device)
        kc = k[b].index_select(0, ti)[None]
        vc = v[b].index_select(0, ti)[None]
        qc = q[b, int(s):int(s) + 1][None]
        g = None if gate is None else gate[b, int(s):int(s) + 1][None]
        idx_c = np.arange(sel.size, dtype=np.int32)[None, None]
        o = O.sparse_attention(qc, kc, vc, idx_c, sm_scale=sm_scale, gate=g, gate_mode=gate_mode,
                               q_off=sel.size - 1)
        out.append(o[0, 0])
    return np.stack(out)


def torch_exact_scores(q_idx, k_idx, w, scale, q_off, rows=None, chunk=256):
    """Whole score matrix [B,S,T] in torch float32 on the device -- exact when the inputs
    are small integers and the scale is a power of two (every partial sum is an integer
    below 2^24).  Used to check full-size score matrices element by element."""
    B, S, HI, DI = q_idx.shape
    T = k_idx.shape[1]
    out = torch.empty((B, S, T), dtype=torch.float32, device=q_idx.device)
    t = torch.arange(T, device=q_idx.device)
    for b in range(B):
        kf = k_idx[b].float()
        for s0 in range(0, S, chunk):
            s1 = min(S, s0 + chunk)
            qf = q_idx[b, s0:s1].float()                       # [n,HI,DI]
            dots = torch.matmul(qf, kf.t())                     # [n,HI,T]
            sc = torch.matmul(w[b, s0:s1, None, :].float(), dots)[:, 0] * scale
            spos = torch.arange(s0, s1, device=q_idx.device)[:, None] + q_off
            out[b, s0:s1] = torch.where(t[None] <= spos, sc, torch.full_like(sc, float("-inf")))
    return out


def check_topk_properties(scores, idx, K, q_off, chunk=1024):
    """Size-independent checks that idx is THE top-k of scores for every row: ascending,
    in range, the right count, -1 padded, every kept key beats every dropped valid key in
    the order (higher score, then lower index)."""
    B, S, T = scores.shape
    dev = scores.device
    t_all = torch.arange(T, device=dev)
    for b in range(B):
        for s0 in range(0, S, chunk):
            s1 = min(S, s0 + chunk)
            sc = scores[b, s0:s1]
            ix = idx[b, s0:s1].long()
            n = torch.clamp(torch.arange(s0, s1, device=dev) + q_off + 1, max=T)  # [r]
            cnt = torch.clamp(n, max=K)
            col = torch.arange(K, device=dev)[None]
            live = col < cnt[:, None]
            assert torch.equal(ix < 0, ~live), "padding / count mismatch"
            assert bool(((ix < n[:, None]) | ~live).all()), "index out of the causal range"
            d = ix[:, 1:] - ix[:, :-1]
            assert bool(((d > 0) | ~live[:, 1:]).all()), "indices not strictly ascending"
            sel = torch.zeros((s1 - s0, T), dtype=torch.bool, device=dev)
            r_of = torch.arange(s1 - s0, device=dev)[:, None].expand_as(ix)
            sel[r_of[live], ix[live]] = True
            valid = t_all[None] < n[:, None]
            v = sc + 0.0  # -0.0 -> +0.0
            tau = torch.where(sel, v, torch.full_like(v, float("inf"))).min(dim=1).values
            drop = valid & ~sel
            mx_drop = torch.where(drop, v, torch.full_like(v, -float("inf"))).max(dim=1).values
            assert bool((mx_drop <= tau).all()), "a dropped key scores above a kept key"
            # ties at tau: every kept tie has a lower index than every dropped tie
            tie = v == tau[:, None]
            last_kept_tie = torch.where(sel & tie, t_all[None], -1).max(dim=1).values
            first_drop_tie = torch.where(drop & tie, t_all[None], T).min(dim=1).values
            assert bool((last_kept_tie < first_drop_tie).all()), "tie-break violated"
