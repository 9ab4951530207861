"""Fused indexer -> top-k (dsa_index_topk, dsa_forward with indexer="fused") against the
oracle: the indices must be bit-exact, both when the candidate filter holds and when it does
not and the full-score fallback runs.

The fallback is forced with inputs the sampled threshold cannot handle: all-equal scores and
scores with two values (every key ties with many others, the candidate lists overflow), and
rows whose sampled tiles score higher than the rest (the threshold lands above the K-th key
and fewer than K keys pass).  Three-value scores put heavy ties at the K-th key inside lists
that hold them (the candidate select breaks the ties by index)."""
import numpy as np
import pytest
import torch

import sparse_attention_15_b200 as dsa
import parity as P
from oracle import dsa_oracle as O
from workloads import dsa_inputs, get_config

DEV = "cuda:0"
pytestmark = pytest.mark.gpu


def _fused(q_idx, k_idx, w, scale, K, relu="none"):
    flag = torch.full((1,), -1, dtype=torch.int32, device=DEV)
    idx = dsa.dsa_index_topk(q_idx, k_idx, w, scale, K, relu=relu, fallback_out=flag)
    torch.cuda.synchronize()
    dsa.dsa_device_status(reset=True)
    return idx, int(flag.item())


def _oracle_all_rows(q_idx, k_idx, w, scale, K, q_off, relu="none"):
    """The oracle's top-k of every row, on the exact scores (float32 on the device is exact
    for these integer inputs and powers-of-two scales; the oracle's own float64 scores are
    compared with them on sampled rows)."""
    sc = P.torch_exact_scores(q_idx, k_idx, w, scale, q_off)
    if relu == "post_sum":
        sc = torch.where(torch.isinf(sc), sc, torch.clamp(sc, min=0.0))
    return O.topk_indices(P.to_np(sc), K, q_off=q_off), sc


def _check_rows_against_oracle_scores(q_idx, k_idx, w, scale, sc, rows, q_off, relu="none"):
    qi, ki, wc = (t.cpu() for t in (q_idx, k_idx, w))
    ref = P.oracle_score_rows(qi, ki, wc, scale, rows, q_off, relu=relu)
    assert np.array_equal(P.to_np(sc[0, rows]), ref.astype(np.float32))


@pytest.mark.parametrize("name,S,relu", [("c2", 4096, "none"), ("c3", 4096, "none"),
                                          ("c3", 8192, "none"), ("c2", 3000, "post_sum")])
def test_fused_index_topk_exact_random(lib, cuda_dev, name, S, relu):
    cfg = get_config(name)
    x = dsa_inputs(cfg, device=DEV, S=S, T=S, need=("q_idx", "k_idx", "w"))
    K = cfg.k_eff
    idx, fell_back = _fused(x["q_idx"], x["k_idx"], x["w"], cfg.scale, K, relu)
    assert fell_back == 0, "the filter should hold on random integer scores"
    ref, sc = _oracle_all_rows(x["q_idx"], x["k_idx"], x["w"], cfg.scale, K, 0, relu)
    assert np.array_equal(P.to_np(idx), ref)
    _check_rows_against_oracle_scores(x["q_idx"], x["k_idx"], x["w"], cfg.scale, sc,
                                      [0, K - 1, K, S // 2, S - 1], 0, relu)


def test_fused_index_topk_full_size_c3(lib, cuda_dev):
    # full-size c3: every row equal to the unfused path, which the full-size parity tests
    # check against the oracle; sampled rows straight against the oracle
    cfg = get_config("c3")
    x = dsa_inputs(cfg, device=DEV, need=("q_idx", "k_idx", "w"))
    K = cfg.k_eff
    idx, fell_back = _fused(x["q_idx"], x["k_idx"], x["w"], cfg.scale, K)
    assert fell_back == 0
    scores = dsa.dsa_index_scores(x["q_idx"], x["k_idx"], x["w"], cfg.scale)
    ref = dsa.dsa_topk(scores, K)
    torch.cuda.synchronize()
    assert torch.equal(idx, ref)
    rows = [0, 1, K - 1, K, K + 1, 7777, cfg.S - 1]
    qi, ki, w = (x[n].cpu() for n in ("q_idx", "k_idx", "w"))
    sc_ref = P.oracle_score_rows(qi, ki, w, cfg.scale, rows, cfg.q_off)
    for i, r in enumerate(rows):
        want = O.topk_indices(sc_ref[i][None, None], K, q_off=r + cfg.q_off)[0, 0]
        assert np.array_equal(P.to_np(idx[0, r]), want), r


def _crafted_case(kind, S, HI=16, DI=64, seed=5):
    """Integer indexer inputs whose scores defeat (or stress) the sampled threshold."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    q = torch.randint(-2, 3, (1, S, HI, DI), generator=g).to(torch.bfloat16)
    k = torch.randint(-2, 3, (1, S, DI), generator=g).to(torch.bfloat16)
    w = torch.randint(1, 5, (1, S, HI), generator=g).to(torch.float32)
    if kind == "all_equal":
        q.zero_()  # every score 0: every key ties
    elif kind in ("two_values", "three_values"):
        q.zero_()
        q[..., 0] = 1
        k.zero_()
        m = 2 if kind == "two_values" else 3  # scores in {0, c} or {-c, 0, c}
        k[0, :, 0] = (torch.arange(S) % m - (m - 2)).to(torch.bfloat16)
    elif kind == "sample_miss":
        # key tile 0 (always sampled) scores high, every other key low: the sampled
        # threshold sits above the K-th key, so fewer than K keys pass it
        q.zero_()
        q[..., 0] = 1
        k.zero_()
        k[0, :, 0] = -1
        k[0, :128, 0] = 2
    return q.to(DEV), k.to(DEV), w.to(DEV)


# (kind, S, K, fallback expected).  The candidate lists hold 2K + 1024 keys: all-equal and
# two-value rows longer than that overflow them; three-value rows fit (ties at the K-th key
# resolved by the candidate select itself); the sample-miss rows pass fewer than K keys.
CRAFTED = [("all_equal", 2048, 256, 1), ("two_values", 4096, 256, 1),
           ("sample_miss", 2048, 256, 1), ("three_values", 2048, 256, 0)]


@pytest.mark.parametrize("kind,S,K,expect", CRAFTED)
def test_fused_index_topk_crafted_exact(lib, cuda_dev, kind, S, K, expect):
    q, k, w = _crafted_case(kind, S)
    idx, fell_back = _fused(q, k, w, 2.0 ** -4, K)
    assert fell_back == expect, f"{kind}: fallback {fell_back}, expected {expect}"
    ref, _ = _oracle_all_rows(q, k, w, 2.0 ** -4, K, 0)
    assert np.array_equal(P.to_np(idx), ref)


def test_fused_forward_matches_per_head_forward(lib, cuda_dev):
    # the whole step with the fused indexer: same indices and the same attention output,
    # bit for bit, as the per-head indexer + top-k (masked-tile attention, gate on)
    cfg = get_config("c3")
    S = 2048
    x = dsa_inputs(cfg, device=DEV, S=S, T=S)
    flag = torch.full((1,), -1, dtype=torch.int32, device=DEV)
    out_f, idx_f = dsa.dsa_forward(x["q_idx"], x["k_idx"], x["w"], cfg.scale, cfg.K, x["q"],
                                   x["k"], x["v"], gate=x["gate"], indexer="fused",
                                   topk_fallback_out=flag)
    out_p, idx_p = dsa.dsa_forward(x["q_idx"], x["k_idx"], x["w"], cfg.scale, cfg.K, x["q"],
                                   x["k"], x["v"], gate=x["gate"])
    torch.cuda.synchronize()
    dsa.dsa_device_status(reset=True)
    assert int(flag.item()) == 0
    assert torch.equal(idx_f, idx_p)
    assert torch.equal(out_f, out_p)
    # and against the oracle on sampled rows
    rows = [0, 5, S // 2, S - 1]
    idx_np = P.to_np(idx_f[0])
    att = P.oracle_attn_rows(x["q"], x["k"], x["v"], idx_np[rows], rows, 0, gate=x["gate"],
                             gate_mode=cfg.gate)
    P.assert_attn_close(out_f[0, rows], att, torch.bfloat16, "fused forward")


def test_fused_forward_with_fallback(lib, cuda_dev):
    # a forward whose candidate filter cannot hold: the fallback gives the oracle's indices
    S, K = 2048, 128  # rows past 2K + 1024 keys overflow their candidate lists
    q, k, w = _crafted_case("all_equal", S, HI=32, DI=128)
    cfg = get_config("c3")
    x = dsa_inputs(cfg, device=DEV, S=S, T=S, need=("q", "k", "v", "gate"))
    flag = torch.full((1,), -1, dtype=torch.int32, device=DEV)
    out, idx = dsa.dsa_forward(q, k, w, 2.0 ** -5, K, x["q"], x["k"], x["v"], gate=x["gate"],
                               indexer="fused", topk_fallback_out=flag)
    torch.cuda.synchronize()
    dsa.dsa_device_status(reset=True)
    assert int(flag.item()) == 1
    ref, _ = _oracle_all_rows(q, k, w, 2.0 ** -5, K, 0)
    assert np.array_equal(P.to_np(idx), ref)
    rows = [0, 200, S - 1]
    att = P.oracle_attn_rows(x["q"], x["k"], x["v"], ref[0][rows], rows, 0, gate=x["gate"],
                             gate_mode=cfg.gate)
    P.assert_attn_close(out[0, rows], att, torch.bfloat16, "fused forward, fallback")
