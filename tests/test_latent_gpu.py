"""GPU parity of the latent (MQA-form) sparse attention against the float64 oracle.

Every head attends over the same cached latent row (keys = the 576-dim row, values = its
first 512 dims).  Index lists are seeded random selections drawn on the CPU (the shape of the
top-k output); the whole-step test takes its indices from the oracle's indexer and top-k.
"""
import numpy as np
import pytest
import torch

import sparse_attention_15_b200 as dsa
from oracle import dsa_oracle as O
import parity as P
from workloads import dsa_inputs, get_config
from workloads.gen import latent_inputs, random_selection

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
DQK, DV = 576, 512


@pytest.fixture(autouse=True)
def _gpu(lib, cuda_dev):
    yield
    torch.cuda.synchronize()
    dsa.dsa_device_status(reset=True)  # raises if a kernel flagged a timeout
    torch.cuda.empty_cache()


def _latent(B, S, T, H, nsink=0, seed=7):
    cfg = get_config("c3")  # bf16, gate logits available
    return latent_inputs(cfg, H=H, B=B, S=S, T=T, nsink=nsink, seed=seed)


def _dev(x):
    return None if x is None else x.to(DEV)


def _oracle_rows(x, idx, rows, gate_mode, b=0):
    """Oracle outputs [len(rows), H, DV] of batch row b, each query over its selected rows,
    restated on the host copies of those rows (all of them causal for the query)."""
    out = []
    T = x["kv"].shape[1]
    S = x["q"].shape[1]
    for s in rows:
        sel = np.asarray(idx[b, s])
        sel = sel[(sel >= 0) & (sel < T) & (sel <= s + T - S)]
        ti = torch.from_numpy(sel.astype(np.int64)).to(x["kv"].device)
        kv_c = x["kv"][b].index_select(0, ti).cpu()[None]
        idx_c = np.arange(sel.size)[None, None]
        g = None if gate_mode == "off" else x["gate"][b:b + 1, s:s + 1].cpu()
        sk = None if x["sink_kv"] is None else x["sink_kv"].cpu()
        o = O.sparse_attention_latent(x["q"][b:b + 1, s:s + 1].cpu(), kv_c, idx_c, DV, gate=g,
                                      gate_mode=gate_mode, q_off=max(sel.size - 1, 0),
                                      sink_kv=sk)
        out.append(o[0, 0])
    return np.stack(out)


CASES = [
    # B, S, T, H, K, nsink, gate
    (1, 300, 300, 128, 64, 0, "off"),        # prefill, ragged last key block
    (1, 77, 500, 128, 200, 0, "sigmoid"),    # queries at the end of a longer cache
    (2, 1, 5000, 128, 2048, 0, "off"),       # decode: split keys + combine
    (2, 40, 260, 16, 96, 7, "silu"),         # 16 heads (padded to the 128-row tile), sinks
    (3, 1, 3000, 64, 512, 128, "sigmoid"),   # decode, 128 sinks, split
    (1, 5, 40, 128, 64, 0, "off"),           # rows with fewer keys than K (-1 padding)
]


@pytest.mark.parametrize("B,S,T,H,K,NS,gm", CASES)
def test_latent_attn_parity(B, S, T, H, K, NS, gm):
    x = _latent(B, S, T, H, NS)
    idx = random_selection(B, S, T, K, seed=B * 1000 + S + T)
    gate = None if gm == "off" else x["gate"]
    got = dsa.dsa_sparse_attn_latent(_dev(x["q"]), _dev(x["kv"]), idx.to(DEV), dv=DV,
                                     sink_kv=_dev(x["sink_kv"]), gate=_dev(gate),
                                     gate_mode=None if gm == "off" else gm)
    ref = O.sparse_attention_latent(x["q"], x["kv"], idx.numpy(), DV, gate=gate,
                                    gate_mode=gm, sink_kv=x["sink_kv"])
    P.assert_attn_close(got, ref, torch.bfloat16, f"latent B={B} S={S} T={T} H={H} NS={NS}")


def test_latent_attn_skips_invalid_and_future_entries():
    B, S, T, H, K = 1, 50, 120, 128, 40
    x = _latent(B, S, T, H)
    rng = np.random.default_rng(3)
    idx = rng.integers(-3, T + 40, size=(B, S, K)).astype(np.int32)  # -1, future, out of range
    for s in range(S):  # valid entries must be distinct: repeats become -1
        seen = set()
        for j in range(K):
            t = int(idx[0, s, j])
            if 0 <= t < T:
                if t in seen:
                    idx[0, s, j] = -1
                seen.add(t)
    got = dsa.dsa_sparse_attn_latent(_dev(x["q"]), _dev(x["kv"]), torch.from_numpy(idx).to(DEV))
    ref = O.sparse_attention_latent(x["q"], x["kv"], idx, DV)
    P.assert_attn_close(got, ref, torch.bfloat16, "latent invalid entries")


def test_latent_attn_deterministic_and_gate_zero_halves():
    B, S, T, H, K = 1, 64, 700, 128, 256
    x = _latent(B, S, T, H)
    idx = random_selection(B, S, T, K, seed=5).to(DEV)
    q, kv = _dev(x["q"]), _dev(x["kv"])
    a = dsa.dsa_sparse_attn_latent(q, kv, idx)
    b = dsa.dsa_sparse_attn_latent(q, kv, idx)
    assert torch.equal(a, b)
    zero = torch.zeros((B, S, H), dtype=torch.bfloat16, device=DEV)
    half = dsa.dsa_sparse_attn_latent(q, kv, idx, gate=zero, gate_mode="sigmoid")
    assert torch.equal(half, (a.float() * 0.5).to(torch.bfloat16))


@pytest.mark.parametrize("name,S,T", [("c2", 333, 333), ("c3", 150, 420)])
def test_forward_latent_parity(name, S, T):
    cfg = get_config(name)
    x = dsa_inputs(cfg, B=1, S=S, T=T, need=("q_idx", "k_idx", "w", "gate"))
    lt = latent_inputs(cfg, H=128, B=1, S=S, T=T, nsink=16)
    K = min(cfg.K, 96)
    gm = cfg.gate
    gate = lt["gate"]
    out, idx = dsa.dsa_forward(_dev(x["q_idx"]), _dev(x["k_idx"]), _dev(x["w"]), cfg.scale, K,
                               _dev(lt["q"]), _dev(lt["kv"]), None, gate=_dev(gate),
                               sink_k=_dev(lt["sink_kv"]), attn_form="latent")
    sc = O.index_scores(x["q_idx"], x["k_idx"], x["w"], cfg.scale)
    idx_ref = O.topk_indices(sc, min(K, T))
    assert np.array_equal(P.to_np(idx), idx_ref)
    ref = O.sparse_attention_latent(lt["q"], lt["kv"], idx_ref, DV, gate=gate, gate_mode=gm,
                                    sink_kv=lt["sink_kv"])
    P.assert_attn_close(out, ref, torch.bfloat16, f"{name} forward latent")


# ------------------------------------------------------------------ full-size workloads
# The latent attention at the sizes the benchmark times (the c2 prefill and c4 decode
# shapes with 128 latent heads), checked on sampled rows.
@pytest.mark.parametrize("name,rows", [("c2", [0, 1, 511, 2047, 4094, 4095]),
                                       ("c4", [0, 1, 17, 31, 32, 47, 62, 63])])
def test_full_size_latent(name, rows):
    cfg = get_config(name)
    x = latent_inputs(cfg, H=128, device=DEV)  # drawn on the GPU: the same tensors feed both
    B, S, T = cfg.B, cfg.S, cfg.T
    idx = random_selection(B, S, T, cfg.k_eff, seed=77)
    got = dsa.dsa_sparse_attn_latent(x["q"], x["kv"], idx.to(DEV))
    got = got.cpu()
    if S == 1:  # decode: batch rows
        for b in rows:
            ref = _oracle_rows(x, idx.numpy(), [0], "off", b=b)
            P.assert_attn_close(got[b, 0:1], ref, torch.bfloat16, f"{name} latent row b={b}")
    else:
        ref = _oracle_rows(x, idx.numpy(), rows, "off")
        P.assert_attn_close(got[0, rows], ref, torch.bfloat16, f"{name} latent rows")
    assert torch.isfinite(got.float()).all()


@pytest.mark.parametrize("NS", [0, 3])
def test_latent_attn_rows_without_valid_keys(NS):
    # rows whose lists hold only -1 or future entries: zeros without sinks, the sinks'
    # softmax alone with them
    B, S, T, H, K = 1, 8, 100, 128, 48
    x = _latent(B, S, T, H, NS, seed=9)
    idx = random_selection(B, S, T, K, seed=19).numpy()
    q_off = T - S
    idx[0, 0, :] = -1
    idx[0, 3, :] = -1
    idx[0, 5, :] = np.arange(K) % 3 + 5 + q_off + 1  # all in the future of query 5
    idx[0, 5, 1::2] = -1
    got = dsa.dsa_sparse_attn_latent(_dev(x["q"]), _dev(x["kv"]), torch.from_numpy(idx).to(DEV),
                                     sink_kv=_dev(x["sink_kv"]))
    ref = O.sparse_attention_latent(x["q"], x["kv"], idx, DV, sink_kv=x["sink_kv"])
    if NS == 0:
        assert float(np.abs(ref[0, [0, 3, 5]]).max()) == 0.0
        assert torch.count_nonzero(got[0, [0, 3, 5]].float()).item() == 0
    P.assert_attn_close(got, ref, torch.bfloat16, f"latent empty rows NS={NS}")


@pytest.mark.parametrize("H", [1, 128])
def test_latent_attn_smallest_shapes(H):
    # one query against one key, one head (127 padded tile rows) or all 128
    x = _latent(1, 1, 1, H, seed=29)
    idx = torch.zeros((1, 1, 1), dtype=torch.int32)
    got = dsa.dsa_sparse_attn_latent(_dev(x["q"]), _dev(x["kv"]), idx.to(DEV))
    ref = O.sparse_attention_latent(x["q"], x["kv"], idx.numpy(), DV)
    P.assert_attn_close(got, ref, torch.bfloat16, f"latent 1x1 H={H}")
