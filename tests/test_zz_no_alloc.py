"""dsa_sparse_attn_noalloc: the workspace-free entry point for callers that cannot allocate
device memory (a runtime plugin whose memory planner owns the device, a fixed-budget decode
loop).  It must give what dsa_sparse_attn gives with a caller workspace, call after call,
although every call reuses the same fixed scratch array.  This file is collected last so
that a failure here stops a -x run only after every other test has run."""
import ctypes

import pytest
import torch

import sparse_attention_15_b200 as dsa
import parity as P
from workloads import dsa_inputs, get_config

DEV = "cuda:0"


def _decode_case(seed, B=4, T=6144):
    """A decode-shaped problem (few query rows, long index lists -> split-key partials)."""
    cfg = get_config("c4")
    x = dsa_inputs(cfg, device=DEV, B=B, T=T, seed=seed, need=("q", "k", "v"))
    g = torch.Generator(device=DEV).manual_seed(seed)
    idx = torch.sort(torch.randperm(T, device=DEV, generator=g)[:cfg.K]).values
    idx = idx.to(torch.int32).expand(B, 1, cfg.K).contiguous()
    return cfg, x, idx


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_two_calls(lib, cuda_dev):
    L = lib.lib()
    assert L.dsa_sparse_attn_noalloc_max_scratch_bytes() == 16 << 20
    outs = []
    for seed in (11, 12):  # two calls in a row, different inputs: no stale partials leak
        cfg, x, idx = _decode_case(seed)
        B, S, H, DQK = x["q"].shape
        T, DV = x["k"].shape[1], x["v"].shape[-1]
        need = dsa.dsa_sparse_attn_workspace_bytes(x["q"].dtype, B, S, T, H, DQK, DV, cfg.K,
                                                   "gather")
        assert 0 < need <= L.dsa_sparse_attn_noalloc_max_scratch_bytes()
        ref = dsa.dsa_sparse_attn(x["q"], x["k"], x["v"], idx, algo="gather")
        out = torch.empty_like(ref)
        st = L.dsa_sparse_attn_noalloc(1, ctypes.c_void_p(x["q"].data_ptr()),
                                       ctypes.c_void_p(x["k"].data_ptr()),
                                       ctypes.c_void_p(x["v"].data_ptr()),
                                       ctypes.c_void_p(idx.data_ptr()), cfg.K, None, 0, 0.0,
                                       B, S, T, H, DQK, DV, ctypes.c_void_p(out.data_ptr()),
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == 0, L.dsa_last_error()
        torch.cuda.synchronize()
        dsa.dsa_device_status(reset=True)
        err = (out.float() - ref.float()).abs().max().item()
        assert err <= P.TOL[torch.bfloat16][0], err
        P.assert_attn_close(out, P.to_np(ref).astype("float64"), torch.bfloat16, f"seed {seed}")
        outs.append(out)
    assert not torch.equal(outs[0], outs[1])


def test_noalloc_rejects_shapes_beyond_its_scratch(lib):
    # rejected on the host before any device work (runs without a GPU)
    L = lib.lib()
    fake = ctypes.c_void_p(0x10000)
    # 200 decode rows x 2048 keys: about 33 MB of split-key partials, over the 16 MiB
    st = L.dsa_sparse_attn_noalloc(1, fake, fake, fake, fake, 2048, None, 0, 0.0,
                                   200, 1, 131072, 32, 192, 128, fake, None)
    assert st == 2
    assert b"more than the fixed" in L.dsa_last_error()
    assert L.dsa_sparse_attn_noalloc(1, None, fake, fake, fake, 8, None, 0, 0.0, 1, 1, 8, 4, 64,
                                     64, fake, None) == 1
