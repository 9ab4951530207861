"""dsa_sparse_attn_noalloc: the workspace-free entry point for callers that cannot allocate
device memory -- a plugin inside an inference runtime whose memory planner owns every device
byte, or a fixed-budget decode loop that must not pay for a fresh allocation.  It keeps the
gather attention's split-key partials in one fixed array of the library instead of a caller
workspace, so it must give exactly what dsa_sparse_attn gives with a workspace (same
kernels, same split), call after call, although every call reuses that array; and no call
may allocate.  This file is collected last so that a failure here stops a -x run only after
every other test has run."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import sparse_attention_15_b200 as dsa
import parity as P
from workloads import dsa_inputs, get_config

DEV = "cuda:0"
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _decode_case(seed, B, K, T=6144):
    """A decode-shaped problem (few query rows, long index lists -> split-key partials):
    B rows of one query each, K distinct causal keys per row, drawn per row."""
    cfg = get_config("c4")
    x = dsa_inputs(cfg, device=DEV, B=B, T=T, seed=seed, need=("q", "k", "v"))
    g = torch.Generator(device="cpu").manual_seed(seed)
    idx = torch.stack([torch.sort(torch.randperm(T, generator=g)[:K]).values
                       for _ in range(B)]).to(torch.int32).view(B, 1, K).contiguous().to(DEV)
    return x, idx


def _noalloc(L, x, idx, out):
    B, S, H, DQK = x["q"].shape
    T, DV = x["k"].shape[1], x["v"].shape[-1]
    return L.dsa_sparse_attn_noalloc(1, ctypes.c_void_p(x["q"].data_ptr()),
                                     ctypes.c_void_p(x["k"].data_ptr()),
                                     ctypes.c_void_p(x["v"].data_ptr()),
                                     ctypes.c_void_p(idx.data_ptr()), idx.shape[-1], None, 0,
                                     0.0, B, S, T, H, DQK, DV, ctypes.c_void_p(out.data_ptr()),
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_two_calls(lib, cuda_dev):
    L = lib.lib()
    assert L.dsa_sparse_attn_noalloc_max_scratch_bytes() == 16 << 20
    # a large call, then a smaller one with a different split count: the second reads the
    # array at other offsets, over whatever the first left there
    cases = [(11, 8, 2048), (12, 2, 1024)]
    splits = []
    for seed, B, K in cases:
        x, idx = _decode_case(seed, B, K)
        _, S, H, DQK = x["q"].shape
        T, DV = x["k"].shape[1], x["v"].shape[-1]
        need = dsa.dsa_sparse_attn_workspace_bytes(x["q"].dtype, B, S, T, H, DQK, DV, K,
                                                   "gather")
        assert 0 < need <= L.dsa_sparse_attn_noalloc_max_scratch_bytes()
        splits.append(need // (B * S * H * (DV + 2) * 4))
        ref = dsa.dsa_sparse_attn(x["q"], x["k"], x["v"], idx, algo="gather")
        out = torch.empty_like(ref)
        assert _noalloc(L, x, idx, out) == 0, L.dsa_last_error()
        torch.cuda.synchronize()
        dsa.dsa_device_status(reset=True)
        # the same kernels and the same split as the workspace path: bit for bit
        assert torch.equal(out, ref), f"B={B} K={K}: differs from dsa_sparse_attn"
        # and against the float64 oracle, row by row, within the bf16 tolerance
        idx_np = P.to_np(idx)
        for b in range(B):
            att_ref = P.oracle_attn_rows(x["q"], x["k"], x["v"], idx_np[b], [0], T - 1, b=b)
            P.assert_attn_close(out[b], att_ref, torch.bfloat16, f"noalloc B={B} K={K} b={b}")
    assert splits[0] != splits[1], splits


@pytest.mark.gpu
def test_noalloc_allocates_nothing(lib, cuda_dev):
    L = lib.lib()
    x, idx = _decode_case(13, 4, 2048)
    out = torch.empty(x["q"].shape[:3] + (x["v"].shape[-1],), dtype=x["q"].dtype, device=DEV)
    # the first call may load the library's device code and look the array up
    assert _noalloc(L, x, idx, out) == 0, L.dsa_last_error()
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(5):
        assert _noalloc(L, x, idx, out) == 0, L.dsa_last_error()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    dsa.dsa_device_status(reset=True)
    assert free1 == free0, f"device free memory changed by {free0 - free1} bytes"


def test_noalloc_source_names_no_allocation_call():
    # the entry point's source calls no device allocator (runs without a GPU)
    src = open(os.path.join(ROOT, "sparse_attention_15_b200", "csrc", "noalloc.cu")).read()
    code = re.sub(r"//[^\n]*", "", src)
    for name in ("cudaMalloc", "cudaMallocAsync", "cudaMallocManaged", "cudaFree",
                 "cudaFreeAsync", "cuMemAlloc", "cuMemCreate"):
        assert not re.search(r"\b" + name + r"\w*\s*\(", code), name


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
    # the same argument checks as dsa_sparse_attn: a finite sm_scale of any size is taken
    # up to the size check, a non-finite one is refused
    assert L.dsa_sparse_attn_noalloc(1, fake, fake, fake, fake, 2048, None, 0,
                                     ctypes.c_float(float("inf")), 200, 1, 131072, 32, 192,
                                     128, fake, None) == 1
    assert L.dsa_sparse_attn_noalloc(1, fake, fake, fake, fake, 2048, None, 0,
                                     ctypes.c_float(3.3e38), 200, 1, 131072, 32, 192, 128,
                                     fake, None) == 2
