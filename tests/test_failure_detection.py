"""Failure detection: every in-kernel wait is bounded, and a wait that runs out records
DSA_ERR_TIMEOUT in the device status word instead of hanging the GPU.  The fault is made on
the host side: dsa_test_arm_wait_timeout() makes the next gather launch's first CTA fill none
of its key slots, so its consumers' wait on a slot that nothing fills runs out (about 2 s).
Nothing faults or traps; the test then checks that the device is still usable: the next
call is correct against the oracle and leaves the status word clean."""
import numpy as np
import pytest
import torch

import sparse_attention_15_b200 as dsa
import parity as P
from workloads import dsa_inputs, get_config

DEV = "cuda:0"
DSA_ERR_TIMEOUT = 4


def _case(seed=21, B=2, K=512, T=2048):
    cfg = get_config("c4")
    x = dsa_inputs(cfg, device=DEV, B=B, T=T, seed=seed, need=("q", "k", "v"))
    g = torch.Generator(device="cpu").manual_seed(seed)
    idx = torch.stack([torch.sort(torch.randperm(T, generator=g)[:K]).values
                       for _ in range(B)]).to(torch.int32).view(B, 1, K).contiguous().to(DEV)
    return x, idx


@pytest.mark.gpu
def test_bounded_wait_runs_out_records_timeout_and_device_stays_usable(lib, cuda_dev):
    L = lib.lib()
    x, idx = _case()
    dsa.dsa_device_status(reset=True)  # a clean word before the fault
    dsa.dsa_test_arm_wait_timeout()
    dsa.dsa_sparse_attn(x["q"], x["k"], x["v"], idx, algo="gather")
    torch.cuda.synchronize()  # returns: the wait gave up, the launch ended
    assert L.dsa_device_status(1) == DSA_ERR_TIMEOUT, L.dsa_last_error()
    assert L.dsa_device_status(0) == 0  # cleared
    # the knob was one-shot, and the context survived: the same call is now correct
    out = dsa.dsa_sparse_attn(x["q"], x["k"], x["v"], idx, algo="gather")
    torch.cuda.synchronize()
    assert L.dsa_device_status(1) == 0
    T = x["k"].shape[1]
    idx_np = P.to_np(idx)
    for b in range(idx.shape[0]):
        ref = P.oracle_attn_rows(x["q"], x["k"], x["v"], idx_np[b], [0], T - 1, b=b)
        P.assert_attn_close(out[b], ref, torch.bfloat16, f"after the timeout, b={b}")

