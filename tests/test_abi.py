"""The C-ABI library: it loads without a GPU, exports every entry point include/dsa.h
declares, and rejects invalid arguments on the host, before any CUDA call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(dsa_[a-z_]+)\s*\(",
                                text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_path():
    names = _declared_functions()
    for required in ("dsa_index_scores", "dsa_topk", "dsa_sparse_attn", "dsa_forward"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    L = lib.lib()
    for name in _declared_functions():
        assert hasattr(L, name), f"libdsa.so does not export {name}"


def test_version_and_status_strings(lib):
    L = lib.lib()
    assert b"sm_100a" in L.dsa_version()
    assert L.dsa_status_string(0) == b"ok"
    assert L.dsa_status_string(4) == b"in-kernel wait timed out"


FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: validation fails first
FAKE_MIS = ctypes.c_void_p(0x10008)  # 8-byte aligned only


def _index(L, **kw):
    a = dict(dtype=1, q=FAKE, k=FAKE, w=FAKE, scale=0.5, relu=0, B=1, S=4, T=4, HI=2, DI=64,
             scores=FAKE)
    a.update(kw)
    return L.dsa_index_scores(a["dtype"], a["q"], a["k"], a["w"], a["scale"], a["relu"], a["B"],
                              a["S"], a["T"], a["HI"], a["DI"], a["scores"], None)


def test_index_scores_rejects_bad_arguments(lib):
    L = lib.lib()
    assert _index(L, q=None) == 1
    assert _index(L, B=0) == 1
    assert _index(L, S=8, T=4) == 1          # queries must be the last S of T keys
    assert _index(L, scale=0.0) == 1
    assert _index(L, scale=float("nan")) == 1
    assert _index(L, relu=7) == 1
    assert _index(L, dtype=5) == 1
    assert _index(L, DI=60) == 2             # not a multiple of 8 for bf16
    assert _index(L, DI=256) == 2
    assert _index(L, q=FAKE_MIS) == 2        # misaligned
    assert b"16-byte" in L.dsa_last_error()
    assert _index(L, dtype=2, HI=16, DI=64) == 2   # e4m3 needs DI == 128
    assert b"e4m3" in L.dsa_last_error()
    assert _index(L, dtype=2, HI=8, DI=128) == 2   # and HI in {16, 32}


def _collapsed(L, ws_bytes=1 << 20, **kw):
    a = dict(dtype=1, q=FAKE, k=FAKE, w=FAKE, scale=0.5, relu=0, B=1, S=4, T=4, HI=16, DI=64,
             scores=FAKE, ws=FAKE)
    a.update(kw)
    return L.dsa_index_scores_collapsed(a["dtype"], a["q"], a["k"], a["w"], a["scale"], a["relu"],
                                        a["B"], a["S"], a["T"], a["HI"], a["DI"], a["scores"],
                                        a["ws"], ws_bytes, None)


def test_index_scores_collapsed_rejects_bad_arguments(lib):
    L = lib.lib()
    assert L.dsa_index_scores_collapsed_workspace_bytes(2, 5, 128) == 2 * 5 * 2 * 128 * 2
    assert _collapsed(L, q=None) == 1
    assert _collapsed(L, S=8, T=4) == 1
    assert _collapsed(L, relu=2) == 2        # a per-head ReLU does not collapse
    assert b"per-head" in L.dsa_last_error()
    assert _collapsed(L, dtype=0, DI=32) == 2  # float32 / DI outside {64, 128}
    assert _collapsed(L, DI=96) == 2
    assert _collapsed(L, ws=None) == 1
    assert _collapsed(L, ws_bytes=4 * 2 * 64 * 2 - 1) == 1  # one byte short
    assert _collapsed(L, ws=FAKE_MIS) == 2


def test_hadamard_rejects_bad_arguments(lib):
    L = lib.lib()

    def call(dtype=1, x=FAKE, rows=4, d=128, out=FAKE):
        return L.dsa_hadamard_rotate(dtype, x, rows, d, out, None)
    assert call(d=32) == 2
    assert call(dtype=2) == 2            # e4m3 is quantised after the rotation
    assert call(rows=0) == 1
    assert call(x=None) == 1
    assert call(out=FAKE_MIS) == 2


def test_topk_rejects_bad_arguments(lib):
    L = lib.lib()
    assert L.dsa_topk(None, 1, 4, 4, 2, FAKE, None) == 1
    assert L.dsa_topk(FAKE, 1, 4, 4, 0, FAKE, None) == 1
    assert L.dsa_topk(FAKE, 1, 5, 4, 2, FAKE, None) == 1
    assert L.dsa_topk(FAKE, 1, 4, 4, 2, FAKE_MIS, None) == 2


def test_index_topk_rejects_bad_arguments(lib):
    L = lib.lib()

    def call(**kw):
        a = dict(dtype=1, q=FAKE, k=FAKE, w=FAKE, scale=0.0625, relu=0, B=1, S=4096, T=4096,
                 HI=16, DI=64, K=512, idx=FAKE, ws=FAKE, wsb=1 << 40, fb=None)
        a.update(kw)
        return L.dsa_index_topk(a["dtype"], a["q"], a["k"], a["w"], a["scale"], a["relu"],
                                a["B"], a["S"], a["T"], a["HI"], a["DI"], a["K"], a["idx"],
                                a["ws"], a["wsb"], a["fb"], None)

    need = L.dsa_index_topk_workspace_bytes(1, 4096, 4096, 512)
    # sampled scores + thresholds + counters + 2 candidate lists + the fallback's scores
    assert need >= 4096 * 4096 * 4 + 2 * 4096 * (2 * 512 + 1024) * 4
    assert L.dsa_index_topk_workspace_bytes(0, 4096, 4096, 512) == 0
    assert call(dtype=0) == 2                 # float32: no tensor-core indexer
    assert call(HI=8) == 2
    assert call(q=None) == 1
    assert call(K=0) == 1
    assert call(S=8192) == 1                  # T < S
    assert call(wsb=need - 1) == 1            # workspace too small
    assert call(ws=None) == 1
    assert call(ws=FAKE_MIS) == 2
    assert call(fb=FAKE_MIS) == 2


def _attn(L, **kw):
    a = dict(dtype=1, q=FAKE, k=FAKE, v=FAKE, idx=FAKE, K=4, gate=None, gm=0, sm=0.0, B=1, S=4,
             T=8, H=4, DQK=64, DV=64, out=FAKE, ws=None, wsb=0)
    a.update(kw)
    return L.dsa_sparse_attn(a["dtype"], a["q"], a["k"], a["v"], a["idx"], a["K"], a["gate"],
                             a["gm"], a["sm"], a["B"], a["S"], a["T"], a["H"], a["DQK"], a["DV"],
                             a.get("algo", 0), a["out"], a["ws"], a["wsb"], None)


def test_sparse_attn_rejects_bad_arguments(lib):
    L = lib.lib()
    assert _attn(L, gm=1) == 1                    # gate on but no gate pointer
    assert _attn(L, gate=FAKE, gm=0) == 1         # gate pointer with the gate off
    assert _attn(L, gate=FAKE, gm=3) == 1         # only sigmoid and silu exist
    assert _attn(L, idx=None) == 1
    assert _attn(L, K=0) == 1
    assert _attn(L, DQK=300) == 2
    assert _attn(L, v=FAKE_MIS) == 2
    assert _attn(L, sm=float("inf")) == 1
    assert _attn(L, algo=7) == 1
    assert _attn(L, dtype=0, DQK=64, DV=64, algo=2) == 2  # masked tile is bf16 only
    # decode-shaped work needs a split-key workspace; too small a workspace is rejected
    need = L.dsa_sparse_attn_workspace_bytes(1, 2, 1, 131072, 32, 192, 128, 2048, 0)
    assert need > 0
    assert _attn(L, B=2, S=1, T=131072, H=32, DQK=192, DV=128, K=2048, ws=FAKE,
                 wsb=need - 1) == 1
    # the cost model: long prefill -> masked tile (bitmask workspace), decode -> gather
    pre = L.dsa_sparse_attn_workspace_bytes(1, 1, 4096, 4096, 20, 128, 128, 512, 0)
    # the selection mask (one bit per key, rows padded to 128 keys) and, after it, the block
    # list: per 128-query block a count (int32) and up to 32 key-block numbers (uint16)
    nqb = nkb = 4096 // 128
    assert pre == 4096 * nkb * 4 * 4 + nqb * 4 + nqb * nkb * 2
    assert L.dsa_sparse_attn_workspace_bytes(1, 1, 4096, 4096, 20, 128, 128, 512, 1) == 0


def test_sparse_attn_sinks_rejects_bad_arguments(lib):
    L = lib.lib()

    def call(nsink=4, sk=FAKE, sv=FAKE, **kw):
        a = dict(dtype=1, B=1, S=4, T=4, H=2, DQK=128, DV=128, K=2)
        a.update(kw)
        return L.dsa_sparse_attn_sinks(a["dtype"], FAKE, FAKE, FAKE, FAKE, a["K"], sk, sv, nsink,
                                       None, 0, 0.0, a["B"], a["S"], a["T"], a["H"], a["DQK"],
                                       a["DV"], 1, FAKE, FAKE, 1 << 20, None)
    assert call(nsink=0) == 1          # use dsa_sparse_attn without sinks
    assert call(nsink=129) == 2        # at most one 128-entry block
    assert call(sk=None) == 1
    assert call(sv=FAKE_MIS) == 2
    assert L.dsa_sparse_attn_sinks_workspace_bytes(1, 1, 4, 4, 2, 128, 128, 2, 4, 1) >= 0


def test_sparse_attn_latent_rejects_bad_arguments(lib):
    L = lib.lib()

    def call(dtype=1, H=128, DQK=576, DV=512, nsink=0, skv=None, q=FAKE, ws_bytes=1 << 30, **kw):
        a = dict(B=2, S=1, T=5000, K=2048)
        a.update(kw)
        return L.dsa_sparse_attn_latent(dtype, q, FAKE, FAKE, a["K"], skv, nsink, None, 0, 0.0,
                                        a["B"], a["S"], a["T"], H, DQK, DV, FAKE, FAKE, ws_bytes,
                                        None)
    assert call(dtype=0) == 2           # float32: no latent kernel
    assert call(dtype=7) == 1
    assert call(DQK=192, DV=128) == 2   # only the 512 + 64 latent row
    assert call(DV=640) == 1            # values longer than the row
    assert call(H=129) == 2
    assert call(H=0) == 1
    assert call(nsink=4) == 1           # sinks without rows
    assert call(nsink=129, skv=FAKE) == 2
    assert call(q=FAKE_MIS) == 2
    assert call(S=2, T=1) == 1
    need = L.dsa_sparse_attn_latent_workspace_bytes(2, 1, 128, 2048, 0)
    assert need > 0                     # decode-shaped: split keys need partials
    assert call(ws_bytes=need - 1) == 1
    assert L.dsa_sparse_attn_latent_workspace_bytes(1, 4096, 128, 2048, 0) == 0


def test_window_attn_sinks_rejects_bad_arguments(lib):
    L = lib.lib()

    def call(nsink=4, sk=FAKE, sv=FAKE):
        return L.dsa_window_attn_sinks(1, FAKE, FAKE, FAKE, sk, sv, nsink, None, 0, 0.0, 8, 1, 4,
                                       4, 4, 2, 128, 128, 1, FAKE, None)
    assert call(nsink=0) == 1
    assert call(nsink=200) == 2
    assert call(sv=None) == 1


def test_window_attn_rejects_bad_arguments(lib):
    L = lib.lib()
    f = L.dsa_window_attn
    assert f(1, FAKE, FAKE, FAKE, None, 0, 0.0, 512, 1, 1024, 1024, 32, 6, 192, 128, 0, FAKE,
             None) == 1  # 32 heads over 6 KV heads
    assert f(1, FAKE, FAKE, FAKE, None, 0, 0.0, 0, 1, 1024, 1024, 32, 8, 192, 128, 0, FAKE,
             None) == 1  # empty window
    assert f(1, FAKE, FAKE, FAKE, None, 0, 0.0, 512, 1, 1024, 1024, 32, 8, 96, 128, 2, FAKE,
             None) == 2  # masked tile needs DQK 128 or 192


def test_forward_workspace_and_validation(lib):
    L = lib.lib()
    a = lib.ForwardArgs(dtype=1, B=1, S=4096, T=4096, HI=16, DI=64, index_scale=2 ** -4,
                        relu=0, K=512, H=20, DQK=128, DV=128, sm_scale=0.0, gate_mode=0,
                        attn_algo=0, q_idx=0x10000, k_idx=0x10000, w=0x10000, q=0x10000,
                        k=0x10000, v=0x10000, gate=None, out=0x10000, scores_out=None,
                        idx_out=None)
    full = lib.dsa_forward_workspace_bytes(a)
    small = lib.dsa_forward_workspace_bytes(a, minimum=True)
    assert full >= 4096 * 4096 * 4 + 4096 * 512 * 4
    assert small < full
    assert L.dsa_forward(ctypes.byref(a), FAKE, small - 1, None) == 1
    a.gate_mode = 1  # gate on without a gate tensor
    assert L.dsa_forward(ctypes.byref(a), FAKE, full, None) == 1
    a.gate_mode = 0
    a.attn_algo = 9
    assert L.dsa_forward(ctypes.byref(a), FAKE, full, None) == 1
    a.attn_algo = 0
    a.indexer = 7
    assert L.dsa_forward(ctypes.byref(a), FAKE, full, None) == 1
    # the collapsed indexer needs room for its query rows and no per-head ReLU
    a.indexer = 1
    full_c = lib.dsa_forward_workspace_bytes(a)
    assert full_c == full + 4096 * 2 * 64 * 2
    assert lib.dsa_forward_workspace_bytes(a, minimum=True) == small + 4096 * 2 * 64 * 2
    a.relu = 2
    assert L.dsa_forward(ctypes.byref(a), FAKE, full_c, None) == 2
    a.relu = 0
    a.index_dtype = 1  # e4m3 indexer inputs: per-head indexer only, DI == 128
    assert L.dsa_forward(ctypes.byref(a), FAKE, full_c, None) == 2
    a.indexer = 0
    assert L.dsa_forward(ctypes.byref(a), FAKE, full, None) == 2  # DI = 64
    a.index_dtype = 5
    assert L.dsa_forward(ctypes.byref(a), FAKE, full, None) == 1
    a.index_dtype = 0
    # the latent attention form: k is the latent cache, v unused; its own shape rules
    a.attn_form = 1
    assert L.dsa_forward(ctypes.byref(a), FAKE, full, None) == 2  # DQK 128 is not 576
    a.H, a.DQK, a.DV, a.v = 128, 576, 512, None
    # prefill: no split partials, and no selection bitmask (4096 rows x 4096 bits) nor its
    # block list (32 counts and 32 x 32 block numbers, the region 256-byte aligned)
    blocks = 32 * 4 + 32 * 32 * 2
    assert lib.dsa_forward_workspace_bytes(a) == full - 4096 * 4096 // 8 - ((blocks + 255) // 256) * 256
    a.attn_form = 3
    assert L.dsa_forward(ctypes.byref(a), FAKE, full, None) == 1


def test_binding_fails_loudly_without_library(monkeypatch):
    import sparse_attention_15_b200 as dsa
    monkeypatch.setattr(dsa, "_LIB", None)
    monkeypatch.setattr(dsa, "LIB_PATH", "/nonexistent/libdsa.so")
    with pytest.raises(RuntimeError, match="no fallback"):
        dsa.lib()
