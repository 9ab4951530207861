"""Python binding of libdsa, the B200 DSA hot path (see include/dsa.h for the contract).

Argument marshalling only: every function here reads sizes off torch tensors, allocates
outputs (device memory plumbing) when the caller gives none, passes raw device pointers
and the current CUDA stream to the C entry point of the same name, and raises DSAError
on a non-OK status.  All compute runs in the library's CUDA kernels; there is no
fallback -- if libdsa.so is missing, importing a function raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "DSAError", "lib", "dsa_index_scores", "dsa_index_scores_collapsed", "dsa_hadamard_rotate",
    "dsa_topk", "dsa_index_topk", "dsa_index_topk_workspace_bytes",
    "dsa_sparse_attn", "dsa_sparse_attn_sinks", "dsa_sparse_attn_workspace_bytes",
    "dsa_sparse_attn_algo", "dsa_forward",
    "dsa_forward_workspace_bytes",
    "dsa_window_attn", "dsa_sparse_attn_noalloc", "dsa_device_status", "dsa_version",
    "dsa_test_arm_wait_timeout", "dsa_test_topk_bucket_floor", "LIB_PATH",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdsa.so")

DTYPE = {torch.float32: 0, torch.bfloat16: 1, torch.float8_e4m3fn: 2}  # e4m3: indexer inputs
RELU = {"none": 0, "post_sum": 1, "per_head": 2}
GATE = {"off": 0, "sigmoid": 1, "silu": 2}
ATTN_ALGO = {"auto": 0, "gather": 1, "masked_tile": 2}
INDEXER = {"per_head": 0, "collapsed": 1, "fused": 2}
ATTN_FORM = {"expanded": 0, "latent": 1}
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "CUDA error", 4: "timeout",
          5: "internal"}


class DSAError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"libdsa status {status} ({STATUS.get(status, '?')}): {message}")
        self.status = status


class ForwardArgs(ctypes.Structure):
    """Mirror of dsa_forward_args (include/dsa.h)."""
    _fields_ = [
        ("dtype", ctypes.c_int), ("B", ctypes.c_int), ("S", ctypes.c_int), ("T", ctypes.c_int),
        ("HI", ctypes.c_int), ("DI", ctypes.c_int), ("index_scale", ctypes.c_float),
        ("relu", ctypes.c_int), ("K", ctypes.c_int), ("H", ctypes.c_int), ("DQK", ctypes.c_int),
        ("DV", ctypes.c_int), ("sm_scale", ctypes.c_float), ("gate_mode", ctypes.c_int),
        ("attn_algo", ctypes.c_int),
        ("q_idx", ctypes.c_void_p), ("k_idx", ctypes.c_void_p), ("w", ctypes.c_void_p),
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("gate", ctypes.c_void_p), ("out", ctypes.c_void_p), ("scores_out", ctypes.c_void_p),
        ("idx_out", ctypes.c_void_p), ("events", ctypes.c_void_p), ("indexer", ctypes.c_int),
        ("index_dtype", ctypes.c_int), ("sink_k", ctypes.c_void_p), ("sink_v", ctypes.c_void_p),
        ("nsink", ctypes.c_int), ("attn_form", ctypes.c_int),
        ("topk_fallback_out", ctypes.c_void_p),
    ]


_LIB = None
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_Z = ctypes.c_size_t

_SIGNATURES = {
    "dsa_index_scores": (_I, [_I, _P, _P, _P, _F, _I, _I, _I, _I, _I, _I, _P, _P]),
    "dsa_index_scores_collapsed_workspace_bytes": (_Z, [_I, _I, _I]),
    "dsa_index_scores_collapsed": (_I, [_I, _P, _P, _P, _F, _I, _I, _I, _I, _I, _I, _P, _P, _Z,
                                        _P]),
    "dsa_hadamard_rotate": (_I, [_I, _P, ctypes.c_longlong, _I, _P, _P]),
    "dsa_topk": (_I, [_P, _I, _I, _I, _I, _P, _P]),
    "dsa_index_topk_workspace_bytes": (_Z, [_I, _I, _I, _I]),
    "dsa_index_topk": (_I, [_I, _P, _P, _P, _F, _I, _I, _I, _I, _I, _I, _I, _P, _P, _Z, _P,
                            _P]),
    "dsa_sparse_attn_workspace_bytes": (_Z, [_I, _I, _I, _I, _I, _I, _I, _I, _I]),
    "dsa_sparse_attn_algo": (_I, [_I, _I, _I, _I, _I, _I, _I, _I, _I]),
    "dsa_sparse_attn": (_I, [_I, _P, _P, _P, _P, _I, _P, _I, _F, _I, _I, _I, _I, _I, _I, _I, _P,
                             _P, _Z, _P]),
    "dsa_sparse_attn_sinks_workspace_bytes": (_Z, [_I, _I, _I, _I, _I, _I, _I, _I, _I, _I]),
    "dsa_sparse_attn_sinks": (_I, [_I, _P, _P, _P, _P, _I, _P, _P, _I, _P, _I, _F, _I, _I, _I,
                                   _I, _I, _I, _I, _P, _P, _Z, _P]),
    "dsa_sparse_attn_latent_workspace_bytes": (_Z, [_I, _I, _I, _I, _I]),
    "dsa_sparse_attn_latent": (_I, [_I, _P, _P, _P, _I, _P, _I, _P, _I, _F, _I, _I, _I, _I, _I,
                                    _I, _P, _P, _Z, _P]),
    "dsa_forward_workspace_bytes": (_Z, [ctypes.POINTER(ForwardArgs)]),
    "dsa_forward_min_workspace_bytes": (_Z, [ctypes.POINTER(ForwardArgs)]),
    "dsa_forward": (_I, [ctypes.POINTER(ForwardArgs), _P, _Z, _P]),
    "dsa_window_attn": (_I, [_I, _P, _P, _P, _P, _I, _F, _I, _I, _I, _I, _I, _I, _I, _I, _I,
                             _P, _P]),
    "dsa_window_attn_sinks": (_I, [_I, _P, _P, _P, _P, _P, _I, _P, _I, _F, _I, _I, _I, _I, _I,
                                   _I, _I, _I, _I, _P, _P]),
    "dsa_sparse_attn_noalloc_max_scratch_bytes": (_Z, []),
    "dsa_sparse_attn_noalloc": (_I, [_I, _P, _P, _P, _P, _I, _P, _I, _F, _I, _I, _I, _I, _I, _I,
                                     _P, _P]),
    "dsa_status_string": (ctypes.c_char_p, [_I]),
    "dsa_last_error": (ctypes.c_char_p, []),
    "dsa_device_status": (_I, [_I]),
    "dsa_version": (ctypes.c_char_p, []),
    "dsa_test_arm_wait_timeout": (_I, []),
    "dsa_test_topk_bucket_floor": (ctypes.c_float, [ctypes.c_uint]),
}


def lib() -> ctypes.CDLL:
    """The loaded libdsa.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m sparse_attention_15_b200.build`"
                " (there is no fallback path)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def _check(status: int):
    if status != 0:
        raise DSAError(status, lib().dsa_last_error().decode(errors="replace"))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("libdsa takes contiguous CUDA tensors")


def _dtype_code(t):
    try:
        return DTYPE[t.dtype]
    except KeyError:
        raise ValueError(f"unsupported dtype {t.dtype}") from None


def dsa_version() -> str:
    return lib().dsa_version().decode()


def dsa_device_status(reset: bool = True) -> int:
    """Reads (and clears) the device status word; raises DSAError on a recorded fault."""
    st = lib().dsa_device_status(1 if reset else 0)
    _check(st)
    return st


def dsa_test_arm_wait_timeout() -> None:
    """Testing aid: the next gather-attention launch runs one bounded wait out on purpose
    (it records DSA_ERR_TIMEOUT; its output is undefined).  One-shot."""
    _check(lib().dsa_test_arm_wait_timeout())


def dsa_test_topk_bucket_floor(b: int) -> float:
    """Testing aid: the top-k's float bound of 12-bit key bucket b (host code)."""
    return float(lib().dsa_test_topk_bucket_floor(b))


def dsa_index_scores(q_idx, k_idx, w, scale, relu="none", scores=None, stream=None):
    """scores[b,s,t] = scale * sum_h w[b,s,h] (q_idx[b,s,h,:] . k_idx[b,t,:]), -inf if t > s+T-S."""
    _dev(q_idx, k_idx, w, scores)
    B, S, HI, DI = q_idx.shape
    T = k_idx.shape[1]
    if scores is None:
        scores = torch.empty((B, S, T), dtype=torch.float32, device=q_idx.device)
    _check(lib().dsa_index_scores(_dtype_code(q_idx), _ptr(q_idx), _ptr(k_idx), _ptr(w),
                                  float(scale), RELU[relu], B, S, T, HI, DI, _ptr(scores),
                                  _stream(stream)))
    return scores


def dsa_index_scores_collapsed(q_idx, k_idx, w, scale, relu="none", scores=None, ws=None,
                               stream=None):
    """The same scores as dsa_index_scores from the head-collapsed query
    sum_h w[b,s,h] q_idx[b,s,h,:] (bf16, no per-head ReLU; see include/dsa.h)."""
    _dev(q_idx, k_idx, w, scores, ws)
    B, S, HI, DI = q_idx.shape
    T = k_idx.shape[1]
    if scores is None:
        scores = torch.empty((B, S, T), dtype=torch.float32, device=q_idx.device)
    nbytes = int(lib().dsa_index_scores_collapsed_workspace_bytes(B, S, DI))
    ws = _workspace(nbytes, q_idx.device, ws)
    _check(lib().dsa_index_scores_collapsed(_dtype_code(q_idx), _ptr(q_idx), _ptr(k_idx), _ptr(w),
                                            float(scale), RELU[relu], B, S, T, HI, DI,
                                            _ptr(scores), _ptr(ws), nbytes, _stream(stream)))
    return scores


def dsa_hadamard_rotate(x, out=None, stream=None):
    """x @ H / sqrt(d) over the last dimension (d in {64, 128}; float32 or bf16); out may be x."""
    _dev(x, out)
    d = x.shape[-1]
    if out is None:
        out = torch.empty_like(x)
    _check(lib().dsa_hadamard_rotate(_dtype_code(x), _ptr(x), x.numel() // d, d, _ptr(out),
                                     _stream(stream)))
    return out


def dsa_topk(scores, K, idx=None, stream=None):
    """int32 [B,S,K]: the kept keys of each query in ascending order, -1 padded."""
    _dev(scores, idx)
    B, S, T = scores.shape
    if idx is None:
        idx = torch.empty((B, S, K), dtype=torch.int32, device=scores.device)
    _check(lib().dsa_topk(_ptr(scores), B, S, T, int(K), _ptr(idx), _stream(stream)))
    return idx



def dsa_index_topk_workspace_bytes(B, S, T, K) -> int:
    return int(lib().dsa_index_topk_workspace_bytes(B, S, T, K))


def dsa_index_topk(q_idx, k_idx, w, scale, K, relu="none", idx=None, ws=None,
                   fallback_out=None, stream=None):
    """Fused indexer -> top-k: the indices dsa_index_scores + dsa_topk give, without the
    score matrix (candidates filtered inside the indexer).  fallback_out: optional int32
    device tensor of one element, set to 1 when the full-score fallback ran."""
    _dev(q_idx, k_idx, w, idx, ws, fallback_out)
    B, S, HI, DI = q_idx.shape
    T = k_idx.shape[1]
    k_eff = min(int(K), T)
    if idx is None:
        idx = torch.empty((B, S, k_eff), dtype=torch.int32, device=q_idx.device)
    nbytes = dsa_index_topk_workspace_bytes(B, S, T, int(K))
    ws = _workspace(nbytes, q_idx.device, ws)
    _check(lib().dsa_index_topk(_dtype_code(q_idx), _ptr(q_idx), _ptr(k_idx), _ptr(w),
                                float(scale), RELU[relu], B, S, T, HI, DI, int(K), _ptr(idx),
                                _ptr(ws), nbytes, _ptr(fallback_out), _stream(stream)))
    return idx

def dsa_sparse_attn_workspace_bytes(dtype, B, S, T, H, DQK, DV, K, algo="auto") -> int:
    code = dtype if isinstance(dtype, int) else DTYPE[dtype]
    return int(lib().dsa_sparse_attn_workspace_bytes(code, B, S, T, H, DQK, DV, K,
                                                     ATTN_ALGO[algo]))


def dsa_sparse_attn_algo(dtype, B, S, T, H, DQK, DV, K, algo="auto") -> str:
    """The algorithm ("gather" / "masked_tile") a request resolves to for this shape."""
    code = dtype if isinstance(dtype, int) else DTYPE[dtype]
    r = int(lib().dsa_sparse_attn_algo(code, B, S, T, H, DQK, DV, K, ATTN_ALGO[algo]))
    return {v: k for k, v in ATTN_ALGO.items()}[r]


def _workspace(nbytes, device, ws):
    if nbytes == 0:
        return ws
    if ws is None or ws.numel() < nbytes:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return ws


def dsa_sparse_attn(q, k, v, idx, gate=None, gate_mode=None, sm_scale=0.0, algo="auto",
                    out=None, ws=None, stream=None):
    """Attention of each query over its selected keys (idx), with the optional gate.
    algo: "auto", "gather" or "masked_tile"."""
    _dev(q, k, v, idx, gate, out, ws)
    B, S, H, DQK = q.shape
    T, DV = k.shape[1], v.shape[-1]
    K = idx.shape[-1]
    gm = GATE[gate_mode or ("sigmoid" if gate is not None else "off")]
    if out is None:
        out = torch.empty((B, S, H, DV), dtype=q.dtype, device=q.device)
    nbytes = dsa_sparse_attn_workspace_bytes(_dtype_code(q), B, S, T, H, DQK, DV, K, algo)
    ws = _workspace(nbytes, q.device, ws)
    _check(lib().dsa_sparse_attn(_dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), K,
                                 _ptr(gate), gm, float(sm_scale), B, S, T, H, DQK, DV,
                                 ATTN_ALGO[algo], _ptr(out), _ptr(ws), nbytes, _stream(stream)))
    return out


def dsa_sparse_attn_sinks(q, k, v, idx, sink_k, sink_v, gate=None, gate_mode=None,
                          sm_scale=0.0, algo="auto", out=None, ws=None, stream=None):
    """dsa_sparse_attn with attention sinks: sink_k [NS,H,DQK], sink_v [NS,H,DV] (NS <= 128)
    join every query's softmax unmasked."""
    _dev(q, k, v, idx, sink_k, sink_v, gate, out, ws)
    B, S, H, DQK = q.shape
    T, DV = k.shape[1], v.shape[-1]
    K = idx.shape[-1]
    NS = sink_k.shape[0]
    gm = GATE[gate_mode or ("sigmoid" if gate is not None else "off")]
    if out is None:
        out = torch.empty((B, S, H, DV), dtype=q.dtype, device=q.device)
    nbytes = int(lib().dsa_sparse_attn_sinks_workspace_bytes(_dtype_code(q), B, S, T, H, DQK, DV,
                                                             K, NS, ATTN_ALGO[algo]))
    ws = _workspace(nbytes, q.device, ws)
    _check(lib().dsa_sparse_attn_sinks(_dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), K,
                                       _ptr(sink_k), _ptr(sink_v), NS, _ptr(gate), gm,
                                       float(sm_scale), B, S, T, H, DQK, DV, ATTN_ALGO[algo],
                                       _ptr(out), _ptr(ws), nbytes, _stream(stream)))
    return out


def dsa_sparse_attn_noalloc(q, k, v, idx, gate=None, gate_mode=None, sm_scale=0.0, out=None,
                            stream=None):
    """dsa_sparse_attn (gather form) with no workspace: the split-key partials live in the
    library's fixed device array (see include/dsa.h).  Allocates nothing but ``out`` when
    the caller gives none."""
    _dev(q, k, v, idx, gate, out)
    B, S, H, DQK = q.shape
    T, DV = k.shape[1], v.shape[-1]
    K = idx.shape[-1]
    gm = GATE[gate_mode or ("sigmoid" if gate is not None else "off")]
    if out is None:
        out = torch.empty((B, S, H, DV), dtype=q.dtype, device=q.device)
    _check(lib().dsa_sparse_attn_noalloc(_dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), K,
                                         _ptr(gate), gm, float(sm_scale), B, S, T, H, DQK, DV,
                                         _ptr(out), _stream(stream)))
    return out


def dsa_sparse_attn_latent(q, kv, idx, dv=512, sink_kv=None, gate=None, gate_mode=None,
                           sm_scale=0.0, out=None, ws=None, stream=None):
    """Sparse attention over a shared latent cache (MQA form): q [B,S,H,DQK], kv [B,T,DQK]
    (keys = whole rows, values = their first ``dv`` dims), idx [B,S,K]; optional latent sink
    rows sink_kv [NS,DQK] (NS <= 128).  bf16, DQK 576, dv 512, H <= 128."""
    _dev(q, kv, idx, sink_kv, gate, out, ws)
    B, S, H, DQK = q.shape
    T = kv.shape[1]
    K = idx.shape[-1]
    NS = 0 if sink_kv is None else int(sink_kv.shape[0])
    gm = GATE[gate_mode or ("sigmoid" if gate is not None else "off")]
    if out is None:
        out = torch.empty((B, S, H, dv), dtype=q.dtype, device=q.device)
    nbytes = int(lib().dsa_sparse_attn_latent_workspace_bytes(B, S, H, K, NS))
    ws = _workspace(nbytes, q.device, ws)
    _check(lib().dsa_sparse_attn_latent(_dtype_code(q), _ptr(q), _ptr(kv), _ptr(idx), K,
                                        _ptr(sink_kv), NS, _ptr(gate), gm, float(sm_scale), B, S,
                                        T, H, DQK, int(dv), _ptr(out), _ptr(ws), nbytes,
                                        _stream(stream)))
    return out


def _forward_args(q_idx, k_idx, w, index_scale, K, q, k, v, gate, gate_mode, relu, sm_scale,
                  attn_algo, out, scores_out, idx_out, indexer="per_head", sink_k=None,
                  sink_v=None, attn_form="expanded", dv=512, topk_fallback_out=None):
    B, S, HI, DI = q_idx.shape
    T = k_idx.shape[1]
    H, DQK = q.shape[2], q.shape[3]
    DV = int(dv) if attn_form == "latent" else v.shape[-1]
    gm = GATE[gate_mode or ("sigmoid" if gate is not None else "off")]
    a = ForwardArgs(
        dtype=_dtype_code(q), B=B, S=S, T=T, HI=HI, DI=DI, index_scale=float(index_scale),
        relu=RELU[relu], K=int(K), H=H, DQK=DQK, DV=DV, sm_scale=float(sm_scale), gate_mode=gm,
        attn_algo=ATTN_ALGO[attn_algo], q_idx=q_idx.data_ptr(), k_idx=k_idx.data_ptr(),
        w=w.data_ptr(), q=q.data_ptr(), k=k.data_ptr(), v=None if v is None else v.data_ptr(),
        gate=None if gate is None else gate.data_ptr(), out=out.data_ptr(),
        scores_out=None if scores_out is None else scores_out.data_ptr(),
        idx_out=None if idx_out is None else idx_out.data_ptr(), indexer=INDEXER[indexer],
        index_dtype=1 if q_idx.dtype == torch.float8_e4m3fn else 0,
        sink_k=None if sink_k is None else sink_k.data_ptr(),
        sink_v=None if sink_v is None else sink_v.data_ptr(),
        nsink=0 if sink_k is None else int(sink_k.shape[0]), attn_form=ATTN_FORM[attn_form],
        topk_fallback_out=None if topk_fallback_out is None else topk_fallback_out.data_ptr())
    return a


def dsa_forward_workspace_bytes(args: ForwardArgs, minimum: bool = False) -> int:
    f = lib().dsa_forward_min_workspace_bytes if minimum else lib().dsa_forward_workspace_bytes
    return int(f(ctypes.byref(args)))


def dsa_forward(q_idx, k_idx, w, index_scale, K, q, k, v, gate=None, gate_mode=None,
                relu="none", sm_scale=0.0, attn_algo="auto", out=None, scores_out=None,
                idx_out=None, ws=None, ws_bytes=None, stream=None, events=None,
                indexer="per_head", sink_k=None, sink_v=None, attn_form="expanded", dv=512,
                topk_fallback_out=None):
    """The whole DSA step (indexer -> top-k -> sparse attention -> gate).
    indexer: "per_head" (the pages' per-head work), "collapsed" (see
    dsa_index_scores_collapsed) or "fused" (see dsa_index_topk; topk_fallback_out, an
    optional int32 device tensor of one element, receives whether its fallback ran).  attn_form "latent": k is the latent cache [B,T,DQK]
    (values = its first ``dv`` dims), v is None, sink_k holds latent sink rows [NS,DQK].

    Returns (out, idx); idx is idx_out if given, else a view of the workspace copy.
    ``ws_bytes`` limits the workspace handed to the library (row blocking below the
    full size)."""
    _dev(q_idx, k_idx, w, q, k, v, gate, out, scores_out, idx_out, ws, sink_k, sink_v,
         topk_fallback_out)
    B, S = q_idx.shape[:2]
    T = k_idx.shape[1]
    if out is None:
        DV = int(dv) if attn_form == "latent" else v.shape[-1]
        out = torch.empty((B, S, q.shape[2], DV), dtype=q.dtype, device=q.device)
    k_eff = min(int(K), T)
    if idx_out is None:
        idx_out = torch.empty((B, S, k_eff), dtype=torch.int32, device=q.device)
    a = _forward_args(q_idx, k_idx, w, index_scale, K, q, k, v, gate, gate_mode, relu, sm_scale,
                      attn_algo, out, scores_out, idx_out, indexer, sink_k, sink_v, attn_form,
                      dv, topk_fallback_out)
    ev_arr = None
    if events is not None:  # 4 torch.cuda.Event, recorded by the library at stage boundaries
        for e in events:
            if e.cuda_event == 0:
                e.record()  # torch creates the CUDA event on first use
        ev_arr = (ctypes.c_void_p * 4)(*[e.cuda_event for e in events])
        a.events = ctypes.cast(ev_arr, ctypes.c_void_p).value
    nbytes = dsa_forward_workspace_bytes(a) if ws_bytes is None else int(ws_bytes)
    ws = _workspace(nbytes, q.device, ws)
    _check(lib().dsa_forward(ctypes.byref(a), _ptr(ws), nbytes, _stream(stream)))
    return out, idx_out


def dsa_window_attn(q, k, v, window, gate=None, gate_mode=None, sm_scale=0.0, algo="auto",
                    out=None, stream=None, sink_k=None, sink_v=None):
    """Sliding-window causal attention with grouped KV heads (window keys incl. self);
    optional attention sinks sink_k [NS,HKV,DQK], sink_v [NS,HKV,DV] (NS <= 128)."""
    _dev(q, k, v, gate, out, sink_k, sink_v)
    B, S, H, DQK = q.shape
    T, HKV, DV = k.shape[1], k.shape[2], v.shape[-1]
    gm = GATE[gate_mode or ("sigmoid" if gate is not None else "off")]
    if out is None:
        out = torch.empty((B, S, H, DV), dtype=q.dtype, device=q.device)
    if sink_k is None:
        _check(lib().dsa_window_attn(_dtype_code(q), _ptr(q), _ptr(k), _ptr(v), _ptr(gate), gm,
                                     float(sm_scale), int(window), B, S, T, H, HKV, DQK, DV,
                                     ATTN_ALGO[algo], _ptr(out), _stream(stream)))
    else:
        _check(lib().dsa_window_attn_sinks(_dtype_code(q), _ptr(q), _ptr(k), _ptr(v),
                                           _ptr(sink_k), _ptr(sink_v), int(sink_k.shape[0]),
                                           _ptr(gate), gm, float(sm_scale), int(window), B, S,
                                           T, H, HKV, DQK, DV, ATTN_ALGO[algo], _ptr(out),
                                           _stream(stream)))
    return out
