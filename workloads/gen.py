"""Seeded synthetic inputs.  Random numbers only: no part of the method is computed here.

Recipe (every config): indexer q_I and k_I are integers drawn uniformly from [-2, 2];
indexer head weights w are integers drawn uniformly from [1, 4] (float32); attention
q, k, v and gate logits are N(0, 1) drawn in float32 and rounded to the compute dtype.
Each tensor has its own torch.Generator seeded with ``16 * seed + slot`` on the device it
is created on, so a tensor's values do not depend on which other tensors were drawn.
CPU and CUDA generators give different streams: a check always feeds the same tensors
to both sides.
"""
from __future__ import annotations

import torch

_SLOTS = {"q_idx": 0, "k_idx": 1, "w": 2, "q": 3, "k": 4, "v": 5, "gate": 6}
# the latent (MQA-form) attention inputs and the random selections use slots of their own
_LATENT_SLOTS = {"q": 8, "kv": 9, "sink": 10, "sel": 11}


def _gen(device, seed, slot):
    g = torch.Generator(device=device)
    g.manual_seed(16 * int(seed) + slot)
    return g


def _dtype(name):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def _ints(shape, lo, hi, dtype, device, g):
    return torch.empty(shape, dtype=dtype, device=device).random_(lo, hi + 1, generator=g)


def _normal(shape, dtype, device, g):
    if dtype == torch.float32:
        return torch.empty(shape, dtype=dtype, device=device).normal_(generator=g)
    # draw in float32, round to bf16; chunked so huge caches need no big fp32 temporary
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(-1)
    step = 1 << 28
    for i in range(0, flat.numel(), step):
        n = min(step, flat.numel() - i)
        flat[i:i + n] = torch.empty(n, dtype=torch.float32, device=device).normal_(generator=g)
    return out


def dsa_inputs(cfg, device="cpu", seed=None, B=None, S=None, T=None, need=None):
    """Inputs of one DSA layer for ``cfg`` (sizes may be overridden for small cases).

    Returns a dict with q_idx [B,S,HI,DI], k_idx [B,T,DI], w [B,S,HI] (float32),
    q [B,S,H,Dqk], k [B,T,H,Dqk], v [B,T,H,Dv], gate [B,S,H] (or None when the gate is off).
    ``need`` restricts which tensors are created.
    """
    seed = cfg.seed if seed is None else seed
    B = cfg.B if B is None else B
    S = cfg.S if S is None else S
    T = cfg.T if T is None else T
    dt = _dtype(cfg.dtype)
    need = set(need) if need is not None else set(_SLOTS)
    out = {}
    if "q_idx" in need:
        out["q_idx"] = _ints((B, S, cfg.HI, cfg.DI), -2, 2, dt, device, _gen(device, seed, 0))
    if "k_idx" in need:
        out["k_idx"] = _ints((B, T, cfg.DI), -2, 2, dt, device, _gen(device, seed, 1))
    if "w" in need:
        out["w"] = _ints((B, S, cfg.HI), 1, 4, torch.float32, device, _gen(device, seed, 2))
    if "q" in need:
        out["q"] = _normal((B, S, cfg.H, cfg.dqk), dt, device, _gen(device, seed, 3))
    if "k" in need:
        out["k"] = _normal((B, T, cfg.H, cfg.dqk), dt, device, _gen(device, seed, 4))
    if "v" in need:
        out["v"] = _normal((B, T, cfg.H, cfg.dv), dt, device, _gen(device, seed, 5))
    if "gate" in need:
        out["gate"] = (_normal((B, S, cfg.H), dt, device, _gen(device, seed, 6))
                       if cfg.gate != "off" else None)
    return out


def swa_inputs(cfg, layer, device="cpu", seed=None, B=None, S=None, T=None):
    """Inputs of sliding-window layer ``layer`` (1-based) of a hybrid block.

    q [B,S,H,Dqk], k [B,T,HKV,Dqk], v [B,T,HKV,Dv], gate [B,S,H] or None.
    """
    seed = (cfg.seed if seed is None else seed) + 1000 * int(layer)
    B = cfg.B if B is None else B
    S = cfg.S if S is None else S
    T = cfg.T if T is None else T
    dt = _dtype(cfg.dtype)
    hkv = cfg.swa_kv_heads
    return {
        "q": _normal((B, S, cfg.H, cfg.dqk), dt, device, _gen(device, seed, 3)),
        "k": _normal((B, T, hkv, cfg.dqk), dt, device, _gen(device, seed, 4)),
        "v": _normal((B, T, hkv, cfg.dv), dt, device, _gen(device, seed, 5)),
        "gate": (_normal((B, S, cfg.H), dt, device, _gen(device, seed, 6))
                 if cfg.gate != "off" else None),
    }


def latent_inputs(cfg, H=128, dqk=576, device="cpu", seed=None, B=None, S=None, T=None,
                  nsink=0):
    """Inputs of the latent (MQA-form) attention of a DSA layer: absorbed queries
    q [B,S,H,dqk], the latent cache kv [B,T,dqk] (one row per token, shared by all heads) and
    optional latent sink rows sink_kv [nsink,dqk] (None when nsink == 0); N(0, 1) drawn in
    float32 and rounded to the compute dtype, like the other attention inputs.  The gate,
    when the config has one, is the config's own ``gate`` tensor (dsa_inputs) resized to H.
    """
    seed = cfg.seed if seed is None else seed
    B = cfg.B if B is None else B
    S = cfg.S if S is None else S
    T = cfg.T if T is None else T
    dt = _dtype(cfg.dtype)
    sl = _LATENT_SLOTS
    out = {
        "q": _normal((B, S, H, dqk), dt, device, _gen(device, seed, sl["q"])),
        "kv": _normal((B, T, dqk), dt, device, _gen(device, seed, sl["kv"])),
        "sink_kv": (_normal((nsink, dqk), dt, device, _gen(device, seed, sl["sink"]))
                    if nsink > 0 else None),
        "gate": (_normal((B, S, H), dt, device, _gen(device, seed, 6))
                 if cfg.gate != "off" else None),
    }
    return out


def random_selection(B, S, T, K, seed, q_off=None):
    """Random index lists shaped like the top-k output, on the CPU: row (b, s) holds
    min(K, n) distinct keys drawn uniformly from the n = s + q_off + 1 causal keys, in
    ascending order, then -1 padding.  int32 [B,S,K]."""
    if q_off is None:
        q_off = T - S
    g = _gen("cpu", seed, _LATENT_SLOTS["sel"])
    idx = torch.full((B, S, K), -1, dtype=torch.int32)
    for b in range(B):
        for s in range(S):
            n = min(s + q_off + 1, T)
            k = min(K, n)
            pick = torch.randperm(n, generator=g)[:k]
            idx[b, s, :k] = torch.sort(pick).values.to(torch.int32)
    return idx
