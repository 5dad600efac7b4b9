"""Shared test helpers: build a cache from a synth layer, the oracle's view of
the same context, and comparison helpers.  Inputs come from ``synth`` only;
expected values from ``oracle`` only."""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import oracle
import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")

ATT_MAX_ABS = 2e-2     # attention: max |O_gpu - O_oracle|
ATT_REL_L2 = 5e-3      # attention: ||O_gpu - O_oracle||_2 / ||O_oracle||_2
KEY_MAX_ABS = 1e-2     # shifted keys (with a one-bf16-ulp allowance)
LSE_MAX_ABS = 1e-3


def seeds() -> dict:
    with open(os.path.join(GOLD, "seeds.json")) as f:
        return json.load(f)


def seed_for(name: str) -> int:
    s = seeds()
    if name in s:
        return s[name]
    return synth.nominal_seed(list(synth.WORKLOADS).index(name))


def build_cache(pf, wl, d, via_append: bool = False, device="cuda", sink_rope_in_attention: bool = False):
    """A one-layer cache holding d's sink, mid pool and recent blocks."""
    cache = pf.PackedKVCache(pf.config_for(wl, layers=1, sink_rope_in_attention=sink_rope_in_attention),
                             device=device)
    dev = lambda t: t.to(device).contiguous()  # noqa: E731
    for s in range(wl.sink_blocks):
        cache.append_block(0, dev(d["sink_K"][:, s]), dev(d["sink_V"][:, s]))
    P = wl.pool_blocks
    if P:
        if via_append:
            zK = torch.zeros_like(dev(d["K_cur"]))
            for p in range(P):
                cache.append_block(0, zK, zK, dev(d["mid_K"][:, p]), dev(d["mid_V"][:, p]))
            # the last pool block is still "recent"; push it into the pool with the recent blocks below
        else:
            cache.load_mid(0, dev(d["mid_K"]), dev(d["mid_V"]))
    for r in range(wl.recent_blocks):
        cache.append_block(0, dev(d["recent_K"][:, r]), dev(d["recent_V"][:, r]),
                           dev(d["recent_Kc"][:, r]), dev(d["recent_Vc"][:, r]))
    return cache


def oracle_context(wl, d, sel):
    """The (K, V) partitions of batch-item-wise context, in context order.

    sel: [B, k] selected mid indices (by age).  Returns a list of (K, V)
    pairs, each [B, L, H, D] (the selected mid blocks gathered per item)."""
    B = wl.batch
    parts = []
    if wl.sink_blocks:
        sK = d["sink_K"].reshape(B, -1, wl.heads, wl.head_dim)
        sV = d["sink_V"].reshape(B, -1, wl.heads, wl.head_dim)
        parts.append((sK, sV))
    if sel is not None and sel.shape[1]:
        idx = torch.as_tensor(np.asarray(sel))
        mK = torch.stack([d["mid_K"][b, idx[b]].reshape(-1, wl.heads, wl.head_dim) for b in range(B)])
        mV = torch.stack([d["mid_V"][b, idx[b]].reshape(-1, wl.heads, wl.head_dim) for b in range(B)])
        parts.append((mK, mV))
    if wl.recent_blocks:
        parts.append((d["recent_K"].reshape(B, -1, wl.heads, wl.head_dim),
                      d["recent_V"].reshape(B, -1, wl.heads, wl.head_dim)))
    parts.append((d["K_cur"], d["V_cur"]))
    return parts


def assert_attention_close(O_gpu, O_ref, what=""):
    o = oracle.to_f64(O_gpu)
    err = np.abs(o - O_ref)
    rel = np.linalg.norm(o - O_ref) / np.linalg.norm(O_ref)
    assert np.all(np.isfinite(o)), f"{what}: non-finite output"
    assert err.max() <= ATT_MAX_ABS, f"{what}: max abs err {err.max():.3e}"
    assert rel <= ATT_REL_L2, f"{what}: rel L2 err {rel:.3e}"
    return float(err.max()), float(rel)


def assert_keys_close(K_gpu, K_ref_f64, what=""):
    """Shifted keys: within 1e-2 or one bf16 ulp of the oracle rounded to bf16."""
    g = oracle.to_f64(K_gpu)
    r = oracle.round_bf16(K_ref_f64)
    ulp = np.ldexp(1.0, np.frexp(np.abs(r))[1] - 8)      # bf16 spacing at |r|
    tol = np.maximum(KEY_MAX_ABS, ulp)
    bad = np.abs(g - r) > tol
    assert not bad.any(), f"{what}: {bad.sum()} keys off, worst {np.abs(g - r).max():.3e}"
    return int((np.abs(g - r) > KEY_MAX_ABS).sum())


def arena_view(cache, ptr: int, shape, dtype=torch.bfloat16):
    """A tensor view of cache memory at device address ptr."""
    base = cache.arena.data_ptr()
    off = ptr - base
    n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
    return cache.arena[off:off + n].view(dtype).view(*shape)
