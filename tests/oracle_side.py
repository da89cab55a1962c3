"""Oracle-side construction of a workload's cache (host numpy), for tests.

Mirrors what the CUDA path does to the same seeded inputs, but only through
oracle/: scales from the pre-filled BF16 tokens, bulk append, then the step's
new token.  Inputs generated on a GPU are copied to the host first; nothing
here reads a value the CUDA path computed.
"""
import numpy as np
import torch

import oracle
from fp8_kv_paged_kvq_b200 import workloads as W

MODE = {W.SCALE_TENSOR: oracle.SCALE_TENSOR, W.SCALE_HEAD: oracle.SCALE_HEAD,
        W.SCALE_TOKEN: oracle.SCALE_TOKEN}


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def new_cache(wl, kv_dtype=None, canary=0xCD):
    s = wl.spec
    dt = kv_dtype or s.kv_dtype
    P, ps, H = wl.num_pages, s.page_size, s.num_kv_heads
    if dt == W.FP8:
        kp = np.full((P, H, ps, s.head_dim_k), canary, np.uint8)
        vp = None if s.v_alias else np.full((P, H, ps, s.head_dim_v), canary, np.uint8)
    else:
        kp = np.zeros((P, H, ps, s.head_dim_k), np.uint16)
        vp = None if s.v_alias else np.zeros((P, H, ps, s.head_dim_v), np.uint16)
    if s.scale_mode == W.SCALE_TOKEN:
        ks = np.ones((P, H, ps), np.float32)
        vs = None if s.v_alias else np.ones((P, H, ps), np.float32)
    else:
        n = 1 if s.scale_mode == W.SCALE_TENSOR else H
        ks, vs = np.ones(n, np.float32), (None if s.v_alias else np.ones(n, np.float32))
    return oracle.Cache(oracle.FP8 if dt == W.FP8 else oracle.BF16, MODE[s.scale_mode], P, ps, H,
                        s.head_dim_k, s.head_dim_v, kp, vp, ks, vs, wl.page_tags.copy())


def fill(wl, cache, chunk_tokens=None):
    """Scales + pre-fill + the step's new token, all through the oracle."""
    s = wl.spec
    hist = [(bf16_bits(k), None if v is None else bf16_bits(v), sl)
            for k, v, sl in wl.hist_chunks(chunk_tokens)]
    if cache.dtype == oracle.FP8 and s.scale_mode != W.SCALE_TOKEN and hist:
        per_head = s.scale_mode == W.SCALE_HEAD
        cache.k_scale[:] = oracle.scales(np.concatenate([h[0] for h in hist]), per_head)
        if cache.v_scale is not None:
            cache.v_scale[:] = oracle.scales(np.concatenate([h[1] for h in hist]), per_head)
    for k, v, slots in hist:
        oracle.append(cache, k, v, slots)
    kn, vn, slots = wl.new_tokens()
    oracle.append(cache, bf16_bits(kn), None if vn is None else bf16_bits(vn), slots)


def decode(wl, cache, abort=None, rows=None):
    return oracle.decode(cache, bf16_bits(wl.q()), wl.block_table, wl.seq_lens, abort,
                         wl.sm_scale, rows=rows)
