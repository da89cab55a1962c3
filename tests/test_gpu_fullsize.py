"""Full-size parity in the launch configuration bench.py times (default CTA
count, same kernels): every E4M3 code of the cache bit-exact against the
oracle's own quantization, abort masks bit-exact, and sampled output rows
(which the oracle computes one by one) within the decode tolerance.

The long workload runs its whole 1,000-step loop: every step's abort mask is
compared with the oracle's, whose expected tags come from the oracle's own
tag state (a page's tag right after the oracle's append reallocated it), not
from the library's host tracker; every output row is compared at three steps.
"""
import numpy as np
import pytest
import torch

import oracle
import fp8_kv_paged_kvq_b200 as kvq
from fp8_kv_paged_kvq_b200 import workloads as W
from fp8_kv_paged_kvq_b200.pipeline import NOCHECK, STALE, DecodeBatch, DecodeLoop
from tests import oracle_side as OS
from tests.test_gpu_parity import assert_decode_close

pytestmark = pytest.mark.gpu


def sample_rows(wl, n, seed):
    r = np.random.default_rng(seed)
    s = wl.spec
    rows = set()
    # first and last query head of the first and last sequences, plus random rows
    for b in (0, s.B - 1):
        rows.update({b * s.num_q_heads, b * s.num_q_heads + s.num_q_heads - 1})
    while len(rows) < n:
        rows.add(int(r.integers(0, s.B * s.num_q_heads)))
    return np.array(sorted(rows), np.int32)


def compare_cache(db, oc):
    c = db.cache
    if c.fp8:
        assert np.array_equal(c.k_pages.cpu().numpy(), oc.k_pages)
        if oc.v_pages is not None:
            assert np.array_equal(c.v_pages.cpu().numpy(), oc.v_pages)
        assert np.array_equal(c.k_scale.cpu().numpy(), oc.k_scale)
        if oc.v_scale is not None:
            assert np.array_equal(c.v_scale.cpu().numpy(), oc.v_scale)
    else:
        assert np.array_equal(c.k_pages.cpu().view(torch.int16).numpy().view(np.uint16), oc.k_pages)
        assert np.array_equal(c.v_pages.cpu().view(torch.int16).numpy().view(np.uint16), oc.v_pages)
    assert np.array_equal(c.page_tags.cpu().numpy().view(np.uint32), oc.page_tags)


@pytest.mark.parametrize("name,kv", [("gqa", W.FP8), ("ragged", W.FP8), ("ragged", W.BF16),
                                     ("wide", W.FP8)])
def test_full_size_step(name, kv):
    spec = W.spec_by_name(name)
    spec.kv_dtype = kv
    wl = W.make_workload(spec, seed=0, device="cuda")
    db = DecodeBatch(wl)
    if db.cache.fp8:
        db.cache.k_pages.fill_(0xCD)
        if db.cache.v_pages is not None:
            db.cache.v_pages.fill_(0xCD)
    db.prefill()
    out, lse = db.step(check_tags=True)
    torch.cuda.synchronize()
    oc = OS.new_cache(wl)
    OS.fill(wl, oc)
    compare_cache(db, oc)
    mask = oracle.validate(oc.page_tags, wl.block_table, wl.expected_tags, wl.seq_lens,
                           spec.page_size)
    assert np.array_equal(db.abort.cpu().numpy(), mask)
    rows = sample_rows(wl, 24, seed=1)
    ro, rl = OS.decode(wl, oc, abort=mask, rows=rows)
    o = out.reshape(-1, spec.head_dim_v)[torch.from_numpy(rows).long().cuda()]
    l = lse.reshape(-1)[torch.from_numpy(rows).long().cuda()]
    assert_decode_close(o, l, ro, rl, f"{name}/{kv}")
    assert kvq.device_error() == 0


def test_wide_whole_sequences_all_heads():
    """The wide batch in the launch configuration bench.py times: every query
    head of four whole sequences, the first and last of the batch among them,
    so that the first and last pieces of the split are covered."""
    spec = W.spec_by_name("wide")
    wl = W.make_workload(spec, seed=0, device="cuda")
    db = DecodeBatch(wl)
    db.prefill()
    out, lse = db.step(check_tags=True)
    torch.cuda.synchronize()
    oc = OS.new_cache(wl)
    OS.fill(wl, oc)
    mask = oracle.validate(oc.page_tags, wl.block_table, wl.expected_tags, wl.seq_lens,
                           spec.page_size)
    assert np.array_equal(db.abort.cpu().numpy(), mask)
    seqs = (0, 1, 31, spec.B - 1)
    rows = np.array([b * spec.num_q_heads + h for b in seqs for h in range(spec.num_q_heads)],
                    np.int32)
    ro, rl = OS.decode(wl, oc, abort=mask, rows=rows)
    ri = torch.from_numpy(rows).long().cuda()
    assert_decode_close(out.reshape(-1, spec.head_dim_v)[ri], lse.reshape(-1)[ri], ro, rl,
                        "wide whole sequences")
    assert kvq.device_error() == 0


def test_long_loop_1000_steps():
    """The 1,000-step loop as bench.py runs it (one CUDA graph per step over
    inputs laid out on the device).  Even steps check the tags with stale
    entries injected, odd steps skip the check.  Every step's abort mask is
    compared with the oracle's; every output row (all 64 sequences x 64
    query heads) is compared at steps 0, 1 and 999; the final tags, block
    tables and codes of the whole cache are compared at the end."""
    spec = W.spec_by_name("long")
    steps = 1000
    wl = W.make_workload(spec, seed=0, device="cuda")
    loop = DecodeLoop(wl, steps)
    loop.batch.cache.k_pages.fill_(0xCD)      # same canary as the oracle's cache
    loop.batch.cache.v_pages.fill_(0xCD)
    loop.batch.prefill()
    torch.cuda.synchronize()
    loop.snapshot_tags()
    kinds = [STALE if i % 2 == 0 else NOCHECK for i in range(steps)]
    stream = torch.cuda.Stream()
    loop.capture(stream, kinds)
    # oracle side: its own cache, block table and expected tags
    oc = OS.new_cache(wl)
    hist = [(OS.bf16_bits(k), OS.bf16_bits(v), sl) for k, v, sl in wl.hist_chunks()]
    oc.k_scale[:] = oracle.scales(np.concatenate([h[0] for h in hist]), True)
    oc.v_scale[:] = oracle.scales(np.concatenate([h[1] for h in hist]), True)
    for k, v, sl in hist:
        oracle.append(oc, k, v, sl)
    del hist
    cap = W.loop_capacity(wl, steps)
    obt = np.full((spec.B, cap), -1, np.int32)
    obt[:, : wl.max_pages] = wl.block_table
    oexp = np.zeros((spec.B, cap), np.uint32)
    oexp[:, : wl.max_pages] = np.where(wl.block_table >= 0,
                                       oc.page_tags[np.maximum(wl.block_table, 0)], 0)
    check_steps = {0, 1, steps - 1}
    q = OS.bf16_bits(wl.q())
    n_aborts = 0
    for ls in W.loop_steps(wl, steps):
        chk = kinds[ls.step] == STALE
        loop.replay_step(ls.step, stream)
        torch.cuda.synchronize()
        # oracle step
        k, v = W.loop_tokens(wl, ls.step)
        pages = [p for _, _, p in ls.new_pages]
        oracle.append(oc, OS.bf16_bits(k), OS.bf16_bits(v), ls.slots,
                      realloc_pages=np.array(pages, np.int32) if pages else None)
        for b, i, p in ls.new_pages:
            obt[b, i] = p
            oexp[b, i] = oc.page_tags[p]
        m = None
        if chk:
            e = oexp.copy()
            for b, i in ls.stale:
                e[b, i] ^= np.uint32(1)
            m = oracle.validate(oc.page_tags, obt, e, ls.seq_lens, spec.page_size)
            got = loop.batch.abort.cpu().numpy()
            assert np.array_equal(got, m), ls.step
            assert set(np.nonzero(m)[0].tolist()) == {b for b, _ in ls.stale}
            n_aborts += int(m.sum())
        if ls.step in check_steps:
            ro, rl = oracle.decode(oc, q, obt, ls.seq_lens, m, wl.sm_scale)
            assert_decode_close(loop.batch.out.reshape(-1, spec.head_dim_v),
                                loop.batch.lse.reshape(-1), ro, rl, f"step {ls.step}")
    assert n_aborts > 0
    assert np.array_equal(loop.batch.cache.page_tags.cpu().numpy().view(np.uint32), oc.page_tags)
    assert np.array_equal(loop.final_tags(), oc.page_tags)
    assert np.array_equal(loop.tracker.block_table, obt)
    assert np.array_equal(loop.tracker.expected, oexp)
    assert np.array_equal(loop.batch.cache.k_pages.cpu().numpy(), oc.k_pages)
    assert np.array_equal(loop.batch.cache.v_pages.cpu().numpy(), oc.v_pages)
    assert kvq.device_error() == 0
