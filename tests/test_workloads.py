"""The seeded synthetic workloads match the configurations they stand for,
and the same seed gives the same inputs (every input of the tests and the
benchmark comes from here; nothing here does quantization or attention)."""
import math

import numpy as np
import pytest
import torch

from fp8_kv_paged_kvq_b200 import workloads as W


@pytest.mark.parametrize("name", ["tiny", "gqa", "ragged", "wide"])
def test_same_seed_same_inputs(name):
    a = W.make_workload(W.spec_by_name(name), seed=7)
    b = W.make_workload(W.spec_by_name(name), seed=7)
    for f in ("seq_lens", "block_table", "page_tags", "expected_tags", "free_pages",
              "hist_slots", "new_slots"):
        assert np.array_equal(getattr(a, f), getattr(b, f)), f
    assert torch.equal(a.q(), b.q())
    ka, va, _ = a.new_tokens()
    kb, vb, _ = b.new_tokens()
    assert torch.equal(ka, kb) and (va is None or torch.equal(va, vb))
    c = W.make_workload(W.spec_by_name(name), seed=8)
    assert not np.array_equal(a.page_tags, c.page_tags)


def _pages_are_a_layout(wl):
    ps = wl.spec.page_size
    n = (wl.seq_lens.astype(np.int64) + ps - 1) // ps
    used = np.concatenate([wl.block_table[b, : n[b]] for b in range(wl.B)])
    assert len(set(used.tolist())) == used.size                       # no page twice
    assert not set(used.tolist()) & set(wl.free_pages.tolist())
    assert used.size + wl.free_pages.size == wl.num_pages             # a permutation of the pool
    assert ((used >= 0) & (used < wl.num_pages)).all()
    return used.size


def test_gqa_batch_configuration():
    wl = W.make_workload(W.spec_by_name("gqa"), seed=0)
    s = wl.spec
    assert (s.B, s.page_size, s.num_q_heads, s.num_kv_heads, s.head_dim_k) == (32, 16, 64, 8, 128)
    assert (wl.seq_lens == 8192).all()
    need = _pages_are_a_layout(wl)
    assert wl.num_pages == math.ceil(1.2 * need)                      # 20% oversized pool
    assert np.array_equal(wl.expected_tags[:, :512], wl.page_tags[wl.block_table[:, :512]])
    k, v, _ = next(wl.hist_chunks(1 << 14))                            # values N(0,1), 1% x8
    x = k.float().abs()
    frac = float((x > 6.0).float().mean())
    assert 0.004 < frac < 0.012                                        # ~1% x8 outliers pass 6
    assert abs(float(wl.q().float().std()) - 1.0) < 0.02


def test_ragged_lengths_log_uniform():
    wl = W.make_workload(W.spec_by_name("ragged"), seed=0)
    L = wl.seq_lens.astype(np.float64)
    assert wl.B == 64 and L.min() >= 1024 and L.max() <= 32768
    u = (np.log(L) - math.log(1024)) / (math.log(32768) - math.log(1024))
    assert 0.35 < u.mean() < 0.65                                      # roughly uniform in log
    _pages_are_a_layout(wl)


def test_wide_and_tiny_configuration():
    w = W.make_workload(W.spec_by_name("wide"), seed=0)
    s = w.spec
    assert (s.B, s.page_size, s.num_q_heads, s.num_kv_heads, s.head_dim_k, s.head_dim_v) == \
        (64, 64, 128, 1, 576, 512)
    assert s.v_alias and s.scale_mode == W.SCALE_TOKEN and (w.seq_lens == 16384).all()
    _pages_are_a_layout(w)
    t = W.make_workload(W.spec_by_name("tiny"), seed=0)
    assert t.seq_lens.tolist() == [37, 100] and t.num_pages == 16 and len(t.stale) == 1
    b, i = t.stale[0]
    assert t.expected_tags[b, i] != t.page_tags[t.block_table[b, i]]    # the one stale entry
    assert t.sm_scale == 1.0 / 8.0
