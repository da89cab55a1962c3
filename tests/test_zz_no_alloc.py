"""kvq_decode_noalloc against kvq_decode.

kvq_decode_noalloc serves callers that cannot allocate device memory (a
plug-in whose host framework owns all device memory, a serving loop that
forbids allocation after start-up): its scratch is a fixed array inside the
library instead of a caller workspace.  This test calls it through the C ABI
twice in a row, on two different batches, and checks each result against the
allocating entry point on the same inputs, within the tolerance the parity
tests use (the two share their kernels, so the results are expected to be
identical).  A third call repeats the first batch after the second has left
its own contents in the shared array.  A batch too large for the array must
be refused with KVQ_ERR_WORKSPACE.

This file is named to be collected after every other test file.
"""
import ctypes

import numpy as np
import pytest
import torch

import fp8_kv_paged_kvq_b200 as kvq
from fp8_kv_paged_kvq_b200 import workloads as W
from fp8_kv_paged_kvq_b200.pipeline import DecodeBatch

pytestmark = pytest.mark.gpu

ATOL, RTOL, REL_FLOOR = 2e-3, 1e-2, 0.2


def _close(a, b):
    a = a.detach().cpu().double().numpy()
    b = b.detach().cpu().double().numpy()
    inf_a, inf_b = np.isneginf(a), np.isneginf(b)
    assert np.array_equal(inf_a, inf_b)
    fa = np.where(inf_a, 0.0, a)
    fb = np.where(inf_b, 0.0, b)
    d = np.abs(fa - fb)
    assert d.max(initial=0.0) <= ATOL
    big = np.abs(fb) >= REL_FLOOR
    if big.any():
        assert (d[big] / np.abs(fb[big])).max() <= RTOL


def _batch(spec, seed, num_ctas=0):
    wl = W.make_workload(spec, seed=seed, device="cuda")
    db = DecodeBatch(wl, num_ctas=num_ctas)
    db.prefill()
    db.append_new()
    db.validate()
    ref_out, ref_lse = [t.clone() for t in db.decode(use_abort=True)]
    return db, ref_out, ref_lse


def _noalloc(db, num_ctas=0):
    out = torch.full_like(db.out, float("nan"))
    lse = torch.full_like(db.lse, float("nan"))
    st = kvq.lib().kvq_decode_noalloc(
        ctypes.byref(db.cache.desc), ctypes.c_void_p(db.q.data_ptr()), db.q.shape[1],
        ctypes.c_void_p(db.block_table.data_ptr()), db.block_table.shape[1],
        ctypes.c_void_p(db.seq_lens.data_ptr()), db.q.shape[0],
        ctypes.c_void_p(db.abort.data_ptr()), ctypes.c_float(db.wl.sm_scale),
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()), num_ctas,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == kvq.KVQ_OK, kvq.lib().kvq_status_string(st)
    return out, lse


def test_noalloc_matches_allocating_decode_on_two_calls_in_a_row():
    spec_a = W.Spec("na_a", [1, 15, 16, 17, 300, 1000, 4097], 16, 16, 2, 128, 128,
                    outlier_p=0.01, n_stale=1)
    spec_b = W.Spec("na_b", [2000, 33, 700], 16, 64, 8, 128, 128)
    db_a, ra_out, ra_lse = _batch(spec_a, seed=21)
    db_b, rb_out, rb_lse = _batch(spec_b, seed=22)
    torch.cuda.synchronize()

    a_out, a_lse = _noalloc(db_a)      # two calls in a row, no host sync in between
    b_out, b_lse = _noalloc(db_b)
    torch.cuda.synchronize()
    _close(a_out, ra_out)
    _close(a_lse, ra_lse)
    _close(b_out, rb_out)
    _close(b_lse, rb_lse)
    assert torch.equal(a_out, ra_out) and torch.equal(b_out, rb_out)

    a2_out, a2_lse = _noalloc(db_a)    # the array now holds batch b's partials
    torch.cuda.synchronize()
    _close(a2_out, ra_out)
    _close(a2_lse, ra_lse)
    assert kvq.device_error() == 0


def test_noalloc_wide_group_matches_allocating_decode_on_two_calls_in_a_row():
    """The same check on the tensor-core shape (128 query heads on one KV
    head, K 576 / V the first 512 dims, per-token scales), whose workspace also
    holds the query images: two calls in a row on two batches.  Its partial
    outputs take 256 KB per CTA pair, so the batch runs on 8 pairs to fit
    the fixed array (the default pair count would be refused)."""
    pairs = 8
    spec_a = W.Spec("na_wide_a", [700, 65], 64, 128, 1, 576, 512, v_alias=True,
                    scale_mode=W.SCALE_TOKEN, n_stale=1)
    spec_b = W.Spec("na_wide_b", [1, 300, 129], 64, 128, 1, 576, 512, v_alias=True,
                    scale_mode=W.SCALE_TOKEN)
    db_a, ra_out, ra_lse = _batch(spec_a, seed=23, num_ctas=pairs)
    db_b, rb_out, rb_lse = _batch(spec_b, seed=24, num_ctas=pairs)
    assert kvq.decode_workspace_size(db_a.cache, 3, 128, pairs) <= (8 << 20)
    torch.cuda.synchronize()
    a_out, a_lse = _noalloc(db_a, pairs)
    b_out, b_lse = _noalloc(db_b, pairs)
    torch.cuda.synchronize()
    _close(a_out, ra_out)
    _close(a_lse, ra_lse)
    _close(b_out, rb_out)
    _close(b_lse, rb_lse)
    assert torch.equal(a_out, ra_out) and torch.equal(b_out, rb_out)
    assert kvq.device_error() == 0


def test_noalloc_rejects_a_batch_beyond_the_fixed_scratch():
    c = kvq.PagedCache(kvq.FP8_E4M3, kvq.SCALE_HEAD, 64, 16, 8, 128, 128)
    B, Hq = 4096, 128                      # workspace far above the 8 MiB array
    assert kvq.decode_workspace_size(c, B, Hq) > (8 << 20)
    q = torch.zeros((B, Hq, 128), dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros((B, 1), dtype=torch.int32, device="cuda")
    sl = torch.ones(B, dtype=torch.int32, device="cuda")
    out = torch.empty((B, Hq, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(kvq.KvqError) as e:
        kvq.decode_noalloc(c, q, bt, sl, None, 1.0, out, None)
    assert e.value.status == kvq.KVQ_ERR_WORKSPACE
