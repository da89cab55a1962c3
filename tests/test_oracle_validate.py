"""Pins of the oracle's tag bump and batched validation: brute force and the
injected-stale-tag property (exactly the requests holding a stale entry abort)."""
import numpy as np
import pytest

import oracle
from fp8_kv_paged_kvq_b200 import workloads as W


def brute_validate(tags, bt, exp, lens, ps):
    B, maxp = bt.shape
    out = []
    for b in range(B):
        n = min(max(int(lens[b]), 0), maxp * ps)
        bad = False
        for i in range(-(-n // ps)):
            p = int(bt[b, i])
            if not (0 <= p < tags.size) or int(tags[p]) != int(exp[b, i]):
                bad = True
        out.append(int(bad))
    return np.array(out, np.uint8)


@pytest.mark.parametrize("name", ["tiny", "ragged5", "long"])
def test_stale_injection_aborts_exactly_the_affected_requests(name):
    if name == "ragged5":
        spec = W.spec_by_name("ragged")
        spec.n_stale = 5
    else:
        spec = W.spec_by_name(name)
    wl = W.make_workload(spec, seed=2)
    m = oracle.validate(wl.page_tags, wl.block_table, wl.expected_tags, wl.seq_lens,
                        wl.spec.page_size)
    want = np.zeros(wl.B, np.uint8)
    for b, _ in wl.stale:
        want[b] = 1
    assert wl.stale, "workload must inject at least one stale tag"
    assert np.array_equal(m, want)
    clean = oracle.validate(wl.page_tags, wl.block_table, wl.page_tags[np.maximum(wl.block_table, 0)],
                            wl.seq_lens, wl.spec.page_size)
    assert not clean.any()


def test_validate_matches_brute_force_random():
    r = np.random.default_rng(0)
    for trial in range(50):
        P, B, maxp, ps = int(r.integers(1, 40)), int(r.integers(1, 9)), int(r.integers(1, 7)), int(r.integers(1, 5))
        tags = r.integers(0, 4, P).astype(np.uint32)
        bt = r.integers(-2, P + 2, (B, maxp)).astype(np.int32)
        exp = r.integers(0, 4, (B, maxp)).astype(np.uint32)
        lens = r.integers(-3, maxp * ps + 5, B).astype(np.int32)
        got = oracle.validate(tags, bt, exp, lens, ps)
        assert np.array_equal(got, brute_validate(tags, bt, exp, lens, ps))


def test_first_bad_index_matches_brute_force():
    """Telemetry: the first failing block-table index of each request (-1 if none),
    against a direct scan in Python."""
    r = np.random.default_rng(7)
    for trial in range(50):
        P, B, maxp, ps = int(r.integers(1, 40)), int(r.integers(1, 9)), int(r.integers(1, 9)), int(r.integers(1, 5))
        tags = r.integers(0, 3, P).astype(np.uint32)
        bt = r.integers(-1, P + 1, (B, maxp)).astype(np.int32)
        exp = r.integers(0, 3, (B, maxp)).astype(np.uint32)
        lens = r.integers(-3, maxp * ps + 5, B).astype(np.int32)
        mask, first = oracle.validate(tags, bt, exp, lens, ps, first_bad=True)
        for b in range(B):
            n = min(max(int(lens[b]), 0), maxp * ps)
            want = -1
            for i in range(-(-n // ps)):
                p = int(bt[b, i])
                if not (0 <= p < P) or int(tags[p]) != int(exp[b, i]):
                    want = i
                    break
            assert first[b] == want and mask[b] == (want >= 0), (trial, b)


def test_entries_beyond_sequence_are_ignored():
    tags = np.arange(10, dtype=np.uint32)
    bt = np.array([[3, 4, 99]], np.int32)          # third entry is garbage
    exp = np.array([[3, 4, 0]], np.uint32)
    assert oracle.validate(tags, bt, exp, np.array([32], np.int32), 16)[0] == 0
    assert oracle.validate(tags, bt, exp, np.array([33], np.int32), 16)[0] == 1


def test_out_of_range_page_aborts():
    tags = np.zeros(4, np.uint32)
    for bad in (-1, 4, 1 << 30):
        bt = np.array([[0, bad]], np.int32)
        assert oracle.validate(tags, bt, np.zeros((1, 2), np.uint32), np.array([20], np.int32), 16)[0] == 1


def test_tag_bump_per_occurrence_with_wraparound():
    P, ps, H, D = 6, 4, 1, 16
    c = oracle.Cache(oracle.FP8, oracle.SCALE_TENSOR, P, ps, H, D, D,
                     np.zeros((P, H, ps, D), np.uint8), np.zeros((P, H, ps, D), np.uint8),
                     np.ones(1, np.float32), np.ones(1, np.float32),
                     np.array([0, 7, 0xFFFFFFFF, 5, 5, 5], np.uint32))
    oracle.append(c, np.zeros((0, H, D), np.uint16), np.zeros((0, H, D), np.uint16),
                  np.zeros(0, np.int32), realloc_pages=np.array([1, 2, 4, 4, -1, 6], np.int32))
    assert c.page_tags.tolist() == [0, 8, 0, 5, 7, 5]


def test_reallocated_page_fails_old_expectation():
    """A request still holding the pre-reallocation tag is aborted after the bump."""
    P, ps, H, D = 4, 4, 1, 8
    tags = np.array([10, 20, 30, 40], np.uint32)
    c = oracle.Cache(oracle.FP8, oracle.SCALE_TENSOR, P, ps, H, D, D,
                     np.zeros((P, H, ps, D), np.uint8), np.zeros((P, H, ps, D), np.uint8),
                     np.ones(1, np.float32), np.ones(1, np.float32), tags.copy())
    bt = np.array([[2, 1], [3, 0]], np.int32)
    exp_before = tags[bt]
    oracle.append(c, np.zeros((0, H, D), np.uint16), np.zeros((0, H, D), np.uint16),
                  np.zeros(0, np.int32), realloc_pages=np.array([1], np.int32))
    m = oracle.validate(c.page_tags, bt, exp_before, np.array([8, 8], np.int32), ps)
    assert m.tolist() == [1, 0]
