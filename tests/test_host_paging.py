"""Host-side page bookkeeping of the long decode loop, checked on the CPU: the
free-list allocator of workloads.loop_steps and the tracker holding each
request's expected (page, tag) pairs (paging.TagTracker).  Tags are
generation counters that kvq_append bumps by one for every reallocated page
("Cloudflare: Kleinere Modellbereitstellung senkt Speicherbedarf, doch
Sicherheit wird zum Prüfstein" (remio.ai), section "Sicherheit gemeinsamer
KV-Caches wird zum Produktionsthema"); the tracker's expectations are checked
with the oracle's validation after that bump is mirrored on a host copy of
the live tags."""
import math

import numpy as np
import pytest

import oracle
from fp8_kv_paged_kvq_b200 import workloads as W
from fp8_kv_paged_kvq_b200.paging import TagTracker


@pytest.fixture(scope="module")
def long_wl():
    return W.make_workload(W.spec_by_name("long"), seed=0, device="cpu")


def test_loop_allocator_invariants(long_wl):
    wl = long_wl
    s, ps = wl.spec, wl.spec.page_size
    npages = (wl.seq_lens.astype(np.int64) + ps - 1) // ps
    owner = {}
    for b in range(s.B):
        for i in range(npages[b]):
            p = int(wl.block_table[b, i])
            assert p not in owner                      # no page held twice
            owner[p] = (b, i)
    free = set(int(p) for p in wl.free_pages)
    assert not free & set(owner)
    bt = {b: [int(p) for p in wl.block_table[b, : npages[b]]] for b in range(s.B)}
    for ls in W.loop_steps(wl, 1000):
        live = wl.seq_lens > 0
        assert np.array_equal(ls.seq_lens[live], wl.seq_lens[live] + ls.step)
        for b, i, page in ls.new_pages:
            assert page in free and page not in owner  # handed out from the free list only
            free.remove(page)
            owner[page] = (b, i)
            assert i == len(bt[b])                     # the next entry of that request
            bt[b].append(page)
        pos = wl.seq_lens.astype(np.int64) - 1 + ls.step
        for b in np.nonzero(live)[0]:
            slot = int(ls.slots[b])
            assert slot // ps == bt[b][pos[b] // ps] and slot % ps == pos[b] % ps
        ent = (ls.seq_lens.astype(np.int64) + ps - 1) // ps
        assert all(len(bt[b]) >= ent[b] for b in range(s.B))
        assert len(ls.stale) == math.ceil(s.stale_frac * ent.sum())
        assert len(set(ls.stale)) == len(ls.stale)
        assert all(0 <= i < ent[b] for b, i in ls.stale)


def test_tracker_expectations_pass_and_stale_entries_abort(long_wl):
    wl = long_wl
    s, ps = wl.spec, wl.spec.page_size
    steps = 200
    live = wl.page_tags.astype(np.uint32).copy()
    tr = TagTracker(live, wl.block_table, wl.seq_lens, ps, W.loop_capacity(wl, steps))
    for ls in W.loop_steps(wl, steps):
        for b, i, page in ls.new_pages:
            tr.hand_out(b, i, page)
            live[page] = np.uint32((int(live[page]) + 1) & 0xFFFFFFFF)   # kvq_append's bump
        assert np.array_equal(tr.tags, live)
        if ls.step % 25:
            continue
        mask = oracle.validate(live, tr.block_table, tr.expected, ls.seq_lens, ps)
        assert not mask.any()
        exp = tr.expected.copy()
        for b, i in ls.stale:
            exp[b, i] ^= 1
        want = np.zeros(s.B, np.uint8)
        want[[b for b, _ in ls.stale]] = 1
        assert np.array_equal(oracle.validate(live, tr.block_table, exp, ls.seq_lens, ps), want)


def test_page_handed_to_another_request_leaves_the_old_holder_stale():
    ps = 16
    live = np.array([7, 7, 7, 7], np.uint32)
    bt = np.array([[0, 1], [2, 3]], np.int32)
    lens = np.array([32, 17], np.int32)
    tr = TagTracker(live, bt, lens, ps, capacity=3)
    assert not oracle.validate(live, tr.block_table, tr.expected, lens, ps).any()
    # page 1 goes to request 1 as its third page; request 0 still lists it
    tr.hand_out(1, 2, 1)
    live[1] += 1
    lens2 = np.array([32, 33], np.int32)
    mask = oracle.validate(live, tr.block_table, tr.expected, lens2, ps)
    assert mask.tolist() == [1, 0]
