"""A decode batch driven end to end through libkvq: cache set-up, pre-fill,
and the per-step hot path (append the new token -> validate tags -> decode).

Only library calls touch the data; torch provides device memory and streams.
"""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch

from . import (BF16, FP8_E4M3, SCALE_HEAD, SCALE_TENSOR, SCALE_TOKEN, PagedCache, alloc_workspace,
               amax, append, decode, scale_from_amax, validate)
from . import workloads as W

_MODE = {W.SCALE_TENSOR: SCALE_TENSOR, W.SCALE_HEAD: SCALE_HEAD, W.SCALE_TOKEN: SCALE_TOKEN}


def _dev_i32(a: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int32)).to(device)


class DecodeBatch:
    """Device state of one decode batch built from a seeded workload."""

    def __init__(self, wl: W.Workload, device="cuda", num_ctas: int = 0,
                 kv_dtype: Optional[str] = None):
        s = wl.spec
        self.wl = wl
        self.device = torch.device(device)
        dt = kv_dtype or s.kv_dtype
        self.cache = PagedCache(FP8_E4M3 if dt == W.FP8 else BF16, _MODE[s.scale_mode],
                                wl.num_pages, s.page_size, s.num_kv_heads, s.head_dim_k,
                                s.head_dim_v, v_alias=s.v_alias, device=self.device,
                                tags=_dev_i32(wl.page_tags, "cpu"))
        self.q = wl.q().to(self.device)
        self.block_table = _dev_i32(wl.block_table, self.device)
        self.seq_lens = _dev_i32(wl.seq_lens, self.device)
        self.expected = _dev_i32(wl.expected_tags, self.device)
        self.abort = torch.zeros(s.B, dtype=torch.uint8, device=self.device)
        self.out = torch.empty((s.B, s.num_q_heads, s.head_dim_v), dtype=torch.float32,
                               device=self.device)
        self.lse = torch.empty((s.B, s.num_q_heads), dtype=torch.float32, device=self.device)
        self.num_ctas = num_ctas
        self.workspace = alloc_workspace(self.cache, s.B, s.num_q_heads, num_ctas, self.device)
        kn, vn, slots = wl.new_tokens()
        self.k_new = kn.to(self.device)
        self.v_new = None if vn is None else vn.to(self.device)
        self.new_slots = _dev_i32(slots, self.device)

    # -- pre-fill --------------------------------------------------------------
    def prefill(self, chunk_tokens: Optional[int] = None) -> None:
        """Scales from the pre-filled tokens (per tensor / per head), then bulk append."""
        s = self.wl.spec
        c = self.cache
        if c.fp8 and s.scale_mode != W.SCALE_TOKEN:
            per_head = s.scale_mode == W.SCALE_HEAD
            n = s.num_kv_heads if per_head else 1
            ak = torch.zeros(n, dtype=torch.float32, device=self.device)
            av = torch.zeros(n, dtype=torch.float32, device=self.device)
            for k, v, _ in self.wl.hist_chunks(chunk_tokens):
                amax(k.to(self.device), per_head, ak)
                if v is not None:
                    amax(v.to(self.device), per_head, av)
            scale_from_amax(ak, out=c.k_scale)
            if c.v_scale is not None:
                scale_from_amax(av, out=c.v_scale)
        for k, v, slots in self.wl.hist_chunks(chunk_tokens):
            append(c, k.to(self.device), None if v is None else v.to(self.device),
                   _dev_i32(slots, self.device))

    # -- the hot path of one decode step ----------------------------------------
    def append_new(self, realloc_pages: Optional[torch.Tensor] = None, stream=None) -> None:
        append(self.cache, self.k_new, self.v_new, self.new_slots, realloc_pages, stream)

    def validate(self, stream=None) -> torch.Tensor:
        return validate(self.cache.page_tags, self.block_table, self.expected, self.seq_lens,
                        self.cache.page_size, self.abort, stream)

    def decode(self, use_abort: bool = True, stream=None):
        return decode(self.cache, self.q, self.block_table, self.seq_lens,
                      self.abort if use_abort else None, self.wl.sm_scale, self.out, self.lse,
                      self.workspace, self.num_ctas, stream)

    def step(self, check_tags: bool = True, stream=None):
        self.append_new(stream=stream)
        if check_tags:
            self.validate(stream)
        return self.decode(use_abort=check_tags, stream=stream)

    def capture_io_step(self, host_in: dict, host_out: dict, stream,
                        check_tags: bool = True) -> torch.cuda.CUDAGraph:
        """One step with its host traffic as a CUDA graph.  host_in maps input
        names (q, k_new, v_new, new_slots, seq_lens, block_table, expected) to
        pinned host tensors copied in first; host_out maps out, lse and abort to
        pinned host tensors filled last.  Every replay moves the host buffers'
        current contents, so a caller refills host_in and replays."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for name, h in host_in.items():
                getattr(self, name).copy_(h, non_blocking=True)
            self.step(check_tags, stream=stream)
            for name, h in host_out.items():
                h.copy_(getattr(self, name), non_blocking=True)
        return g

    IO_IN = ("q", "k_new", "v_new", "new_slots", "seq_lens", "block_table", "expected")
    IO_OUT = ("out", "lse", "abort")

    def capture_io_pipelined(self, host_in: list, host_out: list, stream):
        """Two CUDA graphs, replayed alternately, that keep a stream of steps
        and their host traffic overlapped.  host_in / host_out are two dicts
        each (pinned host tensors keyed by the names in IO_IN / IO_OUT), one per
        device buffer set.  Graph k runs a step on buffer set k while side
        streams copy host_in[1-k] into set 1-k (the next step's inputs) and set
        1-k's results into host_out[1-k] (the previous step's).  Every replay
        thus moves one step's inputs and one step's results across the link."""
        sets = [{n: getattr(self, n) for n in self.IO_IN + self.IO_OUT
                 if getattr(self, n) is not None}]
        sets.append({n: t.clone() for n, t in sets[0].items()})
        side_in, side_out = torch.cuda.Stream(self.device), torch.cuda.Stream(self.device)
        graphs = []
        for k in (0, 1):
            o = 1 - k
            for n, t in sets[k].items():
                setattr(self, n, t)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                fork = torch.cuda.Event()
                fork.record(stream)
                side_in.wait_event(fork)
                side_out.wait_event(fork)
                with torch.cuda.stream(side_in):
                    for n, h in host_in[o].items():
                        sets[o][n].copy_(h, non_blocking=True)
                with torch.cuda.stream(side_out):
                    for n, h in host_out[o].items():
                        h.copy_(sets[o][n], non_blocking=True)
                self.step(True, stream=stream)
                for side in (side_in, side_out):
                    join = torch.cuda.Event()
                    join.record(side)
                    stream.wait_event(join)
            graphs.append(g)
        for n, t in sets[0].items():
            setattr(self, n, t)
        return graphs


STALE, CLEAN, NOCHECK = "stale", "clean", "nocheck"


class DecodeLoop:
    """The long decode loop, with every step's inputs resident in device memory.

    Step s appends one token per sequence (a token that opens a page takes a
    page from the free list, a reallocation whose tag kvq_append bumps),
    checks the requests' expected (page, tag) pairs and decodes.  A step is
    one of three kinds:
      STALE    the check runs with some expected tags made stale for that step
               (those requests abort);
      CLEAN    the check runs and every expected tag is right;
      NOCHECK  the check is skipped (decode ignores the abort mask).
    All steps' inputs (new K/V, slots, sequence lengths, reallocated pages)
    are laid out on the device up front, and the block table and expected
    tags hold every entry the loop will hand out: an entry is read only once
    the sequence has grown into it.  Each step is then a CUDA graph of the
    library calls on its own slice of those inputs, so a pass over the loop
    is a row of graph replays that the host queues without waiting.  A pass
    starts by putting the live tags back to their values before the loop, so
    every pass repeats the same tag history.
    """

    def __init__(self, wl: W.Workload, steps: int, device="cuda", num_ctas: int = 0):
        from .paging import TagTracker
        s = wl.spec
        self.wl, self.steps = wl, steps
        self.device = torch.device(device)
        cap = W.loop_capacity(wl, steps)
        self.cap = cap
        self.plan = list(W.loop_steps(wl, steps))
        # the host tracker hands out every page the loop will hand out: its
        # block table and expected tags are then the loop's final ones
        self.tracker = TagTracker(wl.page_tags, wl.block_table, wl.seq_lens, s.page_size, cap)
        for ls in self.plan:
            for b, i, page in ls.new_pages:
                self.tracker.hand_out(b, i, page)
        self.batch = DecodeBatch(wl, device=device, num_ctas=num_ctas)
        db = self.batch
        db.block_table = _dev_i32(self.tracker.block_table, self.device)
        db.expected = _dev_i32(self.tracker.expected, self.device)
        B = s.B
        rl = np.full((steps, B), -1, np.int32)
        for ls in self.plan:
            pages = [p for _, _, p in ls.new_pages]
            rl[ls.step, : len(pages)] = pages
        self.realloc = _dev_i32(rl, self.device)
        self.seq_lens = _dev_i32(np.stack([ls.seq_lens for ls in self.plan]), self.device)
        self.slots = _dev_i32(np.stack([ls.slots for ls in self.plan]), self.device)
        ks, vs = zip(*(W.loop_tokens(wl, st) for st in range(steps)))
        self.k_new = torch.stack([k.to(self.device) for k in ks]).contiguous()
        self.v_new = None if vs[0] is None else torch.stack([v.to(self.device) for v in vs]).contiguous()
        # stale entries of each step: flat index, corrupted and true expected tag
        exp_flat = self.tracker.expected.reshape(-1)
        self.stale = []
        for ls in self.plan:
            if not ls.stale:
                self.stale.append(None)
                continue
            idx = np.array([b * cap + i for b, i in ls.stale], np.int64)
            true = exp_flat[idx].copy()
            self.stale.append((torch.from_numpy(idx).to(self.device),
                               _dev_i32(true ^ np.uint32(1), self.device),
                               _dev_i32(true, self.device)))
        self.n_aborted = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.tags0 = None
        self.graphs = None

    def snapshot_tags(self) -> None:
        """Record the live tags that every pass starts from (call after pre-fill)."""
        self.tags0 = self.batch.cache.page_tags.clone()

    def final_tags(self) -> np.ndarray:
        """Live tags after one pass, as the host tracker expects them."""
        return self.tracker.tags

    # -- the three parts of step i --------------------------------------------
    def _append(self, i: int, kind: str, stream) -> None:
        db = self.batch
        if kind == STALE and self.stale[i] is not None:
            idx, bad, _ = self.stale[i]
            db.expected.view(-1).index_copy_(0, idx, bad)
        append(db.cache, self.k_new[i], None if self.v_new is None else self.v_new[i],
               self.slots[i], self.realloc[i], stream)

    def _validate(self, i: int, kind: str, stream) -> None:
        if kind == NOCHECK:
            return
        db = self.batch
        validate(db.cache.page_tags, db.block_table, db.expected, self.seq_lens[i],
                 db.cache.page_size, db.abort, stream, n_aborted=self.n_aborted)

    def _decode(self, i: int, kind: str, stream) -> None:
        db = self.batch
        decode(db.cache, db.q, db.block_table, self.seq_lens[i],
               None if kind == NOCHECK else db.abort, self.wl.sm_scale, db.out, db.lse,
               db.workspace, db.num_ctas, stream)
        if kind == STALE and self.stale[i] is not None:
            idx, _, true = self.stale[i]
            db.expected.view(-1).index_copy_(0, idx, true)

    def run_step_eager(self, i: int, kind: str, stream=None) -> None:
        self._append(i, kind, stream)
        self._validate(i, kind, stream)
        self._decode(i, kind, stream)

    def capture(self, stream, kinds, detailed=None) -> None:
        """Capture every step as CUDA graphs.  kinds[i]: STALE, CLEAN or
        NOCHECK.  detailed[i]: capture step i as three graphs (append,
        check, decode) so that events can be recorded between its calls;
        otherwise one graph, in which the calls overlap their launches."""
        assert self.tags0 is not None, "snapshot_tags() after pre-fill first"
        detailed = detailed or [False] * self.steps
        self.kinds, self.detailed = list(kinds), list(detailed)
        # first calls (per-device set-up) outside any capture
        with torch.cuda.stream(stream):
            self.run_step_eager(0, CLEAN, stream)
            self.run_step_eager(0, NOCHECK, stream)
            self.batch.cache.page_tags.copy_(self.tags0)
        torch.cuda.synchronize()
        graphs = []
        parts = (self._append, self._validate, self._decode)
        for i in range(self.steps):
            k = self.kinds[i]
            if self.detailed[i]:
                gs = []
                for part, f in enumerate(parts):
                    if part == 1 and k == NOCHECK:
                        gs.append(None)              # nothing to run between the events
                        continue
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g, stream=stream):
                        f(i, k, stream)
                    gs.append(g)
                graphs.append(gs)
            else:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    for f in parts:
                        f(i, k, stream)
                graphs.append([g])
        self.graphs = graphs

    def reset(self, stream) -> None:
        """Put the live tags back to their values before the loop."""
        with torch.cuda.stream(stream):
            self.batch.cache.page_tags.copy_(self.tags0)

    def replay_step(self, i: int, stream, events=None) -> None:
        """Queue step i.  events: None, or per graph of the step one event
        before it plus one after the last (2 events, or 4 for a detailed step)."""
        with torch.cuda.stream(stream):
            gs = self.graphs[i]
            for j, g in enumerate(gs):
                if events is not None:
                    events[j].record(stream)
                if g is not None:
                    g.replay()
            if events is not None:
                events[len(gs)].record(stream)

    def replay_pass(self, stream, events=None) -> None:
        """Queue one pass: the tag reset, then every step (events[i] per step)."""
        self.reset(stream)
        for i in range(self.steps):
            self.replay_step(i, stream, None if events is None else events[i])

    # -- the loop through the public API with host buffers ----------------------
    def io_setup(self, stream) -> dict:
        """Set up the end-to-end form of the loop: each step's inputs come from
        pinned host memory (query, new K/V, slots, sequence lengths, reallocated
        pages and the block-table / expected-tag entries they fill) and its
        results (out, lse, abort mask, abort count) go back to pinned host
        memory.  Two device buffer sets and two CUDA graphs alternate: graph k
        runs a step on set k while side streams copy the next step's inputs
        into set 1-k and the previous step's results out of set 1-k.  Returns
        the bytes each step moves each way."""
        s = self.wl.spec
        B, dev = s.B, self.device
        db = self.batch
        # host copies of every step's inputs
        self._h_k = self.k_new.cpu()
        self._h_v = None if self.v_new is None else self.v_new.cpu()
        self._h_q = db.q.cpu()
        self._h_lens = self.seq_lens.cpu()
        self._h_slots = self.slots.cpu()
        self._h_rl = self.realloc.cpu()
        # block-table / expected entries each step fills (padded with an
        # entry rewritten with its own value)
        didx = np.zeros((self.steps, B), np.int64)
        dpage = np.zeros((self.steps, B), np.int32)
        dtag = np.zeros((self.steps, B), np.int32)
        bt_f = self.tracker.block_table.reshape(-1)
        ex_f = self.tracker.expected.reshape(-1).view(np.int32)
        dpage[:] = bt_f[0]
        dtag[:] = ex_f[0]
        for ls in self.plan:
            for j, (b, i, page) in enumerate(ls.new_pages):
                didx[ls.step, j] = b * self.cap + i
                dpage[ls.step, j] = bt_f[b * self.cap + i]
                dtag[ls.step, j] = ex_f[b * self.cap + i]
        self._h_didx, self._h_dpage, self._h_dtag = (torch.from_numpy(didx),
                                                     torch.from_numpy(dpage),
                                                     torch.from_numpy(dtag))
        # tables before the loop: entries the loop hands out are not there yet
        bt0 = np.full((B, self.cap), -1, np.int32)
        ex0 = np.zeros((B, self.cap), np.uint32)
        bt0[:, : self.wl.max_pages] = self.wl.block_table
        n0 = (self.wl.seq_lens.astype(np.int64) + s.page_size - 1) // s.page_size
        for b in range(B):
            ex0[b, : n0[b]] = self.wl.page_tags[self.wl.block_table[b, : n0[b]]]
        self._bt0 = _dev_i32(bt0, dev)
        self._ex0 = _dev_i32(ex0, dev)
        self._bt_final = db.block_table.clone()
        self._ex_final = db.expected.clone()

        def dev_set():
            return {"q": torch.empty_like(db.q), "k": torch.empty_like(self.k_new[0]),
                    "v": None if self.v_new is None else torch.empty_like(self.v_new[0]),
                    "lens": torch.empty(B, dtype=torch.int32, device=dev),
                    "slots": torch.empty(B, dtype=torch.int32, device=dev),
                    "rl": torch.empty(B, dtype=torch.int32, device=dev),
                    "didx": torch.empty(B, dtype=torch.int64, device=dev),
                    "dpage": torch.empty(B, dtype=torch.int32, device=dev),
                    "dtag": torch.empty(B, dtype=torch.int32, device=dev),
                    "out": torch.empty_like(db.out), "lse": torch.empty_like(db.lse),
                    "abort": torch.empty_like(db.abort),
                    "nab": torch.zeros(1, dtype=torch.int32, device=dev)}
        IN = ("q", "k", "v", "lens", "slots", "rl", "didx", "dpage", "dtag")
        OUT = ("out", "lse", "abort", "nab")
        self._io_in, self._io_out = IN, OUT
        sets = [dev_set(), dev_set()]
        pin = lambda t: torch.empty(t.shape, dtype=t.dtype).pin_memory()
        self._h_in = [{n: pin(sets[0][n]) for n in IN if sets[0][n] is not None}
                      for _ in range(2)]
        self._h_out = [{n: pin(sets[0][n]) for n in OUT} for _ in range(2)]
        self._sets = sets
        side_in, side_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

        def body(S):
            bt, ex = db.block_table.view(-1), db.expected.view(-1)
            bt.index_copy_(0, S["didx"], S["dpage"])
            ex.index_copy_(0, S["didx"], S["dtag"])
            append(db.cache, S["k"], S["v"], S["slots"], S["rl"], stream)
            validate(db.cache.page_tags, db.block_table, db.expected, S["lens"],
                     db.cache.page_size, S["abort"], stream, n_aborted=S["nab"])
            decode(db.cache, S["q"], db.block_table, S["lens"], S["abort"], self.wl.sm_scale,
                   S["out"], S["lse"], db.workspace, db.num_ctas, stream)

        # warm the per-device set-up outside capture, then restore the tables
        self._fill_host(0, 0)
        with torch.cuda.stream(stream):
            for n, h in self._h_in[0].items():
                sets[0][n].copy_(h)
            body(sets[0])
            db.cache.page_tags.copy_(self.tags0)
            db.block_table.copy_(self._bt_final)
            db.expected.copy_(self._ex_final)
        torch.cuda.synchronize()
        graphs = []
        for k in (0, 1):
            o = 1 - k
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                fork = torch.cuda.Event()
                fork.record(stream)
                side_in.wait_event(fork)
                side_out.wait_event(fork)
                with torch.cuda.stream(side_in):
                    for n, h in self._h_in[o].items():
                        sets[o][n].copy_(h, non_blocking=True)
                with torch.cuda.stream(side_out):
                    for n, h in self._h_out[o].items():
                        h.copy_(sets[o][n], non_blocking=True)
                body(sets[k])
                for side in (side_in, side_out):
                    join = torch.cuda.Event()
                    join.record(side)
                    stream.wait_event(join)
            graphs.append(g)
        self._io_graphs = graphs
        h2d = sum(t.numel() * t.element_size() for t in self._h_in[0].values())
        d2h = sum(t.numel() * t.element_size() for t in self._h_out[0].values())
        return {"h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    def _fill_host(self, slot: int, i: int) -> None:
        h = self._h_in[slot]
        h["q"].copy_(self._h_q)
        h["k"].copy_(self._h_k[i])
        if "v" in h:
            h["v"].copy_(self._h_v[i])
        h["lens"].copy_(self._h_lens[i])
        h["slots"].copy_(self._h_slots[i])
        h["rl"].copy_(self._h_rl[i])
        h["didx"].copy_(self._h_didx[i])
        h["dpage"].copy_(self._h_dpage[i])
        h["dtag"].copy_(self._h_dtag[i])

    def io_pass(self, stream, steps: Optional[int] = None):
        """One pass of the loop with host traffic (every step CLEAN).  Returns
        (start event, end event, each step's abort count as read back)."""
        n = steps or self.steps
        db = self.batch
        sets, graphs = self._sets, self._io_graphs
        if not hasattr(self, "_h_last"):
            self._h_last = {nm: torch.empty(h.shape, dtype=h.dtype).pin_memory()
                            for nm, h in self._h_out[0].items()}
        done = [torch.cuda.Event(), torch.cuda.Event()]
        counts = [None] * n
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            db.cache.page_tags.copy_(self.tags0)
            db.block_table.copy_(self._bt0)
            db.expected.copy_(self._ex0)
            torch.cuda.synchronize()
            self._fill_host(0, 0)
            e0.record(stream)
            for nm, h in self._h_in[0].items():      # the first step's inputs
                sets[0][nm].copy_(h, non_blocking=True)
            done[1].record(stream)                   # host_in[0] is free once this is done
            for i in range(n):
                k, o = i % 2, 1 - i % 2
                # replay i-2 has finished: it read host_in[o] and wrote step
                # i-3's results to host_out[o], which replay i overwrites
                done[k].synchronize()
                if i >= 3:
                    counts[i - 3] = int(self._h_out[o]["nab"][0])
                if i + 1 < n:
                    self._fill_host(o, i + 1)
                graphs[k].replay()
                done[k].record(stream)
            last = sets[(n - 1) % 2]                 # the last step's results
            for nm, h in self._h_last.items():
                h.copy_(last[nm], non_blocking=True)
            e1.record(stream)
        torch.cuda.synchronize()
        if n >= 3:
            counts[n - 3] = int(self._h_out[(n - 1) % 2]["nab"][0])
        if n >= 2:
            counts[n - 2] = int(self._h_out[n % 2]["nab"][0])
        counts[n - 1] = int(self._h_last["nab"][0])
        db.block_table.copy_(self._bt_final)
        db.expected.copy_(self._ex_final)
        return e0, e1, counts
