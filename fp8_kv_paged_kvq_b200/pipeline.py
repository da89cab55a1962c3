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


class DecodeLoop:
    """The long decode loop on the device.  Every step appends one token per
    sequence (pages handed out from the free list are reallocations whose tags
    kvq_append bumps), validates the tracker's expected tags with some entries
    made stale for that step (or skips the check), and decodes.

    The hot path of a step (kvq_append -> kvq_validate -> kvq_decode) is a CUDA
    graph over fixed device buffers, so its kernels run back to back; the
    realloc list is padded to B entries with -1 (skipped by kvq_append).
    Page-table bookkeeping for the step is written into those buffers first."""

    def __init__(self, wl: W.Workload, steps: int, device="cuda", num_ctas: int = 0):
        from .paging import TagTracker
        s = wl.spec
        self.wl, self.steps = wl, steps
        self.device = torch.device(device)
        cap = W.loop_capacity(wl, steps)
        self.cap = cap
        self.tracker = TagTracker(wl.page_tags, wl.block_table, wl.seq_lens, s.page_size, cap)
        self.batch = DecodeBatch(wl, device=device, num_ctas=num_ctas)
        db = self.batch
        db.block_table = _dev_i32(self.tracker.block_table, self.device)
        db.expected = _dev_i32(self.tracker.expected, self.device)
        self.realloc = torch.full((s.B,), -1, dtype=torch.int32, device=self.device)
        self.graphs = {}

    def _path(self, check_tags: bool, stream=None, ev=None):
        """One step.  ev: None, [start, end], or [start, before validate,
        before decode, end] (events between kernels also break the kernels'
        programmatic launch overlap, so the two-event form times the step)."""
        db = self.batch
        st = torch.cuda.current_stream() if stream is None else stream
        inner = ev is not None and len(ev) == 4
        if ev is not None:
            ev[0].record(st)
        append(db.cache, db.k_new, db.v_new, db.new_slots, self.realloc, stream)
        if inner:
            ev[1].record(st)
        if check_tags:
            db.validate(stream)
        if inner:
            ev[2].record(st)
        db.decode(use_abort=check_tags, stream=stream)
        if ev is not None:
            ev[-1].record(st)

    def capture(self, stream) -> None:
        """Capture the step's hot path, with and without the tag check, each
        twice: with timing events only around the step, and with events
        between append, validate and decode as well."""
        for chk in (True, False):
            self._path(chk, stream)          # warm up outside capture
            for n_ev in (2, 4):
                ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(n_ev)]
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    self._path(chk, stream, ev)
                self.graphs[(chk, n_ev == 4)] = (g, ev)

    def _flat(self, entries):
        return torch.tensor([b * self.cap + i for b, i in entries], dtype=torch.long,
                            device=self.device)

    def prepare(self, ls: W.LoopStep, check_tags: bool, inject_stale: bool = True):
        """Write the step's inputs into the fixed buffers; with check_tags and
        inject_stale, the step's stale entries are corrupted in the expected tags.
        Returns the stale-entry index (restore() undoes it after the step)."""
        db = self.batch
        pages, tags, entries = [], [], []
        for b, i, page in ls.new_pages:
            tags.append(self.tracker.hand_out(b, i, page))
            pages.append(page)
            entries.append((b, i))
        if entries:
            idx = self._flat(entries)
            db.block_table.view(-1)[idx] = torch.tensor(pages, dtype=torch.int32,
                                                        device=self.device)
            db.expected.view(-1)[idx] = torch.from_numpy(
                np.array(tags, np.uint32).view(np.int32)).to(self.device)
        rl = np.full(self.wl.spec.B, -1, np.int32)
        rl[: len(pages)] = pages
        self.realloc.copy_(torch.from_numpy(rl))
        db.seq_lens.copy_(torch.from_numpy(ls.seq_lens))
        db.new_slots.copy_(torch.from_numpy(ls.slots))
        k, v = W.loop_tokens(self.wl, ls.step)
        db.k_new.copy_(k)
        if v is not None:
            db.v_new.copy_(v)
        stale_idx = self._flat(ls.stale) if (check_tags and inject_stale and ls.stale) else None
        if stale_idx is not None:
            db.expected.view(-1)[stale_idx] ^= 1
        return stale_idx

    def restore(self, stale_idx) -> None:
        if stale_idx is not None:
            self.batch.expected.view(-1)[stale_idx] ^= 1

    def run(self, check_tags: bool, stream, detailed: bool = False):
        """Replay the step's graph.  Returns its events: (start, end), or with
        detailed=True (before append, before validate, before decode, after
        decode); they are reused by the next replay of the same graph, so read
        them after synchronizing and before replaying again."""
        g, ev = self.graphs[(check_tags, detailed)]
        g.replay()
        return ev
