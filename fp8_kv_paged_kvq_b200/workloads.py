"""Seeded synthetic decode workloads.

This module only draws random inputs and lays out page tables; it holds none
of the method's arithmetic (no quantization, no scales, no attention, no tag
bump).  Both the CUDA path and the CPU oracle consume what it produces.

Shapes follow the five decode workloads the library is measured on:

  tiny    2 sequences (37 and 100 tokens), page 16, 4 query heads on 1 KV
          head, head_dim 64, per-tensor scales, 10 pages out of a
          16-page pool, one stale expected tag.
  gqa     32 x 8,192 tokens, page 16, 64 query / 8 KV heads, head_dim 128,
          per-head scales, K/V N(0,1) with 1% of elements x8, pool 20%
          larger than needed, pages in a random permutation.
  ragged  64 sequences, lengths log-uniform in [1,024, 32,768], otherwise as
          gqa; also run with a BF16 cache.
  wide    64 x 16,384 tokens, page 64, 128 query heads on 1 KV head,
          K dim 576, V = first 512 dims of K, one scale per token.
  long    4 x 262,144 + 60 x 8,192 tokens, otherwise as gqa; 1,000 decode
          steps with page reallocation and 0.01% stale expected tags.

Each decode step attends over exactly seq_len tokens; the token appended in
the step is the last of them, so the cache is pre-filled with seq_len - 1
tokens per sequence.
"""
from __future__ import annotations

import math
import zlib
from dataclasses import dataclass, field
from typing import Iterator, List, Optional, Sequence

import numpy as np
import torch

FP8, BF16 = "fp8", "bf16"
SCALE_TENSOR, SCALE_HEAD, SCALE_TOKEN = "tensor", "head", "token"


@dataclass
class Spec:
    name: str
    seq_lens: Sequence[int]
    page_size: int
    num_q_heads: int
    num_kv_heads: int
    head_dim_k: int
    head_dim_v: int
    v_alias: bool = False          # V is the first head_dim_v dims of K
    kv_dtype: str = FP8
    scale_mode: str = SCALE_HEAD
    pool_factor: float = 1.2       # pool pages / pages needed
    pool_pages: Optional[int] = None
    extra_pages: int = 0           # pages reserved for growth (decode loop)
    outlier_p: float = 0.0
    outlier_mult: float = 8.0
    n_stale: int = 0               # stale expected tags injected
    stale_frac: float = 0.0        # or: fraction of expected entries made stale
    sm_scale: Optional[float] = None

    @property
    def B(self) -> int:
        return len(self.seq_lens)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads


def _rng(seed: int, *tags) -> np.random.Generator:
    # zlib.crc32 rather than hash(): str hashes change from process to process
    return np.random.default_rng([seed, *[zlib.crc32(str(t).encode()) for t in tags]])


def log_uniform_lens(n: int, lo: int, hi: int, seed: int) -> List[int]:
    r = _rng(seed, "lens")
    return [int(x) for x in np.exp(r.uniform(math.log(lo), math.log(hi), size=n)).round()]


def spec_by_name(name: str, seed: int = 0) -> Spec:
    if name == "tiny":
        return Spec("tiny", [37, 100], 16, 4, 1, 64, 64, scale_mode=SCALE_TENSOR,
                    pool_pages=16, n_stale=1, sm_scale=1.0 / 8.0)
    if name == "gqa":
        return Spec("gqa", [8192] * 32, 16, 64, 8, 128, 128, outlier_p=0.01)
    if name == "ragged":
        return Spec("ragged", log_uniform_lens(64, 1024, 32768, seed + 3), 16, 64, 8, 128, 128)
    if name == "ragged_bf16":
        return Spec("ragged_bf16", log_uniform_lens(64, 1024, 32768, seed + 3), 16, 64, 8, 128,
                    128, kv_dtype=BF16)
    if name == "wide":
        return Spec("wide", [16384] * 64, 64, 128, 1, 576, 512, v_alias=True,
                    scale_mode=SCALE_TOKEN)
    if name == "long":
        return Spec("long", [262144] * 4 + [8192] * 60, 16, 64, 8, 128, 128,
                    pool_factor=1.0, extra_pages=8192, stale_frac=1e-4)
    raise KeyError(name)


@dataclass
class Workload:
    spec: Spec
    seed: int
    device: torch.device
    num_pages: int
    seq_lens: np.ndarray            # int32 [B]
    block_table: np.ndarray         # int32 [B][max_pages]
    page_tags: np.ndarray           # uint32 [P] live tags at the start
    expected_tags: np.ndarray       # uint32 [B][max_pages] (stale entries injected)
    stale: List[tuple]              # (b, i) entries made stale
    free_pages: np.ndarray          # int32 pool pages not in any block table
    hist_slots: np.ndarray          # int32 slots of the pre-filled tokens (logical order)
    new_slots: np.ndarray           # int32 [B] slot of the step's new token (-1: none)
    sm_scale: float
    _chunk_tokens: int = 1 << 20
    _q: Optional[torch.Tensor] = None
    _new: Optional[tuple] = None

    # -- dimensions --------------------------------------------------------
    @property
    def B(self):
        return self.spec.B

    @property
    def max_pages(self):
        return self.block_table.shape[1]

    @property
    def kv_row_bytes(self) -> int:
        """Bytes of one cached token row of one KV head (K + V, codes only)."""
        el = 1 if self.spec.kv_dtype == FP8 else 2
        s = self.spec
        return el * (s.head_dim_k + (0 if s.v_alias else s.head_dim_v))

    # -- random tensors (generated on self.device) ---------------------------
    def _normal(self, shape, *tags, outliers=True) -> torch.Tensor:
        g = torch.Generator(device=self.device)
        g.manual_seed(int(_rng(self.seed, *tags).integers(0, 2**62)))
        x = torch.randn(shape, generator=g, device=self.device, dtype=torch.float32)
        if outliers and self.spec.outlier_p > 0:
            m = torch.rand(shape, generator=g, device=self.device) < self.spec.outlier_p
            x = torch.where(m, x * self.spec.outlier_mult, x)
        return x.to(torch.bfloat16)

    def q(self) -> torch.Tensor:
        """Query of the decode step, bf16 [B][Hq][Dk], N(0,1)."""
        if self._q is None:
            s = self.spec
            self._q = self._normal((s.B, s.num_q_heads, s.head_dim_k), "q", outliers=False)
        return self._q

    def new_tokens(self):
        """(k_new [B][Hkv][Dk], v_new [B][Hkv][Dv] or None, slots [B]) of the step."""
        if self._new is None:
            s = self.spec
            k = self._normal((s.B, s.num_kv_heads, s.head_dim_k), "knew")
            v = None if s.v_alias else self._normal((s.B, s.num_kv_heads, s.head_dim_v), "vnew")
            self._new = (k, v, self.new_slots)
        return self._new

    def hist_chunks(self, chunk_tokens: Optional[int] = None) -> Iterator[tuple]:
        """Pre-filled cache contents, in chunks: (k [n][Hkv][Dk], v or None, slots [n])."""
        s = self.spec
        ct = chunk_tokens or self._chunk_tokens
        n = self.hist_slots.size
        for ci, lo in enumerate(range(0, n, ct)):
            hi = min(n, lo + ct)
            k = self._normal((hi - lo, s.num_kv_heads, s.head_dim_k), "khist", ci, ct)
            v = None if s.v_alias else self._normal((hi - lo, s.num_kv_heads, s.head_dim_v),
                                                     "vhist", ci, ct)
            yield k, v, self.hist_slots[lo:hi]

    # -- algorithmic sizes ---------------------------------------------------
    def kv_bytes_read(self) -> int:
        """Cache bytes one decode step reads (codes; + per-token scales in TOKEN mode)."""
        toks = int(self.seq_lens.astype(np.int64).sum())
        b = toks * self.spec.num_kv_heads * self.kv_row_bytes
        if self.spec.scale_mode == SCALE_TOKEN and self.spec.kv_dtype == FP8:
            b += toks * self.spec.num_kv_heads * 4
        return b


def make_workload(spec: Spec, seed: int = 0, device="cpu") -> Workload:
    """Lay out a seeded workload: page permutation, block tables, tags, stale entries."""
    device = torch.device(device)
    r = _rng(seed, spec.name, "layout")
    lens = np.asarray(spec.seq_lens, dtype=np.int32)
    ps = spec.page_size
    npages = (lens.astype(np.int64) + ps - 1) // ps
    need = int(npages.sum())
    if spec.pool_pages is not None:
        P = spec.pool_pages
    else:
        P = int(math.ceil(spec.pool_factor * need)) + spec.extra_pages
    assert P >= need, "pool too small"
    perm = r.permutation(P).astype(np.int32)
    max_pages = max(1, int(npages.max()) if lens.size else 1)
    bt = np.full((spec.B, max_pages), -1, dtype=np.int32)
    pos = 0
    for b in range(spec.B):
        bt[b, : npages[b]] = perm[pos: pos + npages[b]]
        pos += int(npages[b])
    free = perm[pos:].copy()
    tags = r.integers(0, 2**32, size=P, dtype=np.uint64).astype(np.uint32)
    expected = np.zeros((spec.B, max_pages), dtype=np.uint32)
    for b in range(spec.B):
        expected[b, : npages[b]] = tags[bt[b, : npages[b]]]
    # stale expected tags: the entry no longer equals the live tag
    stale = []
    n_entries = need
    n_stale = spec.n_stale or (int(math.ceil(spec.stale_frac * n_entries)) if spec.stale_frac else 0)
    if n_stale:
        flat = r.choice(n_entries, size=n_stale, replace=False)
        starts = np.concatenate([[0], np.cumsum(npages)])
        for f in sorted(flat.tolist()):
            b = int(np.searchsorted(starts, f, side="right") - 1)
            i = int(f - starts[b])
            expected[b, i] ^= np.uint32(1)
            stale.append((b, i))
    # slots: logical token j of sequence b lives at page bt[b][j // ps], offset j % ps
    hist = []
    new_slots = np.full(spec.B, -1, dtype=np.int32)
    for b in range(spec.B):
        L = int(lens[b])
        if L == 0:
            continue
        j = np.arange(L, dtype=np.int64)
        slots = bt[b, j // ps].astype(np.int64) * ps + j % ps
        hist.append(slots[:-1])
        new_slots[b] = slots[-1]
    hist_slots = (np.concatenate(hist) if hist else np.zeros(0, np.int64)).astype(np.int32)
    sm = spec.sm_scale if spec.sm_scale is not None else 1.0 / math.sqrt(spec.head_dim_k)
    return Workload(spec, seed, device, P, lens, bt, tags, expected, stale, free, hist_slots,
                    new_slots, float(sm))


# ---------------------------------------------------------------------------
# The multi-step decode loop (long workload): layout of every step
# ---------------------------------------------------------------------------
@dataclass
class LoopStep:
    step: int
    slots: np.ndarray            # int32 [B]: slot of each sequence's new token
    new_pages: List[tuple]       # (b, i, page): entry i of sequence b handed out this step
    seq_lens: np.ndarray         # int32 [B]: tokens each sequence decodes over this step
    stale: List[tuple]           # (b, i): expected-tag entries made stale for this step


def loop_capacity(wl: Workload, steps: int) -> int:
    """Block-table width that holds every sequence after `steps` steps."""
    ps = wl.spec.page_size
    return int(((wl.seq_lens.astype(np.int64) + steps - 1 + ps - 1) // ps).max())


def loop_steps(wl: Workload, steps: int) -> Iterator[LoopStep]:
    """Step s appends token seq_len-1+s of every sequence (step 0 appends the
    workload's own new token) and decodes over seq_len+s tokens.  A token that
    starts a page takes the next page of the seeded free list.  Each step
    re-draws ceil(stale_frac * entries) stale (request, entry) positions."""
    s = wl.spec
    ps = s.page_size
    free = list(wl.free_pages.tolist())
    npages = ((wl.seq_lens.astype(np.int64) + ps - 1) // ps).astype(np.int64)
    bt = {b: list(wl.block_table[b, : npages[b]]) for b in range(s.B)}
    for st in range(steps):
        pos = wl.seq_lens.astype(np.int64) - 1 + st
        slots = np.full(s.B, -1, np.int32)
        new_pages = []
        for b in range(s.B):
            if wl.seq_lens[b] == 0:
                continue
            i = int(pos[b] // ps)
            if i >= len(bt[b]):
                page = free.pop(0)
                bt[b].append(page)
                new_pages.append((b, i, page))
            slots[b] = bt[b][i] * ps + pos[b] % ps
        lens = np.where(wl.seq_lens > 0, wl.seq_lens + st, 0).astype(np.int32)
        stale = []
        if s.stale_frac:
            ent = ((lens.astype(np.int64) + ps - 1) // ps)
            n = int(math.ceil(s.stale_frac * ent.sum()))
            r = _rng(wl.seed, s.name, "stale", st)
            flat = r.choice(int(ent.sum()), size=n, replace=False)
            starts = np.concatenate([[0], np.cumsum(ent)])
            for f in sorted(flat.tolist()):
                b = int(np.searchsorted(starts, f, side="right") - 1)
                stale.append((b, int(f - starts[b])))
        yield LoopStep(st, slots, new_pages, lens, stale)


def loop_tokens(wl: Workload, step: int):
    """Random K/V of the token each sequence appends at `step` (step 0: the workload's own)."""
    if step == 0:
        k, v, _ = wl.new_tokens()
        return k, v
    s = wl.spec
    k = wl._normal((s.B, s.num_kv_heads, s.head_dim_k), "loopk", step)
    v = None if s.v_alias else wl._normal((s.B, s.num_kv_heads, s.head_dim_v), "loopv", step)
    return k, v
