"""Host-side page-tag tracker.

The server side of the integrity check: it records, for every request, the
physical pages it holds and the tag each page carried when it was handed to
the request ("Cloudflare: Kleinere Modellbereitstellung senkt Speicherbedarf,
doch Sicherheit wird zum Prüfstein" (remio.ai), section "Sicherheit gemeinsamer
KV-Caches wird zum Produktionsthema"; "Công thức của Cloudflare ..."
(manulx.blog), section "Bảo vệ bộ nhớ đệm dùng chung").  Tags are generation
counters: a page handed out again gets tag + 1 (mod 2^32), the value
kvq_append gives it on the device when the page is listed in realloc_pages.
"""
from __future__ import annotations

import numpy as np


class TagTracker:
    def __init__(self, live_tags: np.ndarray, block_table: np.ndarray, seq_lens: np.ndarray,
                 page_size: int, capacity: int):
        """live_tags: u32 [P] as on the device; block_table: i32 [B][>= pages in use]."""
        B = block_table.shape[0]
        self.tags = np.asarray(live_tags, dtype=np.uint32).copy()
        self.block_table = np.full((B, capacity), -1, dtype=np.int32)
        self.expected = np.zeros((B, capacity), dtype=np.uint32)
        n = (np.asarray(seq_lens, np.int64) + page_size - 1) // page_size
        for b in range(B):
            pages = block_table[b, : n[b]]
            self.block_table[b, : n[b]] = pages
            self.expected[b, : n[b]] = self.tags[pages]

    def hand_out(self, b: int, i: int, page: int) -> int:
        """Entry i of request b now holds `page`, a reallocation: returns the expected tag."""
        t = np.uint32((int(self.tags[page]) + 1) & 0xFFFFFFFF)
        self.tags[page] = t
        self.block_table[b, i] = page
        self.expected[b, i] = t
        return int(t)
