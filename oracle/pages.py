"""Page-level model of the two-stream paged KV cache, for bit-exact checks.

Test infrastructure only (see the package docstring).

Physical pool, per transformer block: [max_pages, 2, page_size, H, D]
([P1] "Physical Memory Layout"). Dimension 1 is read as K (0) / V (1); the two
streams are told apart by page-id range: patch pages are [0, Np), special pages
are [Np, max_pages) ([P3] "Constant Memory with Two-Stream Paging": memory is
max_patch_pages + max_special_pages).

Patch stream ([P1] "Patch Stream (Recyclable)"; [P3] same section): one page
per frame, page_size == patches per frame. Pages come from a free list; evicted
pages go back on it. The free list is a LIFO stack that starts as
[Np-1, ..., 1, 0], so the first pops yield 0, 1, 2, ...

Special stream ([P1] "Special Stream (Append-Only)"): NS tokens per frame,
packed back to back with no padding; special token j (0-based over the stream)
lives on page Np + j // page_size at slot j % page_size.

Visible page table ([P1] "Building the Visible Page Table"; [P3] "Visible Page
Table Attention"): scale pages in frame order, window pages oldest to newest,
then the pending page if any, then special pages Np .. Np+k-1. Only the last
page may be partial; last_page_len is the fill of the table's final page.

Without cross-frame special retention ([P2] "Configuration Parameters"), the
special tokens of evicted frames drop out: the visible special tokens are the
runs of the frames whose patches are visible. Evictions always take the
oldest window frame, so those runs form at most two ranges of the stream
(the scale frames' and the window's), and the table lists only special pages
that hold a visible token.

Camera-only ([P2] "Configuration Parameters"; the reading is stated in
frames.py): the pages and free list behave as always, but attention sees only
the camera token (slot 0) of each frame among the special tokens that would
otherwise be visible, and no patch page; the table then lists only special
pages holding a visible camera token.

Shared pool ([P3] "Constant Memory with Two-Stream Paging": memory is bounded
by max_patch_pages + max_special_pages). Several streams can share one pool
per block: the patch pages [0, Np) and one LIFO free list are common, and
each stream owns a fixed range of special pages [sp_base, sp_base + sp_pages)
for its own special stream. Reading: a stream that is reset returns its scale
pages (in frame order), then its window pages (oldest first), then a pending
page to the common free list; nothing else changes for the other streams.

get_cache_stats keys ([P3] "Monitoring Cache Statistics"): frame_count,
scale_pages, live_pages, free_pages, special_tokens.
"""
from __future__ import annotations

import numpy as np


class OracleError(Exception):
    def __init__(self, code: str, msg: str = ""):
        super().__init__(f"{code}: {msg}")
        self.code = code


class SharedPatchPool:
    """Patch pages [0, Np) and their LIFO free list, common to the page
    models of several streams (initially [Np-1, ..., 0]: pops yield 0, 1, ...)."""

    def __init__(self, Np: int):
        self.Np = Np
        self.free = list(range(Np - 1, -1, -1))


class PageModel:
    def __init__(self, S: int, W: int, page_size: int, max_pages: int,
                 NS: int = 6, patch_pages: int | None = None, cross_frame_special: bool = True,
                 camera_only: bool = False, shared: SharedPatchPool | None = None,
                 sp_base: int | None = None, sp_pages: int | None = None):
        """shared: the common patch pool of a group of streams (patch_pages is
        then its size); sp_base, sp_pages: this stream's range of special
        pages (default: every page after the patch pages)."""
        self.S, self.W, self.ps, self.NS = S, W, page_size, NS
        self.cross_frame_special = cross_frame_special
        self.camera_only = camera_only
        self.shared = shared
        self.Np = shared.Np if shared else (patch_pages if patch_pages else S + W + 1)
        self.sp_base = self.Np if sp_base is None else sp_base
        self.sp_pages = max_pages - self.sp_base if sp_pages is None else sp_pages
        if (self.Np < 1 or self.sp_base < self.Np or self.sp_base + self.sp_pages > max_pages
                or self.sp_pages < (1 if NS > 0 else 0)):
            raise OracleError("CAPACITY", "pool too small")
        self.max_pages = max_pages
        self._own_free: list[int] = []
        self.scale, self.window, self.pending = [], [], None
        self.reset()

    @property
    def free(self) -> list[int]:
        return self.shared.free if self.shared else self._own_free

    def reset(self) -> None:
        if self.shared:
            # this stream's patch pages go back to the common free list
            for _, p in self.scale + self.window + ([self.pending] if self.pending else []):
                self.shared.free.append(p)
        else:
            self._own_free = list(range(self.Np - 1, -1, -1))
        self.scale: list[tuple[int, int]] = []    # (frame, page)
        self.window: list[tuple[int, int]] = []   # (frame, page), oldest first
        self.pending: tuple[int, int] | None = None
        self.sp_len = 0
        self.sp_owner: list[tuple[int, int]] = []  # (frame, slot) of special token j
        self.committed = 0
        self.defer = False

    @property
    def special_capacity(self) -> int:
        return self.sp_pages * self.ps

    # -- operations -------------------------------------------------------
    def append(self, f: int) -> tuple[int, int]:
        """New frame f: returns (patch page, first special slot index)."""
        if self.pending is not None:
            raise OracleError("ORDER", "pending frame")
        if not self.free:
            raise OracleError("CAPACITY", "no free patch page")
        if self.sp_len + self.NS > self.special_capacity:
            raise OracleError("CAPACITY", "special stream full")
        page = self.free.pop()
        sp0 = self.sp_len
        self.sp_len += self.NS
        self.sp_owner.extend((f, i) for i in range(self.NS))
        if self.defer:
            self.pending = (f, page)
        else:
            self._commit(f, page)
        return page, sp0

    def _commit(self, f: int, page: int) -> None:
        if len(self.scale) < self.S:
            self.scale.append((f, page))
        else:
            self.window.append((f, page))
        self.committed += 1

    def evict(self) -> list[int]:
        """Frees window pages beyond W, oldest first; returns the freed frames."""
        if self.defer:
            return []
        freed = []
        while len(self.window) > self.W:
            f, p = self.window.pop(0)
            self.free.append(p)
            freed.append(f)
        return freed

    def set_defer(self, on: bool) -> None:
        if not on and self.pending is not None:
            raise OracleError("ORDER", "pending frame")
        self.defer = bool(on)

    def commit(self) -> None:
        if self.pending is None:
            raise OracleError("NO_PENDING")
        f, p = self.pending
        self.pending = None
        self.defer = False
        self._commit(f, p)
        self.evict()

    def rollback(self) -> None:
        if self.pending is None:
            raise OracleError("NO_PENDING")
        _, p = self.pending
        self.pending = None
        self.defer = False
        self.free.append(p)
        self.sp_len -= self.NS
        del self.sp_owner[self.sp_len:]

    # -- queries ----------------------------------------------------------
    def patch_pages_visible(self) -> list[tuple[int, int]]:
        out = self.scale + self.window
        if self.pending is not None:
            out = out + [self.pending]
        return out

    def attended_patch_pages(self) -> list[tuple[int, int]]:
        """(frame, page) of the patch pages attention reads: none with camera-only."""
        return [] if self.camera_only else self.patch_pages_visible()

    def visible_special_index(self) -> list[int]:
        """Stream indices j of the visible special tokens, ascending."""
        if self.cross_frame_special:
            out = list(range(self.sp_len))
        else:
            live = {f for f, _ in self.patch_pages_visible()}
            out = [j for j in range(self.sp_len) if self.sp_owner[j][0] in live]
        if self.camera_only:
            out = [j for j in out if self.sp_owner[j][1] == 0]
        return out

    def page_table(self) -> tuple[list[int], int]:
        """(kv_indices, last_page_len) of the visible page table.

        last_page_len is the number of tokens written to the table's final
        page ([P1] "Frequently Asked Questions": the exact count of valid
        tokens in the final page). The final page is a special page; only
        with cross-frame special retention off can it be an earlier one than
        the stream's last, whose specials are then all hidden. Hidden tokens
        inside a listed page are not expressible by (indices, last_page_len)
        and are read off visible_special_index instead.
        """
        if self.committed == 0 and self.pending is None:
            raise OracleError("EMPTY", "no frame")
        patch = [p for _, p in self.attended_patch_pages()]
        pages = sorted({j // self.ps for j in self.visible_special_index()})
        special = [self.sp_base + i for i in pages]
        table = patch + special
        if not table:   # scale_frames = window = 0 with retention off
            raise OracleError("EMPTY", "no visible token")
        last = min(self.ps, self.sp_len - self.ps * pages[-1]) if pages else self.ps
        return table, last

    def visible_token_count(self) -> int:
        return len(self.attended_patch_pages()) * self.ps + len(self.visible_special_index())

    def stats(self) -> dict:
        pend = 1 if self.pending is not None else 0
        return {
            "frame_count": self.committed + pend,
            "scale_pages": len(self.scale),
            "live_pages": len(self.window) + pend,
            "free_pages": len(self.free),
            "special_tokens": self.sp_len,
        }

    def special_location(self, j: int) -> tuple[int, int]:
        return self.sp_base + j // self.ps, j % self.ps

    def visible_tokens(self) -> set:
        """Visible tokens in the frame simulator's ('p', frame, t) / ('s', frame,
        slot) form, read back through the page table: each listed page and
        slot is mapped to the frame that wrote it."""
        if self.visible_token_count() == 0:
            return set()
        table, last = self.page_table()
        owner = {p: f for f, p in self.attended_patch_pages()}
        vis = set(self.visible_special_index())
        out = set()
        for n, p in enumerate(table):
            cnt = last if n == len(table) - 1 else self.ps
            for t in range(cnt):
                if p < self.Np:
                    out.add(("p", owner[p], t))
                elif (p - self.sp_base) * self.ps + t in vis:
                    out.add(("s",) + self.sp_owner[(p - self.sp_base) * self.ps + t])
        return out

    def snapshot(self):
        return (tuple(self.free), tuple(self.scale), tuple(self.window), self.pending,
                self.sp_len, tuple(self.sp_owner), self.committed, self.defer)


class PoolImage:
    """Expected raw contents of one block's pool: [max_pages, 2, ps, H, D] of
    16-bit bit patterns. `write` mirrors what an append stores."""

    def __init__(self, model: PageModel, H: int, D: int):
        self.m = model
        self.bits = np.zeros((model.max_pages, 2, model.ps, H, D), dtype=np.uint16)

    def write(self, page: int, sp0: int, k_bits: np.ndarray, v_bits: np.ndarray, model=None) -> None:
        """k_bits, v_bits: [NS + P, H, D] uint16. Tokens 0..NS-1 are the frame's
        special tokens, NS.. its patch tokens. model: the stream that appends
        (for a pool shared by several streams), default the image's own."""
        m = model or self.m
        NS, ps = m.NS, m.ps
        for kv, x in ((0, k_bits), (1, v_bits)):
            self.bits[page, kv, :ps] = x[NS:NS + ps]
            for i in range(NS):
                pg, slot = m.special_location(sp0 + i)
                self.bits[pg, kv, slot] = x[i]

    def gather(self, kv_indices, last_page_len):
        """Visible K and V rows in page-table order: two [L, H, D] uint16 arrays."""
        ps = self.m.ps
        ks, vs = [], []
        for n, p in enumerate(kv_indices):
            cnt = last_page_len if n == len(kv_indices) - 1 else ps
            ks.append(self.bits[p, 0, :cnt])
            vs.append(self.bits[p, 1, :cnt])
        return np.concatenate(ks), np.concatenate(vs)
