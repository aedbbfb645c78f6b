"""Pins for the oracle's cache-state models (no GPU).

The page-level model and the frame-list simulator are pinned against the
values the pages print, against closed forms of the retention rule, and
against each other on random operation sequences.
"""
import json
import math
import os

import pytest
from hypothesis import given, settings, strategies as st

from oracle import FrameListSim, PageModel, OracleError

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_stats_example_12_frames():
    g = load("cache_stats_12_frames.json")
    c = g["config"]
    m = PageModel(c["scale_frames"], c["sliding_window"], c["page_size"],
                  max_pages=g["patch_pages"] + 2, NS=c["num_special"],
                  patch_pages=g["patch_pages"])
    for f in range(c["frames"]):
        m.append(f)
        m.evict()
    assert m.stats() == g["expected"]


def test_interval_keyframes_200_frames():
    g = load("keyframe_interval_200.json")
    n, k = g["frames"], g["keyframe_interval"]
    S, W, NS = 8, g["sliding_window"], g["special_tokens_per_frame"]
    m = PageModel(S, W, 256, max_pages=S + W + 1 + 4, NS=NS)
    sim = FrameListSim(S, W, NS)
    for t in range(n):
        key = (t % k) == 0
        for model in (m, sim):
            if key:
                model.append(t)
                model.evict()
            else:
                model.set_defer(True)
                model.append(t)
                model.evict()
                model.rollback()
    assert m.committed == g["expected_keyframes"]
    assert len(sim.C) == g["expected_keyframes"]
    assert m.sp_len == NS * g["expected_keyframes"]
    assert len(sim.SP) == NS * g["expected_keyframes"]


@pytest.mark.parametrize("ps,n,pages,lpl", [
    (16, 12, 5, 8),      # 72 special tokens on 16-token pages: 4 full + 8
    (256, 320, 8, 128),  # 1920 tokens on 256-token pages: 7 full + 128
    (999, 1000, 7, 6),   # 6000 tokens on 999-token pages: 6 full + 6
])
def test_special_stream_worked_sizes(ps, n, pages, lpl):
    m = PageModel(8, 64, ps, max_pages=73 + pages, NS=6)
    for f in range(n):
        m.append(f)
        m.evict()
    table, last = m.page_table()
    special = [p for p in table if p >= m.Np]
    assert len(special) == pages
    assert last == lpl
    assert m.sp_len == 6 * n


@pytest.mark.parametrize("ps", [16, 17, 256, 999])
def test_special_stream_grows_six_per_frame(ps):
    m = PageModel(2, 4, ps, max_pages=7 + 64, NS=6)
    for n in range(1, 120):
        before = m.sp_len
        m.append(n)
        m.evict()
        assert m.sp_len - before == 6
        table, last = m.page_table()
        # continuous packing: 6n tokens fill ceil(6n/ps) pages, the last one
        # holding the remainder (a full page when 6n is a multiple of ps)
        assert len([p for p in table if p >= m.Np]) == math.ceil(6 * n / ps)
        assert last == ((6 * n - 1) % ps) + 1


@pytest.mark.parametrize("S,W", [(8, 64), (2, 4), (0, 3), (3, 0), (1, 1)])
def test_retained_frames_closed_form(S, W):
    """After n keyframes: the first min(n, S) frames plus the latest
    min(n - S, W) others are resident, i.e. min(n, S + W) frames."""
    sim = FrameListSim(S, W, 6)
    m = PageModel(S, W, 16, max_pages=S + W + 1 + 200, NS=6)
    for n in range(1, 200):
        f = n - 1
        sim.append(f)
        sim.evict()
        m.append(f)
        m.evict()
        want = list(range(min(n, S))) + list(range(max(S, n - W), n))
        assert sim.patch_frames() == want
        assert [f for f, _ in m.patch_pages_visible()] == want
        assert len(want) == min(n, S + W)


def test_free_list_pops_in_order_and_reuses_evicted_page():
    m = PageModel(2, 3, 16, max_pages=7, NS=1)
    pages = [m.append(f)[0] for f in range(3)]
    assert pages == [0, 1, 2]
    for f in range(3, 6):
        page, _ = m.append(f)
        m.evict()
        assert page == f
    # window now holds frames 3,4,5 (W=3); frame 2 was evicted -> page 2 freed
    page, _ = m.append(6)
    assert page == 2


def test_capacity_errors():
    with pytest.raises(OracleError) as e:
        PageModel(2, 2, 16, max_pages=5, NS=6)
    assert e.value.code == "CAPACITY"
    m = PageModel(1, 1, 16, max_pages=4, NS=6)   # 1 special page = 16 tokens
    m.append(0); m.evict()
    m.append(1); m.evict()
    with pytest.raises(OracleError) as e:
        m.append(2)
    assert e.value.code == "CAPACITY"
    with pytest.raises(OracleError) as e:
        PageModel(1, 1, 16, max_pages=4).page_table()
    assert e.value.code == "EMPTY"


def test_last_page_len_is_the_fill_of_the_tables_final_page():
    """[P1] "Frequently Asked Questions": last_page_len counts the valid tokens
    in the table's final page. One scale frame, no window, retention off,
    three frames of page size 16: frames 1 and 2 are evicted on arrival, so
    stream tokens 6-17 are hidden and special page 1 (tokens 16-17) drops out
    of the table; its final page is special page 0, written in full."""
    m = PageModel(1, 0, 16, max_pages=6, NS=6, cross_frame_special=False)
    sim = FrameListSim(1, 0, 6, cross_frame_special=False)
    for f in range(3):
        m.append(f); m.evict()
        sim.append(f); sim.evict()
    assert m.page_table() == ([0, 2], 16)
    assert m.visible_special_index() == list(range(6))
    assert m.visible_tokens() == sim.visible_tokens(16)
    # with retention on the final page is the stream's last: 18 - 16 = 2 tokens
    m.cross_frame_special = True
    assert m.page_table() == ([0, 2, 3], 2)


def test_nothing_visible_is_an_empty_table():
    """No scale frame, no window, retention off: a frame is evicted as it is
    appended and its specials hide with it, so the table would be empty."""
    m = PageModel(0, 0, 16, max_pages=4, NS=6, cross_frame_special=False)
    sim = FrameListSim(0, 0, 6, cross_frame_special=False)
    m.append(0); m.evict()
    sim.append(0); sim.evict()
    assert sim.visible_tokens(16) == set() == m.visible_tokens()
    with pytest.raises(OracleError) as e:
        m.page_table()
    assert e.value.code == "EMPTY"


def _invariants(m: PageModel):
    used = [p for _, p in m.scale] + [p for _, p in m.window]
    if m.pending is not None:
        used.append(m.pending[1])
    assert len(used) + len(m.free) == m.Np
    assert sorted(used + m.free) == list(range(m.Np))
    assert len(m.scale) <= m.S
    if not m.defer:
        assert len(m.window) <= m.W
    assert len(m.sp_owner) == m.sp_len


OPS = st.lists(st.sampled_from(["key", "key", "key", "defer_keep", "defer_drop",
                                "evict", "bad_commit", "bad_rollback"]),
               min_size=1, max_size=60)


@settings(max_examples=150, deadline=None)
@given(ops=OPS, S=st.integers(0, 3), W=st.integers(0, 4), ps=st.sampled_from([1, 5, 16]), xs=st.booleans())
def test_page_model_matches_frame_list(ops, S, W, ps, xs):
    NS = 6
    m = PageModel(S, W, ps, max_pages=S + W + 1 + (NS * 64) // ps + 2, NS=NS, cross_frame_special=xs)
    sim = FrameListSim(S, W, NS, cross_frame_special=xs)
    f = 0
    for op in ops:
        if op == "evict":
            m.evict(); sim.evict()
        elif op == "key":
            m.set_defer(False); sim.set_defer(False)
            m.append(f); sim.append(f)
            m.evict(); sim.evict()
            f += 1
        elif op in ("defer_keep", "defer_drop"):
            m.set_defer(True); sim.set_defer(True)
            m.append(f); sim.append(f)
            m.evict(); sim.evict()
            assert m.visible_tokens() == sim.visible_tokens(ps)
            _invariants(m)
            if op == "defer_keep":
                m.commit(); sim.commit()
            else:
                m.rollback(); sim.rollback()
            f += 1
        elif op == "bad_commit":
            with pytest.raises(OracleError):
                m.commit()
            with pytest.raises(ValueError):
                sim.commit()
        elif op == "bad_rollback":
            with pytest.raises(OracleError):
                m.rollback()
            with pytest.raises(ValueError):
                sim.rollback()
        _invariants(m)
        if m.committed or m.pending is not None:
            assert m.visible_tokens() == sim.visible_tokens(ps)
            assert m.visible_token_count() == len(sim.visible_tokens(ps))


@settings(max_examples=100, deadline=None)
@given(n=st.integers(0, 90), S=st.integers(0, 4), W=st.integers(0, 5))
def test_rollback_restores_pre_append_state(n, S, W):
    m = PageModel(S, W, 7, max_pages=S + W + 1 + 100, NS=6)
    sim = FrameListSim(S, W, 6)
    for f in range(n):
        m.append(f); m.evict()
        sim.append(f); sim.evict()
    before_m, before_s = m.snapshot(), sim.snapshot()
    for model in (m, sim):
        model.set_defer(True)
        model.append(n)
        model.evict()
        model.rollback()
    assert m.snapshot() == before_m
    assert sim.snapshot() == before_s


def test_deferred_frame_is_visible_on_top_of_full_window():
    S, W = 2, 3
    m = PageModel(S, W, 16, max_pages=S + W + 1 + 10, NS=6)
    for f in range(10):
        m.append(f); m.evict()
    m.set_defer(True)
    m.append(10)
    m.evict()                                  # no-op while deferred
    assert [f for f, _ in m.patch_pages_visible()] == [0, 1, 7, 8, 9, 10]
    m.commit()                                 # commit runs the eviction
    assert [f for f, _ in m.patch_pages_visible()] == [0, 1, 8, 9, 10]


def test_cross_frame_special_off_worked_example():
    """Tiny config (page 16, S=2, W=4), 12 frames, specials of evicted frames
    dropped: frames 0, 1 (scale) and 8..11 (window) stay, so the visible
    special stream indices are [0, 12) and [48, 72): special pages 0, 3 and 4
    (16 slots each), the last one holding 72 - 64 = 8 tokens. Worked by hand."""
    m = PageModel(2, 4, 16, max_pages=7 + 5, NS=6, cross_frame_special=False)
    sim = FrameListSim(2, 4, 6, cross_frame_special=False)
    for f in range(12):
        m.append(f); m.evict()
        sim.append(f); sim.evict()
    table, lpl = m.page_table()
    Np = 7
    # pages 0..6 go to frames 0..6; from frame 6 on each append evicts the
    # oldest window frame (2, 3, ...) and the next frame reuses its page, so
    # frames 8..11 sit on pages 3, 4, 5, 6
    assert table[:6] == [0, 1, 3, 4, 5, 6]
    assert table[6:] == [Np + 0, Np + 3, Np + 4] and lpl == 8
    assert m.visible_special_index() == list(range(12)) + list(range(48, 72))
    assert m.visible_token_count() == 6 * 16 + 6 * 6
    assert m.visible_tokens() == sim.visible_tokens(16)


@pytest.mark.parametrize("S,W", [(0, 3), (2, 4), (8, 64)])
def test_cross_frame_special_off_closed_form(S, W):
    """Every visible frame keeps exactly its NS special tokens and no other
    frame's: visible tokens = (frames visible) x (P + NS)."""
    P, NS = 16, 6
    on, off = FrameListSim(S, W, NS), FrameListSim(S, W, NS, cross_frame_special=False)
    for n in range(1, 3 * (S + W) + 5):
        for sim in (on, off):
            sim.append(n - 1); sim.evict()
        frames = min(n, S) + min(max(n - S, 0), W)
        assert len(off.visible_tokens(P)) == frames * (P + NS)
        assert len(on.visible_tokens(P)) == frames * P + NS * n
        if n <= S + W:   # nothing evicted yet: the two settings agree
            assert off.visible_tokens(P) == on.visible_tokens(P)


def test_camera_only_worked_example():
    """Tiny config (page 16, S=2, W=4, NS=6), 12 frames, camera-only: the
    camera token is slot 0 of each frame's six, so the visible special stream
    indices are the multiples of 6. With retention on: 0, 6, ..., 66 on
    special pages 0 (0, 6, 12), 1 (18, 24, 30), 2 (36, 42), 3 (48, 54, 60)
    and 4 (66); no patch page; the last page holds 72 - 64 = 8 written
    tokens. With retention off only frames 0, 1 and 8..11 count: indices 0,
    6, 48, 54, 60, 66 on special pages 0, 3, 4. Worked by hand."""
    Np = 7
    for xs, idx, pages in [(True, list(range(0, 72, 6)), [0, 1, 2, 3, 4]),
                           (False, [0, 6, 48, 54, 60, 66], [0, 3, 4])]:
        m = PageModel(2, 4, 16, max_pages=Np + 5, NS=6, cross_frame_special=xs, camera_only=True)
        sim = FrameListSim(2, 4, 6, cross_frame_special=xs, camera_only=True)
        for f in range(12):
            m.append(f); m.evict()
            sim.append(f); sim.evict()
        table, lpl = m.page_table()
        assert table == [Np + p for p in pages] and lpl == 8
        assert m.visible_special_index() == idx
        assert m.visible_token_count() == len(idx)
        assert sim.visible_specials() == [(j // 6, 0) for j in idx]
        assert m.visible_tokens() == sim.visible_tokens(16) == {("s", j // 6, 0) for j in idx}
        # the cache itself is as without camera-only: same pages, stats, free list
        plain = PageModel(2, 4, 16, max_pages=Np + 5, NS=6, cross_frame_special=xs)
        for f in range(12):
            plain.append(f); plain.evict()
        assert m.snapshot() == plain.snapshot() and m.stats() == plain.stats()


@pytest.mark.parametrize("S,W", [(0, 3), (2, 4), (8, 64)])
def test_camera_only_closed_form(S, W):
    """Camera-only sees exactly one token per frame whose special tokens are
    visible: n with retention on, the visible frames with it off."""
    for xs in (True, False):
        sim = FrameListSim(S, W, 6, cross_frame_special=xs, camera_only=True)
        for n in range(1, 3 * (S + W) + 5):
            sim.append(n - 1); sim.evict()
            frames = min(n, S) + min(max(n - S, 0), W)
            assert len(sim.visible_tokens(16)) == (n if xs else frames)
            assert sim.attended_patch_frames() == []


@settings(max_examples=80, deadline=None)
@given(ops=st.lists(st.sampled_from(["key", "key", "defer_keep", "defer_drop"]), min_size=1, max_size=40),
       S=st.integers(0, 3), W=st.integers(0, 4), ps=st.sampled_from([5, 16, 130]), xs=st.booleans())
def test_camera_only_page_model_matches_frame_list(ops, S, W, ps, xs):
    m = PageModel(S, W, ps, max_pages=S + W + 1 + 6 * 40 // ps + 2, NS=6, cross_frame_special=xs,
                  camera_only=True)
    sim = FrameListSim(S, W, 6, cross_frame_special=xs, camera_only=True)
    for f, op in enumerate(ops):
        d = op != "key"
        m.set_defer(d); sim.set_defer(d)
        m.append(f); sim.append(f)
        m.evict(); sim.evict()
        assert m.visible_tokens() == sim.visible_tokens(ps)
        if d:
            if op == "defer_keep":
                m.commit(); sim.commit()
            else:
                m.rollback(); sim.rollback()
        assert m.visible_tokens() == sim.visible_tokens(ps)


def test_shared_pool_worked_example():
    """Two streams A, B share 5 patch pages (S=1, W=1, page 4, NS=2); A's
    special pages are 5-6, B's 7-8. Worked by hand, the common LIFO free
    list starting [4, 3, 2, 1, 0]:
      A0 takes 0, B0 takes 1, A1 takes 2, A2 takes 3 and evicts A1 (2 back),
      B1 takes 2, B2 takes 4 and evicts B1 (2 back): free [2].
      A's table [0, 3, 5, 6] (6 special tokens: 4 + 2), B's [1, 4, 7, 8].
      Reset A: its scale page 0, then window page 3, go back: free [2, 0, 3].
      B3 takes 3 and evicts B2 (4 back): free [2, 0, 4]; B's table [1, 3, 7, 8]
      with the last page full (8 tokens). A0 again takes 4: table [4, 5]."""
    from oracle import SharedPatchPool
    pool = SharedPatchPool(5)
    A = PageModel(1, 1, 4, 9, NS=2, shared=pool, sp_base=5, sp_pages=2)
    B = PageModel(1, 1, 4, 9, NS=2, shared=pool, sp_base=7, sp_pages=2)

    def step(m, f):
        page, sp0 = m.append(f)
        m.evict()
        return page, sp0

    assert [step(A, 0), step(B, 0), step(A, 1), step(A, 2)] == [(0, 0), (1, 0), (2, 2), (3, 4)]
    assert pool.free == [4, 2]
    assert [step(B, 1), step(B, 2)] == [(2, 2), (4, 4)]
    assert pool.free == [2]
    assert A.page_table() == ([0, 3, 5, 6], 2)
    assert B.page_table() == ([1, 4, 7, 8], 2)
    assert A.special_location(4) == (6, 0) and B.special_location(5) == (8, 1)
    A.reset()
    assert pool.free == [2, 0, 3]
    assert step(B, 3) == (3, 6) and pool.free == [2, 0, 4]
    assert B.page_table() == ([1, 3, 7, 8], 4)
    assert step(A, 0) == (4, 0) and A.page_table() == ([4, 5], 2)
    assert A.stats()["free_pages"] == B.stats()["free_pages"] == 2


@settings(max_examples=80, deadline=None)
@given(ops=st.lists(st.tuples(st.integers(0, 2), st.sampled_from(["key", "key", "defer_keep", "defer_drop",
                                                                  "reset"])), min_size=1, max_size=60),
       S=st.integers(0, 2), W=st.integers(0, 3))
def test_shared_pool_partitions_the_patch_pages(ops, S, W):
    """Every patch page is on the common free list or held by exactly one
    stream (scale, window or pending page); each stream's visible set is what
    its own frame-list simulator says; a stream alone in a pool of its own
    size behaves exactly as a standalone page model."""
    from oracle import SharedPatchPool
    n, ps, Np = 3, 5, 3 * (S + W + 1)
    pool = SharedPatchPool(Np)
    ms = [PageModel(S, W, ps, Np + 3 * 20, NS=6, shared=pool, sp_base=Np + 20 * i, sp_pages=20) for i in range(n)]
    sims = [FrameListSim(S, W, 6) for _ in range(n)]
    nxt = [0] * n
    for s_i, op in ops:
        m, sim = ms[s_i], sims[s_i]
        if op == "reset":
            m.reset()
            sims[s_i] = FrameListSim(S, W, 6)
            nxt[s_i] = 0
            continue
        if m.sp_len + 6 > m.special_capacity:
            continue
        d = op != "key"
        m.set_defer(d); sim.set_defer(d)
        f = nxt[s_i]
        m.append(f); sim.append(f)
        m.evict(); sim.evict()
        nxt[s_i] += 1
        if d:
            if op == "defer_keep":
                m.commit(); sim.commit()
            else:
                m.rollback(); sim.rollback()
                nxt[s_i] -= 1
        held = [p for mm in ms for _, p in mm.patch_pages_visible()]
        assert sorted(held + pool.free) == list(range(Np))
        for mm, ss in zip(ms, sims):
            assert mm.visible_tokens() == ss.visible_tokens(ps)
    # one stream alone in a pool of its own size: the standalone model
    solo_pool = SharedPatchPool(S + W + 1)
    a = PageModel(S, W, ps, S + W + 1 + 20, NS=6, shared=solo_pool)
    b = PageModel(S, W, ps, S + W + 1 + 20, NS=6)
    for f in range(15):
        for m in (a, b):
            m.append(f); m.evict()
        assert a.snapshot() == b.snapshot() and a.page_table() == b.page_table()
