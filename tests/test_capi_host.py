"""Host-side tests of the C-ABI library (no GPU, no kernel launches).

The library loads without a GPU; the page state machine, the visible page
table, last_page_len, the free list, the statistics and the K/V tiling are
compared bit for bit with the oracle's page-level model. Appends pass NULL
k/v (state only) and plans are host-only (no workspace).
"""
import json
import math
import os
import re

import pytest
from hypothesis import given, settings, strategies as st

from oracle import PageModel, OracleError

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="session")
def pkv():
    from paged_kv_cache_frame_b200 import build
    build.build()
    import paged_kv_cache_frame_b200 as m
    return m


def declared_functions():
    src = open(os.path.join(ROOT, "include", "kv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]*?\b(kv_\w+)\s*\(", src, flags=re.M)))


def test_library_exports_every_declared_function(pkv):
    import ctypes
    names = declared_functions()
    assert len(names) >= 20
    lib = ctypes.CDLL(pkv.capi.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(pkv.capi.SIGNATURES)


def test_strerror_covers_codes(pkv):
    for code in range(0, -11, -1):
        assert pkv.kv_strerror(code) != "unknown status"
    assert pkv.kv_strerror(-99) == "unknown status"


def mk(pkv, S, W, ps, max_pages, NS=6, B=1, patch_pages=0, H=2, D=64):
    return pkv.kv_init(max_pages, ps, H, D, S, W, B, NS, pkv.KV_BF16, patch_pages)


def step(pkv, c, B=1):
    for b in range(B):
        pkv.kv_append_frame(c, b, None, None)
        pkv.kv_evict_frames(c)


def table(pkv, caches):
    p = pkv.kv_plan(caches)
    try:
        return [pkv.kv_get_page_table(p, i) for i in range(len(caches))]
    finally:
        pkv.kv_plan_free(p)


def assert_same_table(pkv, h, m):
    """The library's page table equals the oracle's; where the oracle finds
    nothing to attend to (no frame, or no visible token), kv_plan refuses
    with KV_ERR_EMPTY."""
    try:
        want = m.page_table()
    except OracleError as e:
        assert e.code == "EMPTY"
        with pytest.raises(pkv.KVError) as ce:
            table(pkv, [h])
        assert ce.value.code == pkv.capi.KV_ERR_EMPTY
        return
    assert table(pkv, [h])[0] == want


def test_stats_example_through_capi(pkv):
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "cache_stats_12_frames.json")))
    c = g["config"]
    h = mk(pkv, c["scale_frames"], c["sliding_window"], c["page_size"], g["patch_pages"] + 2,
           NS=c["num_special"], patch_pages=g["patch_pages"])
    for _ in range(c["frames"]):
        step(pkv, h)
    assert pkv.kv_get_stats(h) == g["expected"]
    pkv.kv_destroy(h)


def test_interval_keyframes_through_capi(pkv):
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "keyframe_interval_200.json")))
    h = mk(pkv, 8, g["sliding_window"], 256, 73 + 4)
    for t in range(g["frames"]):
        if t % g["keyframe_interval"] == 0:
            step(pkv, h)
        else:
            pkv.kv_defer_eviction(h, True)
            step(pkv, h)
            pkv.kv_rollback_last_frame(h)
    s = pkv.kv_get_stats(h)
    assert s["frame_count"] == g["expected_keyframes"]
    assert s["special_tokens"] == g["special_tokens_per_frame"] * g["expected_keyframes"]


@pytest.mark.parametrize("ps,n,pages,lpl", [(16, 12, 5, 8), (256, 320, 8, 128), (999, 1000, 7, 6)])
def test_special_stream_sizes_through_capi(pkv, ps, n, pages, lpl):
    h = mk(pkv, 8, 64, ps, 73 + pages)
    for _ in range(n):
        step(pkv, h)
    (tbl, last), = table(pkv, [h])
    assert len([p for p in tbl if p >= 73]) == pages and last == lpl
    assert len(tbl) == min(n, 72) + pages


def test_error_codes(pkv):
    E = pkv.capi
    h = mk(pkv, 1, 1, 16, 4, B=2)          # 3 patch pages, 1 special page of 16 tokens
    with pytest.raises(pkv.KVError) as e:
        pkv.kv_plan([h])
    assert e.value.code == E.KV_ERR_EMPTY
    with pytest.raises(pkv.KVError) as e:
        pkv.kv_commit_frame(h)
    assert e.value.code == E.KV_ERR_NO_PENDING
    with pytest.raises(pkv.KVError) as e:
        pkv.kv_rollback_last_frame(h)
    assert e.value.code == E.KV_ERR_NO_PENDING
    pkv.kv_append_frame(h, 0, None, None)
    with pytest.raises(pkv.KVError) as e:
        pkv.kv_append_frame(h, 0, None, None)          # block 0 twice in one step
    assert e.value.code == E.KV_ERR_ORDER
    with pytest.raises(pkv.KVError) as e:
        pkv.kv_append_frame(h, 2, None, None)
    assert e.value.code == E.KV_ERR_ARG
    pkv.kv_append_frame(h, 1, None, None)
    pkv.kv_evict_frames(h)
    step(pkv, h, B=2)                                  # 12 special tokens used
    with pytest.raises(pkv.KVError) as e:
        pkv.kv_append_frame(h, 0, None, None)          # 18 > 16: special stream full
    assert e.value.code == E.KV_ERR_CAPACITY
    assert pkv.kv_get_stats(h)["special_tokens"] == 12  # unchanged by the failed append
    # defer: turning it off while a frame is pending is out of order
    h2 = mk(pkv, 1, 1, 16, 8, B=2)
    pkv.kv_defer_eviction(h2, True)
    pkv.kv_append_frame(h2, 0, None, None)
    with pytest.raises(pkv.KVError) as e:
        pkv.kv_defer_eviction(h2, False)
    assert e.value.code == E.KV_ERR_ORDER
    with pytest.raises(pkv.KVError) as e:
        pkv.kv_commit_frame(h2)                        # block 1 not yet appended
    assert e.value.code == E.KV_ERR_ORDER
    pkv.kv_append_frame(h2, 1, None, None)
    pkv.kv_commit_frame(h2)
    # kv_init arguments
    with pytest.raises(pkv.KVError) as e:
        mk(pkv, 2, 2, 16, 5)                           # needs 5 patch + 1 special page
    assert e.value.code == E.KV_ERR_CAPACITY
    with pytest.raises(pkv.KVError) as e:
        pkv.kv_init(10, 0, 2, 64, 1, 1, 1, 6, 0, 0)
    assert e.value.code == E.KV_ERR_ARG
    # a host-only plan cannot run
    p = pkv.kv_plan([h2])
    with pytest.raises(pkv.KVError) as e:
        pkv.kv_run(p, 0, 16, 16)
    assert e.value.code == E.KV_ERR_ARG
    pkv.kv_plan_free(p)
    for x in (h, h2):
        pkv.kv_destroy(x)


def test_frame_step_rule_multi_block(pkv):
    h = mk(pkv, 2, 2, 16, 10, B=3)
    pkv.kv_append_frame(h, 1, None, None)              # any block may open the step
    assert pkv.kv_get_stats(h)["frame_count"] == 1
    pkv.kv_append_frame(h, 0, None, None)
    pkv.kv_append_frame(h, 2, None, None)
    assert pkv.kv_get_stats(h)["frame_count"] == 1
    pkv.kv_append_frame(h, 0, None, None)              # all appended -> new step
    assert pkv.kv_get_stats(h)["frame_count"] == 2
    pkv.kv_destroy(h)


OPS = st.lists(st.sampled_from(["key", "key", "key", "defer_keep", "defer_drop", "evict",
                                "bad_commit", "bad_rollback"]), min_size=1, max_size=50)


@settings(max_examples=120, deadline=None)
@given(ops=OPS, S=st.integers(0, 3), W=st.integers(0, 4), ps=st.sampled_from([1, 5, 16, 130]),
       B=st.integers(1, 3), xs=st.booleans(), NS=st.sampled_from([6, 6, 1, 0]))
def test_state_machine_bit_exact_vs_oracle(pkv, ops, S, W, ps, B, xs, NS):
    max_pages = S + W + 1 + (NS * 60) // ps + 2
    m = PageModel(S, W, ps, max_pages, NS=NS, cross_frame_special=xs)
    h = mk(pkv, S, W, ps, max_pages, NS=NS, B=B)
    pkv.kv_set_cross_frame_special(h, xs)
    E = pkv.capi
    try:
        f = 0
        for op in ops:
            if op == "evict":
                m.evict(); pkv.kv_evict_frames(h)
            elif op == "key":
                m.set_defer(False); pkv.kv_defer_eviction(h, False)
                m.append(f); m.evict()
                step(pkv, h, B)
                f += 1
            elif op in ("defer_keep", "defer_drop"):
                m.set_defer(True); pkv.kv_defer_eviction(h, True)
                m.append(f); m.evict()
                step(pkv, h, B)
                assert_same_table(pkv, h, m)
                if op == "defer_keep":
                    m.commit(); pkv.kv_commit_frame(h)
                else:
                    m.rollback(); pkv.kv_rollback_last_frame(h)
                f += 1
            elif op == "bad_commit":
                with pytest.raises(OracleError):
                    m.commit()
                with pytest.raises(pkv.KVError) as e:
                    pkv.kv_commit_frame(h)
                assert e.value.code == E.KV_ERR_NO_PENDING
            elif op == "bad_rollback":
                with pytest.raises(OracleError):
                    m.rollback()
                with pytest.raises(pkv.KVError) as e:
                    pkv.kv_rollback_last_frame(h)
                assert e.value.code == E.KV_ERR_NO_PENDING
            assert pkv.kv_get_free_list(h) == m.free
            assert pkv.kv_get_stats(h) == m.stats()
            assert_same_table(pkv, h, m)
    finally:
        pkv.kv_destroy(h)


@settings(max_examples=60, deadline=None)
@given(n=st.integers(0, 80), S=st.integers(0, 4), W=st.integers(0, 5))
def test_rollback_restores_state_through_capi(pkv, n, S, W):
    h = mk(pkv, S, W, 7, S + W + 1 + 80, B=2)
    for _ in range(n):
        step(pkv, h, 2)
    before = (pkv.kv_get_free_list(h), pkv.kv_get_stats(h), table(pkv, [h]) if n else None)
    pkv.kv_defer_eviction(h, True)
    step(pkv, h, 2)
    pkv.kv_rollback_last_frame(h)
    after = (pkv.kv_get_free_list(h), pkv.kv_get_stats(h), table(pkv, [h]) if n else None)
    assert before == after
    pkv.kv_destroy(h)


def test_last_page_len_when_retention_off_hides_the_last_special_page(pkv):
    """One scale frame, no window, retention off, 3 frames, page size 16:
    frames 1 and 2 are evicted as soon as they are appended, so their
    specials (stream tokens 6-17) are hidden and special page 1 (tokens
    16-17) holds nothing visible. The table is frame 0's patch page and
    special page 0, which is full: last_page_len = 16, not the fill of the
    stream's last page (2). Only tokens 0-5 of special page 0 are tiled."""
    S, W, ps, max_pages = 1, 0, 16, 6
    Np = S + W + 1
    h = mk(pkv, S, W, ps, max_pages)
    pkv.kv_set_cross_frame_special(h, False)
    for _ in range(3):
        step(pkv, h)
    p = pkv.kv_plan([h])
    assert pkv.kv_get_page_table(p) == ([0, Np], 16)
    got = tile_cover(pkv.kv_get_kv_tiles(p), ps)
    assert sorted(got) == sorted([(0, t) for t in range(ps)] + [(Np, t) for t in range(6)])
    pkv.kv_plan_free(p)
    # retention on: every special is visible; the last page holds 2 tokens
    pkv.kv_set_cross_frame_special(h, True)
    p = pkv.kv_plan([h])
    assert pkv.kv_get_page_table(p) == ([0, Np, Np + 1], 2)
    pkv.kv_plan_free(p)
    pkv.kv_destroy(h)


def test_plan_refuses_a_stream_with_no_visible_token(pkv):
    """No scale frame, no window, retention off: every frame is evicted as it
    is appended and its specials go with it, so nothing is left to attend
    to; kv_plan reports KV_ERR_EMPTY instead of planning an empty softmax."""
    h = mk(pkv, 0, 0, 16, 4)
    pkv.kv_set_cross_frame_special(h, False)
    step(pkv, h)
    with pytest.raises(pkv.KVError) as e:
        pkv.kv_plan([h])
    assert e.value.code == pkv.capi.KV_ERR_EMPTY
    assert "no visible token" in str(e.value)
    pkv.kv_set_cross_frame_special(h, True)   # the specials are visible again
    p = pkv.kv_plan([h])
    assert pkv.kv_get_page_table(p) == ([1], 6)
    pkv.kv_plan_free(p)
    pkv.kv_destroy(h)


def tile_cover(tiles, ps):
    """(page, token) pairs the tiles mark visible, with multiplicity."""
    out = []
    for row, lo, hi in tiles:
        for col in range(lo, hi):
            r = row + col
            page, rem = divmod(r, 2 * ps)
            assert rem < ps, "a visible column must be a K row of its page"
            out.append((page, rem))
    return out


@pytest.mark.parametrize("xs", [True, False])
@pytest.mark.parametrize("ps,n", [(16, 12), (256, 320), (999, 30), (130, 40), (128, 9), (64, 100),
                                  (16, 200), (300, 150)])
def test_kv_tiles_cover_visible_tokens_exactly_once(pkv, ps, n, xs):
    S, W = 8, 64
    pages = math.ceil(6 * n / ps) + 1
    h = mk(pkv, S, W, ps, 73 + pages)
    pkv.kv_set_cross_frame_special(h, xs)
    m = PageModel(S, W, ps, 73 + pages, cross_frame_special=xs)
    for f in range(n):
        step(pkv, h)
        m.append(f); m.evict()
    p = pkv.kv_plan([h])
    tiles = pkv.kv_get_kv_tiles(p)
    assert pkv.kv_get_page_table(p) == m.page_table()
    want = [(pg, t) for _, pg in m.patch_pages_visible() for t in range(ps)]
    want += [(m.Np + j // ps, j % ps) for j in m.visible_special_index()]
    got = tile_cover(tiles, ps)
    assert sorted(got) == sorted(want)
    for row, lo, hi in tiles:
        assert 0 <= lo < hi <= 128
        if ps >= 128:   # long pages: a box never leaves its page's K rows
            assert (row % (2 * ps)) + 128 <= ps
    s = pkv.kv_plan_get_stats(p)
    assert s["visible_tokens"] == m.visible_token_count()
    assert s["n_kv_tiles"] == len(tiles)
    pkv.kv_plan_free(p)


@pytest.mark.parametrize("S,W,NS,xs", [(2, 3, 0, True), (8, 64, 0, True), (2, 0, 6, True), (2, 0, 6, False),
                                        (0, 0, 6, True), (0, 0, 1, True), (1, 0, 1, False)])
def test_kv_tiles_degenerate_configs(pkv, S, W, NS, xs):
    """No special tokens, an empty sliding window, or both scale frames and
    window empty: after every frame the K/V tiles cover exactly the oracle's
    visible tokens (with W = 0 the frame just appended is already evicted)."""
    ps, n = 64, 40
    max_pages = S + W + 1 + math.ceil(NS * n / ps) + 1
    h = mk(pkv, S, W, ps, max_pages, NS=NS)
    pkv.kv_set_cross_frame_special(h, xs)
    m = PageModel(S, W, ps, max_pages, NS=NS, cross_frame_special=xs)
    try:
        for f in range(n):
            step(pkv, h)
            m.append(f)
            m.evict()
            p = pkv.kv_plan([h])
            try:
                want = [(pg, t) for _, pg in m.patch_pages_visible() for t in range(ps)]
                want += [(m.Np + j // ps, j % ps) for j in m.visible_special_index()]
                assert sorted(tile_cover(pkv.kv_get_kv_tiles(p), ps)) == sorted(want), f"frame {f}"
                assert pkv.kv_plan_get_stats(p)["visible_tokens"] == m.visible_token_count() == len(want)
            finally:
                pkv.kv_plan_free(p)
    finally:
        pkv.kv_destroy(h)


def test_unit_beyond_the_shared_tile_cache_host_plan(pkv):
    """The configuration of the GPU test of a CTA with more K/V tiles than its
    shared-memory cache of 512 descriptors: 16-token pages, S = 2, W = 600,
    620 frames, no split."""
    S, W, ps, frames = 2, 600, 16, 620
    h = mk(pkv, S, W, ps, (S + W + 1) + -(-6 * frames // ps), H=1)
    for _ in range(frames):
        step(pkv, h)
    p = pkv.kv_plan([h], tiles_per_split=4096)
    s = pkv.kv_plan_get_stats(p)
    assert s["n_ctas"] == 1 and s["tiles_per_cta"] == s["n_kv_tiles"] == 836 > 512
    assert s["visible_tokens"] == (S + W) * ps + 6 * frames
    pkv.kv_plan_free(p)


def test_in_kernel_merge_takes_at_most_32_chunks(pkv):
    """The attention CTAs merge a split group themselves only while the
    launch fits the device and no group has more than 32 chunks (the kernel
    marks a group's shares in a 32-bit mask): 32 chunks of one tile merge in
    the kernel, 54 run the merge as its own launch although their 108 CTAs
    would fit."""
    for W, frames, tiles, fused in ((20, 30, 32, 1), (40, 50, 54, 0)):
        h = mk(pkv, 8, W, 64, 200)
        for _ in range(frames):
            step(pkv, h)
        p = pkv.kv_plan([h], tiles_per_split=1)
        s = pkv.kv_plan_get_stats(p)
        assert s["n_kv_tiles"] == tiles and s["n_ctas"] == 2 * tiles <= 148
        assert s["fused_merge"] == fused
        pkv.kv_plan_free(p)
        pkv.kv_destroy(h)


def test_split_schedule_covers_each_unit(pkv):
    """Host plan for the 224x224 shape at frame 320: 160 tiles per head
    (71 earlier patch pages x 2, the current frame's page x 2, the earlier
    1914 special tokens in 15 tiles, the current frame's 6 in their own),
    16 heads x 3 query tiles (one pair-plus-tail unit per head); a forced
    split of 10 tiles per CTA."""
    h = pkv.kv_init(81, 256, 16, 64, 8, 64, 1, 6, pkv.KV_BF16, 0)
    for _ in range(320):
        step(pkv, h)
    p = pkv.kv_plan([h], tiles_per_split=10)
    s = pkv.kv_plan_get_stats(p)
    assert s["n_kv_tiles"] == 160
    assert s["visible_tokens"] == 72 * 256 + 6 * 320
    assert s["n_split_units"] == 48          # every (head, query tile) is split
    # per head one unit: query tiles 0-1 plus the 6-row tail tile 2, in
    # ceil(159/10) = 16 chunks
    assert s["n_ctas"] == 16 * 16
    assert s["tiles_per_cta"] <= 10
    assert s["fused_merge"] == 0             # 256 CTAs cannot all be resident: a merge launch
    pkv.kv_plan_free(p)
    p = pkv.kv_plan([h])                   # automatic: fills 148 SMs
    s = pkv.kv_plan_get_stats(p)
    assert 100 <= s["n_ctas"] <= 2 * 148 + 16
    # the automatic schedule fits one CTA per SM, so each split group merges itself
    assert s["n_ctas"] <= 148 and s["fused_merge"] == 1
    pkv.kv_plan_free(p)
    p = pkv.kv_plan([h], tiles_per_split=200)   # no split: nothing to merge
    assert pkv.kv_plan_get_stats(p)["fused_merge"] == 0
    pkv.kv_plan_free(p)
    pkv.kv_destroy(h)


def test_workspace_bytes_and_batch_checks(pkv):
    a = pkv.kv_init(81, 256, 8, 128, 8, 64, 2, 6, pkv.KV_FP16, 0)
    b = pkv.kv_init(81, 256, 8, 128, 8, 64, 2, 6, pkv.KV_FP16, 0)
    c = pkv.kv_init(81, 256, 8, 64, 8, 64, 2, 6, pkv.KV_FP16, 0)
    assert pkv.kv_workspace_bytes([a, b]) > pkv.kv_workspace_bytes([a]) > 0
    assert pkv.kv_workspace_bytes([a, c]) == 0        # mixed head_dim
    for x in (a, b):
        step(pkv, x, 2)
    p = pkv.kv_plan([a, b])
    assert pkv.kv_plan_get_stats(p)["n_streams"] == 2
    pkv.kv_plan_free(p)
    with pytest.raises(pkv.KVError):
        pkv.kv_plan([a, c])
    for x in (a, b, c):
        pkv.kv_destroy(x)


def test_run_static_argument_checks_before_any_device_work(pkv):
    """kv_run_static rejects bad calls on the host, before touching a device
    (so these run without a GPU)."""
    E = pkv.capi
    h = mk(pkv, 2, 4, 16, 12, B=2)
    q = out = 1 << 20                         # 16-byte aligned addresses that are never dereferenced

    def code(*args, **kw):
        with pytest.raises(pkv.KVError) as e:
            pkv.kv_run_static(*args, **kw)
        return e.value.code

    step(pkv, h, 1)                          # only block 0 appended in this step
    assert code([h], 0, None, out) == E.KV_ERR_ARG                  # NULL q
    assert code([h], 0, q, out, tiles_per_split=-1) == E.KV_ERR_ARG
    assert code([h], 0, q + 4, out) == E.KV_ERR_ARG                 # misaligned q
    assert code([h], 5, q, out) == E.KV_ERR_ARG                     # block out of range
    assert code([h], 1, q, out) == E.KV_ERR_NOT_APPENDED            # block 1 not appended yet
    assert code([h], 0, q, out) == E.KV_ERR_ARG                     # no pool bound for block 0
    assert code([], 0, q, out) == E.KV_ERR_ARG                      # no caches
    pkv.kv_destroy(h)


def test_run_static_python_checks_tensors_before_the_call(pkv):
    """The kv_run_static binding takes q and out as tensors and checks them
    against the caches' configuration ([sum of T, H, D], cache dtype,
    contiguous, CUDA) before any library call, as Plan.run does: the library
    would read and write exactly that many rows at their addresses."""
    import torch
    T, H, D = 16 + 6, 2, 64
    c = pkv.PagedKVCache(8, 16, H, D, scale_frames=1, window=2, num_blocks=1)
    c2 = pkv.PagedKVCache(8, 16, H, D, scale_frames=1, window=2, num_blocks=1)
    for bad, what in [(torch.zeros(T + 1, H, D, dtype=torch.bfloat16), "shape"),
                      (torch.zeros(T, H, D, dtype=torch.float16), "dtype"),
                      (torch.zeros(H, T, D, dtype=torch.bfloat16).transpose(0, 1), "contiguous"),
                      (torch.zeros(T, H, D, dtype=torch.bfloat16), "CUDA")]:
        with pytest.raises(ValueError, match=what):
            pkv.kv_run_static([c], 0, bad, bad)
        with pytest.raises(ValueError, match=what):      # raw handles are checked the same way
            pkv.kv_run_static([c.handle], 0, bad, bad)
    # two streams: 2 T rows
    with pytest.raises(ValueError, match="expected \\(44, 2, 64\\)"):
        pkv.kv_run_static([c, c2], 0, torch.zeros(T, H, D, dtype=torch.bfloat16), None)


def test_get_config_reports_what_init_fixed(pkv):
    h = pkv.kv_init(90, 256, 16, 64, 8, 64, 24, num_special=6, dtype=pkv.KV_FP16)
    cfg = pkv.kv_get_config(h)
    assert cfg == {"max_pages": 90, "page_size": 256, "num_heads": 16, "head_dim": 64, "scale_frames": 8,
                   "window": 64, "num_blocks": 24, "num_special": 6, "dtype": pkv.KV_FP16,
                   "patch_pages": 73, "special_base": 73, "special_pages": 17, "tokens_per_frame": 262,
                   "cross_frame_special": 1, "camera_only": 0}
    pkv.kv_set_cross_frame_special(h, False)
    assert pkv.kv_get_config(h)["cross_frame_special"] == 0
    pkv.kv_destroy(h)
    h = pkv.kv_init(100, 16, 2, 64, 2, 4, 1, patch_pages=88)
    assert pkv.kv_get_config(h)["patch_pages"] == 88
    pkv.kv_destroy(h)


def test_cross_frame_special_setting_changes_the_visible_rows(pkv):
    """Switching cross-frame special retention changes what the next plan
    attends to (here: 2 patch frames of 16 plus 24 special tokens, then plus
    only frames 0 and 3's 12); switching to the current value changes nothing."""
    h = mk(pkv, 1, 1, 16, 10)
    for _ in range(4):
        step(pkv, h)

    def visible():
        p = pkv.kv_plan([h])
        try:
            return pkv.kv_plan_get_stats(p)["visible_tokens"], tile_cover(pkv.kv_get_kv_tiles(p), 16)
        finally:
            pkv.kv_plan_free(p)

    n_on, cover_on = visible()
    pkv.kv_set_cross_frame_special(h, True)   # already on: no change
    assert visible() == (n_on, cover_on)
    pkv.kv_set_cross_frame_special(h, False)
    n_off, cover_off = visible()
    assert (n_on, n_off) == (2 * 16 + 24, 2 * 16 + 12)
    m = PageModel(1, 1, 16, 10, cross_frame_special=False)
    for f in range(4):
        m.append(f); m.evict()
    want = [(pg, t) for _, pg in m.patch_pages_visible() for t in range(16)]
    want += [(m.Np + j // 16, j % 16) for j in m.visible_special_index()]
    assert sorted(cover_off) == sorted(want)
    pkv.kv_destroy(h)


def test_object_api_checks_tensors_before_the_call(pkv):
    """The library sees only addresses, so PagedKVCache and Plan check each
    tensor's shape, dtype, layout and device first; a refused call leaves the
    page state untouched."""
    import torch
    T, H, D = 16 + 6, 2, 64
    c = pkv.PagedKVCache(8, 16, H, D, scale_frames=1, window=2, num_blocks=1)
    on_cpu = torch.zeros(T, H, D, dtype=torch.bfloat16)
    for bad, what in [(torch.zeros(T - 1, H, D, dtype=torch.bfloat16), "shape"),
                      (torch.zeros(T, H, D, dtype=torch.float16), "dtype"),
                      (torch.zeros(H, T, D, dtype=torch.bfloat16).transpose(0, 1), "contiguous"),
                      (on_cpu, "CUDA")]:
        with pytest.raises(ValueError, match=what):
            c.append_frame(0, bad, bad)
    assert c.get_stats()["frame_count"] == 0
    with pytest.raises(ValueError, match="bytes"):
        c.bind_pool(0, torch.zeros(16, dtype=torch.uint8))
    c.append_frame(0, None, None)
    p = pkv.Plan([c])
    with pytest.raises(ValueError, match="shape"):
        p.run(0, torch.zeros(T + 1, H, D, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="CUDA"):
        p.run(0, on_cpu)
    # a torch dtype selects the same kernels and pool dtype as its name
    f16 = pkv.PagedKVCache(8, 16, H, D, 1, 2, num_blocks=1, dtype=torch.float16)
    with pytest.raises(ValueError, match="dtype"):
        f16.append_frame(0, on_cpu, on_cpu)
    assert f16.fp16 and not c.fp16


def test_inspection_calls_copy_at_most_cap_and_check_ranges(pkv):
    """kv_get_page_table / kv_get_kv_tiles / kv_get_free_list write at most
    `cap` entries and always report the full count; stream indices are
    range-checked; a batch may hold at most KV_MAX_STREAMS streams."""
    import ctypes
    lib, E = pkv.capi.lib(), pkv.capi
    h = mk(pkv, 2, 3, 16, 12)
    for _ in range(7):
        step(pkv, h)
    p = pkv.kv_plan([h])
    full, lpl_full = pkv.kv_get_page_table(p)
    assert len(full) > 3
    buf = (ctypes.c_int * 8)(*([-7] * 8))
    n, lpl = ctypes.c_int(), ctypes.c_int()
    assert lib.kv_get_page_table(p, 0, buf, 2, ctypes.byref(n), ctypes.byref(lpl)) == 0
    assert n.value == len(full) and lpl.value == lpl_full
    assert list(buf[:2]) == full[:2] and list(buf[2:]) == [-7] * 6
    tiles = pkv.kv_get_kv_tiles(p)
    row, lo, hi, kr, sp = ((ctypes.c_int * 4)(*([-7] * 4)) for _ in range(5))
    assert lib.kv_get_kv_tiles(p, 0, row, lo, hi, kr, sp, 1, ctypes.byref(n)) == 0
    assert n.value == len(tiles) and (row[0], lo[0], hi[0]) == tiles[0] and row[1] == -7 and kr[1] == -7
    assert sp[0] == 1 and sp[1] == -7
    assert lib.kv_get_kv_tiles(p, 0, row, lo, hi, None, None, 1, ctypes.byref(n)) == 0   # krow, step optional
    free = pkv.kv_get_free_list(h)
    fb = (ctypes.c_int * 4)(*([-7] * 4))
    assert lib.kv_get_free_list(h, fb, 1, ctypes.byref(n)) == 0
    assert n.value == len(free) and fb[1] == -7
    for bad in (-1, 1):
        with pytest.raises(pkv.KVError) as e:
            pkv.kv_get_page_table(p, bad)
        assert e.value.code == E.KV_ERR_ARG
        with pytest.raises(pkv.KVError) as e:
            pkv.kv_get_kv_tiles(p, bad)
        assert e.value.code == E.KV_ERR_ARG
    pkv.kv_plan_free(p)
    many = [h] * (pkv.KV_MAX_STREAMS + 1)
    with pytest.raises(pkv.KVError) as e:
        pkv.kv_plan(many)
    assert e.value.code == E.KV_ERR_CAPACITY
    assert pkv.kv_workspace_bytes(many) == 0
    pkv.kv_destroy(h)


def snapshot(pkv, h):
    s = pkv.kv_get_stats(h)
    free = pkv.kv_get_free_list(h)
    try:
        tab = table(pkv, [h])
    except pkv.KVError as e:
        tab = e.value.name if hasattr(e, "value") else e.name
    return s, free, tab


@settings(max_examples=60, deadline=None)
@given(ops=st.lists(st.sampled_from(["key", "key", "defer_keep", "defer_drop"]), min_size=1, max_size=30),
       S=st.integers(0, 2), W=st.integers(0, 3), B=st.integers(1, 3), xs=st.booleans())
def test_begin_frame_is_the_step_opening_append(pkv, ops, S, W, B, xs):
    """A step opened by kv_begin_frame, then every block appended, leaves the
    page state a step opened by the first block's append leaves: same stats,
    free list and page table after every operation."""
    a = mk(pkv, S, W, 16, S + W + 1 + 20, B=B)
    b = mk(pkv, S, W, 16, S + W + 1 + 20, B=B)
    for h in (a, b):
        pkv.kv_set_cross_frame_special(h, xs)
    for op in ops:
        defer = op != "key"
        for h in (a, b):
            pkv.kv_defer_eviction(h, defer)
        pkv.kv_begin_frame(b)
        for blk in range(B):
            pkv.kv_append_frame(a, blk, None, None)
            pkv.kv_append_frame(b, blk, None, None)
            if blk == 0:
                assert snapshot(pkv, a) == snapshot(pkv, b)
        for h in (a, b):
            pkv.kv_evict_frames(h)
            if op == "defer_keep":
                pkv.kv_commit_frame(h)
            elif op == "defer_drop":
                pkv.kv_rollback_last_frame(h)
        assert snapshot(pkv, a) == snapshot(pkv, b)
    pkv.kv_destroy(a)
    pkv.kv_destroy(b)


def test_begin_frame_errors_leave_the_state_unchanged(pkv):
    E = pkv.capi
    h = mk(pkv, 1, 1, 16, 4, B=2)               # patch pool S + W + 1 = 3 pages, 1 special page
    pkv.kv_begin_frame(h)
    before = snapshot(pkv, h)
    with pytest.raises(pkv.KVError) as e:        # the open step still has blocks to append
        pkv.kv_begin_frame(h)
    assert e.value.code == E.KV_ERR_ORDER and snapshot(pkv, h) == before
    pkv.kv_append_frame(h, 0, None, None)
    with pytest.raises(pkv.KVError) as e:        # block 1 still to append
        pkv.kv_begin_frame(h)
    assert e.value.code == E.KV_ERR_ORDER
    pkv.kv_append_frame(h, 1, None, None)
    pkv.kv_evict_frames(h)
    pkv.kv_begin_frame(h)                        # the step is complete: a new one opens
    assert pkv.kv_get_stats(h)["frame_count"] == 2
    for blk in range(2):
        pkv.kv_append_frame(h, blk, None, None)
    pkv.kv_evict_frames(h)
    # 16-token special page: 2 frames of 6 fit, a third does not
    before = snapshot(pkv, h)
    with pytest.raises(pkv.KVError) as e:
        pkv.kv_begin_frame(h)
    assert e.value.code == E.KV_ERR_CAPACITY and snapshot(pkv, h) == before
    # a pending frame of an earlier step must be decided first
    h2 = mk(pkv, 1, 1, 16, 20, B=1)
    pkv.kv_defer_eviction(h2, True)
    pkv.kv_begin_frame(h2)
    pkv.kv_append_frame(h2, 0, None, None)
    with pytest.raises(pkv.KVError) as e:
        pkv.kv_begin_frame(h2)
    assert e.value.code == E.KV_ERR_ORDER
    pkv.kv_rollback_last_frame(h2)
    assert pkv.kv_get_stats(h2)["frame_count"] == 0
    pkv.kv_destroy(h)
    pkv.kv_destroy(h2)


def test_run_append_argument_checks_on_the_host(pkv):
    E = pkv.capi
    h = mk(pkv, 1, 2, 16, 8)
    pkv.kv_begin_frame(h)
    p = pkv.kv_plan([h])                          # host-only plan: no workspace
    a = 1 << 20
    for args, code in [((p, 0, None, a, a, a), E.KV_ERR_ARG),     # NULL k
                       ((p, 0, a, None, a, a), E.KV_ERR_ARG),     # NULL v
                       ((p, 0, a, a, a, a), E.KV_ERR_ARG)]:       # plan without a workspace
        with pytest.raises(pkv.KVError) as e:
            pkv.kv_run_append(*args)
        assert e.value.code == code
    pkv.kv_plan_free(p)
    pkv.kv_destroy(h)


def test_current_frame_tiles_carry_their_k_v_rows(pkv):
    """The open step's frame is tiled on its own, each tile with the k/v row
    of its column 0: its patch page (rows NS.. of k/v) and its NS special
    tokens (rows 0..NS-1); other tiles carry none. Checked through the
    coverage: every visible token once, the frame's tokens on current tiles."""
    ps, S, W = 256, 8, 64
    h = mk(pkv, S, W, ps, 73 + 9, B=2)
    for f in range(100):
        step(pkv, h, B=2)
    pkv.kv_begin_frame(h)                         # frame 100 opens: page and special slots 600..605
    pkv.kv_evict_frames(h)
    p = pkv.kv_plan([h])
    s = pkv.kv_plan_get_stats(p)
    tiles = pkv.kv_get_kv_tiles(p)
    # 71 earlier patch pages (2 tiles each), the frame's page (2), the earlier
    # 600 special tokens (5 tiles), the frame's 6 (1 tile)
    assert s["n_kv_tiles"] == len(tiles) == 142 + 2 + 5 + 1
    cover = tile_cover(tiles, ps)
    assert len(cover) == len(set(cover)) == s["visible_tokens"] == 72 * ps + 606
    # the frame's tokens are exactly the current tiles' columns, mapped to
    # their k/v rows: special token 600 + i is row i, patch slot x row 6 + x
    page = pkv.kv_get_free_list(h)  # noqa: F841  (the page is read from the table below)
    frame_page = pkv.kv_get_page_table(p)[0][71]          # scale 8 + window 64, the newest last
    Np = 73
    got = {}
    for row, lo, hi, kr, _ in pkv.kv_get_kv_tiles(p, with_krow=True):
        for col in range(lo, hi):
            tok = divmod(row + col, 2 * ps)
            if kr == pkv.KV_NOT_CURRENT:
                assert tok[0] != frame_page and not (tok[0] == Np + 2 and 88 <= tok[1] < 94)
            else:
                got[tok] = kr + col
    want = {(frame_page, x): 6 + x for x in range(ps)}
    want.update({(Np + 2, 88 + i): i for i in range(6)})   # tokens 600..605: page 2, slots 88..93
    assert got == want
    pkv.kv_plan_free(p)
    pkv.kv_destroy(h)


def strided_cover(tiles, ps):
    """(page, token) pairs that (row, lo, hi, krow, step) tiles mark visible."""
    out = []
    for row, lo, hi, _, step in tiles:
        for col in range(lo, hi, step):
            page, rem = divmod(row + col, 2 * ps)
            assert rem < ps, "a visible column must be a K row of its page"
            out.append((page, rem))
    return out


@pytest.mark.parametrize("xs", [True, False])
@pytest.mark.parametrize("ps,n", [(16, 12), (256, 320), (999, 40), (130, 150), (64, 100), (7, 30)])
def test_camera_only_tiles_cover_the_camera_tokens(pkv, ps, n, xs):
    """kv_set_camera_only: the tiles cover exactly the oracle's visible camera
    tokens (slot 0 of each frame's six), each once, with the open step's own
    camera token on a current-frame tile that maps it to k/v row 0; the page
    table is the oracle's; the page state is as without camera-only."""
    S, W = 8, 64
    pages = math.ceil(6 * (n + 1) / ps) + 1
    h = mk(pkv, S, W, ps, 73 + pages)
    ref = mk(pkv, S, W, ps, 73 + pages)
    for c in (h, ref):
        pkv.kv_set_cross_frame_special(c, xs)
    pkv.kv_set_camera_only(h, True)
    assert pkv.kv_get_config(h)["camera_only"] == 1
    m = PageModel(S, W, ps, 73 + pages, cross_frame_special=xs, camera_only=True)
    for f in range(n):
        step(pkv, h)
        step(pkv, ref)
        m.append(f); m.evict()
    pkv.kv_begin_frame(h)                     # an open step: the frame's tiles are separate
    pkv.kv_evict_frames(h)
    m.append(n); m.evict()
    p = pkv.kv_plan([h])
    assert pkv.kv_get_page_table(p) == m.page_table()
    tiles = pkv.kv_get_kv_tiles(p, with_krow=True)
    want = sorted((m.Np + j // ps, j % ps) for j in m.visible_special_index())
    assert sorted(strided_cover(tiles, ps)) == want
    assert pkv.kv_plan_get_stats(p)["visible_tokens"] == m.visible_token_count() == len(want)
    own = [(row, lo, hi, kr) for row, lo, hi, kr, _ in tiles if kr != pkv.KV_NOT_CURRENT]
    assert len(own) == 1 and own[0][3] + own[0][1] == 0          # column lo is k/v row 0
    assert divmod(own[0][0] + own[0][1], 2 * ps) == (m.Np + 6 * n // ps, 6 * n % ps)
    pkv.kv_plan_free(p)
    step(pkv, ref)
    for blk in range(1):
        pkv.kv_append_frame(h, blk, None, None)
    assert pkv.kv_get_stats(h) == pkv.kv_get_stats(ref)
    assert pkv.kv_get_free_list(h) == pkv.kv_get_free_list(ref)
    pkv.kv_destroy(h)
    pkv.kv_destroy(ref)


@settings(max_examples=80, deadline=None)
@given(ops=st.lists(st.tuples(st.integers(0, 2), st.sampled_from(["key", "key", "defer_keep", "defer_drop",
                                                                  "reset"])), min_size=1, max_size=60),
       S=st.integers(0, 2), W=st.integers(0, 3), ps=st.sampled_from([5, 16]),
       short=st.booleans())
def test_group_state_bit_exact_vs_oracle(pkv, ops, S, W, ps, short):
    """kv_init_group: three streams over one pool. Free list (common), stats
    and page tables after every operation equal the oracle's shared page
    models; with a common patch pool smaller than the
    streams' sum, an append that finds it empty fails with KV_ERR_CAPACITY
    and changes nothing."""
    from oracle import SharedPatchPool
    n, sp_pages = 3, 12
    Np = n * (S + W + 1) - (2 if short else 0)
    if Np < 1:
        return
    max_pages = Np + n * sp_pages
    hs = pkv.kv_init_group(n, max_pages, ps, 2, 64, S, W, 1, 6, pkv.KV_BF16, Np, sp_pages)
    pool = SharedPatchPool(Np)
    ms = [PageModel(S, W, ps, max_pages, NS=6, shared=pool, sp_base=Np + i * sp_pages, sp_pages=sp_pages)
          for i in range(n)]
    nxt = [0] * n
    for s_i, op in ops:
        h, m = hs[s_i], ms[s_i]
        if op == "reset":
            pkv.kv_reset(h)
            m.reset()
            nxt[s_i] = 0
        elif m.sp_len + 6 <= m.special_capacity:
            d = op != "key"
            pkv.kv_defer_eviction(h, d)
            m.set_defer(d)
            if not pool.free:
                with pytest.raises(pkv.KVError) as e:
                    pkv.kv_append_frame(h, 0, None, None)
                assert e.value.name == "CAPACITY"
                pkv.kv_defer_eviction(h, False)
                m.set_defer(False)
            else:
                pkv.kv_append_frame(h, 0, None, None)
                pkv.kv_evict_frames(h)
                m.append(nxt[s_i])
                m.evict()
                nxt[s_i] += 1
                if d:
                    if op == "defer_keep":
                        pkv.kv_commit_frame(h); m.commit()
                    else:
                        pkv.kv_rollback_last_frame(h); m.rollback()
                        nxt[s_i] -= 1
        for hh, mm in zip(hs, ms):
            assert pkv.kv_get_free_list(hh) == pool.free
            assert pkv.kv_get_stats(hh) == mm.stats()
            assert_same_table(pkv, hh, mm)
    cfg = [pkv.kv_get_config(h) for h in hs]
    assert [c["special_base"] for c in cfg] == [Np + i * sp_pages for i in range(n)]
    assert all(c["patch_pages"] == Np and c["special_pages"] == sp_pages for c in cfg)
    for h in hs:
        pkv.kv_destroy(h)


def test_group_argument_checks(pkv):
    E = pkv.capi
    with pytest.raises(pkv.KVError) as e:          # 3 x (8 + 64 + 1) patch pages + 3 x 10 special > 240
        pkv.kv_init_group(3, 240, 256, 16, 64, 8, 64, 24, special_pages=10)
    assert e.value.code == E.KV_ERR_CAPACITY
    hs = pkv.kv_init_group(3, 3 * 73 + 30, 256, 16, 64, 8, 64, 24)   # defaults: 219 patch, 10 special each
    cfg = pkv.kv_get_config(hs[2])
    assert (cfg["patch_pages"], cfg["special_base"], cfg["special_pages"]) == (219, 239, 10)
    assert pkv.kv_pool_bytes(hs[0]) == (3 * 73 + 30) * 2 * 256 * 16 * 64 * 2
    with pytest.raises(pkv.KVError) as e:
        pkv.kv_init_group(0, 100, 16, 2, 64, 1, 1, 1)
    assert e.value.code == E.KV_ERR_ARG
    for h in hs:
        pkv.kv_destroy(h)
