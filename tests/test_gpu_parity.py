"""GPU parity: the CUDA path through the C-ABI against the CPU oracle.

Bit-exact: pool contents after every append (scatter), page tables.
Attention: max |err| <= 2e-2 and mean |err| <= 2e-3 against the float64
oracle on unit-variance bf16/fp16 inputs.
"""
import dataclasses

import numpy as np
import pytest
import torch

import workload
from oracle import PageModel, PoolImage
from oracle.stream import StreamOracle, bits16

from gpu_drive import Frames, assert_close, new_cache, run_stream, workspace

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pkv():
    from paged_kv_cache_frame_b200 import build
    build.build()
    import paged_kv_cache_frame_b200 as m
    return m


W0 = workload.WORKLOADS[0]


def small(ps, H=2, D=64, S=2, W=3, dtype="bf16", frames=20):
    return dataclasses.replace(W0, name=f"ps{ps}", H=H, D=D, P=ps, page_size=ps, S=S, W=W,
                               frames=frames, dtype=dtype)


# --------------------------------------------------------------- append scatter
@pytest.mark.parametrize("wl", [W0, small(256), small(999, H=1), small(130), small(64, D=128, dtype="fp16")],
                         ids=lambda w: w.name)
def test_append_scatter_pool_bit_exact(pkv, wl):
    fr = Frames(wl, seed=7)
    cache = new_cache(pkv, wl)
    m = PageModel(wl.S, wl.W, wl.page_size, wl.max_pages, NS=wl.NS)
    img = PoolImage(m, wl.H, wl.D)
    rng = np.random.default_rng(3)
    for f in range(14):
        _, k, v = fr.get(f)
        defer = bool(rng.random() < 0.3)
        cache.defer_eviction(defer)
        m.set_defer(defer)
        cache.append_frame(0, k.cuda(), v.cuda())
        cache.evict_frames()
        page, sp0 = m.append(f)
        m.evict()
        img.write(page, sp0, bits16(k), bits16(v))
        pool = cache.pools[0].cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
        np.testing.assert_array_equal(pool, img.bits, err_msg=f"frame {f}")
        if defer:
            if rng.random() < 0.5:
                cache.commit_frame(); m.commit()
            else:
                cache.rollback_last_frame(); m.rollback()
        assert cache.free_list() == m.free


# --------------------------------------------------------------- attention
def test_tiny_config_every_frame_every_row(pkv):
    res = run_stream(pkv, W0, seed=11, n_frames=W0.frames, check=set(range(W0.frames)))
    assert len(res) == W0.frames


@pytest.mark.parametrize("tps", [1, 2, 3])
def test_forced_split_kv_matches_oracle(pkv, tps):
    run_stream(pkv, W0, seed=12, n_frames=12, check={0, 5, 11}, tiles_per_split=tps)
    wl = small(256, frames=9)
    run_stream(pkv, wl, seed=13, n_frames=9, check={8}, tiles_per_split=tps)


def test_split_and_unsplit_agree(pkv):
    wl = small(256, H=3, S=2, W=4, frames=8)
    a, b = {}, {}
    run_stream(pkv, wl, seed=14, n_frames=8, check={7}, collect=a)
    run_stream(pkv, wl, seed=14, n_frames=8, check={7}, tiles_per_split=2, collect=b)
    d = (a[7].float() - b[7].float()).abs()
    assert d.max().item() <= 1e-2


# Frame sizes around the tail limits: T = P + 6 rows make full 128-row query
# tiles plus a remainder r. r <= 16 (head_dim 64) or r <= 8 (head_dim 128)
# runs on the tail warps -- one 8-row group for r <= 8, two above -- and a
# larger remainder is a query tile of its own.
@pytest.mark.parametrize("ps,D", [(123, 64), (131, 64), (138, 64), (139, 64), (259, 64), (266, 64),
                                  (130, 128), (131, 128)],
                         ids=lambda x: str(x))
def test_tail_sizes(pkv, ps, D):
    dtype = "fp16" if D == 128 else "bf16"
    wl = small(ps, H=2, D=D, S=2, W=3, dtype=dtype, frames=7)
    T = ps + 6
    run_stream(pkv, wl, seed=50 + ps + D, n_frames=wl.frames, check={0, 6}, rows=np.arange(T))
    run_stream(pkv, wl, seed=60 + ps + D, n_frames=wl.frames, check={6}, rows=np.arange(T), fused=True)
    run_stream(pkv, wl, seed=70 + ps + D, n_frames=wl.frames, check={6}, rows=np.arange(T), tiles_per_split=1)


class SpikeFrames(Frames):
    """Every query row near one vector u (per head) and a few keys equal to
    c * u, so that their scores stand far above the rest: in log2 units a key
    c * u scores about c * |u|^2 / sqrt(D) * log2(e), about 11.5 c here, while
    the other keys' maximum is about 6."""

    def __init__(self, wl, seed, spikes):
        super().__init__(wl, seed)
        g = torch.Generator().manual_seed(seed)
        self.u = torch.randn(wl.H, wl.D, generator=g)
        self.spikes = spikes   # {(frame, patch token): c}

    def get(self, f):
        if f not in self.cache:
            q, k, v = (x.float() for x in workload.frame_qkv(self.wl, self.seed, f, 0))
            q = self.u.unsqueeze(0) + 0.1 * q
            for (ff, p), c in self.spikes.items():
                if ff == f:
                    k[self.wl.NS + p] = c * self.u
            dt = self.wl.torch_dtype()
            self.cache[f] = (q.to(dt), k.to(dt), v.to(dt))
        return self.cache[f]


@pytest.mark.parametrize("fused,tps", [(False, 4096), (True, 4096), (False, 0)])
def test_running_max_jumps_force_both_rescales(pkv, fused, tps):
    """Spike keys move the running max past the 2^8 lazy threshold. The first
    sits in the second 64-key half of the stream's first tile, so it raises
    the max (by 9 in head 0, 14 in head 1, log2 units) after the first half's
    P was stored, which is then scaled down in TMEM. The second, in a first
    half four frames later, raises it again by 10 in head 1 (O rescaled after
    earlier PVs) and by 7 in head 0 (under the threshold: no rescale). The
    stale terms a rescale scales would otherwise weigh 2^8 times too much.
    Frames 0 and 1 are scale frames, so the first spike stays visible. Without
    a split (tiles_per_split 4096) both jumps fall inside one CTA's tiles."""
    wl = small(256, H=2, S=2, W=3, frames=7)
    fr = SpikeFrames(wl, 77, {(0, 100): 1.4, (5, 10): 2.13})
    run_stream(pkv, wl, seed=77, n_frames=wl.frames, check={1, 5, 6}, rows=np.arange(wl.T), frames=fr,
               fused=fused, tiles_per_split=tps)


def test_unit_with_more_tiles_than_the_shared_tile_cache(pkv):
    """One unsplit CTA over 836 K/V tiles (16-token pages, one tile per page,
    and a 600-frame window; the host plan's tile count is checked in
    test_capi_host). A CTA caches 512 tile descriptors in shared
    memory and reads the rest from global memory; both kinds of tile are
    checked against the oracle, through both frame-step forms."""
    wl = small(16, H=1, S=2, W=600, frames=620)
    run_stream(pkv, wl, seed=41, n_frames=wl.frames, check={wl.frames - 1}, tiles_per_split=4096)
    run_stream(pkv, wl, seed=42, n_frames=wl.frames, check={wl.frames - 1}, tiles_per_split=4096, fused=True)


@pytest.mark.parametrize("ps", [16, 64, 100, 128, 129, 256, 999])
def test_page_sizes_with_eviction(pkv, ps):
    wl = small(ps, H=2, S=2, W=3, frames=12)
    run_stream(pkv, wl, seed=20 + ps, n_frames=12, check={0, 1, 4, 5, 6, 11})


def test_head_dim_128_fp16(pkv):
    wl = small(256, H=2, D=128, dtype="fp16", frames=10)
    run_stream(pkv, wl, seed=31, n_frames=10, check={0, 9})
    run_stream(pkv, wl, seed=32, n_frames=10, check={9}, tiles_per_split=2)


def test_deferred_frames_commit_and_rollback(pkv):
    wl = small(256, H=2, S=2, W=3, frames=24)
    keep = workload.keyframe_mask(dataclasses.replace(wl, keyframes="bernoulli"), seed=5)
    defer = np.ones(wl.frames, dtype=bool)          # every frame deferred, decided after
    run_stream(pkv, wl, seed=33, n_frames=wl.frames, check=set(range(wl.frames)), defer=defer,
               keep=keep)
    # interval mode: non-keyframes deferred then rolled back, keyframes appended directly
    k4 = workload.interval_mask(wl.frames, 4)
    run_stream(pkv, wl, seed=34, n_frames=wl.frames, check=set(range(0, wl.frames, 3)),
               defer=~k4, keep=k4)


def test_patch_pool_size_does_not_change_results(pkv):
    """Relabelling the special pages (a larger patch pool moves them) gives
    bit-identical outputs: the kernel reads pages only through the table."""
    wl = small(256, H=2, S=2, W=3, frames=9)
    a, b = {}, {}
    run_stream(pkv, wl, seed=35, n_frames=9, check={8}, collect=a)
    run_stream(pkv, wl, seed=35, n_frames=9, check={8}, collect=b, patch_pages=wl.patch_pages + 7)
    assert torch.equal(a[8], b[8])


def test_batched_streams_ragged_ages(pkv):
    wl = small(256, H=2, D=128, dtype="fp16", S=2, W=3, frames=16)
    ages = [3, 9, 1, 14]
    caches, oracles, qs = [], [], []
    for s, age in enumerate(ages):
        fr = Frames(wl, seed=40, stream=s)
        c = new_cache(pkv, wl)
        so = StreamOracle(wl.S, wl.W, wl.NS, wl.P, wl.dtype, fr.bits)
        for f in range(age):
            q, k, v = fr.get(f)
            c.append_frame(0, k.cuda(), v.cuda())
            c.evict_frames()
            so.begin_frame(f)
        caches.append(c)
        oracles.append(so)
        qs.append(q)
    ws = workspace(pkv, caches)
    plan = pkv.Plan(caches, ws)
    q = torch.cat(qs).cuda()
    out = plan.run(0, q)
    plan.check_device()
    for s, so in enumerate(oracles):
        assert_close(out[s * wl.T:(s + 1) * wl.T], so.expected(), f"stream {s}")


def test_closed_forms_on_gpu(pkv):
    """Constant V gives that constant; identical keys give the mean of V."""
    wl = small(128, H=2, S=1, W=2, frames=4)
    cache = new_cache(pkv, wl)
    ws = workspace(pkv, [cache])
    g = torch.Generator().manual_seed(0)
    vs = []
    for f in range(3):
        q = torch.randn(wl.T, wl.H, wl.D, generator=g).bfloat16()
        k = torch.full((wl.T, wl.H, wl.D), 0.5).bfloat16()
        v = torch.full((wl.T, wl.H, wl.D), 0.75).bfloat16()
        v[:, 1] = torch.randn(wl.T, wl.D, generator=g).bfloat16()
        vs.append(v)
        cache.append_frame(0, k.cuda(), v.cuda())
        cache.evict_frames()
    out = pkv.Plan([cache], ws).run(0, q.cuda()).float().cpu()
    assert torch.all(out[:, 0] == 0.75)
    # head 1: all keys equal -> uniform weights over the 3 * 134 visible tokens
    allv = torch.cat([x[:, 1].float() for x in vs])
    mean = allv.mean(0)
    assert (out[:, 1] - mean).abs().max().item() < 4e-3


def test_run_errors(pkv):
    wl = small(64, H=2, frames=3)
    cache = new_cache(pkv, wl, num_blocks=1)
    ws = workspace(pkv, [cache])
    fr = Frames(wl, seed=50)
    q, k, v = (x.cuda() for x in fr.get(0))
    cache.append_frame(0, k, v)
    plan = pkv.Plan([cache], ws)
    plan.run(0, q)
    cache.evict_frames()
    q, k, v = (x.cuda() for x in fr.get(1))
    cache.append_frame(0, k, v)                 # state changed: the plan is stale
    with pytest.raises(pkv.KVError) as e:
        plan.run(0, q)
    assert e.value.name == "STALE_PLAN"
    small_ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(pkv.KVError) as e:
        pkv.Plan([cache], small_ws)
    assert e.value.name == "CAPACITY"
    plan = pkv.Plan([cache], ws)
    plan.run(0, q)
    plan.check_device()


# --------------------------------------------------------------- full-size workloads
def sample_rows(T, seed, n=24):
    rng = np.random.default_rng(seed)
    return sorted(set([0, 1, 5, T - 1, 128, 255, 256, T - 6]) | set(rng.integers(0, T, n).tolist()))


def test_cross_frame_special_off_tiny_every_frame(pkv):
    """kv_cache_cross_frame_special = False: evicted frames' special tokens
    leave the visible set (a hidden range that starts and ends inside pages)."""
    wl = dataclasses.replace(W0, frames=30)
    res = run_stream(pkv, wl, seed=41, n_frames=wl.frames, check=set(range(wl.frames)), cross_special=False)
    assert len(res) == wl.frames


def test_cross_frame_special_off_224_with_keyframes(pkv):
    wl = dataclasses.replace(workload.WORKLOADS[2], frames=110)
    keep = workload.keyframe_mask(wl, seed=42)
    run_stream(pkv, wl, seed=42, n_frames=wl.frames, check={8, 72, 80, 109}, rows=sample_rows(wl.T, 42),
               defer=np.ones(wl.frames, dtype=bool), keep=keep, cross_special=False, dense={109})


def test_include_scale_frames_off_is_zero_scale_frames(pkv):
    """kv_cache_include_scale_frames = False is scale_frames = 0: a pure
    sliding window of W frames."""
    run_stream(pkv, dataclasses.replace(W0, S=0, frames=20), seed=43, n_frames=20, check=set(range(20)))
    wl = dataclasses.replace(workload.WORKLOADS[1], S=0, frames=90)
    run_stream(pkv, wl, seed=44, n_frames=wl.frames, check={63, 64, 89}, rows=sample_rows(wl.T, 44),
               dense={89})


@pytest.mark.parametrize("ps,D", [(128, 64), (130, 64), (64, 128), (136, 128)])
@pytest.mark.parametrize("fused", [False, True])
def test_no_special_tokens(pkv, ps, D, fused):
    """num_special = 0: a frame is its patch tokens alone (T = page size), the
    special stream stays empty and only patch pages are visible. 128 rows are
    one full query tile with no tail, 130 and 136 leave a tail of 2 and 8
    rows, 64 rows a partial tile; every row of every frame is checked."""
    wl = dataclasses.replace(small(ps, D=D, dtype="fp16" if D == 128 else "bf16", frames=14), NS=0)
    assert wl.T == ps
    run_stream(pkv, wl, seed=140 + ps, n_frames=wl.frames, check=set(range(wl.frames)), rows=np.arange(wl.T),
               fused=fused)


@pytest.mark.parametrize("S,xs", [(2, True), (2, False), (0, True)])
@pytest.mark.parametrize("fused", [False, True])
def test_empty_window(pkv, S, xs, fused):
    """sliding_window = 0: once the scale frames are set, a frame's patch
    tokens are evicted in the step that appends them, so its queries see the
    scale frames' patches and the special tokens only (with S = 0 the special
    tokens alone). The frame is still written to its page, which the next
    frame takes again."""
    wl = small(64, S=S, W=0, frames=12)
    run_stream(pkv, wl, seed=150 + S, n_frames=wl.frames, check=set(range(wl.frames)), rows=np.arange(wl.T),
               cross_special=xs, fused=fused)


def test_full_224_stream_block0_sampled(pkv):
    """Every row of the last frame against the oracle (and the fp32 gather),
    sampled rows elsewhere."""
    wl = workload.WORKLOADS[1]
    run_stream(pkv, wl, seed=1, n_frames=wl.frames, check={0, 71, 72, 159, 319},
               rows=sample_rows(wl.T, 1), dense={72, 319}, all_rows={319})


def test_full_224_stream_fused_all_rows(pkv):
    """The fused frame step (begin_frame + run_append) over the whole stream:
    every row against the oracle at the end of the window's ramp and at the
    last frame."""
    wl = workload.WORKLOADS[1]
    run_stream(pkv, wl, seed=6, n_frames=wl.frames, check={71, 200, 319}, rows=sample_rows(wl.T, 6),
               fused=True, all_rows={71, 319})


def test_full_224_keyframes_block0_sampled(pkv):
    wl = workload.WORKLOADS[2]
    keep = workload.keyframe_mask(wl, seed=2)
    run_stream(pkv, wl, seed=2, n_frames=wl.frames, check={50, 200, 319}, rows=sample_rows(wl.T, 2),
               defer=np.ones(wl.frames, dtype=bool), keep=keep)


def test_full_518x378_stream_block0_sampled(pkv):
    wl = workload.WORKLOADS[3]
    run_stream(pkv, wl, seed=3, n_frames=wl.frames, check={0, 499, 999},
               rows=sample_rows(wl.T, 3, n=12), dense={999}, fused=True)


def test_full_batched_ragged_sampled(pkv):
    wl = workload.WORKLOADS[4]
    ages = workload.stream_ages(wl, seed=4)
    caches, oracles, qs = [], [], []
    for s, age in enumerate(ages):
        fr = Frames(wl, seed=4, stream=s)
        c = new_cache(pkv, wl)
        so = StreamOracle(wl.S, wl.W, wl.NS, wl.P, wl.dtype, fr.bits)
        for f in range(int(age) + 1):
            q, k, v = fr.get(f)
            c.append_frame(0, k.cuda(), v.cuda())
            c.evict_frames()
            so.begin_frame(f)
        caches.append(c)
        oracles.append(so)
        qs.append(q)
    ws = workspace(pkv, caches)
    plan = pkv.Plan(caches, ws)
    out = plan.run(0, torch.cat(qs).cuda())
    plan.check_device()
    rows = sample_rows(wl.T, 4, n=8)
    full = {int(np.argmax(ages)), int(np.argmin(ages))}   # every row of the oldest and youngest stream
    for s, so in enumerate(oracles):
        r = None if s in full else rows
        got = out[s * wl.T:(s + 1) * wl.T]
        got = got if r is None else got[torch.as_tensor(r)]
        assert_close(got, so.expected(r), f"stream {s} age {ages[s]}")


def test_failed_append_launch_leaves_state_unchanged(pkv):
    """A scatter launch that fails (faked by kv_testing_fail_launches, so no
    GPU fault is involved) leaves the page state exactly as it was, whether
    the append would have opened a new frame step or not; the same call then
    succeeds, and pool and attention match the oracle."""
    wl = small(64, H=2, S=1, W=2, frames=8)
    cache = new_cache(pkv, wl, num_blocks=2)
    m = PageModel(wl.S, wl.W, wl.page_size, wl.max_pages, NS=wl.NS)
    imgs = [PoolImage(m, wl.H, wl.D) for _ in range(2)]
    frames = [Frames(wl, seed=61, block=b) for b in range(2)]

    def state():
        return cache.get_stats(), cache.free_list()

    for f in range(6):
        for b in range(2):
            _, k, v = frames[b].get(f)
            before = state()
            pkv.kv_testing_fail_launches(1)
            with pytest.raises(pkv.KVError) as e:
                cache.append_frame(b, k.cuda(), v.cuda())
            assert e.value.name == "CUDA"
            assert state() == before, f"frame {f} block {b}"
            cache.append_frame(b, k.cuda(), v.cuda())
            if b == 0:
                cache.evict_frames()
                page, sp0 = m.append(f)
                m.evict()
            imgs[b].write(page, sp0, bits16(k), bits16(v))
        assert cache.free_list() == m.free
    for b in range(2):
        pool = cache.pools[b].cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
        np.testing.assert_array_equal(pool, imgs[b].bits, err_msg=f"block {b}")
    pkv.kv_testing_fail_launches(0)
    so = StreamOracle(wl.S, wl.W, wl.NS, wl.P, wl.dtype, frames[1].bits)
    for f in range(6):
        so.begin_frame(f)
    plan = pkv.Plan([cache], workspace(pkv, [cache]))
    q = frames[1].get(5)[0].cuda()
    out = plan.run(1, q)
    plan.check_device()
    assert_close(out, so.expected(), "after failed launches")


@pytest.mark.parametrize("H,W,frames,tiles,fused", [(2, 40, 50, 54, 0), (4, 40, 50, 54, 0), (2, 20, 30, 32, 1)],
                         ids=["54-chunks-H2", "54-chunks-H4", "32-chunks-H2"])
def test_many_chunks_per_split_unit(pkv, H, W, frames, tiles, fused):
    """One K/V tile per CTA, so a unit has as many chunks as visible tiles
    (64-token pages, one tile each; the special tokens on their own pages,
    the open step's frame's 6 on a tile of their own). 54 chunks: more than
    the 32 the in-kernel merge takes (a 32-bit mask of shares), so the merge
    runs as its own launch, past its first 32-lane pass; with H = 4 the 216
    CTAs would not fit on the device at once either. 32 chunks with H = 2 (64
    CTAs): the CTAs merge their groups themselves, the mask full."""
    wl = small(64, H=H, S=8, W=W, frames=frames)
    fr = Frames(wl, seed=70)
    cache = new_cache(pkv, wl)
    so = StreamOracle(wl.S, wl.W, wl.NS, wl.P, wl.dtype, fr.bits)
    for f in range(wl.frames):
        q, k, v = (x.cuda() for x in fr.get(f))
        cache.append_frame(0, k, v)
        cache.evict_frames()
        so.begin_frame(f)
    plan = pkv.Plan([cache], workspace(pkv, [cache]), tiles_per_split=1)
    st = plan.stats()
    assert st["tiles_per_cta"] == 1 and st["n_kv_tiles"] == tiles
    assert st["fused_merge"] == fused
    for rep in range(2):   # the group counters must be back at zero for the second run
        out = plan.run(0, q)
        plan.check_device()
        assert_close(out, so.expected(), f"H={H} run {rep}")


@pytest.mark.parametrize("xs", [True, False])
@pytest.mark.parametrize("fused", [False, True])
def test_camera_only_tiny_every_frame(pkv, xs, fused):
    """kv_cache_camera_only: each frame attends to the camera tokens (slot 0
    of each frame's six) only; strided tiles over the special pages."""
    wl = dataclasses.replace(W0, frames=30)
    res = run_stream(pkv, wl, seed=90, n_frames=wl.frames, check=set(range(wl.frames)),
                     cross_special=xs, camera_only=True, fused=fused)
    assert len(res) == wl.frames


@pytest.mark.parametrize("ps", [16, 100, 256, 999])
def test_camera_only_page_sizes(pkv, ps):
    wl = small(ps, H=1 if ps == 999 else 2, S=2, W=3, frames=40)
    run_stream(pkv, wl, seed=91 + ps, n_frames=wl.frames, check={0, 5, 39}, camera_only=True)
    run_stream(pkv, wl, seed=92 + ps, n_frames=wl.frames, check={39}, camera_only=True, tiles_per_split=1)


@pytest.mark.parametrize("fused", [False, True])
def test_visibility_options_head_dim_128_fp16(pkv, fused):
    """camera_only and cross_frame_special = False on the head_dim 128 fp16
    path (P over S in two rotating buffers, a tail of at most 8 rows): 256
    patch tokens per frame, so each frame adds two full query tiles and a
    6-row tail; every row checked, with and without a split."""
    wl = small(256, H=2, D=128, dtype="fp16", S=2, W=3, frames=14)
    run_stream(pkv, wl, seed=95, n_frames=wl.frames, check={0, 6, 13}, rows=np.arange(wl.T), camera_only=True,
               fused=fused)
    run_stream(pkv, wl, seed=96, n_frames=wl.frames, check={13}, rows=np.arange(wl.T), camera_only=True,
               tiles_per_split=1, fused=fused)
    run_stream(pkv, wl, seed=97, n_frames=wl.frames, check={6, 13}, rows=np.arange(wl.T), cross_special=False,
               fused=fused)


def test_camera_only_224_stream(pkv):
    wl = dataclasses.replace(workload.WORKLOADS[1], frames=200)
    run_stream(pkv, wl, seed=93, n_frames=wl.frames, check={0, 100, 199}, rows=sample_rows(wl.T, 93),
               camera_only=True, fused=True)
