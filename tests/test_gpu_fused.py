"""GPU parity of kv_run_append: a block's K/V appended and its attention
computed in one launch.

Two caches take the same frames. Cache A runs the pages' sequence
append_frame -> evict -> plan -> run, a scatter launch then an attention
launch that reads the frame from the pool. Cache B runs begin_frame -> evict
-> plan -> run_append, one launch that writes the frame into the pool and
reads it from k/v. Both plans tile the frame the same way, so outputs must be
bit-identical, and so must the pools; the oracle checks the outputs and the
pool image on top.
"""
import dataclasses

import numpy as np
import pytest
import torch

import workload
from oracle import PageModel, PoolImage
from oracle.stream import StreamOracle, bits16

from gpu_drive import Frames, assert_close, new_cache, workspace

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


def pool_bits(cache, block=0):
    return cache.pools[block].cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def run_pair(pkv, wl, seed, n_frames, check=(), rows=None, defer=None, keep=None, tiles_per_split=0,
             check_pool=True, num_blocks=1):
    """Frames 0..n_frames-1 through both caches; bit-equal outputs every frame
    (every block), the oracle at frames in `check` (block 0) and the pool image
    after every frame when check_pool."""
    frames = [Frames(wl, seed, block=b) for b in range(num_blocks)]
    a = new_cache(pkv, wl, num_blocks=num_blocks)
    b = new_cache(pkv, wl, num_blocks=num_blocks)
    ws_a, ws_b = workspace(pkv, [a]), workspace(pkv, [b])
    so = StreamOracle(wl.S, wl.W, wl.NS, wl.P, wl.dtype, frames[0].bits)
    m = PageModel(wl.S, wl.W, wl.page_size, wl.max_pages, NS=wl.NS)
    img = PoolImage(m, wl.H, wl.D)
    for f in range(n_frames):
        d = bool(defer[f]) if defer is not None else False
        for c in (a, b):
            c.defer_eviction(d)
        m.set_defer(d)
        b.begin_frame()
        b.evict_frames()
        plan_b = pkv.Plan([b], ws_b, tiles_per_split=tiles_per_split)
        for blk in range(num_blocks):
            q, k, v = (x.cuda() for x in frames[blk].get(f))
            a.append_frame(blk, k, v)
            if blk == 0:
                a.evict_frames()
                plan_a = pkv.Plan([a], ws_a, tiles_per_split=tiles_per_split)
            out_a = plan_a.run(blk, q)
            out_b = plan_b.run_append(blk, k, v, q)
            plan_a.check_device()
            plan_b.check_device()
            assert torch.equal(out_a, out_b), f"frame {f} block {blk}: fused and unfused outputs differ"
            if blk == 0:
                page, sp0 = m.append(f)
                m.evict()
                so.begin_frame(f, d)
                _, k0, v0 = frames[0].get(f)
                img.write(page, sp0, bits16(k0), bits16(v0))
                if f in check:
                    sel = slice(None) if rows is None else torch.as_tensor(rows)
                    assert_close(out_b[sel], so.expected(rows), f"frame {f}")
        if check_pool:
            got = pool_bits(b)
            np.testing.assert_array_equal(got, img.bits, err_msg=f"frame {f}: pool after run_append")
        for blk in range(num_blocks):
            assert np.array_equal(pool_bits(a, blk), pool_bits(b, blk)), f"frame {f} block {blk}: pools differ"
        if d:
            kept = keep is None or bool(keep[f])
            for c in (a, b):
                c.commit_frame() if kept else c.rollback_last_frame()
            m.commit() if kept else m.rollback()
            so.end_frame(kept)
        assert a.free_list() == b.free_list() == m.free
        assert a.get_stats() == b.get_stats()


def test_tiny_every_frame_with_deferred_frames(pkv):
    wl = dataclasses.replace(W0, frames=24)
    keep = workload.keyframe_mask(dataclasses.replace(wl, keyframes="bernoulli"), seed=3)
    defer = np.random.default_rng(4).random(wl.frames) < 0.5
    run_pair(pkv, wl, seed=80, n_frames=wl.frames, check=set(range(wl.frames)), defer=defer, keep=keep)


@pytest.mark.parametrize("ps", [16, 64, 100, 128, 129, 256, 999])
def test_page_sizes(pkv, ps):
    wl = small(ps, H=1 if ps == 999 else 2, S=2, W=3, frames=10)
    run_pair(pkv, wl, seed=81 + ps, n_frames=wl.frames, check={0, 4, 9})


def test_two_blocks(pkv):
    wl = small(130, H=2, S=1, W=2, frames=6)
    run_pair(pkv, wl, seed=88, n_frames=wl.frames, check={5}, num_blocks=2)


def test_head_dim_128_fp16(pkv):
    wl = small(256, H=2, D=128, dtype="fp16", frames=8)
    run_pair(pkv, wl, seed=82, n_frames=wl.frames, check={0, 7})


@pytest.mark.parametrize("tps", [1, 2])
def test_forced_split(pkv, tps):
    """Every CTA appends its slice of the frame and the split groups merge
    themselves (one CTA per SM at these sizes)."""
    wl = small(256, H=2, S=2, W=3, frames=8)
    run_pair(pkv, wl, seed=83 + tps, n_frames=wl.frames, check={3, 7}, tiles_per_split=tps)


def test_full_224_stream_sampled(pkv):
    wl = workload.WORKLOADS[1]
    rows = sorted({0, 1, 5, 127, 128, 255, 256, 261} | set(np.random.default_rng(5).integers(0, 262, 16).tolist()))
    run_pair(pkv, wl, seed=85, n_frames=wl.frames, check={0, 71, 72, 319}, rows=rows, check_pool=False)


def test_batched_streams(pkv):
    """One plan over four streams of different ages: k, v, q rows of the
    streams concatenated; each stream's frame goes to its own pool."""
    wl = small(256, H=2, D=128, dtype="fp16", S=2, W=3, frames=16)
    ages = [3, 9, 1, 14]
    fused, plain, oracles, frs = [], [], [], []
    for s, age in enumerate(ages):
        fr = Frames(wl, seed=86, stream=s)
        ca, cb = new_cache(pkv, wl), new_cache(pkv, wl)
        so = StreamOracle(wl.S, wl.W, wl.NS, wl.P, wl.dtype, fr.bits)
        for f in range(age):
            _, k, v = (x.cuda() for x in fr.get(f))
            for c in (ca, cb):
                c.append_frame(0, k, v)
                c.evict_frames()
            so.begin_frame(f)
        plain.append(ca)
        fused.append(cb)
        oracles.append(so)
        frs.append(fr)
    qkv = [fr.get(age) for fr, age in zip(frs, ages)]
    q, k, v = (torch.cat([x[i] for x in qkv]).cuda() for i in range(3))
    for s, c in enumerate(fused):
        c.begin_frame()
        c.evict_frames()
        plain[s].append_frame(0, k[s * wl.T:(s + 1) * wl.T], v[s * wl.T:(s + 1) * wl.T])
        plain[s].evict_frames()
        oracles[s].begin_frame(ages[s])
    out_b = pkv.Plan(fused, workspace(pkv, fused)).run_append(0, k, v, q)
    out_a = pkv.Plan(plain, workspace(pkv, plain)).run(0, q)
    torch.cuda.synchronize()
    assert torch.equal(out_a, out_b)
    for s, so in enumerate(oracles):
        assert_close(out_b[s * wl.T:(s + 1) * wl.T], so.expected(), f"stream {s}")
        assert np.array_equal(pool_bits(plain[s]), pool_bits(fused[s])), f"stream {s} pool"


def test_run_append_order_errors(pkv):
    wl = small(64, H=2, frames=4)
    c = new_cache(pkv, wl, num_blocks=2)
    ws = workspace(pkv, [c])
    fr = Frames(wl, seed=87)
    q, k, v = (x.cuda() for x in fr.get(0))
    c.append_frame(0, k, v)                     # step opened by an append: block 1 may run_append
    c.evict_frames()
    plan = pkv.Plan([c], ws)
    with pytest.raises(pkv.KVError) as e:       # block 0 is already appended
        plan.run_append(0, k, v, q)
    assert e.value.name == "ORDER"
    plan.run_append(1, k, v, q)
    with pytest.raises(pkv.KVError) as e:       # and now block 1 too
        plan.run_append(1, k, v, q)
    assert e.value.name == "ORDER"
    plan.check_device()
    q, k, v = (x.cuda() for x in fr.get(1))
    c.append_frame(0, k, v)                     # a new step: the old plan is stale
    with pytest.raises(pkv.KVError) as e:
        plan.run_append(1, k, v, q)
    assert e.value.name == "STALE_PLAN"
    # a failed launch (faked) appends nothing; the same call then succeeds
    plan = pkv.Plan([c], ws)
    pkv.kv_testing_fail_launches(1)
    with pytest.raises(pkv.KVError) as e:
        plan.run_append(1, k, v, q)
    assert e.value.name == "CUDA"
    pkv.kv_testing_fail_launches(0)
    plan.run_append(1, k, v, q)
    plan.check_device()



@pytest.mark.parametrize("fused", [False, True])
def test_group_of_streams_sharing_one_pool(pkv, fused):
    """Four streams of a kv_init_group share one pool per block: patch pages
    from one free list, a special range each. Each step plans all four
    together; outputs match the oracle and the shared pool matches the
    oracle's image after every step."""
    from oracle import SharedPatchPool
    wl = small(64, H=2, D=128, dtype="fp16", S=2, W=3, frames=12)
    n, sp_pages = 4, 3
    Np = n * (wl.S + wl.W + 1) - 3          # 3 pages fewer than the streams' sum
    caches = pkv.PagedKVCache.group(n, Np + n * sp_pages, wl.page_size, wl.H, wl.D, wl.S, wl.W,
                                    num_special=wl.NS, dtype=wl.dtype, patch_pages=Np, special_pages=sp_pages)
    caches[2].allocate_pools("cuda")        # binds the one pool of the group
    assert all(c.pools[0] is caches[0].pools[0] for c in caches)
    pool = SharedPatchPool(Np)
    ms = [PageModel(wl.S, wl.W, wl.page_size, Np + n * sp_pages, NS=wl.NS, shared=pool,
                    sp_base=Np + i * sp_pages, sp_pages=sp_pages) for i in range(n)]
    img = PoolImage(ms[0], wl.H, wl.D)
    frs = [Frames(wl, seed=95, stream=i) for i in range(n)]
    sos = [StreamOracle(wl.S, wl.W, wl.NS, wl.P, wl.dtype, fr.bits) for fr in frs]
    ws = workspace(pkv, caches)
    ages = [0, 0, 0, 0]
    for step_i in range(10):
        live = [i for i in range(n) if (step_i + i) % 4 != 3]     # one stream sits each step out
        if step_i == 6:                                           # stream 1 starts over
            caches[1].reset()
            ms[1].reset()
            sos[1] = StreamOracle(wl.S, wl.W, wl.NS, wl.P, wl.dtype, frs[1].bits)
            ages[1] = 0
        qkv = [frs[i].get(ages[i] + 100 * step_i) for i in live]
        for j, i in enumerate(live):
            k, v = qkv[j][1].cuda(), qkv[j][2].cuda()
            if fused:
                caches[i].begin_frame()
            else:
                caches[i].append_frame(0, k, v)
            caches[i].evict_frames()
            page, sp0 = ms[i].append(ages[i])
            ms[i].evict()
            img.write(page, sp0, bits16(qkv[j][1]), bits16(qkv[j][2]), model=ms[i])
            sos[i].fetch = (lambda fr, off: (lambda f: fr.bits(f + off)))(frs[i], 100 * step_i)
            sos[i].begin_frame(ages[i])
            ages[i] += 1
        plan = pkv.Plan([caches[i] for i in live], ws)
        q, k, v = (torch.cat([x[t] for x in qkv]).cuda() for t in range(3))
        out = plan.run_append(0, k, v, q) if fused else plan.run(0, q)
        plan.check_device()
        for j, i in enumerate(live):
            assert_close(out[j * wl.T:(j + 1) * wl.T], sos[i].expected(), f"step {step_i} stream {i}")
        assert np.array_equal(pool_bits(caches[0]), img.bits), f"step {step_i}: shared pool"
        assert caches[0].free_list() == pool.free


def test_two_plans_on_two_streams_at_once(pkv):
    """Two caches whose launches each fill the GPU (about 144 CTAs, split
    merge in the kernel) run on two CUDA streams at the same time, many
    times. Their CTAs interleave on the SMs, so the CTAs of a split group are
    not all resident together: the merge must still complete (the last CTA
    to arrive takes what the others left), outputs match the oracle and the
    device error word stays clear."""
    wl = small(256, H=16, S=2, W=8, frames=12)
    caches = [new_cache(pkv, wl) for _ in range(2)]
    frames = [Frames(wl, 300 + i) for i in range(2)]
    oracles = [StreamOracle(wl.S, wl.W, wl.NS, wl.P, wl.dtype, fr.bits) for fr in frames]
    wss = [workspace(pkv, [c]) for c in caches]
    streams = [torch.cuda.Stream() for _ in range(2)]
    rows = np.arange(0, wl.T, 7)
    for f in range(wl.frames):
        qs = []
        for c, fr, so in zip(caches, frames, oracles):
            q, k, v = (x.cuda() for x in fr.get(f))
            c.append_frame(0, k, v)
            c.evict_frames()
            so.begin_frame(f, False)
            qs.append(q)
        if f == wl.frames - 1:
            plans = [pkv.Plan([c], ws) for c, ws in zip(caches, wss)]
            assert all(p.stats()["fused_merge"] for p in plans)
            assert sum(p.stats()["n_ctas"] for p in plans) > 148
            torch.cuda.synchronize()
            outs = [torch.empty_like(q) for q in qs]
            for _ in range(20):
                for p, q, o, st in zip(plans, qs, outs, streams):
                    with torch.cuda.stream(st):
                        p.run(0, q, o, stream=st)
            torch.cuda.synchronize()
            for p, o, so in zip(plans, outs, oracles):
                p.check_device()
                assert_close(o[torch.as_tensor(rows)], so.expected(rows), "concurrent plans")
        for so in oracles:
            so.end_frame(True)


@pytest.mark.parametrize("fused", [False, True])
def test_batch_at_the_stream_limit(pkv, fused):
    """One plan over KV_MAX_STREAMS streams, the most a batch takes, all of one
    kv_init_group with two blocks (so a block-0 launch also prefetches from
    every stream's block-1 pool). Streams join at different steps: at the last
    steps their windows, scale frames and special streams all differ. Both
    blocks match the oracle for every stream, and each block's shared pool
    matches the oracle's image after every step."""
    from oracle import SharedPatchPool
    n, joins, steps = pkv.KV_MAX_STREAMS, 8, 12
    wl = small(16, H=2, S=1, W=2, frames=steps)
    T = wl.T
    sp_pages = -(-wl.NS * steps // wl.page_size)
    Np = n * wl.patch_pages
    caches = pkv.PagedKVCache.group(n, Np + n * sp_pages, wl.page_size, wl.H, wl.D, wl.S, wl.W,
                                    num_blocks=2, num_special=wl.NS, dtype=wl.dtype,
                                    patch_pages=Np, special_pages=sp_pages)
    caches[0].allocate_pools("cuda")
    pool = SharedPatchPool(Np)
    ms = [PageModel(wl.S, wl.W, wl.page_size, Np + n * sp_pages, NS=wl.NS, shared=pool,
                    sp_base=Np + i * sp_pages, sp_pages=sp_pages) for i in range(n)]
    imgs = [PoolImage(ms[0], wl.H, wl.D) for _ in range(2)]
    frs = [[Frames(wl, seed=131, stream=i, block=b) for b in range(2)] for i in range(n)]
    sos = [[StreamOracle(wl.S, wl.W, wl.NS, wl.P, wl.dtype, fr.bits) for fr in pair] for pair in frs]
    ws = workspace(pkv, caches)
    ages = [0] * n
    for step in range(steps):
        live = [i for i in range(n) if i % joins <= step]
        qkv = [[frs[i][b].get(ages[i]) for b in range(2)] for i in live]
        for j, i in enumerate(live):
            if fused:
                caches[i].begin_frame()
            else:
                caches[i].append_frame(0, qkv[j][0][1].cuda(), qkv[j][0][2].cuda())
            caches[i].evict_frames()
            page, sp0 = ms[i].append(ages[i])
            ms[i].evict()
            for b in range(2):
                imgs[b].write(page, sp0, bits16(qkv[j][b][1]), bits16(qkv[j][b][2]), model=ms[i])
                sos[i][b].begin_frame(ages[i])
            ages[i] += 1
        plan = pkv.Plan([caches[i] for i in live], ws)
        assert plan.stats()["n_streams"] == len(live)
        for b in range(2):
            q, k, v = (torch.cat([x[b][t] for x in qkv]).cuda() for t in range(3))
            if fused:
                out = plan.run_append(b, k, v, q)
            else:
                if b == 1:
                    for j, i in enumerate(live):
                        caches[i].append_frame(1, k[j * T:(j + 1) * T], v[j * T:(j + 1) * T])
                out = plan.run(b, q)
            plan.check_device()
            if step >= steps - 2:
                for j, i in enumerate(live):
                    assert_close(out[j * T:(j + 1) * T], sos[i][b].expected(),
                                 f"step {step} block {b} stream {i}")
            assert np.array_equal(pool_bits(caches[0], b), imgs[b].bits), f"step {step} block {b}: shared pool"
        assert caches[0].free_list() == pool.free
    assert sorted(set(ages)) == list(range(steps - joins + 1, steps + 1))
