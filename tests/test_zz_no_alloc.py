"""kv_run_static: the entry point for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc. An engine may run under a fixed memory
budget, or call in while another allocator holds the device. kv_run_static
plans and runs one block with its scratch in the library's static device
array, so the caller provides only the caches, q and out. These tests run its
output against the ordinary kv_plan + kv_run path on the same inputs, within
the tolerance of the other GPU tests. They make two calls in a row, since the
array keeps the last call's contents. They also check that an oversized call
is turned away before it does any GPU work.

This file is named so that pytest collects it last.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import pytest
import torch

import workload
from gpu_drive import MAX_ABS, MEAN_ABS, new_cache, workspace

pytestmark = pytest.mark.gpu


def _close(a: torch.Tensor, b: torch.Tensor, what: str):
    d = (a.float() - b.float()).abs()
    mx, mean = float(d.max()), float(d.mean())
    assert np.isfinite(mx), f"{what}: non-finite output"
    assert mx <= MAX_ABS and mean <= MEAN_ABS, f"{what}: max {mx:.3e} mean {mean:.3e}"


def _two_block_stream(pkv, wl, n_frames, seed):
    """A 2-block cache with frames 0..n_frames-1 appended to both blocks;
    returns the cache and each block's last-frame q."""
    cache = new_cache(pkv, wl, num_blocks=2)
    qs = {}
    for f in range(n_frames):
        for b in range(2):
            q, k, v = (x.cuda() for x in workload.frame_qkv(wl, seed, f, b))
            cache.append_frame(b, k, v)
            cache.evict_frames()
            qs[b] = q
    return cache, qs


@pytest.mark.parametrize("wl_idx,n_frames,tps", [(1, 20, 0), (1, 20, 3), (0, 12, 1)])
def test_static_matches_workspace_path_two_calls(wl_idx, n_frames, tps):
    import paged_kv_cache_frame_b200 as pkv
    wl = workload.WORKLOADS[wl_idx]
    cache, qs = _two_block_stream(pkv, wl, n_frames, seed=11)
    ws = workspace(pkv, [cache])
    plan = pkv.Plan([cache], ws, tiles_per_split=tps)
    want = {b: plan.run(b, qs[b]) for b in range(2)}
    plan.check_device()
    got = {b: torch.full_like(qs[b], float("nan")) for b in range(2)}
    # Two calls in a row share the static array; the second overwrites the
    # first call's tables and partials after the first has finished on the stream.
    pkv.kv_run_static([cache.handle], 0, qs[0], got[0], tiles_per_split=tps)
    pkv.kv_run_static([cache.handle], 1, qs[1], got[1], tiles_per_split=tps, check=True)
    torch.cuda.synchronize()
    for b in range(2):
        _close(got[b], want[b], f"block {b}")


def test_static_rejects_oversized_call_before_gpu_work():
    import paged_kv_cache_frame_b200 as pkv
    wl = dataclasses.replace(workload.WORKLOADS[1], blocks=1)
    cache = new_cache(pkv, wl)
    for f in range(11):
        q, k, v = (x.cuda() for x in workload.frame_qkv(wl, 5, f, 0))
        cache.append_frame(0, k, v)
        cache.evict_frames()
    out = torch.zeros_like(q)
    # One K/V tile per CTA: 11 frames span 23 tiles, so 16 heads x 3 query
    # tiles x 23 chunks of fp32 partials, about 37 MB, more than the array
    # holds (the workspace path would still accept this schedule).
    with pytest.raises(pkv.KVError) as e:
        pkv.kv_run_static([cache.handle], 0, q, out, tiles_per_split=1)
    assert e.value.name == "CAPACITY"
    torch.cuda.synchronize()
    assert int(out.abs().max()) == 0
    # The same call with the automatic schedule fits.
    pkv.kv_run_static([cache.handle], 0, q, out, check=True)
    ws = workspace(pkv, [cache])
    _close(out, pkv.Plan([cache], ws).run(0, q), "after a rejected call")
