"""Drives streams of frames through the CUDA library and the oracle in lockstep
(used by the GPU parity tests and by `__graft_entry__.smoke`)."""
from __future__ import annotations

import numpy as np
import torch

import workload
from oracle.stream import StreamOracle, bits16

MAX_ABS = 2e-2    # attention tolerance on unit-variance inputs (bf16/fp16 in, fp32 accumulate)
MEAN_ABS = 2e-3


class Frames:
    """Seeded frames of one stream/block, drawn once and kept on the CPU."""

    def __init__(self, wl, seed, stream=0, block=0):
        self.wl, self.seed, self.stream, self.block = wl, seed, stream, block
        self.cache = {}

    def get(self, f):
        if f not in self.cache:
            self.cache = {k: v for k, v in self.cache.items() if k >= f - 1}
            self.cache[f] = workload.frame_qkv(self.wl, self.seed, f, self.block, self.stream)
        return self.cache[f]

    def bits(self, f):
        return tuple(bits16(x) for x in self.get(f))


def errors(out: torch.Tensor, want: np.ndarray):
    got = out.float().cpu().double().numpy()
    d = np.abs(got - want)
    return float(d.max()), float(d.mean())


def assert_close(out, want, what=""):
    mx, mean = errors(out, want)
    assert np.isfinite(mx), f"{what}: non-finite output"
    assert mx <= MAX_ABS and mean <= MEAN_ABS, f"{what}: max {mx:.3e} mean {mean:.3e}"
    return mx, mean


def dense_fp32(cache, plan, block, q, so, Np, stream_idx=0):
    """Every row and head of the frame's attention in fp32 on the GPU: the
    pages of `plan`'s table gathered densely from the block's pool (a check on
    the kernel at full size, next to the oracle's sampled rows).

    Patch pages are read whole. On special pages, stream token j (page
    Np + j // page_size, slot j % page_size) is read when the oracle's frame
    simulator `so.sim` holds it visible: all written tokens with cross-frame
    special retention on, only live frames' tokens with it off (the table
    cannot express those gaps). last_page_len must equal the number of
    tokens written to the table's final page."""
    pool = cache.pools[block]                       # [max_pages, 2, page_size, H, D]
    ps = cache.page_size
    table, lpl = plan.page_table(stream_idx)
    sp = so.sim.SP                                  # special stream, in append order
    vis = set(so.sim.visible_specials())
    rows = []
    for p in table:
        if p < Np:
            rows.extend(p * 2 * ps + t for t in range(ps))
        else:
            i = p - Np
            rows.extend(p * 2 * ps + t for t in range(ps)
                        if i * ps + t < len(sp) and sp[i * ps + t] in vis)
    last = table[-1]
    assert last >= Np and lpl == min(ps, len(sp) - ps * (last - Np)), "last_page_len"
    idx = torch.as_tensor(rows, device=pool.device, dtype=torch.long)
    flat = pool.view(-1, cache.H, cache.D)          # row (page * 2 + kv) * page_size + slot
    k = flat.index_select(0, idx).float()
    v = flat.index_select(0, idx + ps).float()
    out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    scale = cache.D ** -0.5
    for h in range(cache.H):   # one head at a time keeps the score matrix small
        s_ = (q[:, h].float() @ k[:, h].T) * scale
        out[:, h] = torch.softmax(s_, dim=-1) @ v[:, h]
    return out


def assert_close_dense(out, want, what=""):
    d = (out.float() - want).abs()
    mx, mean = float(d.max()), float(d.mean())
    assert np.isfinite(mx), f"{what}: non-finite output"
    assert mx <= MAX_ABS and mean <= MEAN_ABS, f"{what}: max {mx:.3e} mean {mean:.3e}"
    return mx, mean


def new_cache(pkv, wl, num_blocks=1, patch_pages=0, cross_special=True, camera_only=False):
    max_pages = (patch_pages or wl.patch_pages) + wl.special_pages
    c = pkv.PagedKVCache(max_pages, wl.page_size, wl.H, wl.D, wl.S, wl.W, num_blocks=num_blocks,
                         num_special=wl.NS, dtype=wl.dtype, patch_pages=patch_pages,
                         cross_frame_special=cross_special, camera_only=camera_only)
    c.allocate_pools("cuda")
    return c


def workspace(pkv, caches):
    return torch.empty(pkv.workspace_bytes(caches), dtype=torch.uint8, device="cuda")


def run_stream(pkv, wl, seed, n_frames, check, rows=None, defer=None, keep=None,
               tiles_per_split=0, patch_pages=0, collect=None, dense=(), cross_special=True,
               camera_only=False, fused=False, all_rows=(), frames=None):
    """Append frames 0..n_frames-1 of block 0; at frames in `check`, plan + run
    and compare the chosen query rows with the oracle. defer[f] / keep[f]:
    frame f is appended with eviction deferred and then committed (keep) or
    rolled back. At frames in `dense`, every row is also checked against the
    fp32 dense gather of the visible pages; at frames in `all_rows` every row
    is checked against the oracle whatever `rows` says. fused: each frame goes through
    begin_frame + plan + run_append (the append inside the attention launch)
    instead of append_frame + plan + run. frames: a Frames-like source of the
    stream's q, k, v (default: the seeded workload frames). Returns
    {frame: (max_err, mean_err)}."""
    fr = frames if frames is not None else Frames(wl, seed)
    cache = new_cache(pkv, wl, patch_pages=patch_pages, cross_special=cross_special, camera_only=camera_only)
    ws = workspace(pkv, [cache])
    so = StreamOracle(wl.S, wl.W, wl.NS, wl.P, wl.dtype, fr.bits, cross_frame_special=cross_special,
                      camera_only=camera_only)
    res = {}
    for f in range(n_frames):
        q, k, v = (x.cuda() for x in fr.get(f))
        d = bool(defer[f]) if defer is not None else False
        cache.defer_eviction(d)
        if fused:
            cache.begin_frame()
            cache.evict_frames()
            plan = pkv.Plan([cache], ws, tiles_per_split=tiles_per_split)
            out = plan.run_append(0, k, v, q)
        else:
            cache.append_frame(0, k, v)
            cache.evict_frames()
        so.begin_frame(f, d)
        if f in check:
            if not fused:
                plan = pkv.Plan([cache], ws, tiles_per_split=tiles_per_split)
                out = plan.run(0, q)
            plan.check_device()
            r = None if f in all_rows else rows
            sel = slice(None) if r is None else torch.as_tensor(r)
            res[f] = assert_close(out[sel], so.expected(r), f"frame {f}")
            if f in dense:
                want = dense_fp32(cache, plan, 0, q, so, patch_pages or wl.patch_pages)
                assert_close_dense(out, want, f"frame {f} (all rows, fp32 dense)")
            if collect is not None:
                collect[f] = out.clone()
        if d:
            if keep is None or keep[f]:
                cache.commit_frame()
            else:
                cache.rollback_last_frame()
            so.end_frame(keep is None or bool(keep[f]))
        assert cache.get_stats()["special_tokens"] == len(so.sim.SP)
    return res
