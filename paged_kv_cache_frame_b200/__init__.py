"""Per-frame paged-KV prefill attention for streaming video on B200 (sm_100a).

Python binding of the C-ABI in include/kv.h. The functions below carry the
C names and only marshal arguments (torch tensors -> device pointers, torch
streams -> cudaStream_t); every step of the path runs in libpkv.so.

    cache = PagedKVCache(max_pages, page_size, H, D, scale_frames, window, num_blocks)
    cache.allocate_pools("cuda")               # torch owns the memory, library borrows it
    for frame in stream:
        for b in range(num_blocks):
            cache.append_frame(b, k[b], v[b])
            cache.evict_frames()
            if b == 0:
                plan = Plan([cache], workspace)    # once per frame step
            out[b] = plan.run(b, q[b])             # every block

Token order inside a frame: tokens 0..NS-1 are the special tokens, NS..T-1
the patch tokens, for q, k, v and out alike.
"""
from __future__ import annotations

import ctypes

from . import capi
from .capi import KVError, KV_BF16, KV_FP16, KV_MAX_STREAMS, KV_NOT_CURRENT, KV_STATIC_SCRATCH_BYTES

__all__ = [
    "PagedKVCache", "Plan", "KVError", "workspace_bytes", "KV_BF16", "KV_FP16", "KV_MAX_STREAMS",
    "kv_init", "kv_init_group", "kv_destroy", "kv_reset", "kv_pool_bytes", "kv_bind_pool", "kv_append_frame",
    "kv_evict_frames", "kv_defer_eviction", "kv_commit_frame", "kv_rollback_last_frame",
    "kv_get_stats", "kv_get_config", "kv_get_free_list", "kv_workspace_bytes", "kv_plan", "kv_run",
    "kv_run_append", "kv_begin_frame", "kv_plan_free", "kv_get_page_table", "kv_get_kv_tiles",
    "kv_plan_get_stats", "kv_check_device", "kv_testing_fail_launches", "kv_strerror",
    "kv_last_error", "kv_run_static", "kv_set_cross_frame_special", "kv_set_camera_only",
]


def _ptr(x) -> int | None:
    """Device (or host) address of a tensor, or an int address, or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s) -> int | None:
    if s is None:
        import torch
        if torch.cuda.is_available() and torch.cuda.is_initialized():
            return torch.cuda.current_stream().cuda_stream
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


# ---------------------------------------------------------------- C names
def kv_init(max_pages, page_size, num_heads, head_dim, scale_frames, window, num_blocks,
            num_special=6, dtype=KV_BF16, patch_pages=0) -> int:
    h = ctypes.c_void_p()
    capi.check(capi.lib().kv_init(ctypes.byref(h), max_pages, page_size, num_heads, head_dim,
                                  scale_frames, window, num_blocks, num_special, dtype,
                                  patch_pages), "kv_init")
    return h.value


def kv_init_group(n_streams, max_pages, page_size, num_heads, head_dim, scale_frames, window, num_blocks,
                  num_special=6, dtype=KV_BF16, patch_pages=0, special_pages=0) -> list[int]:
    hs = (ctypes.c_void_p * n_streams)()
    capi.check(capi.lib().kv_init_group(hs, n_streams, max_pages, page_size, num_heads, head_dim, scale_frames,
                                        window, num_blocks, num_special, dtype, patch_pages, special_pages),
               "kv_init_group")
    return [hs[i] for i in range(n_streams)]


def kv_destroy(c) -> None:
    capi.lib().kv_destroy(c)


def kv_reset(c) -> None:
    capi.check(capi.lib().kv_reset(c), "kv_reset")


def kv_pool_bytes(c) -> int:
    return capi.lib().kv_pool_bytes(c)


def kv_bind_pool(c, block, pool, stream=None) -> None:
    capi.check(capi.lib().kv_bind_pool(c, block, _ptr(pool), _stream(stream)), "kv_bind_pool")


def kv_append_frame(c, block, k, v, stream=None) -> None:
    capi.check(capi.lib().kv_append_frame(c, block, _ptr(k), _ptr(v), _stream(stream)),
               "kv_append_frame")


def kv_evict_frames(c) -> None:
    capi.check(capi.lib().kv_evict_frames(c), "kv_evict_frames")


def kv_defer_eviction(c, on) -> None:
    capi.check(capi.lib().kv_defer_eviction(c, 1 if on else 0), "kv_defer_eviction")


def kv_commit_frame(c) -> None:
    capi.check(capi.lib().kv_commit_frame(c), "kv_commit_frame")


def kv_rollback_last_frame(c) -> None:
    capi.check(capi.lib().kv_rollback_last_frame(c), "kv_rollback_last_frame")


def kv_set_cross_frame_special(c, on) -> None:
    capi.check(capi.lib().kv_set_cross_frame_special(c, int(bool(on))), "kv_set_cross_frame_special")


def kv_set_camera_only(c, on) -> None:
    capi.check(capi.lib().kv_set_camera_only(c, int(bool(on))), "kv_set_camera_only")


def kv_get_stats(c) -> dict:
    s = capi.kv_stats()
    capi.check(capi.lib().kv_get_stats(c, ctypes.byref(s)), "kv_get_stats")
    return {f: getattr(s, f) for f, _ in s._fields_}


def kv_get_config(c) -> dict:
    s = capi.kv_config()
    capi.check(capi.lib().kv_get_config(c, ctypes.byref(s)), "kv_get_config")
    return {f: getattr(s, f) for f, _ in s._fields_}


def kv_get_free_list(c) -> list[int]:
    n = ctypes.c_int()
    capi.check(capi.lib().kv_get_free_list(c, None, 0, ctypes.byref(n)), "kv_get_free_list")
    buf = (ctypes.c_int * max(1, n.value))()
    capi.check(capi.lib().kv_get_free_list(c, buf, n.value, ctypes.byref(n)), "kv_get_free_list")
    return list(buf[: n.value])


def _handles(caches):
    arr = (ctypes.c_void_p * len(caches))()
    for i, c in enumerate(caches):
        arr[i] = c
    return arr


def kv_workspace_bytes(caches) -> int:
    return capi.lib().kv_workspace_bytes(_handles(caches), len(caches))


def kv_plan(caches, tiles_per_split=0, workspace=None, workspace_bytes=0, stream=None) -> int:
    h = ctypes.c_void_p()
    if workspace is not None and not isinstance(workspace, int):
        workspace_bytes = workspace.numel() * workspace.element_size()
    capi.check(capi.lib().kv_plan(ctypes.byref(h), _handles(caches), len(caches), tiles_per_split,
                                  _ptr(workspace), workspace_bytes,
                                  _stream(stream) if workspace is not None else None), "kv_plan")
    return h.value


def kv_run(plan, block, q, out, stream=None) -> None:
    capi.check(capi.lib().kv_run(plan, block, _ptr(q), _ptr(out), _stream(stream)), "kv_run")


def kv_run_append(plan, block, k, v, q, out, stream=None) -> None:
    capi.check(capi.lib().kv_run_append(plan, block, _ptr(k), _ptr(v), _ptr(q), _ptr(out), _stream(stream)),
               "kv_run_append")


def kv_begin_frame(c) -> None:
    capi.check(capi.lib().kv_begin_frame(c), "kv_begin_frame")


def kv_plan_free(plan) -> None:
    capi.lib().kv_plan_free(plan)


def kv_get_page_table(plan, stream_idx=0):
    n, lpl = ctypes.c_int(), ctypes.c_int()
    capi.check(capi.lib().kv_get_page_table(plan, stream_idx, None, 0, ctypes.byref(n),
                                            ctypes.byref(lpl)), "kv_get_page_table")
    buf = (ctypes.c_int * max(1, n.value))()
    capi.check(capi.lib().kv_get_page_table(plan, stream_idx, buf, n.value, ctypes.byref(n),
                                            ctypes.byref(lpl)), "kv_get_page_table")
    return list(buf[: n.value]), lpl.value


def kv_get_kv_tiles(plan, stream_idx=0, with_krow=False):
    """[(row, lo, hi)] per tile; with_krow: [(row, lo, hi, krow, step)]
    (krow = KV_NOT_CURRENT for tiles that are not the open step's frame; of
    [lo, hi) only lo, lo + step, ... are visible)."""
    n = ctypes.c_int()
    capi.check(capi.lib().kv_get_kv_tiles(plan, stream_idx, None, None, None, None, None, 0, ctypes.byref(n)),
               "kv_get_kv_tiles")
    m = max(1, n.value)
    row, lo, hi, kr, sp = ((ctypes.c_int * m)() for _ in range(5))
    capi.check(capi.lib().kv_get_kv_tiles(plan, stream_idx, row, lo, hi, kr, sp, n.value, ctypes.byref(n)),
               "kv_get_kv_tiles")
    if with_krow:
        return [(row[i], lo[i], hi[i], kr[i], sp[i]) for i in range(n.value)]
    return [(row[i], lo[i], hi[i]) for i in range(n.value)]


def kv_plan_get_stats(plan) -> dict:
    s = capi.kv_plan_stats()
    capi.check(capi.lib().kv_plan_get_stats(plan, ctypes.byref(s)), "kv_plan_get_stats")
    return {f: getattr(s, f) for f, _ in s._fields_}


def kv_check_device(plan, stream=None) -> None:
    capi.check(capi.lib().kv_check_device(plan, _stream(stream)), "kv_check_device")


def kv_run_static(caches, block, q, out, tiles_per_split=0, check=False, stream=None) -> None:
    """kv_plan + kv_run for one block without any allocation: the plan tables
    and split-KV partials go to the library's static device array
    (KV_STATIC_SCRATCH_BYTES). For callers that cannot allocate device memory;
    calls that overlap on the GPU share that array and race.

    caches: PagedKVCache objects or raw handles. Tensor q and out are checked
    against the caches' configuration ([sum of T, H, D], the cache dtype,
    contiguous, on a CUDA device) before the call, since the library would
    read and write exactly that many rows at their addresses."""
    handles = [c.handle if isinstance(c, PagedKVCache) else c for c in caches]
    if handles:
        cfgs = [kv_get_config(h) for h in handles]
        c0 = cfgs[0]
        shape = (sum(c["tokens_per_frame"] for c in cfgs), c0["num_heads"], c0["head_dim"])
        fp16 = c0["dtype"] == KV_FP16
        _check_tensor(q, "q", shape, fp16)
        _check_tensor(out, "out", shape, fp16)
    capi.check(capi.lib().kv_run_static(_handles(handles), len(handles), block, tiles_per_split, _ptr(q),
                                        _ptr(out), int(bool(check)), _stream(stream)), "kv_run_static")


def kv_testing_fail_launches(n) -> None:
    """Error-path tests only: the library's next n kernel launches fail with
    KV_ERR_CUDA without launching (a fake of a failing launch)."""
    capi.lib().kv_testing_fail_launches(int(n))


def kv_strerror(status) -> str:
    return capi.strerror(status)


def kv_last_error() -> str:
    return capi.lib().kv_last_error().decode()


def workspace_bytes(caches) -> int:
    return kv_workspace_bytes([c.handle for c in caches])


# ---------------------------------------------------------------- objects
def _is_fp16(dtype) -> bool:
    return dtype in ("fp16", "float16") or str(dtype) == "torch.float16"


def _torch_dtype(fp16: bool):
    import torch
    return torch.float16 if fp16 else torch.bfloat16


def _check_tensor(x, name, shape, fp16):
    """The library sees only a tensor's address and touches exactly `shape`
    elements of the cache dtype there, so the shape, dtype, layout and device
    are checked here, before the call. Raw int addresses are the caller's
    responsibility."""
    if x is None or isinstance(x, int):
        return
    want = _torch_dtype(fp16)
    if tuple(x.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(x.shape)}, expected {tuple(shape)}")
    if x.dtype != want:
        raise ValueError(f"{name}: dtype {x.dtype}, expected {want}")
    if not x.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if x.device.type != "cuda":
        raise ValueError(f"{name}: must be a CUDA tensor, not on {x.device}")


class PagedKVCache:
    """One video stream's paged cache (all transformer blocks)."""

    def __init__(self, max_pages, page_size, num_heads, head_dim, scale_frames=8, window=64,
                 num_blocks=1, num_special=6, dtype="bf16", patch_pages=0, cross_frame_special=True,
                 camera_only=False, _handle=None, _pools=None):
        self.dtype = dtype
        self.fp16 = _is_fp16(dtype)
        code = KV_FP16 if self.fp16 else KV_BF16
        self.handle = _handle if _handle is not None else kv_init(
            max_pages, page_size, num_heads, head_dim, scale_frames, window, num_blocks, num_special, code,
            patch_pages)
        self.max_pages, self.page_size = max_pages, page_size
        self.H, self.D, self.num_blocks, self.NS = num_heads, head_dim, num_blocks, num_special
        self.T = page_size + num_special
        # the block pools (a list shared by the caches of a group)
        self.pools = _pools if _pools is not None else [None] * num_blocks
        if not cross_frame_special:
            kv_set_cross_frame_special(self.handle, False)
        if camera_only:
            kv_set_camera_only(self.handle, True)

    def __del__(self):
        h = getattr(self, "handle", None)
        if h:
            self.handle = None
            try:
                kv_destroy(h)
            except Exception:   # interpreter shutdown: the library may already be gone
                pass

    @classmethod
    def group(cls, n_streams, max_pages, page_size, num_heads, head_dim, scale_frames=8, window=64,
              num_blocks=1, num_special=6, dtype="bf16", patch_pages=0, special_pages=0,
              cross_frame_special=True, camera_only=False):
        """n_streams caches sharing one pool per block (kv_init_group): common
        patch pages, a special-page range per stream. allocate_pools on any
        of them allocates and binds the pools of all."""
        code = KV_FP16 if _is_fp16(dtype) else KV_BF16
        hs = kv_init_group(n_streams, max_pages, page_size, num_heads, head_dim, scale_frames, window,
                           num_blocks, num_special, code, patch_pages, special_pages)
        pools = [None] * num_blocks
        return [cls(max_pages, page_size, num_heads, head_dim, scale_frames, window, num_blocks, num_special,
                    dtype, cross_frame_special=cross_frame_special, camera_only=camera_only, _handle=h,
                    _pools=pools) for h in hs]

    def pool_bytes(self) -> int:
        return kv_pool_bytes(self.handle)

    def bind_pool(self, block, pool, stream=None):
        if pool is not None and not isinstance(pool, int):
            nbytes = pool.numel() * pool.element_size()
            if nbytes < self.pool_bytes():
                raise ValueError(f"pool: {nbytes} bytes, the cache needs {self.pool_bytes()}")
            if not pool.is_contiguous() or pool.device.type != "cuda":
                raise ValueError("pool: must be a contiguous CUDA tensor")
        kv_bind_pool(self.handle, block, pool, stream)
        self.pools[block] = pool   # shared list: every cache of a group sees it

    def allocate_pools(self, device="cuda", stream=None):
        """Allocate each block's pool [max_pages, 2, page_size, H, D] with torch and bind it."""
        import torch
        dt = _torch_dtype(self.fp16)
        for b in range(self.num_blocks):
            pool = torch.empty((self.max_pages, 2, self.page_size, self.H, self.D), dtype=dt,
                               device=device)
            self.bind_pool(b, pool, stream)
        return self.pools

    def append_frame(self, block, k, v, stream=None):
        """k, v: [T, H, D] of the cache dtype (tokens 0..NS-1 special), or both
        None to advance the page state only."""
        shape = (self.T, self.H, self.D)
        _check_tensor(k, "k", shape, self.fp16)
        _check_tensor(v, "v", shape, self.fp16)
        kv_append_frame(self.handle, block, k, v, stream)

    def begin_frame(self):
        """Open a frame step (take the new frame's page and special slots)
        before its blocks are appended, e.g. by Plan.run_append."""
        kv_begin_frame(self.handle)

    def evict_frames(self):
        kv_evict_frames(self.handle)

    def defer_eviction(self, on=True):
        kv_defer_eviction(self.handle, on)

    def commit_frame(self):
        kv_commit_frame(self.handle)

    def rollback_last_frame(self):
        kv_rollback_last_frame(self.handle)

    def get_stats(self) -> dict:
        return kv_get_stats(self.handle)

    def free_list(self) -> list[int]:
        return kv_get_free_list(self.handle)

    def reset(self):
        kv_reset(self.handle)


class Plan:
    """One frame step's plan over a batch of caches; run() per block."""

    def __init__(self, caches, workspace=None, tiles_per_split=0, stream=None):
        self.caches = list(caches)
        self.workspace = workspace
        self.handle = kv_plan([c.handle for c in self.caches], tiles_per_split, workspace,
                              stream=stream)
        c0 = self.caches[0]
        self.rows = sum(c.T for c in self.caches)
        self.H, self.D, self.dtype, self.fp16 = c0.H, c0.D, c0.dtype, c0.fp16

    def __del__(self):
        h = getattr(self, "handle", None)
        if h:
            self.handle = None
            try:
                kv_plan_free(h)
            except Exception:   # interpreter shutdown: the library may already be gone
                pass

    def run(self, block, q, out=None, stream=None):
        """q (and out): [sum of the streams' T, H, D] of the cache dtype."""
        shape = (self.rows, self.H, self.D)
        _check_tensor(q, "q", shape, self.fp16)
        if out is None:
            import torch
            out = torch.empty_like(q)
        _check_tensor(out, "out", shape, self.fp16)
        kv_run(self.handle, block, q, out, stream)
        return out

    def run_append(self, block, k, v, q, out=None, stream=None):
        """Append block `block`'s K/V of the open frame step and run its
        attention in one launch. k, v, q (and out): [sum of the streams' T,
        H, D] of the cache dtype, streams in plan order."""
        shape = (self.rows, self.H, self.D)
        for x, name in ((k, "k"), (v, "v"), (q, "q")):
            _check_tensor(x, name, shape, self.fp16)
        if out is None:
            import torch
            out = torch.empty_like(q)
        _check_tensor(out, "out", shape, self.fp16)
        kv_run_append(self.handle, block, k, v, q, out, stream)
        return out

    def page_table(self, stream_idx=0):
        return kv_get_page_table(self.handle, stream_idx)

    def kv_tiles(self, stream_idx=0):
        return kv_get_kv_tiles(self.handle, stream_idx)

    def stats(self) -> dict:
        return kv_plan_get_stats(self.handle)

    def check_device(self, stream=None):
        kv_check_device(self.handle, stream)
