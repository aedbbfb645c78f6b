"""Seeded synthetic workloads for the per-frame paged-KV prefill path.

This module only draws inputs: it holds the workload shapes and the seeded
random generators that both the CUDA path (tests, bench) and the CPU oracle
(tests) consume. It contains none of the method's arithmetic: no paging, no
eviction, no attention.

Workload shapes follow the pages:
  * "How the Paged KV Cache Attention Mechanism Enables Long Sequence Inference
    in LingBot-Map", section "Implementation Example": 256 patch + 6 special
    tokens per frame, scale_frames=8, sliding_window=64.
  * "FlashInfer Paged KV Cache Performance Benefits in LingBot-Map", table
    "Quantitative Performance Benchmarks": 224x224 video, 320 frames.
  * "KV Cache Mechanism in LingBot-Map for Streaming Inference: A Deep Dive",
    section "Practical Implementation Examples": 518-pixel frames, patch 14.
  * "How LingBot-Map Achieves ~20 FPS Inference with Its KV Cache", section
    "Implementation Example": keyframe_interval=4 over 200 frames.

Values are unit-variance normals rounded to bf16 (fp16 for the batched
workload); keyframe decisions are Bernoulli(0.3) with frame 0 forced, a
stand-in for the optical-flow test the pages describe, which needs images.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

NUM_SPECIAL = 6


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    H: int
    D: int
    P: int                 # patch tokens per frame (== page_size)
    page_size: int
    S: int                 # scale frames
    W: int                 # sliding window
    blocks: int
    frames: int            # frames per stream (the last frame index + 1)
    dtype: str = "bf16"
    NS: int = NUM_SPECIAL
    streams: int = 1
    keyframes: str = "all"  # "all" | "bernoulli" | "interval"
    keyframe_p: float = 0.3
    keyframe_interval: int = 4
    age_lo: int = 0         # batched: seeded stream ages in [age_lo, age_hi]
    age_hi: int = 0
    steps: int = 0          # batched: timed steps after warming to the ages
    cross_special: bool = True   # special tokens of evicted frames stay visible

    @property
    def T(self) -> int:
        return self.P + self.NS

    @property
    def patch_pages(self) -> int:
        # append pops a page before eviction pushes one back, and a deferred
        # frame needs the same one extra page
        return self.S + self.W + 1

    def max_frames_per_stream(self) -> int:
        return (self.age_hi + self.steps) if self.streams > 1 else self.frames

    @property
    def special_pages(self) -> int:
        return max(1, math.ceil(self.NS * self.max_frames_per_stream() / self.page_size))

    @property
    def max_pages(self) -> int:
        return self.patch_pages + self.special_pages

    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float16


WORKLOADS = {
    0: Workload("tiny-16tok", H=2, D=64, P=16, page_size=16, S=2, W=4, blocks=1, frames=12),
    1: Workload("224x224-320f", H=16, D=64, P=256, page_size=256, S=8, W=64, blocks=24, frames=320),
    2: Workload("224x224-320f-keyframes", H=16, D=64, P=256, page_size=256, S=8, W=64, blocks=24,
                frames=320, keyframes="bernoulli"),
    3: Workload("518x378-1000f", H=16, D=64, P=999, page_size=999, S=8, W=64, blocks=24, frames=1000),
    4: Workload("batched-8x-ragged", H=8, D=128, P=256, page_size=256, S=8, W=64, blocks=24,
                frames=0, dtype="fp16", streams=8, age_lo=10, age_hi=600, steps=32),
    5: Workload("224x224-320f-no-cross-frame-special", H=16, D=64, P=256, page_size=256, S=8, W=64,
                blocks=24, frames=320, cross_special=False),
}


def frame_seed(seed: int, frame: int, block: int, stream: int = 0) -> int:
    return (seed + 1000003 * frame + block + 7919 * 1000003 * stream) % (2 ** 63)


def frame_qkv(wl: Workload, seed: int, frame: int, block: int, stream: int = 0,
              device: str = "cpu"):
    """Q, K, V for one (frame, block) as [T, H, D] tensors of the workload dtype.

    Drawn on the CPU generator so that the same seed gives the same values on
    every machine, then moved to `device`.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(frame_seed(seed, frame, block, stream))
    x = torch.randn((3, wl.T, wl.H, wl.D), generator=g, dtype=torch.float32)
    x = x.to(wl.torch_dtype())
    if device != "cpu":
        x = x.to(device)
    return x[0], x[1], x[2]


def qkv_ring_cuda(wl: Workload, seed: int, ring: int, device="cuda"):
    """A ring of `ring` frame sets [ring, blocks, 3, streams*T, H, D] drawn on the
    GPU generator (fast; values differ from the CPU draw of `frame_qkv`).
    Timing-only input."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    shape = (ring, wl.blocks, 3, wl.streams * wl.T, wl.H, wl.D)
    x = torch.empty(shape, dtype=wl.torch_dtype(), device=device)
    for r in range(ring):
        x[r].copy_(torch.randn(shape[1:], generator=g, device=device, dtype=torch.float32))
    return x


def keyframe_mask(wl: Workload, seed: int, n_frames: int | None = None) -> np.ndarray:
    """Which frames are kept in the cache.

    "all": every frame. "interval": frame t is kept iff t % K == 0.
    "bernoulli": frame 0 kept, others kept with probability p (seeded).
    """
    n = wl.frames if n_frames is None else n_frames
    if wl.keyframes == "all":
        return np.ones(n, dtype=bool)
    if wl.keyframes == "interval":
        return (np.arange(n) % wl.keyframe_interval) == 0
    rng = np.random.default_rng(seed)
    m = rng.random(n) < wl.keyframe_p
    if n:
        m[0] = True
    return m


def interval_mask(n_frames: int, k: int) -> np.ndarray:
    return (np.arange(n_frames) % k) == 0


def stream_ages(wl: Workload, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed + 17)
    return rng.integers(wl.age_lo, wl.age_hi + 1, size=wl.streams)

