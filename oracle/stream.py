"""Expected attention outputs along a stream of frames.

Test infrastructure only (see the package docstring).

Drives the frame-list simulator (`frames.FrameListSim`) through a stream and
gathers the visible K/V straight from each frame's own tensors, with no pages
involved, so that it checks the paged path from the outside: patch tokens of
every visible frame, then the visible special tokens (all of them with
cross-frame special retention, else those of the visible frames). Attention does not
depend on the order of the visible tokens.

Per frame step ([P1] "Runtime Flow for Frame Processing"; [P2] "Flow-Based
Keyframe Selection"): the frame is appended and eviction runs. With eviction
deferred, the frame stays pending through the forward pass and is then
committed (keyframe) or rolled back.
"""
from __future__ import annotations

import numpy as np

from .attention import decode, dense
from .frames import FrameListSim


def bits16(t) -> np.ndarray:
    """uint16 bit patterns of a CPU torch tensor of a 16-bit float type."""
    import torch
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


class StreamOracle:
    """fetch(frame) -> (q, k, v) as [T, H, D] uint16 bit patterns."""

    def __init__(self, S: int, W: int, NS: int, P: int, dtype: str, fetch, cross_frame_special: bool = True,
                 camera_only: bool = False):
        self.sim = FrameListSim(S, W, NS, cross_frame_special, camera_only)
        self.NS, self.P, self.dtype, self.fetch = NS, P, dtype, fetch
        self.patch_kv: dict[int, tuple[np.ndarray, np.ndarray]] = {}
        self.special_kv: dict[int, tuple[np.ndarray, np.ndarray]] = {}
        self.q: np.ndarray | None = None

    def begin_frame(self, f: int, defer: bool = False) -> None:
        """Append frame f (deferred: pending until `end_frame`) and evict."""
        q, k, v = self.fetch(f)
        # bf16/fp16 values are exact in float32; the arithmetic below is float64
        k64 = decode(k, self.dtype).astype(np.float32)
        v64 = decode(v, self.dtype).astype(np.float32)
        self.q = decode(q, self.dtype)
        self.sim.set_defer(defer)
        self.sim.append(f)
        self.sim.evict()
        self.patch_kv[f] = (k64[self.NS:], v64[self.NS:])
        self.special_kv[f] = (k64[: self.NS], v64[: self.NS])
        self._prune()

    def end_frame(self, keep: bool = True) -> None:
        """Resolve a deferred frame: commit it (keyframe) or roll it back."""
        f = self.sim.pending
        if f is None:
            return
        if keep:
            self.sim.commit()
        else:
            self.sim.rollback()
            del self.special_kv[f]
        self._prune()

    def _prune(self) -> None:
        live = set(self.sim.patch_frames())
        for g in list(self.patch_kv):
            if g not in live:
                del self.patch_kv[g]

    def visible_kv(self):
        ks, vs = [], []
        for f in self.sim.attended_patch_frames():
            k, v = self.patch_kv[f]
            ks.append(k)
            vs.append(v)
        for f, j in self.sim.visible_specials():
            k, v = self.special_kv[f]
            ks.append(k[j:j + 1])
            vs.append(v[j:j + 1])
        return np.concatenate(ks), np.concatenate(vs)

    def expected(self, rows=None) -> np.ndarray:
        """Attention output [len(rows), H, D] for the current frame's query rows,
        computed head by head in float64."""
        k, v = self.visible_kv()
        q = self.q if rows is None else self.q[np.asarray(rows)]
        out = np.empty(q.shape)
        for h in range(q.shape[1]):
            out[:, h:h + 1] = dense(q[:, h:h + 1], k[:, h:h + 1].astype(np.float64),
                                    v[:, h:h + 1].astype(np.float64))
        return out
