"""Brute-force frame-list simulator: the semantic definition of what is visible.

Test infrastructure only (see the package docstring).

State is kept as plain lists of frame ids, with no pages at all:
  C        committed frames, in commit order
  resident committed frames whose patch tokens are still cached
  pending  a frame appended while eviction was deferred, or None
  SP       (frame, slot) records of every cached special token, in append order

Rules, each from the pages:
  * A frame contributes NS special tokens to an append-only stream that is
    never evicted ([P1] "Special Stream (Append-Only)"; [P2] "Special Stream
    (Append-Only)": six tokens per frame). With cross-frame special retention
    on (the default, [P2] "Configuration Parameters"), the special tokens of
    evicted frames stay visible; with it off, only the special tokens of
    frames whose patches are still visible are ([P2] "Configuration
    Parameters": kv_cache_cross_frame_special retains the special tokens of
    evicted frames).
  * Scale frames are the first S committed frames and stay resident for good
    ([P2] "Patch Stream (Recyclable)": first kv_cache_scale_frames frames
    remain permanently resident).
  * Eviction runs after each append: while more than W non-scale frames are
    resident, the oldest is dropped ([P2] "Sliding-Window Eviction Strategy").
    The count includes the frame just appended.
  * While eviction is deferred the appended frame is pending: visible, not
    committed. Commit makes it a normal frame and runs eviction; rollback
    discards it and its special tokens ([P2] "Flow-Based Keyframe Selection";
    [P4] "Deferred Eviction and Rollback Mechanism").
  * Camera-only ([P2] "Configuration Parameters": kv_cache_camera_only
    restricts the cache to camera tokens, excluding patches). The pages list
    a frame's six special tokens as camera, register, scale ([P2] "Special
    Stream (Append-Only)"); reading: slot 0 of the six is the camera token.
    With camera-only on, attention sees no patch token and no register or
    scale token: only the camera tokens among the special tokens that would
    otherwise be visible. The frame lists themselves (what is cached, what
    is evicted) do not change.
"""
from __future__ import annotations


class FrameListSim:
    def __init__(self, S: int, W: int, NS: int = 6, cross_frame_special: bool = True,
                 camera_only: bool = False):
        self.S, self.W, self.NS = S, W, NS
        self.cross_frame_special = cross_frame_special
        self.camera_only = camera_only
        self.C: list[int] = []
        self.resident: list[int] = []
        self.pending: int | None = None
        self.SP: list[tuple[int, int]] = []
        self.defer = False

    # -- operations -------------------------------------------------------
    def append(self, f: int) -> None:
        if self.pending is not None:
            raise ValueError("a deferred frame must be committed or rolled back first")
        if self.defer:
            self.pending = f
        else:
            self.C.append(f)
            self.resident.append(f)
        self.SP.extend((f, j) for j in range(self.NS))

    def evict(self) -> None:
        if self.defer:
            return
        scale = set(self.C[: self.S])
        others = [f for f in self.resident if f not in scale]
        keep = set(others[max(0, len(others) - self.W):]) if self.W > 0 else set()
        self.resident = [f for f in self.resident if f in scale or f in keep]

    def set_defer(self, on: bool) -> None:
        if not on and self.pending is not None:
            raise ValueError("pending frame: commit or roll back first")
        self.defer = bool(on)

    def commit(self) -> None:
        if self.pending is None:
            raise ValueError("no pending frame")
        f, self.pending = self.pending, None
        self.defer = False
        self.C.append(f)
        self.resident.append(f)
        self.evict()

    def rollback(self) -> None:
        if self.pending is None:
            raise ValueError("no pending frame")
        self.pending = None
        self.defer = False
        del self.SP[len(self.SP) - self.NS:]

    # -- queries ----------------------------------------------------------
    def patch_frames(self) -> list[int]:
        """Frames whose patch tokens are cached (resident, then pending), oldest
        first: the visible patch frames unless camera-only is on."""
        return self.resident + ([self.pending] if self.pending is not None else [])

    def attended_patch_frames(self) -> list[int]:
        """Frames whose patch tokens attention sees: none with camera-only."""
        return [] if self.camera_only else self.patch_frames()

    def visible_specials(self) -> list[tuple[int, int]]:
        """Visible special tokens as (frame, slot), in stream order."""
        if self.cross_frame_special:
            out = list(self.SP)
        else:
            live = set(self.patch_frames())
            out = [(f, j) for (f, j) in self.SP if f in live]
        if self.camera_only:
            out = [(f, j) for (f, j) in out if j == 0]
        return out

    def visible_tokens(self, P: int) -> set:
        """Visible tokens as ('p', frame, patch_index) / ('s', frame, slot)."""
        out = {("p", f, t) for f in self.attended_patch_frames() for t in range(P)}
        out.update(("s", f, j) for (f, j) in self.visible_specials())
        return out

    def snapshot(self):
        return (tuple(self.C), tuple(self.resident), self.pending, tuple(self.SP), self.defer)
