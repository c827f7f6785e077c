"""Ring-buffer KV cache bookkeeping and storage, as an explicit slot map.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: aidose.in, "Runway explains how it serves a 57B video model in real
time", third paragraph (the cache is a ring buffer that moves forward without
copying); pttl.gr, section "Από οκτώ H100 σε τέσσερις" (a circular buffer).
The pages give neither the window nor the slot rule; the reading used here:

* The cache holds ``P0`` pinned slots (0 or 1) followed by ``C = W + F_max``
  ring slots, W = window frames, F_max = most frames one chunk may stage.
* With ``P0 = 1`` the first chunk is the conditioning frame (one frame,
  absolute index 0); it is staged straight into slot 0 and, once committed,
  never moves.  Generated frames then start at absolute index 1.
* Generated frame ``g`` (0-based, counted after the pinned frame) lives in
  slot ``P0 + (g mod C)``.  Its absolute frame index is ``P0c + g`` where
  ``P0c`` is 1 once the pinned frame is committed, else 0.
* After ``G`` generated frames are committed, the visible window is
  generated frames ``max(0, G - W) .. G - 1``.  A chunk of F frames is staged
  as generated frames ``G .. G + F - 1``; since ``F <= F_max`` these slots
  never hold a frame of the window.
* The key set of an attention call is, in logical order: the pinned frame
  (if committed), the window oldest to newest, then the staged frames.
* Advancing commits the staged frames: ``G += F`` (or marks the pinned frame
  committed).  Nothing is copied.
"""
from __future__ import annotations

import numpy as np


class OracleRing:
    """Integer-only ring state with an explicit ``slot_of_frame`` map."""

    def __init__(self, window: int, max_frames_per_chunk: int, pinned: int):
        assert window >= 0 and max_frames_per_chunk >= 1 and pinned in (0, 1)
        self.W = window
        self.F_max = max_frames_per_chunk
        self.P0 = pinned
        self.C = window + max_frames_per_chunk
        self.n_slots = pinned + self.C
        self.G = 0                       # generated frames committed
        self.pinned_committed = False
        self.slot_of_frame: dict[int, int] = {}   # visible committed frames only
        self.frame_of_slot = [-1] * self.n_slots   # -1: slot holds no visible frame
        self.visible: list[int] = []     # absolute frame indices, logical order

    # -- derived ----------------------------------------------------------
    @property
    def in_pinned_phase(self) -> bool:
        return self.P0 == 1 and not self.pinned_committed

    @property
    def frames_committed(self) -> int:
        return (1 if self.pinned_committed else 0) + self.G

    @property
    def head(self) -> int:
        """Slot that the next generated frame will occupy."""
        return self.P0 + (self.G % self.C)

    def staged_slots(self, n_frames: int) -> list[int]:
        if not 1 <= n_frames <= self.F_max:
            raise ValueError("n_frames out of range")
        if self.in_pinned_phase:
            if n_frames != 1:
                raise ValueError("the pinned conditioning chunk is one frame")
            return [0]
        return [self.P0 + ((self.G + f) % self.C) for f in range(n_frames)]

    def staged_frames(self, n_frames: int) -> list[int]:
        """Absolute frame indices of the frames a chunk of n_frames stages."""
        base = self.frames_committed
        return [base + f for f in range(n_frames)]

    def key_slots(self, n_staged: int) -> list[int]:
        return [self.slot_of_frame[t] for t in self.visible] + self.staged_slots(n_staged)

    # -- transitions ------------------------------------------------------
    def commit(self, n_frames: int) -> None:
        slots = self.staged_slots(n_frames)
        frames = self.staged_frames(n_frames)
        for t, s in zip(frames, slots):
            # a staged frame may only take a slot that holds no visible frame
            if self.frame_of_slot[s] != -1:
                raise AssertionError(f"slot {s} still holds visible frame {self.frame_of_slot[s]}")
            self.frame_of_slot[s] = t
            self.slot_of_frame[t] = s
            self.visible.append(t)
        pinned_now = self.in_pinned_phase
        if pinned_now:
            self.pinned_committed = True
        else:
            self.G += n_frames
        # generated frames that fell out of the window stop being visible
        n_pinned = 1 if self.pinned_committed else 0
        while len(self.visible) - n_pinned > self.W:
            t = self.visible.pop(n_pinned)
            s = self.slot_of_frame.pop(t)
            self.frame_of_slot[s] = -1


class OracleCache:
    """Per-layer FP8 cache contents plus the ring map, driven like the library.

    ``layers`` may list a subset of the model's layers (the oracle then keeps
    only those, to bound host memory for the 48-layer sequence).
    """

    def __init__(self, cfg: dict, layers=None):
        from . import append_tensor  # the oracle's own arithmetic
        self._append_tensor = append_tensor
        self.cfg = cfg
        self.H, self.D = cfg["n_heads"], cfg["head_dim"]
        self.T = cfg["grid_h"] * cfg["grid_w"]
        self.split = (cfg["rope_t"], cfg["rope_h"], cfg["rope_w"])
        self.base = cfg.get("rope_base", 10000.0)
        self.ring = OracleRing(cfg["window_frames"], cfg["max_frames_per_chunk"],
                               cfg["pinned_frames"])
        layers = range(cfg["n_layers"]) if layers is None else layers
        S, H, T, D = self.ring.n_slots, self.H, self.T, self.D
        self.layers = {}
        for l in layers:
            self.layers[l] = dict(
                kc=np.zeros((S, H, T, D), np.uint8), sk=np.zeros((S, H, T), np.float32),
                vc=np.zeros((S, H, T, D), np.uint8), sv=np.zeros((S, H, T), np.float32),
                qc=None, sq=None, staged=0, qnear=None, knear=None, vnear=None)

    def append(self, layer: int, q_bits, k_bits, v_bits, n_frames: int):
        """q/k/v_bits: uint16 [n_frames*T, H, D] bf16 bit patterns."""
        L = self.layers[layer]
        T = self.T
        slots = self.ring.staged_slots(n_frames)
        t0 = self.ring.frames_committed
        gw = self.cfg["grid_w"]
        qc, sq, qn = self._append_tensor(q_bits, T, gw, t0, True, self.split, self.base)
        kc, sk, kn = self._append_tensor(k_bits, T, gw, t0, True, self.split, self.base)
        vc, sv, vn = self._append_tensor(v_bits, T, gw, t0, False, self.split, self.base)
        for f, s in enumerate(slots):
            L["kc"][s] = kc[:, f * T:(f + 1) * T]
            L["sk"][s] = sk[:, f * T:(f + 1) * T]
            L["vc"][s] = vc[:, f * T:(f + 1) * T]
            L["sv"][s] = sv[:, f * T:(f + 1) * T]
        L.update(qc=qc, sq=sq, staged=n_frames, qnear=qn, knear=kn, vnear=vn)
        return slots

    def key_set(self, layer: int):
        L = self.layers[layer]
        slots = self.ring.key_slots(L["staged"])
        kc = np.concatenate([L["kc"][s] for s in slots], axis=1)
        vc = np.concatenate([L["vc"][s] for s in slots], axis=1)
        sk = np.concatenate([L["sk"][s] for s in slots], axis=1)
        sv = np.concatenate([L["sv"][s] for s in slots], axis=1)
        return slots, kc, sk, vc, sv

    def attend(self, layer: int, rows=None, want_psum=False, matmul=False):
        """fp64 attention of the staged chunk over the key set; ``matmul``
        selects the library-matmul form of the same definition (for
        full-shape outputs)."""
        from . import attend, attend_matmul
        L = self.layers[layer]
        if L["staged"] == 0:
            raise RuntimeError("layer has no staged frames")
        _, kc, sk, vc, sv = self.key_set(layer)
        if matmul:
            assert not want_psum
            return attend_matmul(L["qc"], L["sq"], kc, sk, vc, sv, rows=rows)
        return attend(L["qc"], L["sq"], kc, sk, vc, sv, rows=rows, want_psum=want_psum)

    def advance(self):
        ns = {L["staged"] for L in self.layers.values()}
        if len(ns) != 1 or 0 in ns:
            raise RuntimeError("every layer must be staged with the same frame count")
        n = ns.pop()
        self.ring.commit(n)
        for L in self.layers.values():
            L["staged"] = 0
