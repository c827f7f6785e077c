"""Helpers shared by the GPU parity tests: drive the CUDA path (through the
C ABI) and the oracle on the same seeded inputs, and compare them with the
tolerances of the method's definition.

Tolerances (written here once, used by every parity test):
  * ring state: bit-exact (slots, visible frames, head, counts);
  * E4M3 codes: identical, except 0x00 == 0x80 (both zero) and one code step
    between adjacent magnitudes of the same sign where the oracle flags the
    fp32 value as within 1e-6 relative of a rounding midpoint;
  * scales: within 1e-6 relative, or both 0;
  * attention output: max |gpu - oracle| <= 3e-2 and
    ||gpu - oracle||_2 / ||oracle||_2 <= 1e-2 over the compared rows.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from kv_cache_serving_append_b200 import configs, synth

ATOL_MAX = 3e-2
REL_L2 = 1e-2
SCALE_RTOL = 1e-6


def compare_codes(gpu: np.ndarray, ora: np.ndarray, near: np.ndarray) -> dict:
    gpu = gpu.astype(np.int32)
    ora = ora.astype(np.int32)
    same = gpu == ora
    both_zero = ((gpu & 0x7F) == 0) & ((ora & 0x7F) == 0)
    diff = ~(same | both_zero)
    one_step = ((gpu & 0x80) == (ora & 0x80)) & (np.abs((gpu & 0x7F) - (ora & 0x7F)) == 1)
    allowed = diff & one_step & (near != 0)
    bad = diff & ~allowed
    return dict(n=gpu.size, diff=int(diff.sum()), allowed=int(allowed.sum()), bad=int(bad.sum()))


def compare_scales(gpu: np.ndarray, ora: np.ndarray) -> int:
    gpu = gpu.astype(np.float64)
    ora = ora.astype(np.float64)
    ok = (np.abs(gpu - ora) <= SCALE_RTOL * np.abs(ora)) | ((gpu == 0) & (ora == 0))
    return int((~ok).sum())


def attn_errors(gpu: np.ndarray, ora: np.ndarray) -> tuple[float, float]:
    d = gpu.astype(np.float64) - ora
    return float(np.abs(d).max()), float(np.linalg.norm(d) / max(np.linalg.norm(ora), 1e-300))


def ring_state_matches(st, ring: oracle.OracleRing) -> None:
    assert st.frames_committed == ring.frames_committed
    assert st.generated_committed == ring.G
    assert st.pinned_committed == int(ring.pinned_committed)
    assert st.head == ring.head
    assert st.n_slots == ring.n_slots
    assert st.n_visible == len(ring.visible)
    assert list(st.visible_frames[:st.n_visible]) == ring.visible
    assert list(st.visible_slots[:st.n_visible]) == [ring.slot_of_frame[t] for t in ring.visible]
    assert [st.frame_of_slot[s] for s in range(ring.n_slots)] == ring.frame_of_slot


def sample_rows(M: int, n: int, seed: int) -> np.ndarray:
    """About n query rows: the first and last rows and the ragged tail of the
    last 128-row tile, plus random rows drawn from every 128-row tile alike."""
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 127, 128, M - 1, M - 2, M - 48, (M // 128) * 128]
    fixed = [r for r in fixed if 0 <= r < M]
    n_tiles = (M + 127) // 128
    per_tile = max(1, -(-max(0, n - len(fixed)) // n_tiles))
    rest = []
    for t in range(n_tiles):
        lo, hi = 128 * t, min(M, 128 * t + 128)
        rest.extend(rng.choice(np.arange(lo, hi), size=min(per_tile, hi - lo), replace=False))
    return np.unique(np.concatenate([fixed, rest]).astype(np.int32))


class Runner:
    """Drives one workload through the GPU cache and the oracle in lockstep."""

    def __init__(self, cfg_id, cfg=None, oracle_layers=None, device="cuda"):
        from kv_cache_serving_append_b200 import rtv
        self.rtv = rtv
        self.cfg_id = cfg_id
        self.cfg = cfg or configs.get(cfg_id)
        self.cache = rtv.Cache(self.cfg, device)
        self.ora = oracle.OracleCache(self.cfg, layers=oracle_layers)
        self.T = configs.tokens_per_frame(self.cfg)
        self.H, self.D = self.cfg["n_heads"], self.cfg["head_dim"]
        self.device = device

    def append(self, layer: int, step: int, n_frames: int, check=True):
        q, k, v = synth.chunk(self.cfg_id, self.cfg, layer, step, n_frames)
        qd, kd, vd = q.to(self.device), k.to(self.device), v.to(self.device)
        st = self.cache.append(layer, qd, kd, vd, n_frames)
        assert st == 0, self.rtv.status_string(st)
        if layer in self.ora.layers:
            slots = self.ora.append(layer, synth.bf16_bits(q), synth.bf16_bits(k),
                                    synth.bf16_bits(v), n_frames)
            if check:
                self.check_append(layer, slots, n_frames)
        return qd, kd, vd

    def check_append(self, layer: int, slots, n_frames: int):
        torch.cuda.synchronize()
        V = self.cache.views(layer)
        L = self.ora.layers[layer]
        T = self.T
        rows = n_frames * T
        # Q workspace [H][F_max*T][D] -> first n_frames*T rows
        r = compare_codes(V["q_codes"][:, :rows].cpu().numpy(), L["qc"], L["qnear"])
        assert r["bad"] == 0, ("Q codes", r)
        assert compare_scales(V["q_scales"][:, :rows].cpu().numpy(), L["sq"]) == 0
        for f, s in enumerate(slots):
            for name, near_key in (("k", "knear"), ("v", "vnear")):
                g = V[f"{name}_codes"][s].cpu().numpy()
                o = L[f"{name}c"][s]
                near = L[near_key][:, f * T:(f + 1) * T]
                r = compare_codes(g, o, near)
                assert r["bad"] == 0, (name, f, s, r)
                bad = compare_scales(V[f"{name}_scales"][s].cpu().numpy(), L[f"s{name}"][s])
                assert bad == 0, (name, "scales", f, s, bad)
            # V-scale max tag of the frame: largest V scale over its tokens, per head
            vmax = V["v_scale_max"][s].cpu().numpy().astype(np.uint64) & np.uint64(0xffffffff)
            vmax_f = vmax.astype(np.uint32).view(np.float32)
            assert np.array_equal(vmax_f, L["sv"][s].max(axis=1))

    def attend(self, layer: int, rows=None, out_dtype=torch.float32):
        n = self.ora.layers[layer]["staged"]
        M = n * self.T
        out = torch.full((M, self.H, self.D), float("nan"), dtype=out_dtype, device=self.device)
        st = self.cache.attend(layer, out)
        assert st == 0, self.rtv.status_string(st)
        torch.cuda.synchronize()
        assert self.cache.poll_error() == 0
        g = out.float().cpu().numpy()
        # large calls use the oracle's library-matmul form of the same
        # definition (pinned to the C loops by the CPU tests)
        nk = len(self.ora.ring.key_slots(n)) * self.T
        big = (M if rows is None else len(rows)) * nk * self.H > 2e8
        o = self.ora.attend(layer, rows=rows, matmul=big)
        if rows is not None:
            g = g[rows]
        assert np.isfinite(g).all()
        return g, o

    def advance(self):
        assert self.cache.advance() == 0
        self.ora.advance()
        ring_state_matches(self.cache.state(), self.ora.ring)
