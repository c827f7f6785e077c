"""Workload shapes for the cache-append + attention path.

Pure data: no arithmetic of the method lives here.  Each entry gives the
``rtv_cache_config`` fields plus the step count and the input distribution
used by the synthetic generators (``synth.py``).

Shapes follow the serving workload described on the pages: 704x1088 video at
24 fps in 4-frame chunks (aidose.in, "Runway explains how it serves a 57B
video model in real time", second paragraph; pttl.gr, section "Τέσσερα νέα
καρέ κάθε 166,7 χιλιοστά του δευτερολέπτου"); one latent frame of a 16x
spatial reduction is a 44x68 grid of 2992 tokens.  Head count, head_dim,
window, RoPE split and base, chunk size and the pinned slot are not on the
pages; they are the workload definitions below.
"""
from __future__ import annotations

COMMON = dict(rope_base=10000.0)

CONFIGS = {
    # tiny case the oracle finishes in milliseconds
    1: dict(name="tiny: 1 layer, 2 heads, D64, 8x8 grid, F1, W4, 6 steps",
            n_layers=1, n_heads=2, head_dim=64, grid_h=8, grid_w=8,
            max_frames_per_chunk=1, window_frames=4, pinned_frames=0,
            rope_t=16, rope_h=24, rope_w=24, steps=6, dist="normal"),
    # small multi-head case with fixed outlier channels
    2: dict(name="small: 2 layers, 8 heads, D128, 22x32 grid, F1, W6, 10 steps",
            n_layers=2, n_heads=8, head_dim=128, grid_h=22, grid_w=32,
            max_frames_per_chunk=1, window_frames=6, pinned_frames=0,
            rope_t=32, rope_h=48, rope_w=48, steps=10, dist="outlier_channels"),
    # full-shape single layer, timed in steady state with the ring full
    3: dict(name="full-shape layer: 40 heads, D128, 44x68 grid (2992 tok), F1, W8",
            n_layers=1, n_heads=40, head_dim=128, grid_h=44, grid_w=68,
            max_frames_per_chunk=1, window_frames=8, pinned_frames=0,
            rope_t=32, rope_h=48, rope_w=48, steps=12, dist="outlier_tokens"),
    # 48-layer step sequence at the full-layer shape (the 11.8 GB FP8 cache
    # figure of this workload is only reached with the full-layer shape)
    4: dict(name="full-shape sequence: 48 layers x 16 steps, 40 heads, D128, 2992 tok, W8",
            n_layers=48, n_heads=40, head_dim=128, grid_h=44, grid_w=68,
            max_frames_per_chunk=1, window_frames=8, pinned_frames=0,
            rope_t=32, rope_h=48, rope_w=48, steps=16, dist="outlier_tokens"),
    # long window, two frames per chunk, pinned conditioning slot, heavy tails
    5: dict(name="long window: 40 heads, D128, 2992 tok, F2, W16, pinned slot, 24 steps",
            n_layers=1, n_heads=40, head_dim=128, grid_h=44, grid_w=68,
            max_frames_per_chunk=2, window_frames=16, pinned_frames=1,
            rope_t=32, rope_h=48, rope_w=48, steps=24, dist="student_t"),
    # the 48-layer sequence at the small-case shape (cheap extra)
    "4s": dict(name="48 layers x 16 steps at the small-case shape",
               n_layers=48, n_heads=8, head_dim=128, grid_h=22, grid_w=32,
               max_frames_per_chunk=1, window_frames=8, pinned_frames=0,
               rope_t=32, rope_h=48, rope_w=48, steps=16, dist="outlier_channels"),
}

for _c in CONFIGS.values():
    for _k, _v in COMMON.items():
        _c.setdefault(_k, _v)


def get(cfg_id) -> dict:
    if isinstance(cfg_id, str) and cfg_id.isdigit():
        cfg_id = int(cfg_id)
    return dict(CONFIGS[cfg_id])


def tokens_per_frame(cfg: dict) -> int:
    return cfg["grid_h"] * cfg["grid_w"]


def frames_for_step(cfg: dict, step: int) -> int:
    """Frames staged at chunk step ``step``: the pinned conditioning chunk
    (step -1 when the config has a pinned slot) is one frame."""
    if cfg["pinned_frames"] and step < 0:
        return 1
    return cfg["max_frames_per_chunk"]


def first_step(cfg: dict) -> int:
    return -1 if cfg["pinned_frames"] else 0
