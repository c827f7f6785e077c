"""Seeded synthetic Q/K/V chunks (the only module both sides share).

Holds no arithmetic of the method: it only draws random bf16 tensors with the
shapes and value mix of the workloads in ``configs.py``.  Layout of every
tensor: ``[n_frames * T, n_heads, head_dim]`` bf16, token-major with the
hidden dimension (heads x head_dim) contiguous, as a QKV projection writes it.

Seeds: config 1 uses ``100*layer + step`` (so its first chunk is seed 0);
the other configs use ``1000*cfg + 100*layer + step``; Q, K and V use
sub-streams 0, 1 and 2 of that seed.  The pinned conditioning chunk of a
config with a pinned slot is step -1.

Distributions:
  normal            N(0, 1)
  outlier_channels  N(0, 1) with 4 channels per (layer, head), drawn once
                    from the config seed without replacement, scaled x8
                    (the same channels in Q, K and V and at every step)
  outlier_tokens    N(0, 1) with exactly 1% of the chunk's tokens (30 of
                    2992 per frame), drawn per tensor, scaled x4 in all heads
  student_t         K and V Student-t with 3 degrees of freedom, clipped to
                    +-64; Q is N(0, 1)
Every value is rounded to bf16 once, after scaling.
"""
from __future__ import annotations

import torch


_CFG_NUM = {1: 1, 2: 2, 3: 3, 4: 4, 5: 5, "4s": 6}


def seed_of(cfg_id, layer: int, step: int) -> int:
    base = 0 if cfg_id == 1 else 1000 * _CFG_NUM[cfg_id]
    return base + 100 * layer + step


def _gen(seed: int, sub: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(4 * (seed + 1) + sub)
    return g


def _outlier_channels(cfg_id, cfg, layer: int) -> torch.Tensor:
    """[H, 4] channel indices, fixed per (layer, head) for the whole run."""
    g = torch.Generator()
    g.manual_seed(7919 * (1 + layer) + 17 * (_CFG_NUM[cfg_id] + 1))
    H, D = cfg["n_heads"], cfg["head_dim"]
    return torch.stack([torch.randperm(D, generator=g)[:4] for _ in range(H)])


def chunk(cfg_id, cfg: dict, layer: int, step: int, n_frames: int, device="cpu",
          seed_offset: int = 0):
    """Return (q, k, v) bf16 tensors [n_frames*T, H, D] on ``device``."""
    H, D = cfg["n_heads"], cfg["head_dim"]
    T = cfg["grid_h"] * cfg["grid_w"]
    rows = n_frames * T
    seed = seed_of(cfg_id, layer, step) + seed_offset
    dist = cfg["dist"]
    out = []
    for sub in range(3):
        g = _gen(seed, sub, device)
        x = torch.randn((rows, H, D), generator=g, device=device, dtype=torch.float32)
        if dist == "outlier_channels":
            ch = _outlier_channels(cfg_id, cfg, layer).to(device)
            mult = torch.ones((H, D), device=device)
            mult.scatter_(1, ch, 8.0)
            x = x * mult
        elif dist == "outlier_tokens":
            n_out = max(1, round(0.01 * rows))
            idx = torch.randperm(rows, generator=g, device=device)[:n_out]
            x[idx] *= 4.0
        elif dist == "student_t" and sub > 0:
            chi2 = (torch.randn((3, rows, H, D), generator=g, device=device) ** 2).sum(0)
            x = x / torch.sqrt(chi2 / 3.0)
            x = x.clamp_(-64.0, 64.0)
        elif dist not in ("normal", "student_t"):
            raise ValueError(dist)
        out.append(x.to(torch.bfloat16).contiguous())
    return tuple(out)


def bf16_bits(x: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    return x.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")


def projection_inputs(cfg: dict, layer: int, step: int, n_frames: int, hidden: int, exact: bool,
                      seed_offset: int = 0):
    """E4M3 codes and fp32 scales for the fused projection: activations
    x [n_frames*T, hidden] with one scale per row, weights w [3*H*D, hidden]
    with one scale per output feature.  ``exact``: codes only from the binades
    [0.5, 1) and [1, 2) (random sign, some zeros), whose products are
    multiples of 2^-8 below 4, so any fp32 sum of up to 2^14 of them is exact
    whatever the order; otherwise codes of a N(0, 1) draw.  Returns numpy
    (x_codes, x_scales, w_codes, w_scales)."""
    import numpy as np
    T = cfg["grid_h"] * cfg["grid_w"]
    rows, feats = n_frames * T, 3 * cfg["n_heads"] * cfg["head_dim"]
    rng = np.random.default_rng(7 * (seed_of(2, layer, step) + 1) + 3 * hidden + seed_offset)

    def codes(shape):
        if exact:
            c = ((rng.integers(6, 8, shape) << 3) | rng.integers(0, 8, shape)).astype(np.uint8)
            c |= (rng.integers(0, 2, shape) << 7).astype(np.uint8)
            c[rng.random(shape) < 0.02] = 0
            return c
        import torch
        x = torch.from_numpy(rng.standard_normal(shape).astype(np.float32) * 64.0)
        return x.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()

    xc, wc = codes((rows, hidden)), codes((feats, hidden))
    sx = (rng.uniform(0.5, 2.0, rows) / 64.0).astype(np.float32)
    sw = (rng.uniform(0.5, 2.0, feats) / (64.0 * np.sqrt(hidden))).astype(np.float32)
    return xc, sx, wc, sw
