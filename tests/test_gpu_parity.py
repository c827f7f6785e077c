"""GPU parity: the CUDA path through the C ABI against the oracle, on the
seeded workloads, with the tolerances in tests/parity.py.

Every code and scale of every append is compared.  Attention outputs are
compared element by element: at every step for the tiny and small
workloads; for the full-shape layer and the long-window workload the whole
output at steps after the ring has wrapped (the launch configuration the
benchmark times, key range split included), and sampled query rows (first
and last rows, the ragged tail of the last 128-row tile, random rows from
every 128-row tile) at the steps that cover an empty, partly filled and
just-full ring.  Chunks of 1 to 4 frames, with and without the pinned slot,
run on small shapes at every step.
"""
import numpy as np
import pytest
import torch

from kv_cache_serving_append_b200 import configs, synth
from parity import ATOL_MAX, REL_L2, Runner, attn_errors, sample_rows

pytestmark = pytest.mark.gpu


def run_full_compare(cfg_id, steps=None, check_attn_steps=None, rows_per_step=None,
                     full_steps=(), out_dtype=torch.float32, cfg=None):
    """Drive a workload through the GPU cache and the oracle; compare every
    append, and the attention output at ``check_attn_steps`` (all steps if
    None): the whole output at ``full_steps`` or when ``rows_per_step`` is
    None, else ``rows_per_step`` sampled rows."""
    cfg = cfg or configs.get(cfg_id)
    R = Runner(cfg_id, cfg)
    worst = (0.0, 0.0)
    n_steps = cfg["steps"] if steps is None else steps
    for step in range(configs.first_step(cfg), n_steps):
        F = configs.frames_for_step(cfg, step)
        for layer in range(cfg["n_layers"]):
            R.append(layer, step, F)
        for layer in range(cfg["n_layers"]):
            if check_attn_steps is None or step in check_attn_steps or step in full_steps:
                rows = None
                if rows_per_step and step not in full_steps:
                    rows = sample_rows(F * R.T, rows_per_step, 1000 * (step + 2) + layer)
                g, o = R.attend(layer, rows=rows, out_dtype=out_dtype)
                mx, rl = attn_errors(g, o)
                worst = (max(worst[0], mx), max(worst[1], rl))
                print(f"cfg {cfg_id} step {step} layer {layer} rows {'all' if rows is None else len(rows)}: "
                      f"max-abs {mx:.4g} rel-L2 {rl:.4g} splits {R.cache.state().last_attend_splits}")
                assert mx <= ATOL_MAX and rl <= REL_L2, (cfg_id, step, layer, mx, rl)
        R.advance()
    R.cache.close()
    return worst


def test_tiny_every_step_full_output(gpu):
    worst = run_full_compare(1)
    print("config 1 worst max-abs %.3g rel-L2 %.3g" % worst)


def test_small_every_step_full_output(gpu):
    worst = run_full_compare(2)
    print("config 2 worst max-abs %.3g rel-L2 %.3g" % worst)


def test_full_shape_layer_full_output_after_wrap(gpu):
    """Config 3: the whole output (2992 rows x 40 heads) at the first step
    whose ring has wrapped and at the next, sampled rows before."""
    cfg = configs.get(3)
    W = cfg["window_frames"]
    worst = run_full_compare(3, steps=W + 4, check_attn_steps={0, 1, W - 1, W},
                             rows_per_step=256, full_steps=(W + 2, W + 3))
    print("config 3 worst max-abs %.3g rel-L2 %.3g" % worst)


def test_long_window_pinned_full_output_after_wrap(gpu):
    """Config 5: the pinned chunk, the filling ring with 640 sampled rows (every
    128-row tile), and the whole output (5984 rows x 40 heads) at the last
    step, long after the ring wrapped."""
    worst = run_full_compare(5, steps=None, check_attn_steps={-1, 0, 1, 7, 8, 9},
                             rows_per_step=640, full_steps=(23,))
    print("config 5 worst max-abs %.3g rel-L2 %.3g" % worst)


def _variable_chunk_cfg(D: int, pinned: int) -> dict:
    split = dict(rope_t=32, rope_h=48, rope_w=48) if D == 128 else dict(rope_t=16, rope_h=24, rope_w=24)
    return dict(name="variable chunks", n_layers=2, n_heads=3, head_dim=D, grid_h=8, grid_w=22,
                max_frames_per_chunk=4, window_frames=5, pinned_frames=pinned, steps=12,
                dist="outlier_channels", rope_base=10000.0, **split)


@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("pinned", [0, 1])
def test_chunks_of_one_to_four_frames(gpu, D, pinned):
    """F_max = 4: chunk steps stage 1, 2, 3, 4, 3, 1, 4, 2, ... frames (so the
    ring's slots are reused at every offset), with and without the pinned
    conditioning slot, at a token count (176) that is not a multiple of the
    128-row or 64-key tiles; the whole attention output and every append is
    compared at every step."""
    cfg = _variable_chunk_cfg(D, pinned)
    pattern = [1, 2, 3, 4, 3, 1, 4, 2, 2, 4, 1, 3]
    R = Runner(2, cfg)
    worst = 0.0
    if pinned:
        for layer in range(2):
            R.append(layer, -1, 1)
        for layer in range(2):
            g, o = R.attend(layer)
            mx, rl = attn_errors(g, o)
            assert mx <= ATOL_MAX and rl <= REL_L2, (D, "pinned chunk", layer, mx, rl)
        R.advance()
    for step, F in enumerate(pattern):
        for layer in range(2):
            R.append(layer, step, F)
        for layer in range(2):
            g, o = R.attend(layer)
            mx, rl = attn_errors(g, o)
            worst = max(worst, mx)
            assert mx <= ATOL_MAX and rl <= REL_L2, (D, pinned, step, F, layer, mx, rl)
        R.advance()
    R.cache.close()
    print(f"F_max 4, D {D}, pinned {pinned}: worst max-abs {worst:.3g}")


def test_several_denoising_passes_per_chunk(gpu):
    """Several append + attend passes per chunk before one advance (each pass
    with new Q/K/V for the same frames): every pass's append and output match
    the oracle driven through the same passes, and the advance commits the
    last pass's K/V."""
    cfg = configs.get(2)
    R = Runner(2, cfg)
    for step in range(cfg["window_frames"] + 3):
        for p in range(3):
            for layer in range(cfg["n_layers"]):
                R.append(layer, 100 * p + step, 1)
            for layer in range(cfg["n_layers"]):
                g, o = R.attend(layer)
                mx, rl = attn_errors(g, o)
                assert mx <= ATOL_MAX and rl <= REL_L2, (step, p, layer, mx, rl)
        R.advance()
    R.cache.close()


def test_full_shape_48_layer_sequence(gpu):
    """All 48 layers x 16 steps run on the GPU; the oracle follows layers 0
    and 47 (every append checked); attention is compared on sampled rows at
    steps 0 and 8 and over the whole output at the last step (ring wrapped)."""
    cfg = configs.get(4)
    R = Runner(4, cfg, oracle_layers=[0, 47])
    for step in range(cfg["steps"]):
        for layer in range(cfg["n_layers"]):
            R.append(layer, step, 1, check=True)
        for layer in range(cfg["n_layers"]):
            out = torch.empty((R.T, R.H, R.D), dtype=torch.bfloat16, device="cuda")
            assert R.cache.attend(layer, out) == 0
        if step in (0, 8, cfg["steps"] - 1):
            for layer in (0, 47):
                rows = None if step == cfg["steps"] - 1 else sample_rows(R.T, 24, step * 7 + layer)
                g, o = R.attend(layer, rows=rows)
                mx, rl = attn_errors(g, o)
                assert mx <= ATOL_MAX and rl <= REL_L2, (step, layer, mx, rl)
        R.advance()
    R.cache.close()


def test_bf16_output_small(gpu):
    cfg = configs.get(2)
    R = Runner(2, cfg)
    for step in range(3):
        for layer in range(2):
            R.append(layer, step, 1)
        for layer in range(2):
            g, o = R.attend(layer, out_dtype=torch.bfloat16)
            # the bf16 store adds up to half a bf16 ulp (2^-8 relative): the
            # fp32 bound holds after that rounding
            assert np.all(np.abs(g - o) <= ATOL_MAX + 2.0 ** -8 * np.abs(o))
            _, rl = attn_errors(g, o)
            assert rl <= REL_L2
        R.advance()
    R.cache.close()


def _degenerate(x: torch.Tensor, seed: int, large: bool) -> torch.Tensor:
    """Seeded (row, head) items made degenerate: all zero (amax = 0), below
    the reciprocal's range (amax < 2^-119: stored as zero), tiny but in range
    (amax near 2^-108), a single nonzero element, and -- for Q and K -- large
    (scores that outgrow the running reference: the softmax's redo and
    rescale paths)."""
    rows, H, _ = x.shape
    g = torch.Generator().manual_seed(seed)
    y = x.float().clone()
    pick = torch.rand((rows, H), generator=g)
    zero = pick < 0.02
    tiny = (pick >= 0.02) & (pick < 0.04)
    single = (pick >= 0.04) & (pick < 0.06)
    small = (pick >= 0.07) & (pick < 0.09)
    y[zero] = 0.0
    y[tiny] = y[tiny] * 2.0 ** -126
    y[small] = y[small] * 2.0 ** -110
    keep = y[single][:, :1].clone()
    y[single] = 0.0
    y[single, :1] = keep
    if large:
        big = (pick >= 0.06) & (pick < 0.07)
        y[big] = y[big] * 2.0 ** 8
    return y.to(torch.bfloat16)


@pytest.mark.gpu
def test_degenerate_items(gpu):
    """Zero, tiny, single-element and large (row, head) items: every append
    code and scale bit-exact, attention over the whole output after the ring
    wrapped."""
    cfg = configs.get(2)

    class DegenerateRunner(Runner):
        def append(self, layer, step, n_frames, check=True):
            q, k, v = synth.chunk(self.cfg_id, self.cfg, layer, step, n_frames)
            base = 7919 * (step + 1) + 31 * layer
            q = _degenerate(q, base, True)
            k = _degenerate(k, base + 1, True)
            v = _degenerate(v, base + 2, False)
            st = self.cache.append(layer, q.to(self.device), k.to(self.device), v.to(self.device), n_frames)
            assert st == 0, self.rtv.status_string(st)
            if layer in self.ora.layers:
                slots = self.ora.append(layer, synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v),
                                        n_frames)
                if check:
                    self.check_append(layer, slots, n_frames)

    R = DegenerateRunner(2, cfg)
    last = cfg["window_frames"] + 2
    for step in range(last + 1):
        for layer in range(cfg["n_layers"]):
            R.append(layer, step, 1)
        if step in (0, last):
            for layer in range(cfg["n_layers"]):
                g, o = R.attend(layer)
                mx, rl = attn_errors(g, o)
                print(f"degenerate step {step} layer {layer}: max-abs {mx:.4g} rel-L2 {rl:.4g}")
                assert mx <= ATOL_MAX and rl <= REL_L2, (step, layer, mx, rl)
        R.advance()
    R.cache.close()
