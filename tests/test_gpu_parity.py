"""GPU parity: the CUDA path through the C ABI against the oracle, on the
seeded workloads, with the tolerances in tests/parity.py.

Tiny and small workloads are compared element by element on every output at
every step; the full-shape workloads compare every code and scale of every
append and a sample of query rows of the attention output (first and last
rows, the ragged tail of the last 128-row tile, and random rows), at steps
that cover an empty, partly filled, full and wrapped ring.
"""
import numpy as np
import pytest
import torch

from kv_cache_serving_append_b200 import configs
from parity import ATOL_MAX, REL_L2, Runner, attn_errors, sample_rows

pytestmark = pytest.mark.gpu


def run_full_compare(cfg_id, steps=None, check_attn_steps=None, rows_per_step=None,
                     out_dtype=torch.float32):
    cfg = configs.get(cfg_id)
    R = Runner(cfg_id, cfg)
    worst = (0.0, 0.0)
    n_steps = cfg["steps"] if steps is None else steps
    for step in range(configs.first_step(cfg), n_steps):
        F = configs.frames_for_step(cfg, step)
        for layer in range(cfg["n_layers"]):
            R.append(layer, step, F)
        for layer in range(cfg["n_layers"]):
            if check_attn_steps is None or step in check_attn_steps:
                rows = None
                if rows_per_step:
                    rows = sample_rows(F * R.T, rows_per_step, 1000 * (step + 1) + layer)
                g, o = R.attend(layer, rows=rows, out_dtype=out_dtype)
                mx, rl = attn_errors(g, o)
                worst = (max(worst[0], mx), max(worst[1], rl))
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


def test_full_shape_layer_sampled_rows(gpu):
    cfg = configs.get(3)
    W = cfg["window_frames"]
    worst = run_full_compare(3, steps=W + 3, check_attn_steps={0, 1, W - 1, W, W + 2},
                             rows_per_step=48)
    print("config 3 worst max-abs %.3g rel-L2 %.3g" % worst)


def test_long_window_pinned_sampled_rows(gpu):
    worst = run_full_compare(5, steps=None, check_attn_steps={-1, 0, 1, 7, 8, 9, 23},
                             rows_per_step=40)
    print("config 5 worst max-abs %.3g rel-L2 %.3g" % worst)


def test_full_shape_48_layer_sequence(gpu):
    """All 48 layers x 16 steps run on the GPU; the oracle follows layers 0
    and 47 (every append checked) and attention is compared at three steps."""
    cfg = configs.get(4)
    R = Runner(4, cfg, oracle_layers=[0, 47])
    for step in range(cfg["steps"]):
        for layer in range(cfg["n_layers"]):
            R.append(layer, step, 1, check=True)
        for layer in range(cfg["n_layers"]):
            out = torch.empty((R.T, R.H, R.D), dtype=torch.bfloat16, device="cuda")
            assert R.cache.attend(layer, out) == 0
        if step in (0, 8, 15):
            for layer in (0, 47):
                rows = sample_rows(R.T, 24, step * 7 + layer)
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
