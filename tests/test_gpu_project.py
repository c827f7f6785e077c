"""GPU parity of the fused QKV projection + append (rtv_cache_append_project):
an FP8 GEMM on tcgen05 tensor cores whose epilogue does the append.

With inputs whose products and sums are exact in fp32 in any order (codes
from two binades; synth.projection_inputs(exact=True)), the projected bf16
Q/K/V are the oracle's exactly, so every code and scale of every append is
held to the append's own tolerance (bit-exact but for the flagged rounding
boundaries), at the small shape and at the full layer shape with the full
hidden width.  With N(0,1) codes the fp32 accumulation order can move a
projected value across a bf16 rounding boundary; codes then may differ by
one step and scales by one bf16 ulp of the row's largest value, on a small
fraction of rows (one E4M3 step is 1/16 of a value, so the oracle's own
cache is then not the GPU's; the attention check takes the GPU's cache
contents into the oracle first).  Attention over the projected cache meets
the attention tolerance either way."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_serving_append_b200 import configs, synth
from parity import ATOL_MAX, REL_L2, Runner, attn_errors, compare_codes

pytestmark = pytest.mark.gpu


def _project_step(R, layer, step, hidden, exact, n_frames=1):
    from kv_cache_serving_append_b200 import rtv
    cfg = R.cfg
    H, D = cfg["n_heads"], cfg["head_dim"]
    xc, sx, wc, sw = synth.projection_inputs(cfg, layer, step, n_frames, hidden, exact)
    dev = [torch.from_numpy(a).cuda() for a in (xc, sx, wc, sw)]
    assert R.cache.append_project(layer, *dev, n_frames) == rtv.RTV_OK
    bits = oracle.project_qkv(xc, sx, wc, sw)
    rows = bits.shape[0]
    q, k, v = (bits[:, i * H * D:(i + 1) * H * D].reshape(rows, H, D) for i in range(3))
    return R.ora.append(layer, q, k, v, n_frames)


def _adopt_gpu_cache(R, layer, slots, n_frames):
    """Give the oracle the GPU's codes and scales of this append (after the
    relaxed check), so that the attention is compared on the same cache."""
    torch.cuda.synchronize()
    V = R.cache.views(layer)
    L = R.ora.layers[layer]
    rows = n_frames * R.T
    L["qc"] = V["q_codes"][:, :rows].cpu().numpy().copy()
    L["sq"] = V["q_scales"][:, :rows].cpu().numpy().copy()
    for s in slots:
        for name in ("k", "v"):
            L[f"{name}c"][s] = V[f"{name}_codes"][s].cpu().numpy()
            L[f"s{name}"][s] = V[f"{name}_scales"][s].cpu().numpy()


def _relaxed_check(R, layer, slots, n_frames):
    torch.cuda.synchronize()
    V = R.cache.views(layer)
    L = R.ora.layers[layer]
    T = R.T
    bad_rows = 0
    total_rows = 0
    for name in ("k", "v"):
        for f, s in enumerate(slots):
            g = V[f"{name}_codes"][s].cpu().numpy().astype(np.int32)
            o = L[f"{name}c"][s].astype(np.int32)
            step = np.abs((g & 0x7F) - (o & 0x7F))
            assert step.max() <= 1, name
            gs = V[f"{name}_scales"][s].cpu().numpy().astype(np.float64)
            os_ = L[f"s{name}"][s].astype(np.float64)
            assert np.all(np.abs(gs - os_) <= 2.0 ** -7 * np.abs(os_)), name
            bad_rows += int((step.max(axis=-1) > 0).sum())
            total_rows += step.shape[0] * step.shape[1]
    assert bad_rows <= 0.05 * total_rows, (bad_rows, total_rows)


@pytest.mark.parametrize("exact", [True, False])
def test_projected_append_small_shape(gpu, exact):
    cfg = configs.get(2)                      # 2 layers, 8 heads x D128, 704 tokens, W = 6
    R = Runner(2, cfg)
    for step in range(cfg["window_frames"] + 2):
        for layer in range(cfg["n_layers"]):
            slots = _project_step(R, layer, step, 1024, exact)
            if exact:
                R.check_append(layer, slots, 1)
            else:
                _relaxed_check(R, layer, slots, 1)
                _adopt_gpu_cache(R, layer, slots, 1)
        for layer in range(cfg["n_layers"]):
            g, o = R.attend(layer)
            mx, rl = attn_errors(g, o)
            assert mx <= ATOL_MAX and rl <= REL_L2, (exact, step, layer, mx, rl)
        R.advance()
    R.cache.close()


def test_projected_append_full_layer_shape_exact(gpu):
    """40 heads x D128, 2992 tokens, hidden 5120 (a 2992 x 15360 x 5120 FP8
    GEMM): every code and scale of the first two chunks, and the attention."""
    cfg = configs.get(3)
    R = Runner(3, cfg)
    for step in range(2):
        slots = _project_step(R, 0, step, 5120, True)
        R.check_append(0, slots, 1)
        rows = np.arange(0, R.T, 7, dtype=np.int32)
        g, o = R.attend(0, rows=rows)
        mx, rl = attn_errors(g, o)
        assert mx <= ATOL_MAX and rl <= REL_L2, (step, mx, rl)
        R.advance()
    R.cache.close()


def test_projected_append_two_frames_pinned_and_errors(gpu):
    """Chunks of two frames behind a pinned conditioning frame (exact inputs),
    and the shapes the fused epilogue does not implement."""
    from kv_cache_serving_append_b200 import rtv
    cfg = dict(configs.get(2), max_frames_per_chunk=2, window_frames=4, pinned_frames=1, n_layers=1)
    R = Runner(2, cfg)
    slots = _project_step(R, 0, -1, 512, True, n_frames=1)
    R.check_append(0, slots, 1)
    R.advance()
    for step in range(4):
        slots = _project_step(R, 0, step, 512, True, n_frames=2)
        R.check_append(0, slots, 2)
        g, o = R.attend(0)
        mx, rl = attn_errors(g, o)
        assert mx <= ATOL_MAX and rl <= REL_L2
        R.advance()
    R.cache.close()
    c1 = rtv.Cache(configs.get(1))                 # head_dim 64: not implemented
    xc, sx, wc, sw = (torch.from_numpy(a).cuda() for a in synth.projection_inputs(
        configs.get(1), 0, 0, 1, 128, True))
    wc = torch.zeros((3 * 2 * 64, 128), dtype=torch.uint8, device="cuda")
    sw = torch.ones(3 * 2 * 64, dtype=torch.float32, device="cuda")
    assert c1.append_project(0, xc, sx, wc, sw, 1) == rtv.RTV_ERR_UNSUPPORTED
    c1.close()
