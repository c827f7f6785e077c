"""The C-ABI library loads on a CPU-only host, exports every symbol the header
declares, and its host-only calls (sizes, layout, validation, status strings,
the injected allocation failure) behave; no kernel is launched here."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rtv.h")


@pytest.fixture(scope="module")
def rtv():
    from kv_cache_serving_append_b200 import build
    build.build()
    from kv_cache_serving_append_b200 import rtv as mod
    return mod


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^(?:const char\*|rtv_status|int)\s+(rtv_\w+)\s*\(", text, re.M)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ["rtv_cache_create", "rtv_cache_append", "rtv_attend", "rtv_cache_advance",
                 "rtv_cache_destroy", "rtv_cache_get_state", "rtv_poll_error",
                 "rtv_status_string", "rtv_cache_required_bytes", "rtv_cache_export"]:
        assert name in syms


def test_library_exports_every_declared_symbol(rtv):
    lib = ctypes.CDLL(rtv.LIB_PATH)
    missing = [s for s in declared_symbols() if not hasattr(lib, s)]
    assert not missing
    # and the binding wraps each of them under the same name
    assert set(declared_symbols()) <= set(rtv._SIGS)
    out = subprocess.run(["nm", "-D", "--defined-only", rtv.LIB_PATH], capture_output=True,
                         text=True).stdout
    exported = set(re.findall(r"\sT\s(rtv_\w+)", out))
    assert set(declared_symbols()) <= exported


def test_debug_and_release_builds(rtv):
    """librtv_debug.so (RTV_DEBUG: kernels bounds-check slot indices) exports
    the same symbols and says it is the debug build; the release library
    refuses the debug-only test hook."""
    from kv_cache_serving_append_b200 import build
    dbg = ctypes.CDLL(build.build(debug=True))
    assert dbg.rtv_debug_build() == 1
    assert rtv.lib.rtv_debug_build() == 0
    assert not [s for s in declared_symbols() if not hasattr(dbg, s)]
    assert rtv.lib.rtv_debug_corrupt_next_attend(None, 3) == rtv.RTV_ERR_INVALID_ARG


def test_status_strings(rtv):
    assert rtv.status_string(7) == "slot index out of range (debug build)"
    for s in range(7):
        assert rtv.status_string(s)
    assert rtv.status_string(5) == "kernel wait timed out"


def test_required_bytes_and_layout(rtv):
    from kv_cache_serving_append_b200 import configs
    cfg = configs.get(3)
    n = rtv.required_bytes(cfg)
    H, D, T = 40, 128, 2992
    S = 0 + 8 + 1
    codes = 2 * S * H * T * D
    # key-range split partials: 4 splits x F*T rows x H x (D O values + 2 statistics), fp32
    split = 4 * T * H * (D + 2) * 4
    assert n >= codes + H * T * D + split
    assert n < (codes + split) * 1.2
    L0 = rtv.layer_layout(cfg, 0)
    for f in ("k_codes", "v_codes", "k_scales", "v_scales", "q_codes", "q_scales", "v_scale_max"):
        assert getattr(L0, f) % 1024 == 0
    assert L0.scale_pitch % 16 == 0 and L0.scale_pitch >= T
    c4 = configs.get(4)
    L1 = rtv.layer_layout(c4, 1)
    L0 = rtv.layer_layout(c4, 0)
    assert L1.k_codes - L0.k_codes == L1.q_codes - L0.q_codes > 0
    assert rtv.required_bytes(c4) > 48 * 2 * S * H * T * D


@pytest.mark.parametrize("change,status", [
    (dict(head_dim=96, rope_t=32, rope_h=32, rope_w=32), 6),
    (dict(rope_t=30, rope_h=50, rope_w=48), 6),
    (dict(rope_t=31), 1),
    (dict(rope_t=16), 1),
    (dict(n_layers=0), 1),
    (dict(pinned_frames=2), 1),
    (dict(max_frames_per_chunk=5), 6),
    (dict(window_frames=70), 6),
    (dict(n_heads=300), 6),
    (dict(rope_base=0.0), 1),
])
def test_invalid_configs_are_rejected(rtv, change, status):
    from kv_cache_serving_append_b200 import configs
    cfg = configs.get(2)
    cfg.update(change)
    c = rtv.make_config(cfg)
    n = ctypes.c_size_t()
    assert rtv.lib.rtv_cache_required_bytes(ctypes.byref(c), ctypes.byref(n)) == status


def test_null_arguments(rtv):
    assert rtv.lib.rtv_cache_required_bytes(None, None) == rtv.RTV_ERR_INVALID_ARG
    assert rtv.lib.rtv_cache_destroy(None) == rtv.RTV_ERR_INVALID_ARG
    assert rtv.lib.rtv_cache_advance(None) == rtv.RTV_ERR_INVALID_ARG
    assert rtv.lib.rtv_attend(None, 0, None, 0, None) == rtv.RTV_ERR_INVALID_ARG
    assert rtv.lib.rtv_cache_append(None, 0, None, None, None, 1, None) == rtv.RTV_ERR_INVALID_ARG
    assert rtv.lib.rtv_poll_error(None) == rtv.RTV_ERR_INVALID_ARG


def test_injected_allocation_failure_returns_oom():
    """The out-of-memory path, injected on the host (no device call is made)."""
    code = (
        "import ctypes\n"
        "from kv_cache_serving_append_b200 import rtv, configs\n"
        "c = rtv.make_config(configs.get(1)); h = ctypes.c_void_p()\n"
        "print(rtv.lib.rtv_cache_create(ctypes.byref(c), None, 0, ctypes.byref(h)), h.value)\n")
    env = dict(os.environ, RTV_INJECT_ALLOC_FAILURE="1", PYTHONPATH=ROOT)
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env,
                         cwd=ROOT, timeout=300)
    assert out.returncode == 0, out.stderr
    assert out.stdout.split() == ["2", "None"]


def test_split_plan_choices_and_invariants(rtv):
    """The key-range split rtv_attend uses (host arithmetic, no device)."""
    # full-shape layer, ring full: 12 row blocks x 40 heads, 9 frames x 47 tiles, 148 SMs:
    # 480 CTAs = 3.24 waves unsplit; 4 splits of <= 106 tiles -> 13 waves of quarter CTAs
    assert rtv.split_plan(480, 9 * 47, 148) == (4, 106)
    # the same layer's first step (one frame of keys): still 4 splits, of 12 tiles (last 11)
    assert rtv.split_plan(480, 47, 148) == (4, 12)
    # two frames per chunk, W=16 + pinned: 24 x 40 units, 19 x 47 tiles -> 2 splits
    assert rtv.split_plan(960, 19 * 47, 148) == (2, 447)
    # 704-token frames, 8 heads, 7 frames of 11 tiles: 24 units fill a fraction of the GPU
    assert rtv.split_plan(24, 77, 148) == (4, 20)
    # too few tiles to split (fewer than 8 per split)
    assert rtv.split_plan(2, 5, 148) == (1, 5)
    assert rtv.split_plan(480, 15, 148) == (1, 15)
    for units in (1, 7, 148, 149, 296, 480, 960, 1500):
        for tiles in (1, 8, 15, 16, 17, 47, 423, 1000):
            s, tps = rtv.split_plan(units, tiles, 148)
            assert 1 <= s <= 4
            assert (s - 1) * tps < tiles <= s * tps          # every split non-empty, all tiles covered
            if s > 1:
                assert tps >= 8
    n, t = ctypes.c_int(), ctypes.c_int()
    for bad in ((0, 1, 148), (1, 0, 148), (1, 1, 0)):
        assert rtv.lib.rtv_split_plan(*bad, ctypes.byref(n), ctypes.byref(t)) == 1
    assert rtv.lib.rtv_split_plan(1, 1, 1, None, ctypes.byref(t)) == 1


def test_binding_rejects_bad_tensors_before_the_library(rtv):
    """The binding checks dtype, contiguity, device and element count of every
    tensor it would pass as a bare pointer, and answers RTV_ERR_INVALID_ARG
    itself; here on CPU tensors against a cache object that has no library
    handle (so nothing could be launched even if a check were missing)."""
    import torch
    from kv_cache_serving_append_b200 import configs
    cfg = configs.get(1)
    c = object.__new__(rtv.Cache)
    c.cfg, c.T, c.handle, c._staged = cfg, 64, None, {}
    c.device = torch.device("cpu")
    n = 64 * cfg["n_heads"] * cfg["head_dim"]
    good = torch.zeros((64, cfg["n_heads"], cfg["head_dim"]), dtype=torch.bfloat16)
    assert c.tensor_status(good, n, (torch.bfloat16,)) == rtv.RTV_OK
    assert c.tensor_status(good.float(), n, (torch.bfloat16,)) == rtv.RTV_ERR_INVALID_ARG   # dtype
    assert c.tensor_status(good.transpose(0, 1), n, (torch.bfloat16,)) == rtv.RTV_ERR_INVALID_ARG  # strided
    assert c.tensor_status(good[:32], n, (torch.bfloat16,)) == rtv.RTV_ERR_INVALID_ARG     # too short
    assert c.tensor_status(None, n, (torch.bfloat16,)) == rtv.RTV_ERR_INVALID_ARG
    c.device = torch.device("cuda", 0)
    assert c.tensor_status(good, n, (torch.bfloat16,)) == rtv.RTV_ERR_INVALID_ARG          # device
    # the hot-path calls answer from those checks
    assert c.append(0, good, good, good, 1) == rtv.RTV_ERR_INVALID_ARG
    assert c.append(0, good, good, good, 0) == rtv.RTV_ERR_INVALID_ARG
    assert c.append(0, good, good, good, 2) == rtv.RTV_ERR_INVALID_ARG    # > max_frames_per_chunk
    c._staged[0] = 1
    out = torch.zeros((64, cfg["n_heads"], cfg["head_dim"]), dtype=torch.float32)
    assert c.attend(0, out) == rtv.RTV_ERR_INVALID_ARG                     # CPU tensor
    assert c.attend(0, out.half()) == rtv.RTV_ERR_INVALID_ARG
    assert c.attend_static_scratch(0, out[:10]) == rtv.RTV_ERR_INVALID_ARG
