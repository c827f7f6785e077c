"""GPU tests of the debug build (librtv_debug.so, RTV_DEBUG) and of guard
bytes around the cache buffer.

The debug build's kernels check every ring slot they are given against the
cache's slot count before touching memory.  Run in a child process with
RTV_LIBRARY=debug: normal workloads pass parity with no error recorded; a key
set that names an out-of-range slot (planted through the debug-only hook, so
no real memory is ever misaddressed) is caught, reported as RTV_ERR_BOUNDS by
rtv_poll_error, and the context stays usable.  The guard test runs the
release library with the cache inside a larger caller-owned buffer whose
margins hold a pattern, and checks that no kernel wrote outside the cache."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from kv_cache_serving_append_b200 import configs, synth

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys
sys.path[:0] = [ROOT, ROOT + "/tests"]
import torch
from kv_cache_serving_append_b200 import rtv, configs
from parity import ATOL_MAX, REL_L2, Runner, attn_errors
assert rtv.lib.rtv_debug_build() == 1
for cfg_id in (1, 2):
    cfg = configs.get(cfg_id)
    R = Runner(cfg_id, cfg)
    for step in range(cfg["window_frames"] + 2):
        for layer in range(cfg["n_layers"]):
            R.append(layer, step, 1)
        for layer in range(cfg["n_layers"]):
            g, o = R.attend(layer)
            mx, rl = attn_errors(g, o)
            assert mx <= ATOL_MAX and rl <= REL_L2, (cfg_id, step, mx, rl)
        R.advance()
    assert R.cache.poll_error() == rtv.RTV_OK
    # plant an out-of-range slot in the next attention's key set
    n_slots = R.cache.state().n_slots
    for layer in range(cfg["n_layers"]):
        R.append(layer, 99, 1)
    out = torch.full((R.T, R.H, R.D), 7.0, device="cuda")
    assert rtv.lib.rtv_debug_corrupt_next_attend(R.cache.handle, n_slots + 5) == rtv.RTV_OK
    assert R.cache.attend(0, out) == rtv.RTV_OK
    assert R.cache.poll_error() == rtv.RTV_ERR_BOUNDS
    assert R.cache.poll_error() == rtv.RTV_OK          # the word was cleared
    g, o = R.attend(0)                                 # same context, normal call
    mx, rl = attn_errors(g, o)
    assert mx <= ATOL_MAX and rl <= REL_L2
    R.cache.close()
print("debug build ok")
""".replace("ROOT", repr(ROOT))


def test_debug_build_checks_slots_and_reports_bounds(gpu):
    env = dict(os.environ, RTV_LIBRARY="debug")
    out = subprocess.run([sys.executable, "-c", CHILD], capture_output=True, text=True, env=env,
                         cwd=ROOT, timeout=900)
    assert out.returncode == 0, out.stdout[-3000:] + out.stderr[-3000:]
    assert "debug build ok" in out.stdout


def test_guard_bytes_around_a_caller_owned_cache_buffer(gpu):
    """The cache sits 1 MiB into a caller-owned buffer with 1 MiB of pattern on
    each side; a full workload (appends, split attention, advances) leaves the
    pattern intact."""
    from kv_cache_serving_append_b200 import rtv
    import ctypes
    cfg = configs.get(2)
    need = rtv.required_bytes(cfg)
    guard = 1 << 20
    big = torch.full((need + 2 * guard,), 0xA5, dtype=torch.uint8, device="cuda")
    c = rtv.make_config(cfg)
    h = ctypes.c_void_p()
    assert rtv.lib.rtv_cache_create(ctypes.byref(c), ctypes.c_void_p(big.data_ptr() + guard), need,
                                    ctypes.byref(h)) == rtv.RTV_OK
    T, H, D = 704, 8, 128
    out = torch.empty((T, H, D), dtype=torch.float32, device="cuda")
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    splits = set()
    for step in range(cfg["window_frames"] + 3):
        for layer in range(2):
            q, k, v = (t.cuda() for t in synth.chunk(2, cfg, layer, step, 1))
            assert rtv.lib.rtv_cache_append(h, layer, ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                            ctypes.c_void_p(v.data_ptr()), 1, s) == rtv.RTV_OK
            assert rtv.lib.rtv_attend(h, layer, ctypes.c_void_p(out.data_ptr()), rtv.RTV_OUT_F32, s) == rtv.RTV_OK
            st = rtv.rtv_cache_state()
            rtv.lib.rtv_cache_get_state(h, ctypes.byref(st))
            splits.add(st.last_attend_splits)
        assert rtv.lib.rtv_cache_advance(h) == rtv.RTV_OK
    assert rtv.lib.rtv_poll_error(h) == rtv.RTV_OK
    assert rtv.lib.rtv_cache_destroy(h) == rtv.RTV_OK
    torch.cuda.synchronize()
    assert bool((big[:guard] == 0xA5).all()), "a kernel wrote below the cache buffer"
    assert bool((big[guard + need:] == 0xA5).all()), "a kernel wrote above the cache buffer"
    assert max(splits) > 1, "the split attention path did not run"
