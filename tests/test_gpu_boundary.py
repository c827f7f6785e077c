"""GPU tests of the C-ABI boundary: error statuses and call order, staging
overwrite, that calls write only what they own, and the bounded-wait failure
path (a wait that nothing completes runs out, the kernel reports
RTV_ERR_TIMEOUT through the error word and the context stays usable)."""
import ctypes

import numpy as np
import pytest
import torch

from kv_cache_serving_append_b200 import configs, synth
from parity import ATOL_MAX, REL_L2, Runner, attn_errors

pytestmark = pytest.mark.gpu


def test_call_order_and_argument_errors(gpu):
    from kv_cache_serving_append_b200 import rtv
    cfg = configs.get(2)
    c = rtv.Cache(cfg)
    T, H, D = 704, 8, 128
    q, k, v = (t.cuda() for t in synth.chunk(2, cfg, 0, 0, 1))
    out = torch.empty((T, H, D), dtype=torch.float32, device="cuda")
    assert c.attend(0, out) == rtv.RTV_ERR_STATE          # nothing staged
    assert c.advance() == rtv.RTV_ERR_STATE               # nothing staged
    assert c.append(2, q, k, v, 1) == rtv.RTV_ERR_INVALID_ARG    # no such layer
    assert c.append(0, q, k, v, 0) == rtv.RTV_ERR_INVALID_ARG    # n_frames < 1
    assert c.append(0, q, k, v, 2) == rtv.RTV_ERR_INVALID_ARG    # > F_max
    qb = torch.empty(q.numel() * 2 + 8, dtype=torch.uint8, device="cuda")
    mis = qb[2:2 + q.numel() * 2].view(torch.bfloat16)           # 2-byte aligned only
    assert c.append(0, mis, k, v, 1) == rtv.RTV_ERR_INVALID_ARG
    assert c.append(0, q, k, v, 1) == rtv.RTV_OK
    assert c.advance() == rtv.RTV_ERR_STATE               # layer 1 not staged
    assert c.attend(0, out) == rtv.RTV_OK
    assert c.attend(1, out) == rtv.RTV_ERR_STATE
    bad_out = torch.empty((T, H, D), dtype=torch.float16, device="cuda")
    assert c.attend(0, bad_out) == rtv.RTV_ERR_INVALID_ARG
    assert c.append(1, q, k, v, 1) == rtv.RTV_OK
    assert c.advance() == rtv.RTV_OK
    st = c.state()
    assert st.frames_committed == 1 and st.n_visible == 1 and st.staged_layers == 0
    assert c.poll_error() == rtv.RTV_OK
    c.close()


def test_pinned_chunk_is_one_frame(gpu):
    from kv_cache_serving_append_b200 import rtv
    cfg = configs.get(5)
    cfg.update(n_heads=2, grid_h=4, grid_w=8)
    c = rtv.Cache(cfg)
    q, k, v = (t.cuda() for t in synth.chunk(5, cfg, 0, -1, 2))
    assert c.append(0, q, k, v, 2) == rtv.RTV_ERR_INVALID_ARG
    assert c.append(0, q, k, v, 1) == rtv.RTV_OK
    assert c.advance() == rtv.RTV_OK
    st = c.state()
    assert st.pinned_committed == 1 and st.visible_slots[0] == 0 and st.frame_of_slot[0] == 0
    assert c.append(0, q, k, v, 2) == rtv.RTV_OK
    c.close()


def test_staging_overwrite_and_untouched_memory(gpu):
    """A second append before advance replaces the staged frame; appends
    touch only the staged slot; attention writes only its output rows."""
    cfg = configs.get(2)
    R = Runner(2, cfg)
    for step in range(3):
        for layer in range(2):
            R.append(layer, step, 1)
        R.advance()
    V = R.cache.views(0)
    before = {k: v.clone() for k, v in V.items()}
    R.append(0, 50, 1)   # first pass of the chunk
    R.append(0, 51, 1)   # second pass overwrites it; the oracle follows the second
    staged = R.ora.ring.staged_slots(1)[0]
    after = R.cache.views(0)
    for name in ("k_codes", "v_codes", "k_scales", "v_scales"):
        for s in range(after[name].shape[0]):
            if s != staged:
                assert torch.equal(before[name][s], after[name][s]), (name, s)
    # attention into the middle of a larger canary buffer
    T, H, D = R.T, R.H, R.D
    big = torch.full((T + 64, H, D), 12345.0, device="cuda")
    out = big[32:32 + T]
    assert R.cache.attend(0, out) == 0
    torch.cuda.synchronize()
    assert torch.all(big[:32] == 12345.0) and torch.all(big[32 + T:] == 12345.0)
    o = R.ora.attend(0)
    mx, rl = attn_errors(out.cpu().numpy(), o)
    assert mx <= ATOL_MAX and rl <= REL_L2
    R.cache.close()


def test_bounded_wait_times_out_and_context_survives(gpu):
    from kv_cache_serving_append_b200 import rtv
    cfg = configs.get(1)
    R = Runner(1, cfg)
    R.append(0, 0, 1)
    out = torch.full((R.T, R.H, R.D), 7.0, device="cuda")
    # a wait that nothing completes: ~10 ms limit per wait
    assert R.cache.set_wait_fault(True, 20_000_000) == 0
    assert R.cache.attend(0, out) == 0
    assert R.cache.poll_error() == rtv.RTV_ERR_TIMEOUT
    assert torch.all(out == 7.0)                        # nothing written
    assert R.cache.poll_error() == rtv.RTV_OK           # the word was cleared
    assert R.cache.set_wait_fault(False, 0) == 0
    g, o = R.attend(0)                                  # same context, normal run
    mx, rl = attn_errors(g, o)
    assert mx <= ATOL_MAX and rl <= REL_L2
    R.cache.close()


def test_library_allocated_buffer_and_export(gpu):
    """rtv_cache_create with a NULL buffer (library cudaMalloc) and the
    host export of one slot."""
    from kv_cache_serving_append_b200 import rtv
    cfg = configs.get(1)
    c = rtv.make_config(cfg)
    h = ctypes.c_void_p()
    assert rtv.lib.rtv_cache_create(ctypes.byref(c), None, 0, ctypes.byref(h)) == 0
    q, k, v = (t.cuda() for t in synth.chunk(1, cfg, 0, 0, 1))
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert rtv.lib.rtv_cache_append(h, 0, ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                    ctypes.c_void_p(v.data_ptr()), 1, s) == 0
    kc = np.zeros((2, 64, 64), np.uint8)
    sk = np.zeros((2, 64), np.float32)
    assert rtv.lib.rtv_cache_export(h, 0, 0, kc.ctypes.data_as(ctypes.c_void_p), None,
                                    sk.ctypes.data_as(ctypes.c_void_p), None, s) == 0
    import oracle
    oc, osk, near = oracle.append_tensor(synth.bf16_bits(k.cpu()), 64, 8, 0, True, (16, 24, 24))
    assert np.array_equal(kc, oc) or np.all((kc == oc) | (near != 0))
    assert np.array_equal(sk, osk)
    ptr, nb = ctypes.c_void_p(), ctypes.c_size_t()
    assert rtv.lib.rtv_cache_device_buffer(h, ctypes.byref(ptr), ctypes.byref(nb)) == 0
    assert nb.value == rtv.required_bytes(cfg) and ptr.value
    assert rtv.lib.rtv_cache_destroy(h) == 0
