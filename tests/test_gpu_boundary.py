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
    T = cfg["grid_h"] * cfg["grid_w"]
    assert c.append(0, q, k, v, 2) == rtv.RTV_ERR_INVALID_ARG       # the library refuses 2 frames
    assert c.append(0, q, k, v, 1) == rtv.RTV_ERR_INVALID_ARG       # the binding: 2 frames of rows
    assert c.append(0, q[:T], k[:T], v[:T], 1) == rtv.RTV_OK
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
    """rtv_cache_create with a NULL buffer (library cudaMalloc), then the
    host export (rtv_cache_export, through the C ABI) of the staged slot's K
    and V codes and scales and of the Q workspace, each held to the parity
    tolerance against the oracle: codes identical except one code step where
    the oracle flags a rounding boundary, scales within 1e-6 relative."""
    import oracle
    from kv_cache_serving_append_b200 import rtv
    from parity import compare_codes, compare_scales
    cfg = configs.get(1)
    H, D, T = cfg["n_heads"], cfg["head_dim"], 64
    split = (cfg["rope_t"], cfg["rope_h"], cfg["rope_w"])
    c = rtv.make_config(cfg)
    h = ctypes.c_void_p()
    assert rtv.lib.rtv_cache_create(ctypes.byref(c), None, 0, ctypes.byref(h)) == 0
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    a = lambda x: x.ctypes.data_as(ctypes.c_void_p)   # noqa: E731
    for step in range(2):            # slot 0 at frame 0, then slot 1 at frame 1
        q, k, v = (t.cuda() for t in synth.chunk(1, cfg, 0, step, 1))
        assert rtv.lib.rtv_cache_append(h, 0, ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                        ctypes.c_void_p(v.data_ptr()), 1, s) == 0
        kc, vc = np.zeros((H, T, D), np.uint8), np.zeros((H, T, D), np.uint8)
        sk, sv = np.zeros((H, T), np.float32), np.zeros((H, T), np.float32)
        qc, sq = np.zeros((H, T, D), np.uint8), np.zeros((H, T), np.float32)
        assert rtv.lib.rtv_cache_export(h, 0, step, a(kc), a(vc), a(sk), a(sv), a(qc), a(sq), s) == 0
        for name, x, g, sg, rope in (("q", q, qc, sq, True), ("k", k, kc, sk, True), ("v", v, vc, sv, False)):
            oc, osc, near = oracle.append_tensor(synth.bf16_bits(x.cpu()), T, cfg["grid_w"], step, rope, split)
            r = compare_codes(g, oc, near)
            assert r["bad"] == 0, (name, step, r)
            assert compare_scales(sg, osc) == 0, (name, step)
        assert rtv.lib.rtv_cache_advance(h) == 0
    assert rtv.lib.rtv_cache_export(h, 0, 99, None, None, None, None, None, None, s) == rtv.RTV_ERR_INVALID_ARG
    ptr, nb = ctypes.c_void_p(), ctypes.c_size_t()
    assert rtv.lib.rtv_cache_device_buffer(h, ctypes.byref(ptr), ctypes.byref(nb)) == 0
    assert nb.value == rtv.required_bytes(cfg) and ptr.value
    assert rtv.lib.rtv_cache_destroy(h) == 0
