"""GPU tests of rtv_attend_static_scratch, the attention entry point whose
key-range split partials live in the library's fixed device array instead of
the cache buffer: on two calls in a row it gives rtv_attend's output bit for
bit, with the split path in use, and a plan whose partials exceed the array is
rejected before anything is launched.  The file name sorts last, so in a full
run these tests also run after every other GPU test."""
import pytest
import torch

from kv_cache_serving_append_b200 import configs, synth

pytestmark = pytest.mark.gpu


def test_static_scratch_matches_rtv_attend_on_two_calls(gpu):
    from kv_cache_serving_append_b200 import rtv
    cfg = configs.get(2)                    # 8 heads x D128, 704 tokens per frame, W = 6
    c = rtv.Cache(cfg)
    T, H, D = cfg["grid_h"] * cfg["grid_w"], cfg["n_heads"], cfg["head_dim"]
    ref = torch.empty((T, H, D), dtype=torch.float32, device="cuda")
    got = [torch.empty_like(ref) for _ in range(2)]
    split_seen = False
    for step in range(cfg["window_frames"] + 2):
        q, k, v = (t.cuda() for t in synth.chunk(2, cfg, 0, step, 1))
        for layer in range(cfg["n_layers"]):
            assert c.append(layer, q, k, v, 1) == rtv.RTV_OK
        assert c.attend(0, ref) == rtv.RTV_OK
        splits = c.state().last_attend_splits
        for g in got:                       # two calls in a row on the same staged chunk
            g.fill_(float("nan"))
            assert c.attend_static_scratch(0, g) == rtv.RTV_OK
            assert c.state().last_attend_splits == splits
        torch.cuda.synchronize()
        assert c.poll_error() == rtv.RTV_OK
        for i, g in enumerate(got):
            assert torch.equal(g, ref), f"step {step}, call {i}: output differs from rtv_attend"
        split_seen |= splits > 1
        assert c.advance() == rtv.RTV_OK
    assert split_seen, "the split path (partials in the static array) never ran"
    c.close()


def test_static_scratch_rejects_partials_over_capacity(gpu):
    from kv_cache_serving_append_b200 import rtv
    cfg = configs.get(3)                    # 40 heads x 2992 rows: 4-way partials need ~250 MB
    c = rtv.Cache(cfg)
    T, H, D = cfg["grid_h"] * cfg["grid_w"], cfg["n_heads"], cfg["head_dim"]
    q, k, v = (t.cuda() for t in synth.chunk(3, cfg, 0, 0, 1))
    assert c.append(0, q, k, v, 1) == rtv.RTV_OK
    out = torch.full((T, H, D), 7.0, dtype=torch.float32, device="cuda")
    assert c.attend_static_scratch(0, out) == rtv.RTV_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert bool((out == 7.0).all()), "a rejected call wrote to the output"
    ref = torch.empty_like(out)
    assert c.attend(0, ref) == rtv.RTV_OK
    assert c.state().last_attend_splits > 1
    torch.cuda.synchronize()
    assert c.poll_error() == rtv.RTV_OK
    assert bool(torch.isfinite(ref).all())
    c.close()
