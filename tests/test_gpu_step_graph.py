"""GPU tests of the whole-step CUDA graph (rtv_step_graph_*): the kernels of
a captured steady-state step read the ring state from device memory, so one
graph replays every later step.  Each replayed step is held to the oracle
like a direct step -- every append's codes and scales, every layer's
attention output, and the host ring state -- also when direct calls move the
ring between replays."""
import numpy as np
import pytest
import torch

from kv_cache_serving_append_b200 import configs, synth
from parity import ATOL_MAX, REL_L2, Runner, attn_errors, ring_state_matches

pytestmark = pytest.mark.gpu


def _oracle_step(R, step, outs, F=1):
    """Follow one replayed step in the oracle and compare."""
    cfg = R.cfg
    for layer in range(cfg["n_layers"]):
        q, k, v = synth.chunk(R.cfg_id, cfg, layer, step, F)
        slots = R.ora.append(layer, synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v), F)
        R.check_append(layer, slots, F)
    worst = 0.0
    for layer in range(cfg["n_layers"]):
        o = R.ora.attend(layer)
        g = outs[layer].float().cpu().numpy()
        mx, rl = attn_errors(g, o)
        worst = max(worst, mx)
        assert mx <= ATOL_MAX and rl <= REL_L2, (step, layer, mx, rl)
    R.ora.advance()
    ring_state_matches(R.cache.state(), R.ora.ring)
    return worst


@pytest.mark.parametrize("cfg_id,F", [(2, 1), ("pinned2", 2)])
def test_step_graph_replays_match_oracle(gpu, cfg_id, F):
    from kv_cache_serving_append_b200 import rtv
    if cfg_id == "pinned2":
        cfg = dict(configs.get(2), name="2 frames per chunk, pinned slot", max_frames_per_chunk=2,
                   window_frames=4, pinned_frames=1)
        seed_id = 2
    else:
        cfg, seed_id = configs.get(cfg_id), cfg_id
    R = Runner(seed_id, cfg)
    L, T, H, D = cfg["n_layers"], R.T, R.H, R.D
    stream = torch.cuda.Stream()
    step = configs.first_step(cfg)
    qs = [torch.empty((F * T, H, D), dtype=torch.bfloat16, device="cuda") for _ in range(L)]
    ks = [torch.empty_like(x) for x in qs]
    vs = [torch.empty_like(x) for x in qs]
    outs = [torch.empty((F * T, H, D), dtype=torch.float32, device="cuda") for _ in range(L)]
    with pytest.raises(rtv.RtvError) as e:           # the ring is not full yet
        rtv.StepGraph(R.cache, F, qs, ks, vs, outs, stream)
    assert e.value.status == rtv.RTV_ERR_STATE
    while not (R.ora.ring.G >= cfg["window_frames"] and (not cfg["pinned_frames"] or R.ora.ring.pinned_committed)):
        n = configs.frames_for_step(cfg, step) if step < 0 else F
        for layer in range(L):
            R.append(layer, step, n)
        R.advance()
        step += 1
    g = rtv.StepGraph(R.cache, F, qs, ks, vs, outs, stream)
    worst = 0.0
    for i in range(8):
        if i == 4:
            # a direct step between replays; the next launch re-uploads the state
            for layer in range(L):
                R.append(layer, step, F)
            for layer in range(L):
                gg, o = R.attend(layer)
                mx, rl = attn_errors(gg, o)
                assert mx <= ATOL_MAX and rl <= REL_L2
            R.advance()
            step += 1
            continue
        with torch.cuda.stream(stream):
            for layer in range(L):
                q, k, v = synth.chunk(seed_id, cfg, layer, step, F)
                qs[layer].copy_(q, non_blocking=False)
                ks[layer].copy_(k, non_blocking=False)
                vs[layer].copy_(v, non_blocking=False)
            for o in outs:
                o.fill_(float("nan"))
        assert g.launch(stream) == rtv.RTV_OK
        stream.synchronize()
        assert R.cache.poll_error() == rtv.RTV_OK
        worst = max(worst, _oracle_step(R, step, outs, F))
        step += 1
    # a layer staged by a direct call blocks the replay
    q, k, v = (t.cuda() for t in synth.chunk(seed_id, cfg, 0, step, F))
    assert R.cache.append(0, q, k, v, F) == rtv.RTV_OK
    assert g.launch(stream) == rtv.RTV_ERR_STATE
    g.close()
    R.cache.close()
    print(f"step graph {cfg_id}: worst max-abs {worst:.3g}")
