"""Pins for the oracle's ring map and fp64 attention (CPU only).

Ring: the closed form of the window (after G generated commits the visible
frames are G-W .. G-1, plus the pinned frame), asserted at every step of
every workload's (W, F, pinned) and of extra combinations, against a
brute-force simulation that keeps a physical slot array and the list of
frames written so far.

Attention: softmax rows sum to 1; all-equal keys give the mean of V exactly;
a dominant key returns its value; key order does not matter; and on the tiny
workload it matches PyTorch's float64 scaled_dot_product_attention run on the
dequantised tensors (an independent implementation).
"""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_serving_append_b200 import configs, synth

RING_CASES = [(4, 1, 0), (6, 1, 0), (8, 1, 0), (16, 2, 1), (0, 1, 0), (3, 2, 0), (5, 3, 1),
              (1, 1, 1), (2, 4, 0)]


@pytest.mark.parametrize("W,F_max,P0", RING_CASES)
def test_ring_closed_form_and_brute_force(W, F_max, P0):
    ring = oracle.OracleRing(W, F_max, P0)
    rng = np.random.default_rng(W * 31 + F_max * 7 + P0)
    memory = [None] * ring.n_slots    # what each physical slot holds
    written = []                       # every frame ever written, in order
    G = 0
    pinned = False
    for step in range(40):
        if P0 and not pinned:
            F = 1
        else:
            F = int(rng.integers(1, F_max + 1))
        slots = ring.staged_slots(F)
        frames = ring.staged_frames(F)
        # staged frames must not land on a visible frame's slot
        visible_slots = {ring.slot_of_frame[t] for t in ring.visible}
        assert not (set(slots) & visible_slots)
        assert len(set(slots)) == F
        # absolute frame index of the staged frames
        assert frames == list(range(len(written), len(written) + F))
        # key set = visible (logical order) + staged
        assert ring.key_slots(F) == [ring.slot_of_frame[t] for t in ring.visible] + slots
        for t, s in zip(frames, slots):
            memory[s] = t
        written += frames
        ring.commit(F)
        if P0 and not pinned:
            pinned = True
        else:
            G += F
        # closed form of the visible set
        gen0 = 1 if P0 else 0
        want = ([0] if P0 else []) + [gen0 + g for g in range(max(0, G - W), G)]
        assert ring.visible == want
        assert ring.G == G and ring.frames_committed == len(written)
        assert ring.head == P0 + (G % (W + F_max))
        # brute force: every visible frame is still physically in its slot
        for t in ring.visible:
            assert memory[ring.slot_of_frame[t]] == t
        if P0:
            assert ring.slot_of_frame[0] == 0


@pytest.mark.parametrize("cfg_id", [1, 2, 3, 5])
def test_ring_workloads_first_reuse(cfg_id):
    cfg = configs.get(cfg_id)
    ring = oracle.OracleRing(cfg["window_frames"], cfg["max_frames_per_chunk"], cfg["pinned_frames"])
    seen = set()
    reused = False
    for step in range(configs.first_step(cfg), cfg["steps"]):
        F = configs.frames_for_step(cfg, step)
        for s in ring.staged_slots(F):
            reused |= s in seen
            seen.add(s)
        ring.commit(F)
    n_gen = cfg["steps"] * cfg["max_frames_per_chunk"]
    assert reused == (n_gen > cfg["window_frames"] + cfg["max_frames_per_chunk"])


def _rand_codes(rng, shape):
    c = rng.integers(0, 256, shape).astype(np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x38   # no NaN codes
    return c


def test_softmax_rows_sum_to_one():
    rng = np.random.default_rng(0)
    H, M, NK, D = 2, 9, 77, 64
    qc, kc, vc = _rand_codes(rng, (H, M, D)), _rand_codes(rng, (H, NK, D)), _rand_codes(rng, (H, NK, D))
    sq, sk, sv = [rng.uniform(1e-3, 1e-2, s).astype(np.float32) for s in [(H, M), (H, NK), (H, NK)]]
    out, psum = oracle.attend(qc, sq, kc, sk, vc, sv, want_psum=True)
    assert np.all(np.abs(psum - 1.0) <= 1e-12)
    assert np.all(np.isfinite(out))


def test_equal_keys_give_mean_of_values():
    rng = np.random.default_rng(1)
    H, M, NK, D = 2, 5, 64, 64
    qc = _rand_codes(rng, (H, M, D))
    kc = np.repeat(_rand_codes(rng, (H, 1, D)), NK, axis=1)
    vc = _rand_codes(rng, (H, NK, D))
    sq = np.full((H, M), 0.01, np.float32)
    sk = np.full((H, NK), 0.02, np.float32)
    sv = rng.uniform(0.1, 1, (H, NK)).astype(np.float32)
    out = oracle.attend(qc, sq, kc, sk, vc, sv)
    vhat = oracle.e4m3_decode(vc) * sv[..., None].astype(np.float64)
    mean = vhat.mean(axis=1)          # [H, D]
    assert np.allclose(out, mean[None], rtol=0, atol=1e-12 * np.abs(vhat).max())


def test_dominant_key_returns_its_value():
    H, M, NK, D = 1, 3, 50, 64
    rng = np.random.default_rng(2)
    qc = np.full((H, M, D), 0x38, np.uint8)       # q = 1 everywhere
    kc = np.zeros((H, NK, D), np.uint8)
    kc[0, 17] = 0x38                               # only key 17 aligns with q
    vc = _rand_codes(rng, (H, NK, D))
    sq = np.ones((H, M), np.float32)
    sk = np.ones((H, NK), np.float32) * 4.0        # s_17 = 64*4/8 = 32, others 0
    sv = np.ones((H, NK), np.float32)
    out = oracle.attend(qc, sq, kc, sk, vc, sv)
    v17 = oracle.e4m3_decode(vc[0, 17])
    assert np.allclose(out[:, 0], v17[None], atol=np.abs(oracle.e4m3_decode(vc)).max() * NK * np.exp(-32) * 2)


def test_key_order_does_not_matter_and_row_sampling():
    rng = np.random.default_rng(3)
    H, M, NK, D = 2, 11, 90, 64
    qc, kc, vc = _rand_codes(rng, (H, M, D)), _rand_codes(rng, (H, NK, D)), _rand_codes(rng, (H, NK, D))
    sq, sk, sv = [rng.uniform(1e-3, 3e-3, s).astype(np.float32) for s in [(H, M), (H, NK), (H, NK)]]
    out = oracle.attend(qc, sq, kc, sk, vc, sv)
    perm = rng.permutation(NK)
    out2 = oracle.attend(qc, sq, kc[:, perm], sk[:, perm], vc[:, perm], sv[:, perm])
    assert np.allclose(out, out2, rtol=1e-12, atol=1e-14)
    rows = np.array([10, 0, 4], np.int32)
    out3 = oracle.attend(qc, sq, kc, sk, vc, sv, rows=rows)
    assert np.array_equal(out3, out[rows])


def test_tiny_workload_matches_torch_sdpa_fp64():
    """Config 1 end to end in the oracle, every step, against torch float64 SDPA
    on the oracle's own dequantised cache (mask is full over the key set)."""
    cfg = configs.get(1)
    cache = oracle.OracleCache(cfg)
    D = cfg["head_dim"]
    for step in range(cfg["steps"]):
        q, k, v = synth.chunk(1, cfg, 0, step, 1)
        cache.append(0, synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v), 1)
        out = cache.attend(0)
        L = cache.layers[0]
        _, kc, sk, vc, sv = cache.key_set(0)
        qh = torch.from_numpy(oracle.e4m3_decode(L["qc"]) * L["sq"][..., None].astype(np.float64))
        kh = torch.from_numpy(oracle.e4m3_decode(kc) * sk[..., None].astype(np.float64))
        vh = torch.from_numpy(oracle.e4m3_decode(vc) * sv[..., None].astype(np.float64))
        ref = torch.nn.functional.scaled_dot_product_attention(qh[None], kh[None], vh[None])[0]
        ref = ref.permute(1, 0, 2).numpy()        # [M, H, D]
        assert np.max(np.abs(out - ref)) <= 1e-12 * max(1.0, np.abs(ref).max())
        assert kc.shape[1] == (min(step, cfg["window_frames"]) + 1) * 64
        cache.advance()


def test_matmul_form_agrees_with_the_loops():
    """The library-matmul form of the attention gives the C loops' result to
    fp64 rounding, on random codes with spread scales, all rows and a row
    sample, and with a key count that is not a multiple of anything."""
    rng = np.random.default_rng(4)
    for H, M, NK, D in [(2, 37, 301, 64), (3, 129, 1000, 128)]:
        qc, kc, vc = _rand_codes(rng, (H, M, D)), _rand_codes(rng, (H, NK, D)), _rand_codes(rng, (H, NK, D))
        sq, sk, sv = [rng.uniform(1e-3, 2e-2, s).astype(np.float32) for s in [(H, M), (H, NK), (H, NK)]]
        ref = oracle.attend(qc, sq, kc, sk, vc, sv)
        got = oracle.attend_matmul(qc, sq, kc, sk, vc, sv, block_rows=50)
        assert np.max(np.abs(got - ref)) <= 1e-12 * max(1.0, np.abs(ref).max())
        rows = np.array([M - 1, 0, M // 2], np.int32)
        sub = oracle.attend_matmul(qc, sq, kc, sk, vc, sv, rows=rows, block_rows=50)
        assert np.max(np.abs(sub - got[rows])) <= 1e-12 * max(1.0, np.abs(ref).max())


def test_matmul_form_invariants():
    """Equal keys give the mean of V; a dominant key gives its value."""
    rng = np.random.default_rng(5)
    H, M, NK, D = 1, 4, 96, 64
    qc = _rand_codes(rng, (H, M, D))
    kc = np.repeat(_rand_codes(rng, (H, 1, D)), NK, axis=1)
    vc = _rand_codes(rng, (H, NK, D))
    sq = np.full((H, M), 0.01, np.float32)
    sk = np.full((H, NK), 0.02, np.float32)
    sv = rng.uniform(0.1, 1, (H, NK)).astype(np.float32)
    vhat = oracle.e4m3_decode(vc) * sv[..., None].astype(np.float64)
    out = oracle.attend_matmul(qc, sq, kc, sk, vc, sv)
    assert np.allclose(out, vhat.mean(axis=1)[None], rtol=0, atol=1e-12 * np.abs(vhat).max())
    qc = np.full((H, M, D), 0x38, np.uint8)
    kc = np.zeros((H, NK, D), np.uint8)
    kc[0, 17] = 0x38
    out = oracle.attend_matmul(qc, np.ones((H, M), np.float32), kc, np.full((H, NK), 4.0, np.float32),
                               vc, np.ones((H, NK), np.float32))
    v17 = oracle.e4m3_decode(vc[0, 17])
    assert np.allclose(out[:, 0], v17[None], atol=np.abs(oracle.e4m3_decode(vc)).max() * NK * np.exp(-32) * 2)


def test_matmul_form_matches_torch_sdpa_fp64_on_the_small_workload():
    """Config 2 (8 heads, 704 tokens, outlier channels) after the ring has
    wrapped, against PyTorch's float64 scaled_dot_product_attention on the
    oracle's dequantised tensors."""
    cfg = configs.get(2)
    cache = oracle.OracleCache(cfg, layers=[0])
    for step in range(cfg["window_frames"] + 2):
        q, k, v = synth.chunk(2, cfg, 0, step, 1)
        cache.append(0, synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v), 1)
        if step < cfg["window_frames"] + 1:
            cache.advance()
    L = cache.layers[0]
    _, kc, sk, vc, sv = cache.key_set(0)
    out = cache.attend(0, matmul=True)
    qh = torch.from_numpy(oracle.e4m3_decode(L["qc"]) * L["sq"][..., None].astype(np.float64))
    kh = torch.from_numpy(oracle.e4m3_decode(kc) * sk[..., None].astype(np.float64))
    vh = torch.from_numpy(oracle.e4m3_decode(vc) * sv[..., None].astype(np.float64))
    ref = torch.nn.functional.scaled_dot_product_attention(qh[None], kh[None], vh[None])[0]
    ref = ref.permute(1, 0, 2).numpy()
    assert np.max(np.abs(out - ref)) <= 1e-12 * max(1.0, np.abs(ref).max())
