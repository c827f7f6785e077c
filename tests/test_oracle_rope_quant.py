"""Pins for the oracle's 3D axial RoPE, per-row quantisation and chunk append.

RoPE is pinned by properties a rotary embedding must have, none of which
re-types the oracle's formula: zero position is the identity; each pair keeps
its norm; q.k depends only on the position difference along every axis; a
one-hot input moves only within its rotate-half pair, by the textbook angle
cos(1)/sin(1) at position 1, pair 0; each axis touches only its own segment;
and the angle per unit position falls geometrically across pairs by
base^(-2/n) with n the segment size (not head_dim).
"""
import math

import numpy as np
import pytest

import oracle

SPLITS = {64: (16, 24, 24), 128: (32, 48, 48)}


def rand_x(n, D, seed=0):
    return np.random.default_rng(seed).standard_normal((n, D)).astype(np.float32)


@pytest.mark.parametrize("D", [64, 128])
def test_zero_position_is_identity(D):
    x = rand_x(50, D)
    y = oracle.rope3d(x, SPLITS[D], np.zeros((50, 3), np.int64))
    assert np.array_equal(x, y)


@pytest.mark.parametrize("D", [64, 128])
def test_pair_norms_preserved(D):
    x = rand_x(200, D, 1)
    rng = np.random.default_rng(2)
    pos = np.stack([rng.integers(0, 50, 200), rng.integers(0, 44, 200), rng.integers(0, 68, 200)], 1)
    y = oracle.rope3d(x, SPLITS[D], pos)
    off = 0
    for n in SPLITS[D]:
        h = n // 2
        a = x[:, off:off + h].astype(np.float64) ** 2 + x[:, off + h:off + n].astype(np.float64) ** 2
        b = y[:, off:off + h].astype(np.float64) ** 2 + y[:, off + h:off + n].astype(np.float64) ** 2
        # two fp32 products and one fp32 add per output: a few ulp of relative error
        assert np.all(np.abs(np.sqrt(b) - np.sqrt(a)) <= 4 * 2.0 ** -24 * np.sqrt(a) + 1e-30)
        off += n


@pytest.mark.parametrize("axis", [0, 1, 2])
@pytest.mark.parametrize("D", [64, 128])
def test_dot_product_depends_on_relative_position(axis, D):
    rng = np.random.default_rng(3 + axis)
    q = rand_x(64, D, 10)
    k = rand_x(64, D, 11)
    p1 = np.stack([rng.integers(0, 20, 64), rng.integers(0, 20, 64), rng.integers(0, 20, 64)], 1)
    p2 = np.stack([rng.integers(0, 20, 64), rng.integers(0, 20, 64), rng.integers(0, 20, 64)], 1)
    shift = np.zeros(3, np.int64)
    shift[axis] = 7
    d0 = np.sum(oracle.rope3d(q, SPLITS[D], p1).astype(np.float64)
                * oracle.rope3d(k, SPLITS[D], p2), axis=1)
    d1 = np.sum(oracle.rope3d(q, SPLITS[D], p1 + shift).astype(np.float64)
                * oracle.rope3d(k, SPLITS[D], p2 + shift), axis=1)
    scale = np.sum(np.abs(q.astype(np.float64) * k), axis=1)
    assert np.all(np.abs(d0 - d1) <= 1e-5 * scale)


def test_one_hot_rotates_within_its_pair_textbook_angle():
    D = 128
    n_t = SPLITS[D][0]
    x = np.zeros((1, D), np.float32)
    x[0, 0] = 1.0
    y = oracle.rope3d(x, SPLITS[D], np.array([[1, 0, 0]]))
    nz = set(np.flatnonzero(y[0]))
    assert nz == {0, n_t // 2}, "rotate-half pairs dim j with j + n/2 of its own segment"
    assert y[0, 0] == np.float32(math.cos(1.0))
    assert y[0, n_t // 2] == np.float32(math.sin(1.0))
    # the second member of the pair rotates the other way: (0, 1) -> (-sin, cos)
    x2 = np.zeros((1, D), np.float32)
    x2[0, n_t // 2] = 1.0
    y2 = oracle.rope3d(x2, SPLITS[D], np.array([[1, 0, 0]]))
    assert y2[0, 0] == -np.float32(math.sin(1.0)) and y2[0, n_t // 2] == np.float32(math.cos(1.0))


@pytest.mark.parametrize("D", [64, 128])
def test_axes_touch_only_their_segment(D):
    x = rand_x(8, D, 5)
    n_t, n_h, n_w = SPLITS[D]
    seg = [(0, n_t), (n_t, n_t + n_h), (n_t + n_h, D)]
    for axis in range(3):
        pos = np.zeros((8, 3), np.int64)
        pos[:, axis] = 5
        y = oracle.rope3d(x, SPLITS[D], pos)
        changed = np.flatnonzero(np.any(y != x, axis=0))
        lo, hi = seg[axis]
        assert changed.min() >= lo and changed.max() < hi


@pytest.mark.parametrize("D", [64, 128])
def test_frequencies_geometric_in_segment_size(D):
    base = 10000.0
    off = 0
    for axis, n in enumerate(SPLITS[D]):
        h = n // 2
        angles = []
        for j in range(h):
            x = np.zeros((1, D), np.float32)
            x[0, off + j] = 1.0
            pos = np.zeros((1, 3), np.int64)
            pos[0, axis] = 1
            y = oracle.rope3d(x, SPLITS[D], pos, base)
            angles.append(math.atan2(float(y[0, off + j + h]), float(y[0, off + j])))
        angles = np.array(angles)
        assert abs(angles[0] - 1.0) < 1e-6        # pair 0 turns one radian per unit
        ratio = angles[1:] / angles[:-1]
        assert np.allclose(ratio, base ** (-2.0 / n), rtol=1e-4)
        off += n


def test_quantize_row_error_bound_and_zero_row():
    rng = np.random.default_rng(6)
    x = (rng.standard_normal((500, 128)) * np.exp(rng.uniform(-8, 8, (500, 1)))).astype(np.float32)
    x[7] = 0.0
    codes, scales, _ = oracle.quantize_rows(x)
    assert np.all(codes[7] & 0x7F == 0) and scales[7] == 0.0
    deq = oracle.e4m3_decode(codes) * scales[:, None].astype(np.float64)
    err = np.abs(deq - x)
    # relative half-step 2^-4 for normals, absolute half-step 2^-10 * scale for subnormals,
    # plus the fp32 roundings of x*inv and amax/448
    bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * 448 * scales[:, None] / 448) * 1.0001
    assert np.all(err <= bound + 1e-30)


def test_append_tensor_v_unrotated_and_positions():
    T, gw, H, D = 12, 4, 2, 64
    rng = np.random.default_rng(7)
    x = rng.standard_normal((2 * T, H, D)).astype(np.float32)
    import torch
    bits = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    xf = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    # V: no rotation -> quantisation of the raw rows
    vc, vs, _ = oracle.append_tensor(bits, T, gw, 9, False, SPLITS[D])
    c2, s2, _ = oracle.quantize_rows(xf.transpose(1, 0, 2).reshape(-1, D))
    assert np.array_equal(vc.reshape(-1, D), c2) and np.array_equal(vs.reshape(-1), s2)
    # K: rows rotated at (t0 + frame, token // grid_w, token % grid_w)
    kc, ks, _ = oracle.append_tensor(bits, T, gw, 9, True, SPLITS[D])
    r = np.arange(2 * T)
    pos = np.stack([9 + r // T, (r % T) // gw, (r % T) % gw], 1)
    for h in range(H):
        rot = oracle.rope3d(xf[:, h], SPLITS[D], pos)
        c3, s3, _ = oracle.quantize_rows(rot)
        assert np.array_equal(kc[h], c3) and np.array_equal(ks[h], s3)


def test_bf16_rounding_matches_torch():
    """The oracle's fp32 -> bf16 rounding against PyTorch's cast (an
    independent implementation of round-to-nearest-even), including ties."""
    import torch
    rng = np.random.default_rng(11)
    v = rng.standard_normal(200000).astype(np.float32) * np.float32(3.0)
    u = v.view(np.uint32)
    ties = ((u & 0xFFFF0000) | 0x8000).view(np.float32)            # exactly halfway
    both = np.concatenate([v, ties, np.float32([0.0, -0.0, 1.0, 65504.0, 1e-38])])
    ref = torch.from_numpy(both).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.bf16_rne_bits(both), ref)


def test_projection_definition_on_a_brute_force_case():
    """project_qkv against a per-element loop over the definition (decode,
    products summed in fp64, two fp32 scale multiplies, bf16 rounding)."""
    rng = np.random.default_rng(12)
    xc = rng.integers(0, 256, (5, 16)).astype(np.uint8)
    wc = rng.integers(0, 256, (7, 16)).astype(np.uint8)
    for c in (xc, wc):
        c[(c & 0x7F) == 0x7F] = 0x40
    sx = rng.uniform(0.1, 1, 5).astype(np.float32)
    sw = rng.uniform(0.1, 1, 7).astype(np.float32)
    got = oracle.project_qkv(xc, sx, wc, sw)
    dx, dw = oracle.e4m3_decode(xc), oracle.e4m3_decode(wc)
    for r in range(5):
        for n in range(7):
            acc = 0.0
            for k in range(16):
                acc += dx[r, k] * dw[n, k]
            v = np.float32(np.float32(np.float32(acc) * sx[r]) * sw[n])
            import torch
            ref = torch.tensor([float(v)], dtype=torch.float32).to(torch.bfloat16).view(torch.int16).item() & 0xFFFF
            assert got[r, n] == ref, (r, n)


def test_quantize_row_below_the_reciprocal_range_is_zero():
    """Below amax = 2^-119 the fp32 reciprocal 448/amax would overflow (and a
    zero times it would be NaN): such an item is stored as zero, scale 0.  At
    and above 2^-119 the item quantises as usual, with its amax element on the
    largest code and a finite, exact scale."""
    rng = np.random.default_rng(12)
    base = rng.standard_normal(128).astype(np.float32)
    base[3] = 0.0
    base /= np.abs(base).max()                       # amax = 1
    rows = np.stack([base * np.float32(2.0 ** e) for e in (-126, -120, -119, -110)]).astype(np.float32)
    codes, scales, _ = oracle.quantize_rows(rows)
    for i in (0, 1):                                 # amax 2^-126, 2^-120: zero
        assert np.all(codes[i] & 0x7F == 0) and scales[i] == 0.0
    for i, e in ((2, -119), (3, -110)):              # amax 2^-119, 2^-110: quantised
        amax = np.float32(2.0 ** e)
        assert scales[i] == np.float32(amax / np.float32(448.0))
        assert codes[i][np.argmax(np.abs(rows[i]))] & 0x7F == 0x7E
        assert codes[i][3] & 0x7F == 0               # the zero element stays zero, not NaN
        assert not np.any((codes[i] & 0x7F) == 0x7F)
