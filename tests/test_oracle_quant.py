"""Pins of the oracle's FP8 / NVFP4 / residual quantisation."""

import math

import numpy as np

from oracle import formats as F
from oracle import quant as Qz


def test_fp8_tile_scale_is_smallest_power_of_two():
    rng = np.random.default_rng(0)
    for amax in np.concatenate([10.0 ** rng.uniform(-8, 8, 2000), [448.0, 449.0, 224.0, 1.0]]):
        s = Qz.fp8_tile_scale(amax)
        m, _ = math.frexp(s)
        assert m == 0.5                        # a power of two
        assert amax <= 448.0 * s
        assert amax > 448.0 * s / 2            # the next smaller one does not cover amax
    assert Qz.fp8_tile_scale(0.0) == 1.0
    assert Qz.fp8_tile_scale(448.0) == 1.0
    assert Qz.fp8_tile_scale(449.0) == 2.0
    assert Qz.fp8_tile_scale(5.0) == 2.0 ** -6    # 448/64 = 7 >= 5 > 3.5


def test_fp8_tiles_scale_invariance():
    rng = np.random.default_rng(1)
    X = rng.normal(size=(200, 32))
    c0, s0 = Qz.quant_fp8_tiles(X, 64)
    for k in (-3, 5):
        c1, s1 = Qz.quant_fp8_tiles(X * 2.0 ** k, 64)
        np.testing.assert_array_equal(c0, c1)
        np.testing.assert_array_equal(s1, s0 * 2.0 ** k)
    # ragged tail: 200 = 3*64 + 8 rows; its scale uses only its own 8 rows
    assert s0[3] == Qz.fp8_tile_scale(np.abs(X[192:]).max())


def test_fp8_grid_exact_round_trip():
    rng = np.random.default_rng(2)
    codes = rng.integers(0, 0x7E, size=(128, 64)).astype(np.uint8) | (rng.integers(0, 2, (128, 64)) << 7).astype(np.uint8)
    X = F.e4m3_decode(codes)
    X[0, 0] = 448.0                             # amax = 448 -> scale 1
    X[64, 0] = 448.0
    c, s = Qz.quant_fp8_tiles(X, 64)
    np.testing.assert_array_equal(s, [1.0, 1.0])
    np.testing.assert_array_equal(Qz.dequant_fp8_tiles(c, s, 64), X)


def test_nvfp4_group_hand_worked():
    x = np.zeros(16)
    x[:4] = [6.0, 3.0, -1.2, 0.4]
    codes, sc = Qz.nvfp4_quant_groups(x)
    # amax/6 = 1 -> scale 1.0 = ue4m3 0x38; codes: 6 -> 7, 3 -> 5, -1.2 -> -1 (0xA), 0.4 -> 0.5 (1)
    assert int(sc) == 0x38
    np.testing.assert_array_equal(codes[:4], [0x7, 0x5, 0xA, 0x1])
    np.testing.assert_array_equal(codes[4:], 0)
    y = np.zeros(16)
    y[0] = 10.0
    codes, sc = Qz.nvfp4_quant_groups(y)
    # fp32(10/6) = 1.6666666 -> ue4m3 1.625 (0x3D); 10 * fp32(1/1.625) = 6.1538 -> saturates to 6
    assert int(sc) == 0x3D
    assert int(codes[0]) == 0x7
    assert Qz.nvfp4_dequant_groups(codes, sc)[0] == 9.75


def test_nvfp4_zero_group():
    codes, sc = Qz.nvfp4_quant_groups(np.zeros(16))
    assert int(sc) == 0 and not codes.any()
    tiny = np.full(16, 1e-6)                    # amax/6 rounds to ue4m3 zero
    codes, sc = Qz.nvfp4_quant_groups(tiny)
    assert int(sc) == 0 and not codes.any()


def _grid_exact_groups(rng, shape_groups):
    """Groups of 16 on the NVFP4 grid whose scale is an exact power of two."""
    vals = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    g = vals[rng.integers(0, 8, size=shape_groups + (16,))] * rng.choice([-1.0, 1.0], size=shape_groups + (16,))
    g[..., 0] = 6.0 * rng.choice([-1.0, 1.0], size=shape_groups)
    sc = 2.0 ** rng.integers(-4, 3, size=shape_groups)
    return g * sc[..., None]


def test_nvfp4_rows_and_cols_grid_exact():
    rng = np.random.default_rng(3)
    X = _grid_exact_groups(rng, (40, 4)).reshape(40, 64)
    c, s = Qz.quant_nvfp4_rows(X)
    np.testing.assert_array_equal(Qz.dequant_nvfp4_rows(c, s), X)
    Vt = _grid_exact_groups(rng, (24, 3)).reshape(24, 48)  # [d, N]: groups of 16 tokens
    V = Vt.T.copy()                                          # [N=48, d=24]
    c, s = Qz.quant_nvfp4_cols(V)
    assert c.shape == (48, 24) and s.shape == (3, 24)
    np.testing.assert_array_equal(Qz.dequant_nvfp4_cols(c, s), V)


def test_nvfp4_cols_padding_and_alignment():
    rng = np.random.default_rng(4)
    V = rng.normal(size=(40, 8))                 # 40 = 2*16 + 8: last group half padding
    c, s = Qz.quant_nvfp4_cols(V)
    assert c.shape == (48, 8)
    assert not c[40:].any()
    for col in range(8):
        for g in range(3):
            seg = np.zeros(16)
            rows = V[16 * g:min(40, 16 * g + 16), col]
            seg[:len(rows)] = rows
            cc, ss = Qz.nvfp4_quant_groups(seg)
            assert ss == s[g, col]
            np.testing.assert_array_equal(cc, c[16 * g:16 * g + 16, col])


def test_residual_reduces_error():
    rng = np.random.default_rng(5)
    X = F.bf16_rne(rng.normal(size=(64, 128)))
    qt = Qz.quantize_head(X, X, X, Qz.LOW_NVFP4_RES, 64, 64)
    e1 = np.abs(X - qt["dq"]).max()
    e2 = np.abs(X - qt["dq"] - qt["rq"]).max()
    assert e2 < e1 / 4
    # the residual copy is the NVFP4 of fp32(x - deq(x)), row groups along d
    r = F.fp32_rne(X - qt["dq"])
    c, s = Qz.quant_nvfp4_rows(r)
    np.testing.assert_array_equal(c, qt["rq_codes"])


def _nearest_even(v, grid_vals, grid_codes):
    """Brute force: the grid value nearest to v; on an exact tie the one whose
    code is even (the encoding's last mantissa bit 0)."""
    d = np.abs(grid_vals - v)
    best = np.nonzero(d == d.min())[0]
    if len(best) > 1:
        best = [b for b in best if grid_codes[b] % 2 == 0]
    return grid_codes[best[0]], grid_vals[best[0]]


def test_nvfp4_groups_match_brute_force_nearest():
    # The whole group rule restated by exhaustive search over the two grids,
    # with no bit manipulation: sc = the ue4m3 value nearest fp32(amax / 6)
    # (ties to the even code, saturating at 448), then each element's e2m1
    # value nearest fp32(x * fp32(1 / sc)) (ties to even, saturating at 6,
    # sign kept), and every code 0 when sc = 0.
    rng = np.random.default_rng(21)
    e4 = [(c, F.e4m3_decode(np.array([c], dtype=np.uint8))[0]) for c in range(0x7F)]
    e4_codes = np.array([c for c, _ in e4])
    e4_vals = np.array([v for _, v in e4])
    e2_vals = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    e2_codes = np.arange(8)
    f32 = lambda v: float(np.float32(v))
    groups = []
    for _ in range(3000):
        mag = 2.0 ** rng.uniform(-14, 12)                    # subnormal to saturated scales
        g = rng.normal(size=16) * mag
        g[rng.random(16) < 0.2] = 0.0
        groups.append(F.bf16_rne(g))
    groups.append(np.zeros(16))
    G = np.stack(groups)
    codes, sc_code = Qz.nvfp4_quant_groups(G)
    for k in range(G.shape[0]):
        x = G[k]
        q = f32(f32(np.abs(x).max()) / 6.0)
        want_sc, sc = _nearest_even(min(q, 448.0), e4_vals, e4_codes)
        assert int(sc_code[k]) == want_sc, (k, q)
        if sc == 0.0:
            assert not codes[k].any()
            continue
        inv = f32(1.0 / sc)
        for i in range(16):
            y = f32(x[i] * inv)
            c, _ = _nearest_even(min(abs(y), 6.0), e2_vals, e2_codes)
            want = c | (8 if y < 0 or (y == 0 and np.signbit(y)) else 0)
            assert int(codes[k, i]) == want, (k, i, x[i], y)


def test_fp8_tiles_match_brute_force_nearest():
    # One tile: s = the smallest power of two with amax <= 448 s (found by
    # stepping through powers of two), codes = the e4m3 value nearest x / s
    # (exact: s is a power of two), ties to the even code, sign kept.
    rng = np.random.default_rng(22)
    e4 = [(c, F.e4m3_decode(np.array([c], dtype=np.uint8))[0]) for c in range(0x7F)]
    e4_codes = np.array([c for c, _ in e4])
    e4_vals = np.array([v for _, v in e4])
    for t in range(200):
        X = F.bf16_rne(rng.normal(size=(8, 16)) * 2.0 ** rng.uniform(-20, 20))
        codes, scales = Qz.quant_fp8_tiles(X, 8)
        amax = np.abs(X).max()
        k = -200
        while amax > 448.0 * 2.0 ** k:
            k += 1
        assert scales[0] == 2.0 ** k
        for idx in np.ndindex(X.shape):
            y = X[idx] / 2.0 ** k
            c, _ = _nearest_even(abs(y), e4_vals, e4_codes)
            want = c | (0x80 if y < 0 else 0)
            assert int(codes[idx]) == want, (t, idx, y)
