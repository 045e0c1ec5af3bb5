"""Pins for the NVFP4 oracle (oracle/nvfp4.py), each against something other than itself.

* the E2M1 value table and its halfway cases, written out from the format definition;
* a worked example whose scale bytes, codes and values are derived by hand below;
* exact invariances: a power-of-two scaling of a whole tensor leaves every code and scale
  byte unchanged; halving one line of an operand halves only the GEMM results that line
  feeds, which holds only if every rounding runs along the axis the reading names;
* the rounding error bound of the two-level format;
* with every rounding replaced by the identity, the layer is the plain fp64 layer.
"""
import numpy as np
import pytest

import oracle as O
import oracle.nvfp4 as N


def test_e2m1_codes_round_trip():
    # magnitudes by code, sign in bit 3 (E2M1: bias 1, one mantissa bit, subnormal 0.5)
    want = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for c in range(16):
        v = N.e2m1_decode(np.array([c]))[0]
        assert abs(v) == want[c & 7] and (np.signbit(v) == bool(c & 8))
        assert N.e2m1_encode(np.array([v]))[0] == c


def test_e2m1_halfway_cases_and_saturation():
    # each midpoint between neighbours goes to the code whose mantissa bit is 0
    cases = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6,
             0.2501: 1, 0.7499: 1, 0.7501: 2, 1.2501: 3, 1.7499: 3, 2.4999: 4, 2.5001: 5,
             3.4999: 5, 4.9999: 6, 5.0001: 7, 6.0: 7, 6.5: 7, 1e9: 7}
    for x, c in cases.items():
        assert N.e2m1_encode(np.array([x]))[0] == c, x
        assert N.e2m1_encode(np.array([-x]))[0] == c | 8, -x


def test_nvfp4_worked_example_by_hand():
    # Tensor amax 6 -> gs = 2688 / 6 = 448.
    # Block 0 (amax 6): s = 6/6 * 448 = 448 = 1.75 * 2^8 -> E4M3 byte 0 1111 110 = 0x7E;
    #   gs / s = 1, codes e2m1(6, 3, 1.5, 0.75) = 7, 5, 3, 2 (0.75 ties to 1.0), values 6, 3, 1.5, 1.
    # Block 1 (amax 3): s = 224 = 1.75 * 2^7 -> 0 1110 110 = 0x76; gs / s = 2:
    #   3 -> 6 (code 7), 1.25 -> 2.5 ties to 2 (code 4) -> value 1, 1.3 -> 2.6 -> 3 (code 5) -> 1.5.
    # Block 2 (amax 0.1): s = 0.1/6 * 448 = 7.4667 -> E4M3 step 0.5 in [4, 8): 7.5 = 1.875 * 2^2
    #   -> 0 1001 111 = 0x4F; gs / s = 59.7333: 0.1 -> 5.973 -> 6 (code 7) -> 6 * 7.5 / 448,
    #   0.05 -> 2.987 -> 3 (code 5) -> 3 * 7.5 / 448.
    v = np.zeros((3, 16))
    v[0, :4] = [6, 3, 1.5, 0.75]
    v[1, :3] = [3, 1.25, 1.3]
    v[2, :2] = [0.1, 0.05]
    gs = N.nv_global_scale(v)
    assert gs == np.float32(448.0)
    codes, sb = N.nv_quantize(v, gs, axis=1)
    assert sb.ravel().tolist() == [0x7E, 0x76, 0x4F]
    assert codes[0, :4].tolist() == [7, 5, 3, 2]
    assert codes[1, :3].tolist() == [7, 4, 5]
    assert codes[2, :2].tolist() == [7, 5]
    assert not codes[:, 4:].any() and not codes[1, 3] and not codes[2, 2:].any()
    deq = N.nv_dequantize(codes, sb, gs, axis=1)
    np.testing.assert_allclose(deq[0, :4], [6, 3, 1.5, 1.0], rtol=0, atol=0)
    np.testing.assert_allclose(deq[1, :3], [3, 1.0, 1.5], rtol=0, atol=0)
    np.testing.assert_allclose(deq[2, :2], [6 * 7.5 / 448, 3 * 7.5 / 448], rtol=1e-15)


def test_nvfp4_zero_and_underflowing_blocks():
    v = np.zeros((2, 32))
    assert N.nv_global_scale(v) == np.float32(1.0)
    c, s = N.nv_quantize(v, N.nv_global_scale(v), axis=1)
    assert not c.any() and not s.any()
    # a block 2^-20 below the tensor's amax: its scale underflows E4M3 (below 2^-9 / 2) -> zeros
    v[0, 0] = 1.0
    v[0, 16] = 2.0 ** -20
    gs = N.nv_global_scale(v)
    c, s = N.nv_quantize(v, gs, axis=1)
    assert s[0, 1] == 0 and not c[0, 16:].any()


@pytest.mark.parametrize("k", [-5, -1, 1, 3])
def test_global_scale_power_of_two_invariance(k):
    rng = np.random.default_rng(7)
    v = rng.standard_normal((8, 64)).astype(np.float32).astype(np.float64)
    c0, s0 = N.nv_quantize(v, N.nv_global_scale(v), axis=1)
    w = v * 2.0 ** k
    c1, s1 = N.nv_quantize(w, N.nv_global_scale(w), axis=1)
    assert (c0 == c1).all() and (s0 == s1).all()
    np.testing.assert_array_equal(N.nv_round(w, N.nv_global_scale(w), 1), N.nv_round(v, N.nv_global_scale(v), 1) * 2.0 ** k)


def test_rounding_error_within_the_format_bound():
    # |q - v gs / s| <= 1 (half the widest E2M1 gap, 4..6; saturation stays inside it because
    # s is at most 1/16 below amax gs / 6), so |value - v| <= s / gs <= (amax_block / 6)(1 + 1/16)
    rng = np.random.default_rng(3)
    v = rng.standard_normal((64, 256)) * np.exp(rng.uniform(-4, 4, (64, 1)))
    gs = N.nv_global_scale(v)
    r = N.nv_round(v, gs, axis=1)
    amax = np.repeat(np.abs(v).reshape(64, 16, 16).max(axis=2), 16, axis=1)
    assert np.all(np.abs(r - v) <= amax / 6 * (1 + 1 / 16) * (1 + 1e-6))
    assert np.mean(np.abs(r - v)) < 0.1 * np.mean(np.abs(v))


def test_codes_are_the_nearest_grid_points():
    # brute force over the eight magnitudes on the scaled fp32 values
    rng = np.random.default_rng(11)
    v = rng.standard_normal((4, 64)).astype(np.float32).astype(np.float64)
    gs = N.nv_global_scale(v)
    codes, sb = N.nv_quantize(v, gs, axis=1)
    sdec = O.e4m3_decode(sb).astype(np.float32)
    for r in range(4):
        for j in range(64):
            x = float(np.float32(np.float32(v[r, j]) * np.float32(gs / sdec[r, j // 16])))
            a = min(abs(x), 6.0)
            best = min(range(8), key=lambda c: (abs(a - N.E2M1_GRID[c]), c & 1))
            assert codes[r, j] & 7 == best


def test_rounding_runs_along_the_named_axis():
    # halving one column of v (not the one holding amax): along axis 0 only that column's
    # blocks change, and exactly by 1/2; along axis 1 its neighbours in each block move too
    rng = np.random.default_rng(5)
    v = rng.standard_normal((32, 32))
    v[0, 0] = 10.0
    w = v.copy()
    w[:, 5] *= 0.5
    gs = N.nv_global_scale(v)
    a, b = N.nv_round(v, gs, 0), N.nv_round(w, gs, 0)
    np.testing.assert_array_equal(b[:, 5], a[:, 5] * 0.5)
    np.testing.assert_array_equal(np.delete(b, 5, axis=1), np.delete(a, 5, axis=1))
    a1, b1 = N.nv_round(v, gs, 1), N.nv_round(w, gs, 1)
    assert not np.array_equal(np.delete(b1, 5, axis=1), np.delete(a1, 5, axis=1))


def _layer(seed, T=32, d=64, E=4, I=64, k=2):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((T, d))
    W_r = np.zeros((d, E))  # routing fixed by the bias alone, so X can change without moving it
    bias = rng.standard_normal(E)
    Wg = rng.standard_normal((E, d, I)) / np.sqrt(d)
    Wu = rng.standard_normal((E, d, I)) / np.sqrt(d)
    Wd = rng.standard_normal((E, I, d)) / np.sqrt(I)
    return X, W_r, bias, Wg, Wu, Wd, k


def _A(info):
    return {el: (e[0], e[3]) for el, e in enumerate(info["experts"]) if e is not None}


def test_layer_x_rounded_along_d():
    X, W_r, bias, Wg, Wu, Wd, k = _layer(1)
    X[0, 0] = 50.0  # amax(X) held by token 0
    _, i0 = N.forward_nv(X, W_r, bias, Wg, Wu, Wd, k)
    X2 = X.copy()
    X2[7] *= 0.5
    _, i1 = N.forward_nv(X2, W_r, bias, Wg, Wu, Wd, k)
    a0, a1 = _A(i0), _A(i1)
    for el in a0:
        toks, A0 = a0[el]
        A1 = a1[el][1]
        for r, t in enumerate(toks):
            np.testing.assert_array_equal(A1[r], A0[r] * (0.5 if t == 7 else 1.0))


def test_layer_w_gate_rounded_along_d():
    X, W_r, bias, Wg, Wu, Wd, k = _layer(2)
    Wg[0, 0, 0] = 5.0  # amax(W_gate) in column 0
    _, i0 = N.forward_nv(X, W_r, bias, Wg, Wu, Wd, k)
    Wg2 = Wg.copy()
    Wg2[:, :, 9] *= 0.5
    _, i1 = N.forward_nv(X, W_r, bias, Wg2, Wu, Wd, k)
    a0, a1 = _A(i0), _A(i1)
    for el in a0:
        A0, A1 = a0[el][1], a1[el][1]
        np.testing.assert_array_equal(A1[:, 9], A0[:, 9] * 0.5)
        np.testing.assert_array_equal(np.delete(A1, 9, axis=1), np.delete(A0, 9, axis=1))


def test_layer_w_up_rounded_along_d():
    X, W_r, bias, Wg, Wu, Wd, k = _layer(9)
    Wu[0, 0, 0] = 5.0  # amax(W_up) in column 0
    _, i0 = N.forward_nv(X, W_r, bias, Wg, Wu, Wd, k)
    Wu2 = Wu.copy()
    Wu2[:, :, 21] *= 0.5
    _, i1 = N.forward_nv(X, W_r, bias, Wg, Wu2, Wd, k)
    for e0, e1 in zip(i0["experts"], i1["experts"]):
        if e0 is None:
            continue
        B0, B1 = e0[4], e1[4]
        np.testing.assert_array_equal(B1[:, 21], B0[:, 21] * 0.5)
        np.testing.assert_array_equal(np.delete(B1, 21, axis=1), np.delete(B0, 21, axis=1))


def test_layer_w_down_rounded_along_i():
    X, W_r, bias, Wg, Wu, Wd, k = _layer(3)
    Wd[0, 0, 0] = 5.0  # amax(W_down) in output column 0
    Y0, _ = N.forward_nv(X, W_r, bias, Wg, Wu, Wd, k)
    Wd2 = Wd.copy()
    Wd2[:, :, 13] *= 0.5
    Y1, _ = N.forward_nv(X, W_r, bias, Wg, Wu, Wd2, k)
    np.testing.assert_array_equal(Y1[:, 13], Y0[:, 13] * 0.5)
    np.testing.assert_array_equal(np.delete(Y1, 13, axis=1), np.delete(Y0, 13, axis=1))


def test_layer_h_rounded_along_i():
    # one expert, every token on it: changing token 7's X changes only token 7's H row; with H
    # rounded along I (and amax(X), amax(H) held by token 0) every other token's Y is unchanged
    X, W_r, bias, Wg, Wu, Wd, k = _layer(4, E=1, k=1)
    X[0] *= 8.0
    Y0, i0 = N.forward_nv(X, W_r, bias, Wg, Wu, Wd, k)
    H0 = i0["experts"][0][2]
    assert np.argmax(np.abs(H0).max(axis=1)) == 0
    X2 = X.copy()
    X2[7] *= 0.5
    Y1, _ = N.forward_nv(X2, W_r, bias, Wg, Wu, Wd, k)
    np.testing.assert_array_equal(np.delete(Y1, 7, axis=0), np.delete(Y0, 7, axis=0))
    assert not np.array_equal(Y1[7], Y0[7])


def test_layer_without_rounding_is_the_plain_layer(monkeypatch):
    X, W_r, bias, Wg, Wu, Wd, k = _layer(6)
    W_r = np.random.default_rng(0).standard_normal(W_r.shape) * 0.5
    monkeypatch.setattr(N, "nv_round", lambda v, gs, axis: np.asarray(v, dtype=np.float64))
    Y, _ = N.forward_nv(X, W_r, bias, Wg, Wu, Wd, k)
    Yp, _ = O.forward(X, W_r, bias, Wg, Wu, Wd, k)
    np.testing.assert_allclose(Y, Yp, rtol=1e-13, atol=1e-13)


def test_nvfp4_layer_error_against_exact_layer():
    # the format's error through both GEMMs: a few percent of the output's scale, not more
    X, W_r, bias, Wg, Wu, Wd, k = _layer(8, T=64, d=256, E=4, I=256)
    Y, _ = N.forward_nv(X, W_r, bias, Wg, Wu, Wd, k)
    Yp, _ = O.forward(X, W_r, bias, Wg, Wu, Wd, k)
    err = np.max(np.abs(Y - Yp)) / np.max(np.abs(Yp))
    assert 0.01 < err < 0.5


# ---------------------------------------------------------------- backward
def _bwd_case(seed, T=32, d=64, E=4, I=64, k=2):
    X, W_r, bias, Wg, Wu, Wd, k = _layer(seed, T, d, E, I, k)
    dY = np.random.default_rng(seed + 100).standard_normal((T, d))
    dY[0, 0] = 40.0  # amax(dY) held by token 0
    return X, W_r, bias, Wg, Wu, Wd, k, dY


def test_backward_without_rounding_is_the_plain_backward(monkeypatch):
    X, W_r, bias, Wg, Wu, Wd, k, dY = _bwd_case(21)
    W_r = np.random.default_rng(1).standard_normal(W_r.shape) * 0.5
    import oracle.moe_oracle as M
    monkeypatch.setattr(N, "nv_round", lambda v, gs, axis: np.asarray(v, dtype=np.float64))
    monkeypatch.setattr(M, "bf16_round", lambda v: np.asarray(v, dtype=np.float64))
    _, info = N.forward_nv(X, W_r, bias, Wg, Wu, Wd, k)
    g = N.backward_nv(info, X, W_r, Wg, Wu, Wd, dY)
    _, ctx = O.forward(X, W_r, bias, Wg, Wu, Wd, k)
    gp = O.backward(ctx, dY)
    for n in ("dX", "dW_r"):
        np.testing.assert_allclose(g[n], gp[n], rtol=1e-12, atol=1e-12)
    for n in ("dW_gate", "dW_up", "dW_down"):
        for e in range(4):
            np.testing.assert_allclose(g[n][e], gp[n][e], rtol=1e-12, atol=1e-12)


def test_backward_dy_and_da_db_rounded_along_the_features():
    # halving token 7's dY halves its dH' exactly (dY rows rounded along d), hence its dA, dB, its
    # router-gate gradient, and (dA, dB rounded along I) its dX row; every other token's dX stays
    X, W_r, bias, Wg, Wu, Wd, k, dY = _bwd_case(22)
    _, info = N.forward_nv(X, W_r, bias, Wg, Wu, Wd, k)
    g0 = N.backward_nv(info, X, W_r, Wg, Wu, Wd, dY)
    dY2 = dY.copy()
    dY2[7] *= 0.5
    g1 = N.backward_nv(info, X, W_r, Wg, Wu, Wd, dY2)
    assert g1["gs_ab"] == g0["gs_ab"]
    np.testing.assert_array_equal(g1["dg"][7], g0["dg"][7] * 0.5)
    np.testing.assert_array_equal(np.delete(g1["dg"], 7, axis=0), np.delete(g0["dg"], 7, axis=0))
    np.testing.assert_array_equal(g1["dX"][7], g0["dX"][7] * 0.5)
    np.testing.assert_array_equal(np.delete(g1["dX"], 7, axis=0), np.delete(g0["dX"], 7, axis=0))


def test_backward_w_down_rounded_along_d():
    # halving row i of every W_down (one I index) halves column i of dH', dA, dB and so of dW_gate
    X, W_r, bias, Wg, Wu, Wd, k, dY = _bwd_case(23)
    Wd[0, 0, 0] = 6.0  # amax(W_down) in row 0
    _, info = N.forward_nv(X, W_r, bias, Wg, Wu, Wd, k)
    g0 = N.backward_nv(info, X, W_r, Wg, Wu, Wd, dY)
    Wd2 = Wd.copy()
    Wd2[:, 11, :] *= 0.5
    g1 = N.backward_nv(info, X, W_r, Wg, Wu, Wd2, dY)
    for e in g0["dW_gate"]:
        np.testing.assert_array_equal(g1["dW_gate"][e][:, 11], g0["dW_gate"][e][:, 11] * 0.5)
        np.testing.assert_array_equal(np.delete(g1["dW_gate"][e], 11, axis=1), np.delete(g0["dW_gate"][e], 11, axis=1))


@pytest.mark.parametrize("which", ["gate", "up"])
def test_backward_w_gate_up_rounded_along_i(which):
    # the dgrad of gate/up reads W_gate, W_up along I: halving row j (one d index) of every expert's
    # W_gate (or W_up) moves only column j of dX
    X, W_r, bias, Wg, Wu, Wd, k, dY = _bwd_case(24)
    Wg[0, 0, 0] = 6.0
    Wu[0, 0, 0] = 6.0  # the joint amax of [W_gate | W_up] in row 0
    _, info = N.forward_nv(X, W_r, bias, Wg, Wu, Wd, k)
    g0 = N.backward_nv(info, X, W_r, Wg, Wu, Wd, dY)
    W2 = (Wg if which == "gate" else Wu).copy()
    W2[:, 19, :] *= 0.5
    g1 = N.backward_nv(info, X, W_r, W2 if which == "gate" else Wg, W2 if which == "up" else Wu, Wd, dY)
    assert not np.array_equal(g1["dX"][:, 19], g0["dX"][:, 19])
    np.testing.assert_array_equal(np.delete(g1["dX"], 19, axis=1), np.delete(g0["dX"], 19, axis=1))


def test_weight_layout_caches_give_the_same_layer():
    # the bench's CPU baseline rounds the weights once (nv_weight_layouts, nv_weight_layouts_bwd);
    # the layer through those caches equals the layer rounding them inline
    X, W_r, bias, Wg, Wu, Wd, k, dY = _bwd_case(25)
    gs_w = N.nv_weight_scales(Wg, Wu, Wd)
    gs_b = N.nv_weight_scales_bwd(Wg, Wu, Wd)
    fw = {e: N.nv_weight_layouts(Wg[e], Wu[e], Wd[e], gs_w) for e in range(4)}
    bw = {e: N.nv_weight_layouts_bwd(Wg[e], Wu[e], Wd[e], gs_b) for e in range(4)}
    Y0, i0 = N.forward_nv(X, W_r, bias, Wg, Wu, Wd, k)
    Y1, i1 = N.forward_nv(X, W_r, bias, Wg, Wu, Wd, k, gs_w=gs_w, rounded=fw.__getitem__)
    np.testing.assert_array_equal(Y0, Y1)
    g0 = N.backward_nv(i0, X, W_r, Wg, Wu, Wd, dY)
    g1 = N.backward_nv(i1, X, W_r, Wg, Wu, Wd, dY, gs_bwd=gs_b, rounded=bw.__getitem__)
    for n in ("dX", "dW_r"):
        np.testing.assert_array_equal(g0[n], g1[n])
