"""Pins for the fp64 oracle, each against something other than the oracle itself.

* central finite differences of the forward (brute force) pin every gradient;
* torch autograd / torch.topk / torch float8 casts (library routines) pin the
  closed-form special cases (identical experts, k = E, E = 1) and the encoders;
* invariants of the routing table (counts, prefix sums, a stable bijection).
"""
import numpy as np
import pytest
import torch

import oracle as O


def _rand_layer(rng, T, d, E, I, k, scale_r=0.5):
    X = rng.standard_normal((T, d))
    W_r = rng.standard_normal((d, E)) * scale_r
    Wg = rng.standard_normal((E, d, I)) / np.sqrt(d)
    Wu = rng.standard_normal((E, d, I)) / np.sqrt(d)
    Wd = rng.standard_normal((E, I, d)) / np.sqrt(I)
    dY = rng.standard_normal((T, d))
    return X, W_r, Wg, Wu, Wd, dY


def _loss(X, W_r, b, Wg, Wu, Wd, k, dY):
    Y, _ = O.forward(X, W_r, b, Wg, Wu, Wd, k)
    return float(np.sum(Y * dY))


def _margin_ok(X, W_r, b, k, tol):
    l = O.router_logits(X, W_r, b)
    s = -np.sort(-l, axis=1)
    return np.all(s[:, k - 1] - s[:, k] > tol) if k < l.shape[1] else True


# --------------------------------------------------------------------------
# finite differences (brute force) on a tiny layer
# --------------------------------------------------------------------------
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_gradients_match_central_differences(seed):
    rng = np.random.default_rng(seed)
    T, d, E, I, k = 4, 8, 4, 16, 2
    X, W_r, Wg, Wu, Wd, dY = _rand_layer(rng, T, d, E, I, k)
    b = rng.standard_normal(E) * 0.1
    assert _margin_ok(X, W_r, b, k, 1e-3), "selection too close to a tie for FD"
    _, ctx = O.forward(X, W_r, b, Wg, Wu, Wd, k)
    gr = O.backward(ctx, dY)
    h = 1e-6

    def fd(arr, idx):
        old = arr[idx]
        arr[idx] = old + h
        lp = _loss(X, W_r, b, Wg, Wu, Wd, k, dY)
        arr[idx] = old - h
        lm = _loss(X, W_r, b, Wg, Wu, Wd, k, dY)
        arr[idx] = old
        return (lp - lm) / (2 * h)

    def check(arr, grad):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            num[idx] = fd(arr, idx)
        err = np.max(np.abs(num - grad)) / max(np.max(np.abs(num)), 1e-30)
        assert err < 1e-6, err

    check(X, gr["dX"])
    check(W_r, gr["dW_r"])
    check(Wg, np.stack([gr["dW_gate"][e] for e in range(E)]))
    check(Wu, np.stack([gr["dW_up"][e] for e in range(E)]))
    check(Wd, np.stack([gr["dW_down"][e] for e in range(E)]))


# --------------------------------------------------------------------------
# closed forms, against torch autograd in float64
# --------------------------------------------------------------------------
def _dense_swiglu_torch(X, Wg, Wu, Wd, dY):
    x = torch.tensor(X, requires_grad=True)
    wg = torch.tensor(Wg, requires_grad=True)
    wu = torch.tensor(Wu, requires_grad=True)
    wd = torch.tensor(Wd, requires_grad=True)
    y = (torch.nn.functional.silu(x @ wg) * (x @ wu)) @ wd
    (y * torch.tensor(dY)).sum().backward()
    return y.detach().numpy(), x.grad.numpy(), wg.grad.numpy(), wu.grad.numpy(), wd.grad.numpy()


def test_identical_experts_equal_one_dense_swiglu_mlp():
    rng = np.random.default_rng(3)
    T, d, E, I, k = 37, 16, 6, 24, 3
    X, W_r, Wg, Wu, Wd, dY = _rand_layer(rng, T, d, E, I, k)
    Wg[:] = Wg[0]; Wu[:] = Wu[0]; Wd[:] = Wd[0]
    Y, ctx = O.forward(X, W_r, None, Wg, Wu, Wd, k)
    gr = O.backward(ctx, dY)
    y, dx, dwg, dwu, dwd = _dense_swiglu_torch(X, Wg[0], Wu[0], Wd[0], dY)
    np.testing.assert_allclose(Y, y, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(gr["dX"], dx, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(sum(gr["dW_gate"].values()), dwg, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(sum(gr["dW_up"].values()), dwu, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(sum(gr["dW_down"].values()), dwd, rtol=1e-10, atol=1e-11)
    # every selected expert returns the same output, so the router gets no gradient
    assert np.max(np.abs(gr["dl"])) < 1e-12
    assert np.max(np.abs(gr["dW_r"])) < 1e-11


def test_single_expert_is_dense_mlp_with_unit_gate():
    rng = np.random.default_rng(4)
    T, d, E, I, k = 9, 8, 1, 16, 1
    X, W_r, Wg, Wu, Wd, dY = _rand_layer(rng, T, d, E, I, k)
    Y, ctx = O.forward(X, W_r, None, Wg, Wu, Wd, k)
    assert np.all(ctx["g"] == 1.0)
    gr = O.backward(ctx, dY)
    y, dx, dwg, dwu, dwd = _dense_swiglu_torch(X, Wg[0], Wu[0], Wd[0], dY)
    np.testing.assert_allclose(Y, y, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(gr["dX"], dx, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(gr["dW_gate"][0], dwg, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(gr["dW_down"][0], dwd, rtol=1e-10, atol=1e-11)
    assert np.all(gr["dW_r"] == 0)


def test_k_equals_E_is_dense_softmax_mixture():
    """With every expert selected the gates are a full softmax and differentiable."""
    rng = np.random.default_rng(5)
    T, d, E, I = 11, 8, 4, 12
    X, W_r, Wg, Wu, Wd, dY = _rand_layer(rng, T, d, E, I, E)
    b = rng.standard_normal(E) * 0.3
    Y, ctx = O.forward(X, W_r, b, Wg, Wu, Wd, E)
    gr = O.backward(ctx, dY)
    x = torch.tensor(X, requires_grad=True)
    wr = torch.tensor(W_r, requires_grad=True)
    wg = torch.tensor(Wg, requires_grad=True)
    wu = torch.tensor(Wu, requires_grad=True)
    wd = torch.tensor(Wd, requires_grad=True)
    p = torch.softmax(x @ wr + torch.tensor(b), dim=1)  # [T, E]
    outs = torch.stack([(torch.nn.functional.silu(x @ wg[e]) * (x @ wu[e])) @ wd[e] for e in range(E)], 1)
    y = (p[:, :, None] * outs).sum(1)
    (y * torch.tensor(dY)).sum().backward()
    np.testing.assert_allclose(Y, y.detach().numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(gr["dX"], x.grad.numpy(), rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(gr["dW_r"], wr.grad.numpy(), rtol=1e-10, atol=1e-11)
    for e in range(E):
        np.testing.assert_allclose(gr["dW_gate"][e], wg.grad[e].numpy(), rtol=1e-10, atol=1e-11)
        np.testing.assert_allclose(gr["dW_up"][e], wu.grad[e].numpy(), rtol=1e-10, atol=1e-11)
        np.testing.assert_allclose(gr["dW_down"][e], wd.grad[e].numpy(), rtol=1e-10, atol=1e-11)


def test_topk_gating_matches_torch_autograd_through_selected_softmax():
    """k < E: torch autograd through topk-selected softmax equals the oracle."""
    rng = np.random.default_rng(6)
    T, d, E, I, k = 13, 8, 7, 12, 3
    X, W_r, Wg, Wu, Wd, dY = _rand_layer(rng, T, d, E, I, k)
    Y, ctx = O.forward(X, W_r, None, Wg, Wu, Wd, k)
    gr = O.backward(ctx, dY)
    x = torch.tensor(X, requires_grad=True)
    wr = torch.tensor(W_r, requires_grad=True)
    logits = x @ wr
    vals, idx = torch.topk(logits, k, dim=1)
    assert np.array_equal(idx.numpy(), ctx["ids"])
    g = torch.softmax(vals, dim=1)
    y = torch.zeros(T, d, dtype=torch.float64)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            xt = x[t:t + 1]
            o = (torch.nn.functional.silu(xt @ torch.tensor(Wg[e])) * (xt @ torch.tensor(Wu[e]))) @ torch.tensor(Wd[e])
            y = y.index_add(0, torch.tensor([t]), g[t, j] * o)
    (y * torch.tensor(dY)).sum().backward()
    np.testing.assert_allclose(Y, y.detach().numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(gr["dX"], x.grad.numpy(), rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(gr["dW_r"], wr.grad.numpy(), rtol=1e-10, atol=1e-11)


def test_sonicmoe_identity_router_grad_from_swiglu_backward():
    """<dY, H W_down> == <dY W_down^T, H>: the fused form of the router gradient."""
    rng = np.random.default_rng(7)
    T, d, E, I, k = 40, 16, 5, 32, 2
    X, W_r, Wg, Wu, Wd, dY = _rand_layer(rng, T, d, E, I, k)
    _, ctx = O.forward(X, W_r, None, Wg, Wu, Wd, k)
    gr = O.backward(ctx, dY)
    ids = ctx["ids"]
    for t in range(T):
        for j in range(k):
            e = ids[t, j]
            a, b_ = X[t] @ Wg[e], X[t] @ Wu[e]
            h = O.silu(a) * b_
            fused = float((dY[t] @ Wd[e].T) @ h)
            assert abs(fused - gr["dg"][t, j]) < 1e-12 * max(1.0, abs(fused))


def test_token_path_equals_full_layer():
    rng = np.random.default_rng(8)
    T, d, E, I, k = 21, 8, 6, 16, 3
    X, W_r, Wg, Wu, Wd, dY = _rand_layer(rng, T, d, E, I, k)
    b = rng.standard_normal(E) * 0.2
    for fl, nl in [(0, None), (2, 3)]:
        Y, ctx = O.forward(X, W_r, b, Wg, Wu, Wd, k, first_local=fl, num_local=nl)
        gr = O.backward(ctx, dY)
        for t in [0, 5, 20]:
            y, dx, dl, ids, g = O.token_forward_backward(t, X, W_r, b, Wg, Wu, Wd, k, dY, fl, nl)
            np.testing.assert_allclose(y, Y[t], rtol=1e-13, atol=1e-13)
            np.testing.assert_allclose(dx, gr["dX"][t], rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(dl, gr["dl"][t], rtol=1e-12, atol=1e-13)


def test_local_expert_slices_sum_to_full_layer():
    """Y, dX, dl and dW_r are linear in the experts' contributions: slices add up."""
    rng = np.random.default_rng(9)
    T, d, E, I, k = 30, 8, 6, 16, 3
    X, W_r, Wg, Wu, Wd, dY = _rand_layer(rng, T, d, E, I, k)
    Yf, cf = O.forward(X, W_r, None, Wg, Wu, Wd, k)
    gf = O.backward(cf, dY)
    Ys, dXs, dWrs = 0, 0, 0
    for fl in range(0, E, 2):
        Y, c = O.forward(X, W_r, None, Wg, Wu, Wd, k, first_local=fl, num_local=2)
        g = O.backward(c, dY)
        Ys, dXs, dWrs = Ys + Y, dXs + g["dX"], dWrs + g["dW_r"]
        for e in range(fl, fl + 2):
            np.testing.assert_allclose(g["dW_gate"][e], gf["dW_gate"][e], rtol=1e-12, atol=1e-13)
    # the router term dl W_r^T is added once per slice; the dense part sums exactly
    np.testing.assert_allclose(Ys, Yf, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dWrs, gf["dW_r"], rtol=1e-11, atol=1e-12)


def test_slice_router_gradient_lives_on_tokens_with_a_local_assignment():
    """In an expert slice a token with no local assignment has dg = 0 on every slot, so its
    dl row is exactly zero and dW_r = X^T dl is the same sum over the other tokens alone."""
    rng = np.random.default_rng(10)
    T, d, E, I, k = 40, 8, 12, 16, 2
    X, W_r, Wg, Wu, Wd, dY = _rand_layer(rng, T, d, E, I, k)
    fl, nl = 3, 2
    Y, c = O.forward(X, W_r, None, Wg, Wu, Wd, k, first_local=fl, num_local=nl)
    g = O.backward(c, dY)
    ids = O.topk_ids(O.router_logits(X, W_r, None), k)
    listed = np.any((ids >= fl) & (ids < fl + nl), axis=1)
    assert 0 < listed.sum() < T
    assert np.all(g["dl"][~listed] == 0.0)
    assert np.any(g["dl"][listed] != 0.0)
    np.testing.assert_allclose(X[listed].T @ g["dl"][listed], g["dW_r"], rtol=1e-13, atol=1e-14)
    assert np.all(Y[~listed] == 0.0)  # nothing of theirs is computed in this slice
    assert np.all(g["dX"][~listed] == 0.0)


# --------------------------------------------------------------------------
# routing: selection, ties, invariants of the table
# --------------------------------------------------------------------------
def test_topk_matches_torch_topk_on_distinct_values():
    rng = np.random.default_rng(10)
    l = rng.standard_normal((200, 64))
    for k in [1, 2, 8, 64]:
        ids = O.topk_ids(l, k)
        _, ti = torch.topk(torch.tensor(l), k, dim=1, sorted=True)
        assert np.array_equal(ids, ti.numpy())


def test_topk_tie_break_lower_id_and_signed_zero_and_nan():
    l = np.array([
        [1.0, 1.0, 1.0, 1.0],          # all tied -> 0,1,2
        [0.0, -0.0, 0.5, -0.0],        # -0 == +0 -> 2,0,1
        [np.nan, -np.inf, 3.0, np.nan],  # NaN lowest, below -inf
        [2.0, 5.0, 5.0, 1.0],          # tie at top -> 1,2,0
    ])
    ids = O.topk_ids(l, 3)
    assert ids.tolist() == [[0, 1, 2], [2, 0, 1], [2, 1, 0], [1, 2, 0]]


def test_gates_sum_to_one_and_equal_renormalised_full_softmax():
    rng = np.random.default_rng(11)
    l = rng.standard_normal((50, 16)) * 3
    ids = O.topk_ids(l, 4)
    g = O.gates(l, ids)
    assert np.max(np.abs(g.sum(1) - 1)) < 1e-15
    p = torch.softmax(torch.tensor(l), dim=1).numpy()
    ps = np.take_along_axis(p, ids.astype(np.int64), 1)
    np.testing.assert_allclose(g, ps / ps.sum(1, keepdims=True), rtol=1e-13)
    assert np.all(np.diff(g, axis=1) <= 0)  # descending logits -> descending gates


@pytest.mark.parametrize("T,E,k,fl,nl", [(300, 16, 4, 0, None), (257, 8, 2, 0, None),
                                          (100, 12, 3, 4, 5), (64, 1, 1, 0, None)])
def test_schedule_invariants_and_brute_force(T, E, k, fl, nl):
    rng = np.random.default_rng(T + E)
    l = rng.standard_normal((T, E))
    l[:, 0] += 1.5  # a hot expert: some segments span several padded tiles
    ids = O.topk_ids(l, k)
    s = O.schedule(ids, E, fl, nl)
    El = s["num_local"]
    # exactly k distinct ids per token
    assert all(len(set(r)) == k for r in ids.tolist())
    loc = (ids >= fl) & (ids < fl + El)
    assert s["counts"].sum() == loc.sum()
    if nl is None:
        assert s["counts"].sum() == T * k
    assert np.array_equal(s["offsets"], np.concatenate([[0], np.cumsum(s["counts"])]))
    pc = -(-s["counts"] // O.P_PAD) * O.P_PAD
    assert np.array_equal(s["padded_offsets"], np.concatenate([[0], np.cumsum(pc)]))
    # brute force: a stable sort of (expert, token) pairs gives perm
    pairs = sorted((int(ids[t, j]) - fl, t) for t in range(T) for j in range(k) if loc[t, j])
    assert [t for _, t in pairs] == s["perm"].tolist()
    # slot_row points to the row holding that token inside its expert's padded segment
    for t in range(T):
        for j in range(k):
            r = s["slot_row"][t, j]
            if not loc[t, j]:
                assert r == -1
                continue
            e = ids[t, j] - fl
            assert s["padded_offsets"][e] <= r < s["padded_offsets"][e] + s["counts"][e]
            pos = r - s["padded_offsets"][e]
            assert s["perm"][s["offsets"][e] + pos] == t
    # tokens strictly increasing inside each segment
    for e in range(El):
        seg = s["perm"][s["offsets"][e]:s["offsets"][e + 1]]
        assert np.all(np.diff(seg) > 0)


# --------------------------------------------------------------------------
# MX (E4M3 + E8M0) quantiser
# --------------------------------------------------------------------------
def test_e4m3_decode_matches_torch_float8():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = O.e4m3_decode(codes)
    both_nan = np.isnan(ref) & np.isnan(mine)
    assert np.all(both_nan | (ref == mine))
    assert O.e4m3_decode([0x7E])[0] == 448.0 and O.e4m3_decode([0x01])[0] == 2.0 ** -9


def test_e4m3_encode_round_trips_and_matches_torch_rne():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = O.e4m3_decode(codes)
    back = O.e4m3_encode(vals)
    assert np.array_equal(back, codes)
    rng = np.random.default_rng(12)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.05, 1, 30, 120)])
    x = x[np.abs(x) < 440]
    # exact midpoints between neighbours exercise ties-to-even
    mids = (vals[:-1] + vals[1:]) / 2
    mids = mids[np.isfinite(mids) & (np.abs(mids) < 440)]
    x = np.concatenate([x, mids, -mids])
    ref = torch.tensor(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_encode(x), ref)


def test_e4m3_saturates():
    assert O.e4m3_encode([500.0, -1e9, 449.0])[0] == 0x7E
    assert O.e4m3_encode([-1e9])[0] == 0xFE


def test_mx_quantize_scale_rule_and_edges():
    v = np.zeros((2, 64))
    v[0, :32] = np.linspace(-3, 3, 32)          # amax 3 -> floor(log2 3) - 8 = -7
    v[0, 32:] = 0.0                              # all-zero block
    v[1, :32] = 2.0 ** 5                         # amax a power of two -> -3, value 256
    v[1, 32:] = np.linspace(-1, 1, 32) * 2.0 ** -20
    codes, sc = O.mx_quantize(v, axis=1)
    assert sc.tolist() == [[127 - 7, 0], [127 - 3, 127 - 20 - 8]]
    assert np.all(codes[0, 32:] == 0)
    assert np.all(O.e4m3_decode(codes[1, :32]) == 256.0)
    back = O.mx_dequantize(codes, sc, axis=1)
    # E4M3 has 3 mantissa bits: relative error at most 2^-4 inside the normal range
    nz = np.abs(v) > 2.0 ** -6 * 2.0 ** (sc.repeat(32, axis=1).astype(int) - 127)
    assert np.all(np.abs(back - v)[nz] <= np.abs(v)[nz] * 2.0 ** -4 + 1e-30)
    # amax * 2^-s lies in [256, 512): the largest element may saturate to 448
    big = np.full((1, 32), 1.0); big[0, 0] = 1.99
    c2, s2 = O.mx_quantize(big, axis=1)
    assert s2[0, 0] == 127 - 8 and c2[0, 0] == 0x7E


def test_mx_quantize_axis0_equals_transposed_axis1():
    rng = np.random.default_rng(13)
    v = rng.standard_normal((64, 96))
    c0, s0 = O.mx_quantize(v, axis=0)
    c1, s1 = O.mx_quantize(v.T, axis=1)
    assert np.array_equal(c0, c1.T) and np.array_equal(s0, s1.T)


# --------------------------------------------------------------------------
# MXFP8 layer of the oracle: with MX rounding replaced by the identity it must
# be the bf16 layer exactly (operands, axes and the fused router gradient wired
# as the unquantised definition); the rounding itself is pinned above.
# --------------------------------------------------------------------------
@pytest.mark.parametrize("mx_wgrad", [False, True])
def test_mx_layer_reduces_to_the_plain_layer_without_rounding(monkeypatch, mx_wgrad):
    import oracle.moe_oracle as M
    rng = np.random.default_rng(14)
    T, d, E, I, k = 40, 64, 6, 96, 2
    X, W_r, Wg, Wu, Wd, dY = _rand_layer(rng, T, d, E, I, k)
    Y, ctx = O.forward(X, W_r, None, Wg, Wu, Wd, k)
    g = O.backward(ctx, dY)
    monkeypatch.setattr(M, "mx_round", lambda v, axis: np.asarray(v, dtype=np.float64))
    monkeypatch.setattr(M, "bf16_round", lambda v: np.asarray(v, dtype=np.float64))
    Yq, cq = M.forward_mx(X, W_r, None, Wg, Wu, Wd, k)
    gq = M.backward_mx(cq, dY, mx_wgrad=mx_wgrad)
    np.testing.assert_allclose(Yq, Y, rtol=1e-13, atol=1e-13)
    for n in ("dX", "dW_r", "dl", "dg"):
        np.testing.assert_allclose(gq[n], g[n], rtol=1e-11, atol=1e-12)
    for n in ("dW_gate", "dW_up", "dW_down"):
        for e in range(E):
            np.testing.assert_allclose(gq[n][e], g[n][e], rtol=1e-11, atol=1e-12)


def test_bf16_round_equals_torch_bfloat16_conversion():
    # the saved-activation rounding of the MX backward: fp64 -> fp32 -> bf16, nearest even each
    # time, against torch's conversions (halfway cases, signs, subnormals, large values)
    import torch
    rng = np.random.default_rng(16)
    v = np.concatenate([rng.standard_normal(4000) * 10.0 ** rng.integers(-40, 38, 4000),
                        [0.0, -0.0, 1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 2.0 ** -130,
                         3.0e38, 1.0 + 2.0 ** -8 + 2.0 ** -30]])
    want = torch.from_numpy(v).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.bf16_round(v)
    assert np.array_equal(np.signbit(got), np.signbit(want))
    assert np.array_equal(got, want)


@pytest.mark.parametrize("mx_wgrad", [False, True])
def test_mx_backward_reads_the_saved_activations_as_bf16(mx_wgrad):
    # Moving each saved A, B entry halfway towards its bf16 value keeps that value: the MX
    # backward, which reads them as bf16, returns the same bits; the unrounded values differ.
    X, W_r, Wg, Wu, Wd, dY = _mx_case()
    _, ctx = O.forward_mx(X, W_r, None, Wg, Wu, Wd, _MX_SHAPE["k"])
    g = O.backward_mx(ctx, dY, mx_wgrad=mx_wgrad)
    saved = [None if it is None else (it[0], it[1], (it[2] + O.bf16_round(it[2])) / 2, (it[3] + O.bf16_round(it[3])) / 2)
             for it in ctx["saved"]]
    assert any(it is not None and not np.array_equal(it[2], ctx["saved"][e][2]) for e, it in enumerate(saved))
    g2 = O.backward_mx(dict(ctx, saved=saved), dY, mx_wgrad=mx_wgrad)
    for n in ("dX", "dg", "dl", "dW_r"):
        assert np.array_equal(g[n], g2[n]), n
    for n in ("dW_gate", "dW_up", "dW_down"):
        for e in g[n]:
            assert np.array_equal(g[n][e], g2[n][e]), (n, e)


def test_mx_round_error_bound_and_idempotence():
    rng = np.random.default_rng(15)
    v = rng.standard_normal((16, 256))
    r = O.mx_round(v, axis=1)
    assert np.array_equal(O.mx_round(r, axis=1), r)  # MX values are fixed points
    # per 32-block: |error| <= half an E4M3 ulp of the block's top binade after saturation at 448
    vb, rb = v.reshape(16, 8, 32), r.reshape(16, 8, 32)
    amax = np.abs(vb).max(-1, keepdims=True)
    step = 2.0 ** (np.floor(np.log2(amax)) - 8)  # scale; codes are <= 448 = 1.75 * 2^8
    assert np.all(np.abs(vb - rb) <= np.maximum(amax - 448 * step, 0) + 16 * step + 1e-300)


# --------------------------------------------------------------------------
# MX layer: every operand is rounded in blocks along its own GEMM's contraction
# dimension (d for X, W_gate, W_up and, in the dgrad of W_down, for dY and W_down;
# I for H, W_down in the forward, dA, dB and W_gate / W_up in the dgrad of gate/up).
# Rounding in blocks along one axis commutes with scaling a single line across the
# other axis by a power of two, so a line scaled that way changes its own results
# (by that power exactly) and nothing else, bit for bit.  With any operand rounded
# along the other axis the scaled line would become the amax of its blocks there and
# change how its neighbours round.  The checks below hold one line of each operand
# against that, and so fail if any rounding axis of forward_mx / backward_mx flips.
# --------------------------------------------------------------------------
_MX_SHAPE = dict(T=96, d=64, E=3, I=64, k=2)
_P2 = 32.0  # a power of two large enough to become the amax of any block it joins


def _mx_case(seed=40):
    rng = np.random.default_rng(seed)
    s = _MX_SHAPE
    X, W_r, Wg, Wu, Wd, dY = _rand_layer(rng, s["T"], s["d"], s["E"], s["I"], s["k"])
    return X, W_r, Wg, Wu, Wd, dY


def _mx_run(X, W_r, Wg, Wu, Wd, dY, k=_MX_SHAPE["k"]):
    Y, ctx = O.forward_mx(X, W_r, None, Wg, Wu, Wd, k)
    return Y, ctx, O.backward_mx(ctx, dY)


def _same_except(a, b, axis, line):
    """a and b equal bit for bit outside index `line` of `axis`, and different on it."""
    a, b = np.moveaxis(a, axis, 0), np.moveaxis(b, axis, 0)
    keep = np.ones(a.shape[0], dtype=bool)
    keep[line] = False
    return np.array_equal(a[keep], b[keep]) and not np.array_equal(a[line], b[line])


def test_mx_token_rows_are_independent():
    # X, H, dY, dA and dB are rounded per token row (along d or I): scaling one token's X and
    # dY rows leaves every other token's Y, dX and router gradient bit-identical.
    X, W_r, Wg, Wu, Wd, dY = _mx_case()
    Y, ctx, g = _mx_run(X, W_r, Wg, Wu, Wd, dY)
    t = 37
    X2, dY2 = X.copy(), dY.copy()
    X2[t] *= _P2
    dY2[t] *= _P2
    Y2, ctx2, g2 = _mx_run(X2, W_r, Wg, Wu, Wd, dY2)
    assert np.array_equal(ctx["ids"], ctx2["ids"])  # a positive scale keeps the selection
    assert _same_except(Y, Y2, 0, t)
    assert _same_except(g["dX"], g2["dX"], 0, t)
    assert _same_except(g["dl"], g2["dl"], 0, t)
    # the forward alone, with dY unchanged: the other tokens' dX stays put as well
    _, _, g3 = _mx_run(X2, W_r, Wg, Wu, Wd, dY)
    assert _same_except(g["dX"], g3["dX"], 0, t)
    # dY alone: the backward's dY rounding (along d) keeps tokens apart
    _, _, g4 = _mx_run(X, W_r, Wg, Wu, Wd, dY2)
    assert _same_except(g["dX"], g4["dX"], 0, t)


@pytest.mark.parametrize("name,slot", [("W_gate", 2), ("W_up", 3)])
def test_mx_forward_gate_up_weight_columns_are_independent(name, slot):
    # W_gate and W_up are rounded along d (the forward's contraction): scaling column j of one
    # expert's matrix scales that expert's A (or B) column j exactly and no other column.
    X, W_r, Wg, Wu, Wd, dY = _mx_case()
    _, ctx = O.forward_mx(X, W_r, None, Wg, Wu, Wd, _MX_SHAPE["k"])
    e, j = 1, 21
    W2 = (Wg if name == "W_gate" else Wu).copy()
    W2[e][:, j] *= _P2
    args = (W2, Wu) if name == "W_gate" else (Wg, W2)
    _, ctx2 = O.forward_mx(X, W_r, None, *args, Wd, _MX_SHAPE["k"])
    a, a2 = ctx["saved"][e][slot], ctx2["saved"][e][slot]
    assert _same_except(a, a2, 1, j)
    assert np.array_equal(a2[:, j], a[:, j] * _P2)


def test_mx_forward_down_weight_columns_are_independent():
    # W_down is rounded along I in the forward: scaling its column c (of d) changes column c of
    # Y only.
    X, W_r, Wg, Wu, Wd, dY = _mx_case()
    Y, _ = O.forward_mx(X, W_r, None, Wg, Wu, Wd, _MX_SHAPE["k"])
    Wd2 = Wd.copy()
    Wd2[0][:, 9] *= _P2
    Y2, _ = O.forward_mx(X, W_r, None, Wg, Wu, Wd2, _MX_SHAPE["k"])
    assert _same_except(Y, Y2, 1, 9)


@pytest.mark.parametrize("mx_wgrad", [False, True])
def test_mx_dgrad_down_weight_rows_are_independent(mx_wgrad):
    # In the dgrad of W_down (contraction over d) W_down is rounded along d: scaling its row i
    # (of I) in the backward alone scales dH'[:, i], hence dA[:, i] and dB[:, i], exactly, so
    # column i of dW_gate and dW_up scales exactly and no other column moves.  With mx_wgrad
    # the same holds only if dA and dB are rounded along the rows (tokens): rounded along I,
    # the scaled column would become the amax of its blocks and move its neighbours.
    X, W_r, Wg, Wu, Wd, dY = _mx_case()
    _, ctx = O.forward_mx(X, W_r, None, Wg, Wu, Wd, _MX_SHAPE["k"])
    g = O.backward_mx(ctx, dY, mx_wgrad=mx_wgrad)
    e, i = 2, 45
    Wd2 = Wd.copy()
    Wd2[e][i, :] *= _P2
    g2 = O.backward_mx(dict(ctx, W_down=Wd2), dY, mx_wgrad=mx_wgrad)
    for n in ("dW_gate", "dW_up"):
        assert _same_except(g[n][e], g2[n][e], 1, i), n
        assert np.array_equal(g2[n][e][:, i], g[n][e][:, i] * _P2), n


@pytest.mark.parametrize("name", ["W_gate", "W_up"])
def test_mx_dgrad_gate_up_weight_rows_are_independent(name):
    # In the dgrad of gate/up (contraction over I) W_gate and W_up are rounded along I: scaling
    # row r (of d) in the backward alone changes column r of dX and no other column.
    X, W_r, Wg, Wu, Wd, dY = _mx_case()
    _, ctx = O.forward_mx(X, W_r, None, Wg, Wu, Wd, _MX_SHAPE["k"])
    g = O.backward_mx(ctx, dY)
    W2 = ctx[name].copy()
    W2[0][13, :] *= _P2
    g2 = O.backward_mx(dict(ctx, **{name: W2}), dY)
    assert _same_except(g["dX"], g2["dX"], 1, 13)


def test_mx_layer_worked_example_by_hand():
    # tests/golden/mx_layer_worked_example.json: a one-expert MXFP8 layer whose every rounding
    # is worked out by hand there (the values differ if X, H or dA were rounded along tokens).
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "mx_layer_worked_example.json")) as f:
        G = json.load(f)
    s = G["shape"]
    T, d, E, k, I = s["T"], s["d"], s["E"], s["top_k"], s["I"]
    arrays = {"X": np.zeros((T, d)), "W_gate[0]": np.zeros((d, I)), "W_up[0]": np.zeros((d, I)),
              "W_down[0]": np.zeros((I, d)), "dY": np.zeros((T, d)), "W_r": np.zeros((d, E))}
    for name, entries in G["inputs_nonzero"].items():
        for r, c, v in entries:
            arrays[name][r, c] = v
    Y, ctx = O.forward_mx(arrays["X"], arrays["W_r"], None, arrays["W_gate[0]"][None], arrays["W_up[0]"][None],
                          arrays["W_down[0]"][None], k)
    g = O.backward_mx(ctx, arrays["dY"])
    got = {"Y": Y, "dX": g["dX"], "dg": g["dg"], "dW_gate[0]": g["dW_gate"][0], "dW_up[0]": g["dW_up"][0],
           "dW_down[0]": g["dW_down"][0]}
    for name, entries in G["expected"].items():
        want = np.zeros_like(got[name])
        for r, c, v in entries:
            want[r, c] = v
        np.testing.assert_allclose(got[name], want, rtol=1e-13, atol=0, err_msg=name)
    assert not np.any(g["dW_r"])


# --------------------------------------------------------------------------
# MX weight gradients (mx_wgrad): X, dA, dB, Hg = g H and dY rounded along the expert's
# rows in blocks of 32.  Blocks along the rows commute with scaling one column by a power
# of two, so a column scaled that way moves its own row (or column) of the gradient, by
# that power exactly, and nothing else; rounded along d or I instead, the scaled column
# would become the amax of its blocks and move its neighbours.
# --------------------------------------------------------------------------
def test_mx_wgrad_x_columns_are_independent():
    # X scaled in the backward alone (its weight gradients): column j of X moves row j of
    # every expert's dW_gate and dW_up
    X, W_r, Wg, Wu, Wd, dY = _mx_case()
    _, ctx = O.forward_mx(X, W_r, None, Wg, Wu, Wd, _MX_SHAPE["k"])
    g = O.backward_mx(ctx, dY, mx_wgrad=True)
    j = 29
    X2 = X.copy()
    X2[:, j] *= _P2
    g2 = O.backward_mx(dict(ctx, X=X2), dY, mx_wgrad=True)
    for e in range(_MX_SHAPE["E"]):
        for n in ("dW_gate", "dW_up"):
            assert _same_except(g[n][e], g2[n][e], 0, j), (n, e)
            assert np.array_equal(g2[n][e][j], g[n][e][j] * _P2), (n, e)


def test_mx_wgrad_dy_columns_are_independent():
    # dY column j moves column j of every expert's dW_down and no other (its dgrad changes
    # too, but dW_down reads only Hg, from the forward, and dY itself)
    X, W_r, Wg, Wu, Wd, dY = _mx_case()
    _, ctx = O.forward_mx(X, W_r, None, Wg, Wu, Wd, _MX_SHAPE["k"])
    g = O.backward_mx(ctx, dY, mx_wgrad=True)
    j = 50
    dY2 = dY.copy()
    dY2[:, j] *= _P2
    g2 = O.backward_mx(ctx, dY2, mx_wgrad=True)
    for e in range(_MX_SHAPE["E"]):
        assert _same_except(g["dW_down"][e], g2["dW_down"][e], 1, j), e
        assert np.array_equal(g2["dW_down"][e][:, j], g["dW_down"][e][:, j] * _P2), e


def test_mx_wgrad_hg_columns_are_independent():
    # W_up column i of one expert (rounded along d in the forward) scales B[:, i], hence
    # H[:, i], Hg[:, i] and dA[:, i], exactly: row i of dW_down and column i of dW_gate move,
    # by that power, and nothing else of the expert's weight gradients
    X, W_r, Wg, Wu, Wd, dY = _mx_case()
    k = _MX_SHAPE["k"]
    _, ctx = O.forward_mx(X, W_r, None, Wg, Wu, Wd, k)
    g = O.backward_mx(ctx, dY, mx_wgrad=True)
    e, i = 1, 7
    Wu2 = Wu.copy()
    Wu2[e][:, i] *= _P2
    _, ctx2 = O.forward_mx(X, W_r, None, Wg, Wu2, Wd, k)
    g2 = O.backward_mx(ctx2, dY, mx_wgrad=True)
    assert _same_except(g["dW_down"][e], g2["dW_down"][e], 0, i)
    assert np.array_equal(g2["dW_down"][e][i], g["dW_down"][e][i] * _P2)
    assert _same_except(g["dW_gate"][e], g2["dW_gate"][e], 1, i)
    assert np.array_equal(g2["dW_gate"][e][:, i], g["dW_gate"][e][:, i] * _P2)
    assert np.array_equal(g2["dW_up"][e], g["dW_up"][e])


def test_mx_round_rows_in_groups():
    # Runs of rows rounded on their own (a ring-streamed layer's segments): 20 rows holding 0.005
    # and then 20 rows whose first is 256.  As one run, the block of rows 0-31 has amax 256 and
    # 0.005 falls below E4M3's normal range: 2.56 steps of 2^-9 -> 3 -> 0.005859375.  In runs of
    # 20 + 20, rows 0-19 are their own block (amax 0.005, scale 2^-16): 0.005 * 65536 = 327.68,
    # step 32 -> 320 -> 0.0048828125, and 256 stays 256.
    v = np.zeros((40, 32))
    v[:20, 3] = 0.005
    v[20, 3] = 256.0
    one = O.mx_round_rows(v)
    two = O.mx_round_rows(v, [20, 20])
    assert np.all(one[:20, 3] == 0.005859375) and one[20, 3] == 256.0
    assert np.all(two[:20, 3] == 0.0048828125) and two[20, 3] == 256.0
    # runs that are whole multiples of 32 rows give the blocks of one run; empty runs add nothing
    rng = np.random.default_rng(17)
    w = rng.standard_normal((96, 64)) * np.exp(rng.standard_normal((96, 1)))
    assert np.array_equal(O.mx_round_rows(w, [32, 0, 64]), O.mx_round_rows(w))
    assert np.array_equal(O.mx_round_rows(w, [96]), O.mx_round_rows(w))
    with pytest.raises(ValueError):
        O.mx_round_rows(w, [32, 32])


def test_mx_wgrad_row_groups_reach_every_operand():
    # backward_mx with row groups rounds all five weight-gradient operands by run: runs that
    # split at multiples of 32 reproduce the one-run gradients bit for bit, runs that do not move
    # every gradient
    X, W_r, Wg, Wu, Wd, dY = _mx_case()
    _, ctx = O.forward_mx(X, W_r, None, Wg, Wu, Wd, _MX_SHAPE["k"])
    g = O.backward_mx(ctx, dY, mx_wgrad=True)
    rows = {el: len(ctx["saved"][el][0]) for el in range(_MX_SHAPE["E"]) if ctx["saved"][el] is not None}
    aligned = O.backward_mx(ctx, dY, mx_wgrad=True, row_groups=lambda el: [32, rows[el] - 32])
    split = O.backward_mx(ctx, dY, mx_wgrad=True, row_groups=lambda el: [13, rows[el] - 13])
    for n in ("dW_gate", "dW_up", "dW_down"):
        for e in rows:
            assert np.array_equal(aligned[n][e], g[n][e]), (n, e)
            assert not np.array_equal(split[n][e], g[n][e]), (n, e)
    for n in ("dX", "dg", "dW_r"):
        assert np.array_equal(split[n], g[n]), n


def test_mx_wgrad_worked_example_by_hand():
    # tests/golden/mx_wgrad_worked_example.json: the weight gradients of a two-expert MXFP8
    # layer with MX weight-gradient GEMMs, every rounding worked out by hand there (row blocks
    # of 32 from the expert's first row; Hg = g H and dY as the W_down operands)
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "mx_wgrad_worked_example.json")) as f:
        G = json.load(f)
    s = G["shape"]
    T, d, E, k, I = s["T"], s["d"], s["E"], s["top_k"], s["I"]
    arrays = {"X": np.zeros((T, d)), "dY": np.zeros((T, d)), "W_r": np.zeros((d, E))}
    W = {n: np.zeros((E,) + shp) for n, shp in (("W_gate", (d, I)), ("W_up", (d, I)), ("W_down", (I, d)))}
    for name, entries in G["inputs_nonzero"].items():
        for r, c, v in entries:
            if "[" in name:
                W[name.split("[")[0]][int(name.split("[")[1][:-1])][r, c] = v
            else:
                arrays[name][r, c] = v
    bias = np.array(G["bias"], dtype=np.float32)
    Y, ctx = O.forward_mx(arrays["X"], arrays["W_r"], bias, W["W_gate"], W["W_up"], W["W_down"], k)
    g = O.backward_mx(ctx, arrays["dY"], mx_wgrad=True)
    for name, entries in G["expected"].items():
        n, e = name.split("[")[0], int(name.split("[")[1][:-1])
        want = np.zeros_like(g[n][e])
        for r, c, v in entries:
            want[r, c] = v
        np.testing.assert_allclose(g[n][e], want, rtol=1e-15, atol=0, err_msg=name)


def test_mx_token_path_and_slices_equal_the_full_mx_layer():
    # token_forward_backward_mx is the MX layer on one row; forward_mx / backward_mx over expert
    # slices add up to the full layer; precomputed weight layouts give the same numbers.
    X, W_r, Wg, Wu, Wd, dY = _mx_case(41)
    k, E = _MX_SHAPE["k"], _MX_SHAPE["E"]
    Y, ctx, g = _mx_run(X, W_r, Wg, Wu, Wd, dY)
    cache = {e: O.mx_weight_layouts(Wg[e], Wu[e], Wd[e]) for e in range(E)}
    for t in (0, 17, 95):
        y, dx, dl, ids, gt = O.token_forward_backward_mx(t, X, W_r, None, cache.__getitem__, k, dY)
        np.testing.assert_allclose(y, Y[t], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(dx, g["dX"][t], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(dl, g["dl"][t], rtol=1e-12, atol=1e-14)
    Ys, dXs, dls = np.zeros_like(Y), np.zeros_like(X), np.zeros_like(g["dl"])
    for e in range(E):
        Ye, ce = O.forward_mx(X, W_r, None, Wg, Wu, Wd, k, first_local=e, num_local=1, rounded=cache.__getitem__)
        ge = O.backward_mx(ce, dY)
        Ys += Ye
        dXs += ge["dX"] - ge["dl"] @ W_r.T  # expert parts; the router term once below
        dls += ge["dl"]
        for n in ("dW_gate", "dW_up", "dW_down"):
            np.testing.assert_allclose(ge[n][e], g[n][e], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(Ys, Y, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dls, g["dl"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dXs + dls @ W_r.T, g["dX"], rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("R,Ts,E,k", [(2, (40, 33), 8, 2), (4, (16, 20, 1, 30), 16, 4), (3, (0, 50, 7), 12, 3)])
def test_ep_plan_is_the_single_layer_schedule_of_the_rank_major_batch(R, Ts, E, k):
    # Pull dispatch in source-rank order, each source's tokens ascending, gives every owner the
    # rows the one-GPU schedule of the concatenated (rank-major) batch gives its expert slice;
    # every assignment has exactly one destination row, and the rows are a bijection.
    rng = np.random.default_rng(sum(Ts) + E)
    ids_ranks = [np.array([rng.choice(E, size=k, replace=False) for _ in range(T)], dtype=np.int32).reshape(T, k)
                 for T in Ts]
    plan = O.ep_plan(ids_ranks, E)
    El = E // R
    off = np.concatenate([[0], np.cumsum(Ts)])
    ids_all = np.concatenate(ids_ranks, axis=0)
    for q, own in enumerate(plan["owners"]):
        s = O.schedule(ids_all, E, first_local=q * El, num_local=El)
        assert np.array_equal(own["counts"], s["counts"])
        assert np.array_equal(own["padded_offsets"], s["padded_offsets"])
        glob = [off[src] + t for (src, t, j) in own["rows"]]
        assert np.array_equal(np.array(glob, dtype=np.int64), s["perm"])
        for el in range(El):
            assert own["base"][el, R] == own["counts"][el]
            for src in range(R):
                n = own["base"][el, src + 1] - own["base"][el, src]
                assert n == np.sum(ids_ranks[src] == q * El + el)
    for src in range(R):
        T = Ts[src]
        for t in range(T):
            for j in range(k):
                q, row = plan["dest"][src][t, j]
                assert q == ids_ranks[src][t, j] // El
                sq = O.schedule(ids_all, E, first_local=q * El, num_local=El)
                assert row == sq["slot_row"][off[src] + t, j]
