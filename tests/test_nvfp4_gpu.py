"""NVFP4 layer forward and backward on the GPU, against the NVFP4 oracle (oracle/nvfp4.py).

* global scales: the three weight scales and X's equal the oracle's bit for bit (both
  compute 2688 / amax in fp32 on the same bf16 values);
* prepared weights and the dispatched X: E2M1 codes and E4M3 scale bytes bit-exact against
  the oracle's quantiser, in every prepared layout and every padded row (pad rows zero);
* H: the device's H codes equal the oracle's quantiser applied to the device's own fp32 H
  under the device's H scale, which equals the oracle's scale of that H;
* Y within 2e-2 (max |gpu - ref| / max |ref|) of forward_nv: both sides take the same
  quantisation decisions except where the fp32 accumulation order moves an H value across
  a rounding boundary, so the bf16 tolerance holds; against the exact fp64 layer the error
  is the format's own (reported, bounded loosely);
* two runs are bit-identical; an expert slice, a hot expert spanning tiles, an empty
  expert and T = 0 run;
* backward: the backward's weight layouts and the dispatched dY bit-exact against the oracle
  quantiser, dY's scale bit for bit, [dA | dB]'s within 1e-5 (fp32 against fp64 values), dX,
  dW_r and the (bf16-operand) expert weight gradients within 2e-2 of backward_nv.
"""
import numpy as np
import pytest
import torch

import oracle as O
import oracle.nvfp4 as N
from mixture_experts_layer_27_b200 import binding as B

from _util import TOL_BF16, make_case, relerr, to64

pytestmark = pytest.mark.gpu


def _gate_up_rows(Wg_codes, Wu_codes):
    """Rows of the prepared gate/up operand for one expert: blocks of 64 gate columns, then the
    same 64 up columns (each column one row, K = d)."""
    I = Wg_codes.shape[1]
    rows = []
    for j in range(I // 64):
        rows.append(Wg_codes[:, j * 64:(j + 1) * 64].T)
        rows.append(Wu_codes[:, j * 64:(j + 1) * 64].T)
    return np.concatenate(rows, axis=0)


def test_nvfp4_prepared_weights_only():
    # the weight quantiser alone (no forward), so a failure here is the quantiser's
    T, d, E, k, I = 64, 256, 4, 2, 512
    w, x = make_case(T, d, E, k, I, seed=41)
    lay = B.MoELayerNVFP4(T, d, E, I, k)
    lay.prepare(x["W_gate"], x["W_up"], x["W_down"])
    torch.cuda.synchronize()
    Wg64, Wu64, Wd64 = to64(x["W_gate"]), to64(x["W_up"]), to64(x["W_down"])
    gsw = N.nv_weight_scales(Wg64, Wu64, Wd64)
    assert [np.float32(v) for v in lay.scales()[1]] == list(gsw) + [N.nv_weight_scales_bwd(Wg64, Wu64, Wd64)[0]]
    reg = lay.weight_regions()
    cg, sg = zip(*[N.nv_quantize(Wg64[e], gsw[0], axis=0) for e in range(E)])
    cu, su = zip(*[N.nv_quantize(Wu64[e], gsw[1], axis=0) for e in range(E)])
    cd, sd = zip(*[N.nv_quantize(Wd64[e], gsw[2], axis=0) for e in range(E)])
    assert np.array_equal(reg["Wgu"][0], np.concatenate([_gate_up_rows(cg[e], cu[e]) for e in range(E)]))
    assert np.array_equal(reg["Wgu"][1], np.concatenate([_gate_up_rows(sg[e], su[e]) for e in range(E)]))
    assert np.array_equal(reg["Wd2"][0], np.concatenate([c.T for c in cd]))
    assert np.array_equal(reg["Wd2"][1], np.concatenate([c.T for c in sd]))


def _run(T, d, E, k, I, seed=0, bias=None, first=0, num=0):
    w, x = make_case(T, d, E, k, I, seed=seed, bias=bias)
    El = num or (E - first)
    lay = B.MoELayerNVFP4(T, d, E, I, k, first_local_expert=first, num_local_experts=num)
    Wg = x["W_gate"][first:first + El].contiguous()
    Wu = x["W_up"][first:first + El].contiguous()
    Wd = x["W_down"][first:first + El].contiguous()
    lay.prepare(Wg, Wu, Wd)
    Y = lay.forward(x["X"], x["W_r"], x["bias"])
    torch.cuda.synchronize()
    assert lay.error() == B.MOE_OK
    return lay, x, Y, (Wg, Wu, Wd)


def _check(T, d, E, k, I, seed=0, bias=None, first=0, num=0):
    lay, x, Y, (Wg, Wu, Wd) = _run(T, d, E, k, I, seed, bias, first, num)
    El = lay.El
    f = {n: (None if x[n] is None else to64(x[n])) for n in ("X", "W_r", "bias")}
    Wg64, Wu64, Wd64 = to64(Wg), to64(Wu), to64(Wd)

    # global scales, bit for bit
    (gsx, gsh), gsw = lay.scales()
    want_w = N.nv_weight_scales(Wg64, Wu64, Wd64)
    assert [np.float32(v) for v in gsw[:3]] == list(want_w)
    assert np.float32(gsx) == N.nv_global_scale(f["X"])

    # prepared weights, bit for bit
    reg = lay.weight_regions()
    gu_c, gu_s, d2_c, d2_s = [], [], [], []
    for e in range(El):
        cg, sg = N.nv_quantize(Wg64[e], want_w[0], axis=0)  # [d, I], [d/16, I]
        cu, su = N.nv_quantize(Wu64[e], want_w[1], axis=0)
        cd, sd = N.nv_quantize(Wd64[e], want_w[2], axis=0)  # [I, d], [I/16, d]
        gu_c.append(_gate_up_rows(cg, cu))
        gu_s.append(_gate_up_rows(sg, su))
        d2_c.append(cd.T)
        d2_s.append(sd.T)
    assert np.array_equal(reg["Wgu"][0], np.concatenate(gu_c)), "Wgu codes"
    assert np.array_equal(reg["Wgu"][1], np.concatenate(gu_s)), "Wgu scales"
    assert np.array_equal(reg["Wd2"][0], np.concatenate(d2_c)), "Wd2 codes"
    assert np.array_equal(reg["Wd2"][1], np.concatenate(d2_s)), "Wd2 scales"

    # dispatched X, bit for bit, row by row (pad rows up to the next multiple of 16: zero)
    r = lay.routing()
    counts = r["counts"].cpu().numpy()
    offs = r["offsets"].cpu().numpy()
    poff = r["padded_offsets"].cpu().numpy()
    perm = r["perm"].cpu().numpy()
    xc, xs = lay.x_operand()
    cx, sx = N.nv_quantize(f["X"], gsx, axis=1)
    live = []
    for e in range(El):
        toks = perm[offs[e]:offs[e + 1]]
        rows = poff[e] + np.arange(counts[e])
        assert np.array_equal(xc[rows], cx[toks]) and np.array_equal(xs[rows], sx[toks]), e
        pad = poff[e] + np.arange(counts[e], (counts[e] + 15) // 16 * 16)
        assert not xc[pad].any() and not xs[pad].any(), e
        live.append(rows)
    live = np.concatenate(live) if live else np.zeros(0, dtype=np.int64)

    # H: the device's codes are the oracle's quantiser on the device's fp32 H and scale
    if live.size:
        H = lay.h_fp32()[live].astype(np.float64)  # live rows only: dead pad rows hold stale bytes
        assert np.float32(gsh) == N.nv_global_scale(H)
        hc, hs = lay.h_operand()
        qc, qs = N.nv_quantize(H, gsh, axis=1)
        assert np.array_equal(hc[live], qc) and np.array_equal(hs[live], qs)

    # Y against the NVFP4 oracle
    Yq, info = N.forward_nv(f["X"], f["W_r"], f["bias"], to64(x["W_gate"]), to64(x["W_up"]), to64(x["W_down"]),
                            k, first_local=first, num_local=El, gs_w=want_w)
    assert np.array_equal(r["ids"].cpu().numpy(), info["ids"])
    err = relerr(to64(Y), Yq)
    assert err <= TOL_BF16, err
    Yo, _ = O.forward(f["X"], f["W_r"], f["bias"], to64(x["W_gate"]), to64(x["W_up"]), to64(x["W_down"]), k,
                      first_local=first, num_local=El)
    assert relerr(to64(Y), Yo) < 0.5
    return lay, x, Y


def test_nvfp4_tiny_config():
    _check(128, 256, 8, 2, 512, seed=0)


def test_nvfp4_hot_expert_multi_tile_and_empty_expert():
    bias = np.zeros(4, dtype=np.float32)
    bias[0] = 8.0
    bias[3] = -40.0
    _check(600, 512, 4, 2, 512, bias=bias, seed=42)


def test_nvfp4_expert_slice_ragged_tokens():
    _check(328, 768, 8, 3, 512, seed=7, first=2, num=4)


def test_nvfp4_runs_are_bit_identical():
    lay, x, Y = _check(256, 512, 8, 2, 768, seed=3)
    Y2 = lay.forward(x["X"], x["W_r"], x["bias"])
    torch.cuda.synchronize()
    assert torch.equal(Y, Y2)


def test_nvfp4_empty_batch():
    lay = B.MoELayerNVFP4(0, 256, 4, 512, 2)
    w, x = make_case(8, 256, 4, 2, 512, seed=1)
    lay.prepare(x["W_gate"], x["W_up"], x["W_down"])
    Y = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    B.check(B.moe_fwd_nvfp4(lay.shape, x["X"][:0], x["W_r"], x["bias"], lay.wq, Y, lay.ctx, lay.ws), "empty")
    torch.cuda.synchronize()
    assert lay.error() == B.MOE_OK


def test_nvfp4_full_size_ep64_slice():
    # The EP64 per-rank slice at full size, as the bench runs it (epnv_n2368: 32768 tokens routed
    # top-8 over 384 experts, 6 local experts with 2368 rows each, one batch): every token's Y
    # (but the few near-tie tokens, whose fp64 routing differs) against the NVFP4 oracle's full
    # forward, routing bit-exact on the GPU's logits, the global scales; then the backward.
    from mixture_experts_layer_27_b200 import inputs as IN
    w = IN.WORKLOADS["epnv_n2368"]
    x = IN.make_inputs(w, device="cuda")
    El = w.El
    lay = B.MoELayerNVFP4(w.T, w.d, w.E, w.I, w.k, w.first_local, w.num_local)
    Wg, Wu, Wd = (x[n][:El].contiguous() for n in ("W_gate", "W_up", "W_down"))
    lay.prepare(Wg, Wu, Wd)
    Y = lay.forward(x["X"], x["W_r"], x["bias"])
    torch.cuda.synchronize()
    assert lay.error() == B.MOE_OK
    f = {n: to64(x[n]) for n in ("X", "W_r", "bias")}
    W64 = [to64(t) for t in (Wg, Wu, Wd)]
    gs_w = N.nv_weight_scales(*W64)
    assert [np.float32(v) for v in lay.scales()[1][:3]] == list(gs_w)
    Yq, info = N.forward_nv(f["X"], f["W_r"], f["bias"], W64[0], W64[1], W64[2], w.k, first_local=0,
                            num_local=El, gs_w=gs_w)
    r = lay.routing()
    gids = r["ids"].cpu().numpy()
    # routing bit-exact on the GPU's fp32 logits; against the fp64 logits the ids may differ only
    # at near-ties (fp32 vs fp64 logits of 7168-term dot products), and those tokens are left out
    lg = to64(lay.logits())
    assert np.array_equal(gids, O.topk_ids(lg, w.k))
    lg64 = O.router_logits(f["X"], f["W_r"], f["bias"])
    # selection differences (the order inside a token's top k only orders the combine's sum)
    differ = np.nonzero(np.any(np.sort(gids, 1) != np.sort(info["ids"], 1), axis=1))[0]
    srt = -np.sort(-lg64[differ], axis=1)
    assert np.all(srt[:, w.k - 1] - srt[:, w.k] < 1e-3), differ
    keep = np.setdiff1d(np.arange(w.T), differ)
    assert differ.size < 64
    # H's scale: the device's H (fp32 accumulation) and the oracle's (fp64) share their amax to ~1e-6
    assert abs(float(lay.scales()[0][1]) / float(info["gs_h"]) - 1.0) < 1e-5
    err = relerr(to64(Y)[keep], Yq[keep])
    assert err <= TOL_BF16, err
    # the backward at full size: dX off the near-tie tokens, dW_r and the local experts' weight
    # gradients against backward_nv
    g = lay.backward(x["X"], x["W_r"], x["dY"])
    torch.cuda.synchronize()
    assert lay.error() == B.MOE_OK
    dY64 = to64(x["dY"])
    go = N.backward_nv(info, f["X"], f["W_r"], W64[0], W64[1], W64[2], dY64)
    assert np.float32(lay.bwd_scales()[0]) == go["gs_dy"]
    errs = {"dX": relerr(to64(g["dX"])[keep], go["dX"][keep]), "dW_r": relerr(to64(g["dW_r"]), go["dW_r"])}
    for n in ("dW_gate", "dW_up", "dW_down"):
        errs[n] = relerr(to64(g[n]), np.stack([go[n][e] for e in range(El)]))
    assert all(v <= TOL_BF16 for v in errs.values()), errs


def test_nvfp4_backward_weights_only():
    T, d, E, k, I = 64, 256, 4, 2, 512
    w, x = make_case(T, d, E, k, I, seed=43)
    lay = B.MoELayerNVFP4(T, d, E, I, k)
    lay.prepare(x["W_gate"], x["W_up"], x["W_down"])
    torch.cuda.synchronize()
    Wg64, Wu64, Wd64 = to64(x["W_gate"]), to64(x["W_up"]), to64(x["W_down"])
    gs_gu, gs_d = N.nv_weight_scales_bwd(Wg64, Wu64, Wd64)
    reg = lay.bwd_weight_regions()
    for name, W, gs in (("Wd3", Wd64, gs_d), ("Wg4", Wg64, gs_gu), ("Wu4", Wu64, gs_gu)):
        c, sc = zip(*[N.nv_quantize(W[e], gs, axis=1) for e in range(E)])
        assert np.array_equal(reg[name][0], np.concatenate(c)), name
        assert np.array_equal(reg[name][1], np.concatenate(sc)), name


def _check_bwd(T, d, E, k, I, seed=0, bias=None, first=0, num=0):
    lay, x, Y, (Wg, Wu, Wd) = _run(T, d, E, k, I, seed, bias, first, num)
    El = lay.El
    g = lay.backward(x["X"], x["W_r"], x["dY"])
    torch.cuda.synchronize()
    assert lay.error() == B.MOE_OK
    f = {n: (None if x[n] is None else to64(x[n])) for n in ("X", "W_r", "bias", "dY")}
    W64 = [to64(t) for t in (x["W_gate"], x["W_up"], x["W_down"])]
    _, info = N.forward_nv(f["X"], f["W_r"], f["bias"], *W64, k, first_local=first, num_local=El)
    go = N.backward_nv(info, f["X"], f["W_r"], *W64, f["dY"])
    gs_dy, gs_ab = lay.bwd_scales()
    assert np.float32(gs_dy) == go["gs_dy"]
    assert abs(float(gs_ab) / float(go["gs_ab"]) - 1.0) < 1e-5
    # dispatched dY codes, bit for bit
    r = lay.routing()
    counts, offs = r["counts"].cpu().numpy(), r["offsets"].cpu().numpy()
    poff, perm = r["padded_offsets"].cpu().numpy(), r["perm"].cpu().numpy()
    yc, ys = lay.dy_operand()
    cy, sy = N.nv_quantize(f["dY"], gs_dy, axis=1)
    for e in range(El):
        rows = poff[e] + np.arange(counts[e])
        toks = perm[offs[e]:offs[e + 1]]
        assert np.array_equal(yc[rows], cy[toks]) and np.array_equal(ys[rows], sy[toks]), e
    errs = {"dX": relerr(to64(g["dX"]), go["dX"]), "dW_r": relerr(to64(g["dW_r"]), go["dW_r"])}
    for n in ("dW_gate", "dW_up", "dW_down"):
        errs[n] = relerr(to64(g[n]), np.stack([go[n][e + first] for e in range(El)]))
    assert all(v <= TOL_BF16 for v in errs.values()), errs
    g2 = lay.backward(x["X"], x["W_r"], x["dY"])
    torch.cuda.synchronize()
    for n in ("dX", "dW_gate", "dW_up", "dW_down", "dW_r"):
        assert torch.equal(g[n], g2[n]), n
    return errs


def test_nvfp4_backward_tiny_config():
    _check_bwd(128, 256, 8, 2, 512, seed=0)


def test_nvfp4_backward_hot_expert_and_empty_expert():
    bias = np.zeros(4, dtype=np.float32)
    bias[0] = 8.0
    bias[3] = -40.0
    _check_bwd(600, 512, 4, 2, 512, bias=bias, seed=42)


def test_nvfp4_backward_expert_slice_ragged_tokens():
    _check_bwd(328, 768, 8, 3, 512, seed=7, first=2, num=4)


def test_nvfp4_backward_empty_batch():
    lay = B.MoELayerNVFP4(0, 256, 4, 512, 2)
    w, x = make_case(8, 256, 4, 2, 512, seed=1)
    lay.prepare(x["W_gate"], x["W_up"], x["W_down"])
    g = {n: torch.full_like(x[n], 1.0) for n in ("W_gate", "W_up", "W_down")}
    dWr = torch.ones(256, 4, dtype=torch.float32, device="cuda")
    dX = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    B.check(B.moe_bwd_nvfp4(lay.shape, x["X"][:0], x["W_r"], lay.wq, x["dY"][:0], lay.ctx, dX, g["W_gate"], g["W_up"],
                            g["W_down"], dWr, lay.ws), "empty")
    torch.cuda.synchronize()
    assert not dWr.any() and all(not t.any() for t in g.values())


def test_nvfp4_step_replays_from_a_cuda_graph():
    # the layer only enqueues work (no host sync, no allocation): one fwd+bwd step captured as a
    # CUDA graph and replayed gives the direct launches' results bit for bit
    lay, x, Y, _ = _run(256, 512, 8, 2, 512, seed=5)
    g = lay.backward(x["X"], x["W_r"], x["dY"])
    torch.cuda.synchronize()
    ref = {"Y": Y.clone(), **{n: t.clone() for n, t in g.items()}}
    Y2 = torch.empty_like(Y)
    g2 = {n: torch.empty_like(t) for n, t in g.items()}
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm the capture stream
        lay.forward(x["X"], x["W_r"], x["bias"], Y=Y2)
        lay.backward(x["X"], x["W_r"], x["dY"], out=g2)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        lay.forward(x["X"], x["W_r"], x["bias"], Y=Y2)
        lay.backward(x["X"], x["W_r"], x["dY"], out=g2)
    Y2.zero_()
    for t in g2.values():
        t.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert lay.error() == B.MOE_OK
    assert torch.equal(Y2, ref["Y"])
    for n in g2:
        assert torch.equal(g2[n], ref[n]), n
