"""MXFP8 mode on the GPU.

* prepared weights: E4M3 codes and E8M0 scale bytes bit-exact against the
  oracle's MX quantiser (OCP MX rule), for every prepared layout;
* layer: forward + backward within 6e-2 (max |gpu - ref| / max |ref|) of the
  MXFP8 oracle (fp64 with every quantised GEMM operand rounded to MX along its
  contraction dimension); against the unquantised fp64 oracle, within the
  format's own error (MXFP8 oracle vs unquantised oracle, 5-9% at these shapes)
  plus 2e-2; routing table bit-exact (the router stays bf16);
* two runs are bit-identical.
"""
import numpy as np
import pytest
import torch

import oracle as O
from mixture_experts_layer_27_b200 import binding as B

from _util import make_case, relerr, run_oracle, to64

pytestmark = pytest.mark.gpu
TOL_MX = 6e-2


def _pairs(Wg, Wu):
    """[El*2I, d]: per expert, blocks of 64 W_gate columns then the same 64 W_up columns (as rows)."""
    El, d, I = Wg.shape
    rows = []
    for e in range(El):
        for j in range(I // 64):
            rows.append(Wg[e][:, j * 64:(j + 1) * 64].T)
            rows.append(Wu[e][:, j * 64:(j + 1) * 64].T)
    return np.concatenate(rows, axis=0)


def test_prepared_weights_match_the_oracle_quantiser_bit_for_bit():
    T, d, E, k, I = 64, 256, 4, 2, 512
    w, x = make_case(T, d, E, k, I, seed=41)
    lay = B.MoELayerMX(T, d, E, I, k)
    lay.prepare(x["W_gate"], x["W_up"], x["W_down"])
    torch.cuda.synchronize()
    reg = lay.weight_regions()
    Wg, Wu, Wd = to64(x["W_gate"]), to64(x["W_up"]), to64(x["W_down"])
    src = {"Wgu": _pairs(Wg, Wu), "Wd2": Wd.transpose(0, 2, 1).reshape(E * d, I),
           "Wd3": Wd.reshape(E * I, d), "Wg4": Wg.reshape(E * d, I), "Wu4": Wu.reshape(E * d, I)}
    for name, ref in src.items():
        codes, chunks, R, K = reg[name]
        qc, qs = O.mx_quantize(ref, axis=1)
        assert np.array_equal(codes, qc), name
        assert np.array_equal(B.unchunk_scales(chunks, R, K), qs), name


def _check_layer_mx(T, d, E, k, I, bias=None, seed=0):
    w, x = make_case(T, d, E, k, I, seed=seed, bias=bias)
    lay = B.MoELayerMX(T, d, E, I, k)
    lay.prepare(x["W_gate"], x["W_up"], x["W_down"])
    Y = lay.forward(x["X"], x["W_r"], x["bias"])
    g = lay.backward(x["X"], x["W_r"], x["dY"])
    torch.cuda.synchronize()
    assert lay.error() == B.MOE_OK
    r = lay.routing()
    lg = to64(lay.logits())
    ids = O.topk_ids(lg, k)
    assert np.array_equal(r["ids"].cpu().numpy(), ids)
    f64 = {n: (None if x[n] is None else to64(x[n])) for n in ("X", "W_r", "bias", "W_gate", "W_up", "W_down", "dY")}
    Yq, cq = O.forward_mx(f64["X"], f64["W_r"], f64["bias"], f64["W_gate"], f64["W_up"], f64["W_down"], k)
    gq = O.backward_mx(cq, f64["dY"])
    Yo, ctx, go = run_oracle(x, k)

    def errs_vs(Yr, gr):
        return {
            "Y": relerr(to64(Y), Yr),
            "dX": relerr(to64(g["dX"]), gr["dX"]),
            "dW_r": relerr(to64(g["dW_r"]), gr["dW_r"]),
            "dW_gate": relerr(to64(g["dW_gate"]), np.stack([gr["dW_gate"][e] for e in range(E)])),
            "dW_up": relerr(to64(g["dW_up"]), np.stack([gr["dW_up"][e] for e in range(E)])),
            "dW_down": relerr(to64(g["dW_down"]), np.stack([gr["dW_down"][e] for e in range(E)])),
        }

    errs_q = errs_vs(Yq, gq)
    assert all(v <= TOL_MX for v in errs_q.values()), errs_q
    errs_u = errs_vs(Yo, go)
    fmt = {"Y": relerr(Yq, Yo), "dX": relerr(gq["dX"], go["dX"]), "dW_r": relerr(gq["dW_r"], go["dW_r"])}
    for n in ("dW_gate", "dW_up", "dW_down"):
        fmt[n] = relerr(np.stack([gq[n][e] for e in range(E)]), np.stack([go[n][e] for e in range(E)]))
    assert all(errs_u[n] <= fmt[n] + 2e-2 for n in fmt), (errs_u, fmt)
    return lay, x, Y, g


def test_mxfp8_tiny_config():
    _check_layer_mx(128, 256, 8, 2, 512, seed=0)


def test_mxfp8_hot_expert_multi_tile_and_empty_expert():
    bias = np.zeros(4, dtype=np.float32)
    bias[0] = 8.0
    bias[3] = -40.0
    _check_layer_mx(600, 512, 4, 2, 512, bias=bias, seed=42)


def test_mxfp8_many_experts_ragged_tokens():
    _check_layer_mx(333, 768, 48, 6, 768, seed=43)


def test_mxfp8_bit_identical_runs():
    lay, x, Y, g = _check_layer_mx(256, 512, 8, 2, 512, seed=44)
    Y2 = lay.forward(x["X"], x["W_r"], x["bias"])
    g2 = lay.backward(x["X"], x["W_r"], x["dY"])
    torch.cuda.synchronize()
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))
    for n in ("dX", "dW_gate", "dW_up", "dW_down"):
        assert torch.equal(g[n].view(torch.int16), g2[n].view(torch.int16)), n
    assert torch.equal(g["dW_r"].view(torch.int32), g2["dW_r"].view(torch.int32))


def test_mxfp8_results_do_not_depend_on_stale_ctx_and_workspace_contents():
    T, d, E, k, I = 333, 512, 12, 3, 512
    w, x = make_case(T, d, E, k, I, seed=45)
    outs = []
    for fill in (0, 255):
        lay = B.MoELayerMX(T, d, E, I, k)
        lay.ctx.fill_(fill)
        lay.ws.fill_(fill)
        lay.prepare(x["W_gate"], x["W_up"], x["W_down"])
        Y = lay.forward(x["X"], x["W_r"], x["bias"])
        g = lay.backward(x["X"], x["W_r"], x["dY"])
        torch.cuda.synchronize()
        assert lay.error() == B.MOE_OK
        assert torch.isfinite(Y.float()).all()
        outs.append((Y, g))
    (Y0, g0), (Y1, g1) = outs
    assert torch.equal(Y0.view(torch.int16), Y1.view(torch.int16))
    for n in ("dX", "dW_gate", "dW_up", "dW_down"):
        assert torch.equal(g0[n].view(torch.int16), g1[n].view(torch.int16)), n
    assert torch.equal(g0["dW_r"].view(torch.int32), g1["dW_r"].view(torch.int32))


def _run_mx(x, T, d, E, k, I, first=0, num=0):
    El = num or E - first
    lay = B.MoELayerMX(T, d, E, I, k, first_local_expert=first, num_local_experts=num)
    lay.prepare(x["W_gate"][first:first + El].contiguous(), x["W_up"][first:first + El].contiguous(),
                x["W_down"][first:first + El].contiguous())
    Y = lay.forward(x["X"], x["W_r"], x["bias"])
    g = lay.backward(x["X"], x["W_r"], x["dY"])
    torch.cuda.synchronize()
    assert lay.error() == B.MOE_OK
    return Y, g


def test_mxfp8_local_expert_slices():
    # A rank's slice computes its experts exactly as the full layer does (the router is the
    # full router, so routing and every expert's rows are the same); the slices' outputs add
    # up to the full layer's.
    T, d, E, k, I = 200, 256, 16, 4, 256
    w, x = make_case(T, d, E, k, I, seed=46)
    Yf, gf = _run_mx(x, T, d, E, k, I)
    Y0, g0 = _run_mx(x, T, d, E, k, I, first=0, num=7)
    Y1, g1 = _run_mx(x, T, d, E, k, I, first=7, num=9)
    for n in ("dW_gate", "dW_up", "dW_down"):
        assert torch.equal(g0[n].view(torch.int16), gf[n][:7].view(torch.int16)), n
        assert torch.equal(g1[n].view(torch.int16), gf[n][7:].view(torch.int16)), n
    assert relerr(to64(Y0) + to64(Y1), to64(Yf)) <= 1e-2
    assert relerr(to64(g0["dX"]) + to64(g1["dX"]), to64(gf["dX"])) <= 1e-2
    assert relerr(to64(g0["dW_r"]) + to64(g1["dW_r"]), to64(gf["dW_r"])) <= 1e-2


def test_mxfp8_no_tokens():
    T, d, E, k, I = 0, 256, 4, 2, 256
    lay = B.MoELayerMX(T, d, E, I, k)
    W = {n: torch.randn(*s, device="cuda").to(torch.bfloat16) for n, s in
         dict(W_r=(d, E), W_gate=(E, d, I), W_up=(E, d, I), W_down=(E, I, d)).items()}
    lay.prepare(W["W_gate"], W["W_up"], W["W_down"])
    X0 = torch.empty(0, d, device="cuda", dtype=torch.bfloat16)
    lay.forward(X0, W["W_r"], None, Y=torch.empty(0, d, device="cuda", dtype=torch.bfloat16))
    g = lay.backward(X0, W["W_r"], X0,
                     out=dict(dX=torch.empty(0, d, device="cuda", dtype=torch.bfloat16),
                              dW_gate=torch.full((E, d, I), 7.0, device="cuda", dtype=torch.bfloat16),
                              dW_up=torch.full((E, d, I), 7.0, device="cuda", dtype=torch.bfloat16),
                              dW_down=torch.full((E, I, d), 7.0, device="cuda", dtype=torch.bfloat16),
                              dW_r=torch.full((d, E), 7.0, device="cuda")))
    torch.cuda.synchronize()
    assert lay.error() == B.MOE_OK
    for n in ("dW_gate", "dW_up", "dW_down", "dW_r"):
        assert torch.count_nonzero(g[n]) == 0, n
