"""MXFP8 weight gradients on the GPU (MOE_MXFP8_ALL).

The two weight-gradient GEMMs run on MXFP8 tensor cores, their operands (X, dA, dB,
Hg = g H, dY of each expert) quantised along the expert's rows in blocks of 32 rows:

* the quantised X_perm and dY_perm operands (codes and scale bytes) are bit-exact against
  the oracle's MX quantiser applied along the rows of each expert's bf16 rows;
* the expert weight gradients are within 6e-2 of the MXFP8 oracle with MX weight
  gradients (`backward_mx(..., mx_wgrad=True)`), in bf16 and in fp32;
* the GEMMs themselves: each expert's gradient equals the product of the dequantised operands
  the device quantised (fp64 matmul here) within the fp32-sum and bf16-output rounding, so the
  tile walk, the ragged last K block and the scale placement are checked apart from the
  quantisation;
* Y, dX and dW_r are the plain MXFP8 mode's bits (only the weight-gradient GEMMs differ);
* results do not depend on what ctx and the workspace held, and reruns are bit-identical.
"""
import numpy as np
import pytest
import torch

import oracle as O
from mixture_experts_layer_27_b200 import binding as B

from _util import make_case, relerr, to64

pytestmark = pytest.mark.gpu
TOL_MX = 6e-2


def _step(lay, x, first, El, poison=None):
    if poison is not None:
        lay.ctx.fill_(poison)
        lay.ws.fill_(poison)
    W = [x[n][first:first + El].contiguous() for n in ("W_gate", "W_up", "W_down")]
    lay.prepare(*W)
    Y = lay.forward(x["X"], x["W_r"], x["bias"])
    g = lay.backward(x["X"], x["W_r"], x["dY"])
    torch.cuda.synchronize()
    assert lay.error() == B.MOE_OK
    return Y, g


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


def _check(T, d, E, k, I, seed, bias=None, first=0, num=0, wgrad_dtype=None):
    w, x = make_case(T, d, E, k, I, seed=seed, bias=bias)
    El = num or (E - first)
    plain = B.MoELayerMX(T, d, E, I, k, first_local_expert=first, num_local_experts=num, wgrad_dtype=wgrad_dtype)
    full = B.MoELayerMX(T, d, E, I, k, first_local_expert=first, num_local_experts=num, wgrad_dtype=wgrad_dtype,
                        mx_wgrad=True)
    Y0, g0 = _step(plain, x, first, El)
    Y1, g1 = _step(full, x, first, El, poison=0xFF)
    # only the weight-gradient GEMMs differ between the two modes
    assert torch.equal(_bits(Y1), _bits(Y0))
    for n in ("dX", "dW_r"):
        assert torch.equal(_bits(g1[n]), _bits(g0[n])), n
    _check_gemm_consistency(full, g1, El)
    # the weight gradients against the MX oracle with MX weight gradients
    f64 = {n: (None if x[n] is None else to64(x[n])) for n in ("X", "W_r", "bias", "W_gate", "W_up", "W_down", "dY")}
    Yq, cq = O.forward_mx(f64["X"], f64["W_r"], f64["bias"], f64["W_gate"], f64["W_up"], f64["W_down"], k,
                          first_local=first, num_local=num or None)
    gq = O.backward_mx(cq, f64["dY"], mx_wgrad=True)
    errs = {}
    for n in ("dW_gate", "dW_up", "dW_down"):
        want = np.stack([gq[n][e] for e in range(first, first + El)])
        errs[n] = relerr(to64(g1[n]), want)
    assert all(v <= TOL_MX for v in errs.values()), errs
    # a second run over the same buffers: the same bits
    Y2, g2 = _step(full, x, first, El)
    assert torch.equal(_bits(Y2), _bits(Y1))
    for n in g1:
        assert torch.equal(_bits(g2[n]), _bits(g1[n])), n
    return full, x, g1


def _operand_values(lay, which):
    codes, scales = lay.wgrad_operand(which)
    return O.mx_dequantize(codes, scales, axis=1)  # [C, RP]


def _check_gemm_consistency(lay, g, El):
    r = lay.routing()
    cnt = r["counts"].cpu().numpy()
    poff = r["padded_offsets"].cpu().numpy()
    Xv, dYv, dAv, dBv, Hgv = (_operand_values(lay, i) for i in range(5))
    got = {n: to64(g[n]) for n in ("dW_gate", "dW_up", "dW_down")}
    want = {n: np.zeros_like(got[n]) for n in got}
    for e in range(El):
        n = int(cnt[e])
        if n == 0:
            continue
        rows = slice(int(poff[e]), int(poff[e]) + n)
        want["dW_gate"][e] = Xv[:, rows] @ dAv[:, rows].T
        want["dW_up"][e] = Xv[:, rows] @ dBv[:, rows].T
        want["dW_down"][e] = Hgv[:, rows] @ dYv[:, rows].T
    errs = {n: relerr(got[n], want[n]) for n in got}
    assert all(v <= 8e-3 for v in errs.values()), errs


def _check_operands_exact(lay, x, first, El):
    """X_perm and dY_perm as quantised along the rows: bit-exact vs the oracle quantiser."""
    r = lay.routing()
    cnt = r["counts"].cpu().numpy()
    off = r["offsets"].cpu().numpy()
    poff = r["padded_offsets"].cpu().numpy()
    perm = r["perm"].cpu().numpy()
    for which, src in ((0, x["X"]), (1, x["dY"])):
        codes, sc = lay.wgrad_operand(which)  # [C, RP], [C, RP / 32]
        C = codes.shape[0]
        s64 = to64(src)
        for e in range(El):
            n = int(cnt[e])
            if n == 0:
                continue
            rows = s64[perm[off[e]:off[e] + n]]
            n32 = (n + 31) // 32 * 32
            rows = np.concatenate([rows, np.zeros((n32 - n, C))], axis=0)
            qc, qs = O.mx_quantize(rows, axis=0)
            p0 = int(poff[e])
            assert np.array_equal(codes[:, p0:p0 + n32], qc.T), (which, e)
            assert np.array_equal(sc[:, p0 // 32:(p0 + n32) // 32], qs.T), (which, e)


def test_mx_wgrad_tiny_and_operands_bit_exact():
    lay, x, _ = _check(128, 256, 8, 2, 512, seed=61)
    _check_operands_exact(lay, x, 0, 8)


def test_mx_wgrad_hot_expert_ragged_rows_and_empty_expert():
    # a hot expert with several 128-row K blocks and a ragged last block, an expert with none
    bias = np.zeros(6, dtype=np.float32)
    bias[0] = 8.0
    bias[4] = -40.0
    lay, x, g = _check(600, 512, 6, 2, 512, seed=62, bias=bias)
    _check_operands_exact(lay, x, 0, 6)
    for n in ("dW_gate", "dW_up", "dW_down"):
        assert not torch.any(g[n][4]), n  # no rows: a zero gradient


def test_mx_wgrad_many_experts_few_rows_each():
    # rows per expert from a handful to a few dozen: last blocks of 1 .. 4 K = 32 steps
    lay, x, _ = _check(333, 768, 48, 6, 768, seed=63)
    _check_operands_exact(lay, x, 0, 48)


def test_mx_wgrad_expert_slice():
    lay, x, _ = _check(400, 512, 16, 4, 512, seed=64, first=5, num=6)
    _check_operands_exact(lay, x, 5, 6)


def test_mx_wgrad_fp32_gradients_round_to_the_bf16_mode():
    # fp32 weight gradients are the same sums unrounded: bf16 of them is the bf16 mode's dW
    _, x, g32 = _check(300, 512, 8, 2, 512, seed=65, wgrad_dtype=torch.float32)
    lay16 = B.MoELayerMX(300, 512, 8, 512, 2, mx_wgrad=True)
    _, g16 = _step(lay16, x, 0, 8)
    for n in ("dW_gate", "dW_up", "dW_down"):
        assert g32[n].dtype == torch.float32
        assert torch.equal(_bits(g32[n].to(torch.bfloat16)), _bits(g16[n])), n
