"""The ring-streamed layer in MXFP8 (moe_fwd_stream_mx / moe_bwd_stream_mx) on the GPU.

With MXFP8 weight gradients (MOE_MXFP8_ALL) the stream quantises each (macrobatch, expert)
segment along its rows on its own, so its weight gradients are checked against the MX oracle
with the device plan's segments as row groups (`backward_mx(..., row_groups=...)`).

The stream changes where rows live and when each macrobatch runs, not the arithmetic of a row:
every GEMM output row, its quantisation along d or I, the combine and the reverse dispatch are
row-local, so Y, dX and dW_r must equal the one-batch MXFP8 layer's over the same M*T tokens bit
for bit.  The weight gradients contract over rows in chunks with an fp32 accumulator, so they
differ from the one-batch layer's by fp32 summation order only (checked at 1e-2), and they are
checked against the MXFP8 oracle at 6e-2.  Small rings force replay and several backward
chunks; a large ring keeps everything resident; a local expert slice; reruns are bit-identical.
"""
import numpy as np
import pytest
import torch

import oracle as O
from mixture_experts_layer_27_b200 import binding as B

from _util import make_case, relerr, to64

pytestmark = pytest.mark.gpu
TOL_MX = 6e-2


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


def _one_batch(x, T, d, E, I, k, first, num, El):
    lay = B.MoELayerMX(T, d, E, I, k, first_local_expert=first, num_local_experts=num)
    lay.prepare(*(x[n][first:first + El].contiguous() for n in ("W_gate", "W_up", "W_down")))
    Y = lay.forward(x["X"], x["W_r"], x["bias"])
    g = lay.backward(x["X"], x["W_r"], x["dY"])
    torch.cuda.synchronize()
    assert lay.error() == B.MOE_OK
    return Y, g


@pytest.mark.parametrize("T_mb,M,d,E,k,I,first,num,ring_mult,seed", [
    (128, 8, 256, 16, 4, 256, 0, 0, 1.0, 71),    # smallest legal ring: replay, several chunks
    (128, 8, 256, 16, 4, 256, 0, 0, 100.0, 72),  # everything stays resident
    (64, 10, 512, 24, 6, 512, 3, 6, 1.5, 73),    # a local expert slice (6 of 24)
])
def test_mx_streamed_layer(T_mb, M, d, E, k, I, first, num, ring_mult, seed):
    T = T_mb * M
    w, x = make_case(T, d, E, k, I, seed=seed)
    El = num or E - first
    shape = B.make_shape(T_mb, d, E, I, k, prec=B.MOE_MXFP8, first_local_expert=first, num_local_experts=num)
    ring_bytes = int(B.moe_stream_min_ring_bytes(shape) * ring_mult)  # bf16 rows, their codes and scales
    s = B.MoEStreamMX(T_mb, d, E, I, k, M, ring_bytes, first, num)
    s.ctx.fill_(0xFF)  # NaN patterns wherever the step reads before it writes
    s.ws.fill_(0xFF)
    s.ring.fill_(0xFF)
    s.prepare(*(x[n][first:first + El].contiguous() for n in ("W_gate", "W_up", "W_down")))

    def run():
        Y = s.forward(x["X"], x["W_r"], x["bias"])
        g = s.backward(x["X"], x["W_r"], x["dY"])
        torch.cuda.synchronize()
        assert s.error() == B.MOE_OK
        return Y, g

    Y, g = run()
    Y1, g1 = _one_batch(x, T, d, E, I, k, first, num, El)
    assert torch.equal(_bits(Y), _bits(Y1))
    for n in ("dX", "dW_r"):
        assert torch.equal(_bits(g[n]), _bits(g1[n])), n
    for n in ("dW_gate", "dW_up", "dW_down"):
        assert relerr(to64(g[n]), to64(g1[n])) <= 1e-2, n
    # against the MXFP8 oracle (bf16 weight gradients)
    f64 = {n: (None if x[n] is None else to64(x[n])) for n in ("X", "W_r", "bias", "W_gate", "W_up", "W_down", "dY")}
    Yq, cq = O.forward_mx(f64["X"], f64["W_r"], f64["bias"], f64["W_gate"], f64["W_up"], f64["W_down"], k,
                          first_local=first, num_local=num or None)
    gq = O.backward_mx(cq, f64["dY"])
    errs = {"Y": relerr(to64(Y), Yq), "dX": relerr(to64(g["dX"]), gq["dX"])}
    for n in ("dW_gate", "dW_up", "dW_down"):
        errs[n] = relerr(to64(g[n]), np.stack([gq[n][first + e] for e in range(El)]))
    assert all(v <= TOL_MX for v in errs.values()), errs
    plan = s.plan()["plan"]
    if ring_mult == 1.0:
        assert plan[1] > 1  # several backward chunks: the ring was overwritten and replayed
    # a second run over the same buffers: the same bits
    Y2, g2 = run()
    assert torch.equal(_bits(Y2), _bits(Y))
    for n in g:
        assert torch.equal(_bits(g2[n]), _bits(g[n])), n


def _plan_row_groups(plan, counts, El):
    """Rows of local expert el in each macrobatch of the device plan (cum = rows before)."""
    nm = int(plan["plan"][0])
    cum = plan["cum"]

    def groups(el):
        out = []
        for m in range(nm):
            hi = int(cum[(m + 1) * El + el]) if m + 1 < nm else int(counts[el])
            out.append(hi - int(cum[m * El + el]))
        return out
    return groups


@pytest.mark.parametrize("T_mb,M,d,E,k,I,first,num,ring_mult,seed", [
    (128, 8, 256, 16, 4, 256, 0, 0, 1.0, 75),    # smallest ring: several macrobatches
    (64, 10, 512, 24, 6, 512, 3, 6, 1.5, 76),    # a local expert slice (6 of 24)
])
def test_mx_streamed_layer_with_mx_weight_gradients(T_mb, M, d, E, k, I, first, num, ring_mult, seed):
    T = T_mb * M
    w, x = make_case(T, d, E, k, I, seed=seed)
    El = num or E - first
    shape = B.make_shape(T_mb, d, E, I, k, prec=B.MOE_MXFP8_ALL, first_local_expert=first, num_local_experts=num)
    ring_bytes = int(B.moe_stream_min_ring_bytes(shape) * ring_mult)
    s = B.MoEStreamMX(T_mb, d, E, I, k, M, ring_bytes, first, num, mx_wgrad=True)
    s.ctx.fill_(0xFF)
    s.ws.fill_(0xFF)
    s.ring.fill_(0xFF)
    s.prepare(*(x[n][first:first + El].contiguous() for n in ("W_gate", "W_up", "W_down")))

    def run():
        Y = s.forward(x["X"], x["W_r"], x["bias"])
        g = s.backward(x["X"], x["W_r"], x["dY"])
        torch.cuda.synchronize()
        assert s.error() == B.MOE_OK
        return Y, g

    Y, g = run()
    plan = s.plan()
    if ring_mult == 1.0:
        assert int(plan["plan"][0]) > 1  # several macrobatches: the experts' rows come in segments
    # Y, dX, dW_r: the one-batch MXFP8 layer's bits (only the weight gradients see the segments)
    Y1, g1 = _one_batch(x, T, d, E, I, k, first, num, El)
    assert torch.equal(_bits(Y), _bits(Y1))
    for n in ("dX", "dW_r"):
        assert torch.equal(_bits(g[n]), _bits(g1[n])), n
    f64 = {n: (None if x[n] is None else to64(x[n])) for n in ("X", "W_r", "bias", "W_gate", "W_up", "W_down", "dY")}
    Yq, cq = O.forward_mx(f64["X"], f64["W_r"], f64["bias"], f64["W_gate"], f64["W_up"], f64["W_down"], k,
                          first_local=first, num_local=num or None)
    groups = _plan_row_groups(plan, cq["sched"]["counts"], El)
    gq = O.backward_mx(cq, f64["dY"], mx_wgrad=True, row_groups=groups)
    errs = {n: relerr(to64(g[n]), np.stack([gq[n][first + e] for e in range(El)]))
            for n in ("dW_gate", "dW_up", "dW_down")}
    assert all(v <= TOL_MX for v in errs.values()), errs
    Y2, g2 = run()
    assert torch.equal(_bits(Y2), _bits(Y))
    for n in g:
        assert torch.equal(_bits(g2[n]), _bits(g[n])), n


def test_mx_stream_fp32_weight_gradients_round_to_the_bf16_mode():
    # fp32 weight gradients are the same sums unrounded: bf16 of them is the bf16 mode's dW
    T_mb, M, d, E, k, I = 128, 6, 256, 16, 4, 256
    w, x = make_case(T_mb * M, d, E, k, I, seed=74)
    shape = B.make_shape(T_mb, d, E, I, k, prec=B.MOE_MXFP8)
    ring_bytes = B.moe_stream_min_ring_bytes(shape)  # the smallest ring: replay and several chunks
    out = []
    for wdt in (torch.bfloat16, torch.float32):
        s = B.MoEStreamMX(T_mb, d, E, I, k, M, ring_bytes, wgrad_dtype=wdt)
        s.prepare(x["W_gate"], x["W_up"], x["W_down"])
        s.forward(x["X"], x["W_r"], x["bias"])
        g = s.backward(x["X"], x["W_r"], x["dY"])
        torch.cuda.synchronize()
        assert s.error() == B.MOE_OK
        out.append(g)
    for n in ("dW_gate", "dW_up", "dW_down"):
        assert out[1][n].dtype == torch.float32
        assert torch.equal(_bits(out[1][n].to(torch.bfloat16)), _bits(out[0][n])), n
    assert torch.equal(_bits(out[1]["dX"]), _bits(out[0]["dX"]))
