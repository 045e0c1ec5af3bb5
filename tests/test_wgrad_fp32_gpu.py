"""fp32 expert weight gradients (moe_shape.wgrad_dtype = MOE_WGRAD_FP32) on the GPU.

The option writes the fp32 sums that the bf16 mode rounds to nearest even, so
for each backward entry point (moe_bwd, moe_bwd_mx, and moe_bwd_stream with
one backward chunk and with several):
* bf16(fp32 dW) equals the bf16 mode's dW bit for bit;
* dX and dW_r are the same bits in both modes;
* the fp32 dW is within the bf16-mode tolerance of the fp64 oracle, and
  closer to it on average than the bf16 dW (the output rounding is gone);
* a backward with no tokens zero-fills the fp32 buffers.
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_27_b200 import binding as B

from _util import TOL_BF16, make_case, relerr, run_oracle, to64

pytestmark = pytest.mark.gpu

WNAMES = ("dW_gate", "dW_up", "dW_down")


def _same_bits(a, b):
    return torch.equal(a.contiguous().view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32),
                       b.contiguous().view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32))


def _check_modes(g16, g32):
    for n in WNAMES:
        assert g32[n].dtype == torch.float32 and g16[n].dtype == torch.bfloat16
        assert _same_bits(g32[n].to(torch.bfloat16), g16[n]), n
    assert _same_bits(g32["dX"], g16["dX"])
    assert _same_bits(g32["dW_r"], g16["dW_r"])


@pytest.mark.parametrize("T,d,E,k,I,first,num,seed", [
    (300, 512, 8, 2, 512, 0, 0, 71),   # several tiles, ragged tail
    (257, 256, 12, 3, 768, 2, 7, 72),  # a local expert slice
])
def test_fp32_weight_gradients_moe_bwd(T, d, E, k, I, first, num, seed):
    w, x = make_case(T, d, E, k, I, seed=seed)
    El = num or E - first
    Wg = x["W_gate"][first:first + El].contiguous()
    Wu = x["W_up"][first:first + El].contiguous()
    Wd = x["W_down"][first:first + El].contiguous()
    g = {}
    for dt in (torch.bfloat16, torch.float32):
        lay = B.MoELayer(T, d, E, I, k, first_local_expert=first, num_local_experts=num, wgrad_dtype=dt)
        lay.forward(x["X"], x["W_r"], x["bias"], Wg, Wu, Wd)
        g[dt] = lay.backward(x["X"], x["W_r"], Wg, Wu, Wd, x["dY"])
        torch.cuda.synchronize()
        assert lay.error() == B.MOE_OK
    _check_modes(g[torch.bfloat16], g[torch.float32])
    _, _, go = run_oracle(x, k, first, num or None)
    for n in WNAMES:
        ref = np.stack([go[n][first + e] for e in range(El)])
        e32 = relerr(to64(g[torch.float32][n]), ref)
        assert e32 <= TOL_BF16, (n, e32)
        # without the output rounding the gradient is closer to the oracle on average
        m32 = np.mean(np.abs(to64(g[torch.float32][n]) - ref))
        m16 = np.mean(np.abs(to64(g[torch.bfloat16][n]) - ref))
        assert m32 < m16, (n, m32, m16)


def test_fp32_weight_gradients_moe_bwd_mx():
    T, d, E, k, I = 200, 256, 8, 2, 512
    w, x = make_case(T, d, E, k, I, seed=73)
    g = {}
    for dt in (torch.bfloat16, torch.float32):
        lay = B.MoELayerMX(T, d, E, I, k, wgrad_dtype=dt)
        lay.prepare(x["W_gate"], x["W_up"], x["W_down"])
        lay.forward(x["X"], x["W_r"], x["bias"])
        g[dt] = lay.backward(x["X"], x["W_r"], x["dY"])
        torch.cuda.synchronize()
        assert lay.error() == B.MOE_OK
    _check_modes(g[torch.bfloat16], g[torch.float32])


@pytest.mark.parametrize("ring_mult,several_chunks", [(1.0, True), (100.0, False)])
def test_fp32_weight_gradients_moe_bwd_stream(ring_mult, several_chunks):
    T_mb, M, d, E, k, I = 128, 8, 256, 16, 4, 256
    w, x = make_case(T_mb * M, d, E, k, I, seed=74)
    shape = B.make_shape(T_mb, d, E, I, k)
    ring_bytes = int(B.moe_stream_min_ring_bytes(shape) * ring_mult) // (2 * d) * (2 * d)
    g = {}
    for dt in (torch.bfloat16, torch.float32):
        s = B.MoEStream(T_mb, d, E, I, k, M, ring_bytes, wgrad_dtype=dt)
        s.forward(x["X"], x["W_r"], x["bias"], x["W_gate"], x["W_up"], x["W_down"])
        g[dt] = s.backward(x["X"], x["W_r"], x["W_gate"], x["W_up"], x["W_down"], x["dY"])
        torch.cuda.synchronize()
        assert s.error() == B.MOE_OK
        assert (int(s.plan()["plan"][1]) > 1) == several_chunks
    _check_modes(g[torch.bfloat16], g[torch.float32])


def test_fp32_weight_gradients_no_tokens():
    T, d, E, k, I = 0, 256, 4, 2, 256
    lay = B.MoELayer(T, d, E, I, k, wgrad_dtype=torch.float32)
    W = {n: torch.randn(*s, device="cuda").to(torch.bfloat16) for n, s in
         dict(W_r=(d, E), W_gate=(E, d, I), W_up=(E, d, I), W_down=(E, I, d)).items()}
    X0 = torch.empty(0, d, device="cuda", dtype=torch.bfloat16)
    lay.forward(X0, W["W_r"], None, W["W_gate"], W["W_up"], W["W_down"], Y=X0.clone())
    g = lay.backward(X0, W["W_r"], W["W_gate"], W["W_up"], W["W_down"], X0,
                     out=dict(dX=X0.clone(),
                              dW_gate=torch.full((E, d, I), 7.0, device="cuda"),
                              dW_up=torch.full((E, d, I), 7.0, device="cuda"),
                              dW_down=torch.full((E, I, d), 7.0, device="cuda"),
                              dW_r=torch.full((d, E), 7.0, device="cuda")))
    torch.cuda.synchronize()
    for n in WNAMES + ("dW_r",):
        assert torch.count_nonzero(g[n]) == 0, n
