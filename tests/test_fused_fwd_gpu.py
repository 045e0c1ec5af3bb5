"""Pairs of grouped GEMMs in one persistent launch (`moe_fwd_persistent`, `moe_bwd_persistent`).

The forward's gate/up GEMM (SwiGLU epilogue) and down GEMM (gate multiply), and the backward's
dgrad of W_down (SwiGLU backward, router-gate gradient) and dgrad of gate/up, each run as work
units of one kernel, taken by CTAs in one global order and claimed through Cluster Launch Control;
a tile of the second GEMM waits for the first GEMM's tiles of its rows.  Each unit computes what
the separate launches compute, with the same tiles and epilogues, so Y, everything saved in ctx
and every gradient must be the same bits as `moe_fwd` + `moe_bwd`, in either combination.  Y and
the gradients must also match the fp64 oracle within the bf16 tolerance, and repeated runs must
be bit-identical.
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_27_b200 import binding as B

from _util import TOL_BF16, make_case, relerr, run_oracle, to64

pytestmark = pytest.mark.gpu


def _step(layer, x, first, El, persistent, poison=False, bwd_persistent=None):
    if poison:  # every byte the step may read before writing it holds a NaN pattern
        layer.ctx.fill_(0xFF)
        layer.ws.fill_(0xFF)
    W = [x[n][first:first + El].contiguous() for n in ("W_gate", "W_up", "W_down")]
    Y = layer.forward(x["X"], x["W_r"], x["bias"], *W, persistent=persistent)
    g = layer.backward(x["X"], x["W_r"], *W, x["dY"],
                       persistent=persistent if bwd_persistent is None else bwd_persistent)
    torch.cuda.synchronize()
    assert layer.error() == B.MOE_OK
    return Y, g


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


def _check(T, d, E, k, I, seed, bias=None, first=0, num=0, oracle=True):
    w, x = make_case(T, d, E, k, I, seed=seed, bias=bias)
    El = num or (E - first)
    ref = B.MoELayer(T, d, E, I, k, first_local_expert=first, num_local_experts=num)
    fus = B.MoELayer(T, d, E, I, k, first_local_expert=first, num_local_experts=num)
    Y0, g0 = _step(ref, x, first, El, persistent=False)
    Y1, g1 = _step(fus, x, first, El, persistent=True, poison=True)
    assert torch.equal(_bits(Y1), _bits(Y0))
    for n in g0:
        assert torch.equal(_bits(g1[n]), _bits(g0[n])), n
    r0, r1 = ref.routing(), fus.routing()
    for n in r0:
        assert torch.equal(r0[n], r1[n]), n
    # run to run: a second persistent step over the same buffers
    Y2, g2 = _step(fus, x, first, El, persistent=True)
    assert torch.equal(_bits(Y2), _bits(Y1))
    for n in g1:
        assert torch.equal(_bits(g2[n]), _bits(g1[n])), n
    # the mixed combinations: each persistent half pairs with the other's multi-launch half
    for fp, bp in ((True, False), (False, True)):
        Y3, g3 = _step(fus, x, first, El, persistent=fp, bwd_persistent=bp)
        assert torch.equal(_bits(Y3), _bits(Y0))
        for n in g0:
            assert torch.equal(_bits(g3[n]), _bits(g0[n])), (fp, bp, n)
    if oracle:
        Yo, _, go = run_oracle(x, k, first=first, num=num or None)
        assert relerr(to64(Y1), Yo) <= TOL_BF16
        assert relerr(to64(g1["dX"]), go["dX"]) <= TOL_BF16
        for n in ("W_gate", "W_up", "W_down"):
            want = np.stack([go["d" + n][e] for e in range(first, first + El)])
            assert relerr(to64(g1["d" + n]), want) <= TOL_BF16, n
    return fus


def test_persistent_forward_equals_moe_fwd_several_tiles_per_expert():
    # 600 tokens x 4 over 16 experts: about 150 rows each, two m-tiles, ragged last tiles
    _check(600, 512, 16, 4, 512, seed=81)


def test_persistent_forward_uneven_load_idle_experts_and_a_slice():
    E = 16
    bias = np.zeros(E, dtype=np.float32)
    bias[3] = 4.0   # one hot expert: many m-tiles
    bias[8:12] = -40.0  # idle experts: empty segments between full ones
    _check(500, 256, E, 3, 256, seed=82, bias=bias)
    _check(500, 256, E, 3, 256, seed=83, bias=bias, first=2, num=9)


def test_persistent_forward_one_token_and_many_tiles():
    _check(1, 256, 8, 2, 256, seed=84)
    _check(1500, 256, 32, 8, 256, seed=85)  # more tiles than two per SM


def test_persistent_forward_full_size_deepseek_v3_like_equals_moe_fwd():
    # T = 2048, d = 7168, E = 256, top-8, I = 2048: bit for bit against the multi-launch forward
    # (the oracle comparisons at this size live in test_fullsize_gpu.py)
    _check(2048, 7168, 256, 8, 2048, seed=0, oracle=False)


def test_persistent_forward_ep64_slice_equals_moe_fwd():
    # 6 of 384 experts, 32,768 tokens (the per-rank slice as one batch)
    _check(32768, 7168, 384, 8, 2048, seed=86, first=0, num=6, oracle=False)


def test_persistent_pair_wait_for_rows_nobody_writes_times_out_and_recovers():
    # The debug hook leaves the gate/up tiles out of the persistent launch: every down tile waits
    # for H rows that are never counted.  The first bounded wait to run out (about 2 s) records
    # MOE_ERR_DEVICE_TIMEOUT, every other CTA stops, and the next step on the same buffers is
    # again bit-identical to moe_fwd + moe_bwd.
    T, d, E, k, I = 300, 256, 8, 2, 256
    w, x = make_case(T, d, E, k, I, seed=87)
    ref = B.MoELayer(T, d, E, I, k)
    Y0, g0 = _step(ref, x, 0, E, persistent=False)
    lay = B.MoELayer(T, d, E, I, k)
    Y = torch.empty_like(Y0)
    W = [x[n].contiguous() for n in ("W_gate", "W_up", "W_down")]
    assert B.moe_debug_pair_wait(lay.shape, x["X"], x["W_r"], x["bias"], *W, Y, lay.ctx, lay.ws) == B.MOE_OK
    torch.cuda.synchronize()
    assert lay.error() == B.MOE_ERR_DEVICE_TIMEOUT
    assert lay.error() == B.MOE_OK  # read and cleared
    Y1, g1 = _step(lay, x, 0, E, persistent=True)
    assert torch.equal(_bits(Y1), _bits(Y0))
    for n in g0:
        assert torch.equal(_bits(g1[n]), _bits(g0[n])), n


def test_persistent_pairs_with_fp32_weight_gradients():
    # the dgrad pair feeds the fp32 weight-gradient path exactly as the separate launches do
    T, d, E, k, I = 400, 256, 8, 2, 256
    w, x = make_case(T, d, E, k, I, seed=88)
    W = [x[n].contiguous() for n in ("W_gate", "W_up", "W_down")]
    out = []
    for persistent in (False, True):
        lay = B.MoELayer(T, d, E, I, k, wgrad_dtype=torch.float32)
        Y = lay.forward(x["X"], x["W_r"], x["bias"], *W, persistent=persistent)
        g = lay.backward(x["X"], x["W_r"], *W, x["dY"], persistent=persistent)
        torch.cuda.synchronize()
        assert lay.error() == B.MOE_OK
        assert g["dW_gate"].dtype == torch.float32
        out.append((Y, g))
    assert torch.equal(_bits(out[1][0]), _bits(out[0][0]))
    for n in out[0][1]:
        assert torch.equal(_bits(out[1][1][n]), _bits(out[0][1][n])), n


def test_persistent_forward_without_tokens_clears_the_status():
    T, d, E, k, I = 0, 256, 8, 2, 256
    lay = B.MoELayer(1, d, E, I, k)  # buffers of a one-token layer; the call below has no tokens
    shape0 = B.make_shape(T, d, E, I, k)
    lay.ctx.fill_(0xFF)  # a stale status word
    W = [torch.zeros(E, d, I, dtype=torch.bfloat16, device="cuda"), torch.zeros(E, d, I, dtype=torch.bfloat16,
                                                                                     device="cuda"),
         torch.zeros(E, I, d, dtype=torch.bfloat16, device="cuda")]
    W_r = torch.zeros(d, E, dtype=torch.bfloat16, device="cuda")
    assert B.moe_fwd_persistent(shape0, None, W_r, None, *W, None, lay.ctx, lay.ws) == B.MOE_OK
    torch.cuda.synchronize()
    assert B.moe_get_error(lay.ctx) == B.MOE_OK


def test_persistent_pairs_full_size_kimi_zipf_equals_the_launches():
    # T = 4096, E = 384, top-8 under the Zipf(1.2) bias (hottest expert about 10x the mean): hot
    # experts with several m-tiles, so down tiles wait on many gate/up tiles of their rows
    from mixture_experts_layer_27_b200 import inputs as IN
    w = IN.WORKLOADS["kimi"]
    x = IN.make_inputs(w, device="cuda")
    out = []
    for persistent in (False, True):
        lay = B.MoELayer(w.T, w.d, w.E, w.I, w.k)
        Y = lay.forward(x["X"], x["W_r"], x["bias"], x["W_gate"], x["W_up"], x["W_down"], persistent=persistent)
        g = lay.backward(x["X"], x["W_r"], x["W_gate"], x["W_up"], x["W_down"], x["dY"], persistent=persistent)
        torch.cuda.synchronize()
        assert lay.error() == B.MOE_OK
        out.append((Y, g))
        del lay
    assert torch.equal(_bits(out[1][0]), _bits(out[0][0]))
    for n in out[0][1]:
        assert torch.equal(_bits(out[1][1][n]), _bits(out[0][1][n])), n
    del out, x
    torch.cuda.empty_cache()
