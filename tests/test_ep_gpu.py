"""Expert parallelism across R ranks, run on one device.

Every rank's exchange buffer, ctx and workspace sit in this GPU's memory, and each phase of a
step runs for every rank before the next phase starts, so every bounded wait in a phase is on
flags that earlier phases of the same step have already set: no kernel waits for one that has
not run.  The exchange kernels read and write the other ranks' buffers through their
addresses exactly as they do peer memory across GPUs.

Row order on an owner equals the one-device layer's order for the rank-major concatenation of
the ranks' tokens, and the router GEMM's fixed K split is the same at these sizes, so the
routing, Y, dX and every expert weight gradient must equal the one-device layer's bit for bit;
the router weight gradient is each rank's part (summed over ranks it matches to fp32 rounding).
The device's exchange plan must equal the oracle's; the layer must match the fp64 oracle.
"""
import numpy as np
import pytest
import torch

import oracle as O
from mixture_experts_layer_27_b200 import binding as B

from _util import TOL_BF16, make_case, relerr, run_gpu, run_oracle, to64

pytestmark = pytest.mark.gpu


def _ep_layers(R, T, d, E, I, k):
    shape = B.make_shape(T, d, E, I, k)
    nb = B.moe_ep_buffer_size(shape, R)
    assert nb > 0
    bufs = [torch.zeros(nb, dtype=torch.uint8, device="cuda") for _ in range(R)]
    ranks = [B.MoEExpertParallel(T, d, E, I, k, R, r, bufs) for r in range(R)]
    return bufs, ranks


def _ep_step(ranks, x, R, T, epoch):
    El = ranks[0].El
    sl = [slice(r * T, (r + 1) * T) for r in range(R)]
    ex = [slice(r * El, (r + 1) * El) for r in range(R)]
    X, dY = x["X"], x["dY"]
    Y = torch.empty_like(X)
    dX = torch.empty_like(X)
    dW = {n: torch.empty_like(x[n]) for n in ("W_gate", "W_up", "W_down")}
    dWr = [torch.empty(x["W_r"].shape, dtype=torch.float32, device="cuda") for _ in range(R)]
    W = {n: [x[n][ex[r]].contiguous() for r in range(R)] for n in ("W_gate", "W_up", "W_down")}
    for r in range(R):
        ranks[r].fwd_route(X[sl[r]], x["W_r"], x["bias"], epoch)
    for r in range(R):
        ranks[r].fwd_experts(W["W_gate"][r], W["W_up"][r], W["W_down"][r], epoch)
    for r in range(R):
        ranks[r].fwd_combine(Y[sl[r]], epoch)
    for r in range(R):
        ranks[r].bwd_publish(dY[sl[r]].contiguous(), epoch)
    gW = {n: [torch.empty_like(W[n][r]) for r in range(R)] for n in W}
    for r in range(R):
        ranks[r].bwd_experts(W["W_gate"][r], W["W_up"][r], W["W_down"][r], gW["W_gate"][r], gW["W_up"][r],
                             gW["W_down"][r], epoch)
    for r in range(R):
        ranks[r].bwd_finish(X[sl[r]], x["W_r"], dX[sl[r]], dWr[r], epoch)
    torch.cuda.synchronize()
    for r in range(R):
        assert ranks[r].error() == B.MOE_OK, r
        for n in W:
            dW[n][ex[r]] = gW[n][r]
    return Y, dX, dW, dWr


def _check_against_one_device_layer(R, T, d, E, k, I, seed, bias=None):
    w, x = make_case(R * T, d, E, k, I, seed=seed, bias=bias)
    bufs, ranks = _ep_layers(R, T, d, E, I, k)
    Y, dX, dW, dWr = _ep_step(ranks, x, R, T, epoch=1)
    layer, Y1, g1, st = run_gpu(x, R * T, d, E, k, I)
    assert st == B.MOE_OK

    # the device's exchange plan against the oracle's, on the one-device layer's routing
    ids = layer.routing()["ids"].cpu().numpy()
    plan = O.ep_plan([ids[r * T:(r + 1) * T] for r in range(R)], E)
    for q in range(R):
        got = ranks[q].plan()
        own = plan["owners"][q]
        assert np.array_equal(got["counts"].cpu().numpy(), own["counts"])
        assert np.array_equal(got["padded_offsets"].cpu().numpy(), own["padded_offsets"])
        src = got["row_src"].cpu().numpy()
        poff = own["padded_offsets"]
        i = 0
        for el in range(E // R):
            for row in range(int(poff[el]), int(poff[el]) + int(own["counts"][el])):
                s, t, j = own["rows"][i]
                assert src[row] == s * T * k + t * k + j, (q, el, row)
                i += 1
            assert np.all(src[int(poff[el]) + int(own["counts"][el]):int(poff[el + 1])] < 0)

    # bit for bit against the one-device layer on the rank-major batch
    assert torch.equal(Y.view(torch.int16), Y1.view(torch.int16))
    assert torch.equal(dX.view(torch.int16), g1["dX"].view(torch.int16))
    for n in ("W_gate", "W_up", "W_down"):
        assert torch.equal(dW[n].view(torch.int16), g1["d" + n].view(torch.int16)), n
    assert relerr(to64(sum(dWr)), to64(g1["dW_r"])) <= 1e-4

    # and against the fp64 oracle
    Yo, ctx, go = run_oracle(x, k)
    assert relerr(to64(Y), Yo) <= TOL_BF16
    assert relerr(to64(dX), go["dX"]) <= TOL_BF16
    assert relerr(to64(sum(dWr)), go["dW_r"]) <= TOL_BF16
    for n in ("W_gate", "W_up", "W_down"):
        assert relerr(to64(dW[n]), np.stack([go["d" + n][e] for e in range(E)])) <= TOL_BF16, n
    return x, bufs, ranks, (Y, dX, dW, dWr)


def test_expert_parallel_four_ranks_equal_the_one_device_layer():
    R, T = 4, 96
    x, bufs, ranks, first = _check_against_one_device_layer(R, T, 256, 16, 4, 256, seed=51)
    # a second step (next epoch) over the same buffers is bit-identical
    again = _ep_step(ranks, x, R, T, epoch=2)
    assert torch.equal(first[0].view(torch.int16), again[0].view(torch.int16))
    assert torch.equal(first[1].view(torch.int16), again[1].view(torch.int16))
    for n in first[2]:
        assert torch.equal(first[2][n].view(torch.int16), again[2][n].view(torch.int16)), n


def test_expert_parallel_uneven_load_and_idle_owners():
    # the bias sends most assignments to rank 1's experts and none to rank 2's: ragged segments,
    # an owner with no rows, sources whose tokens all go elsewhere
    R, T, E = 4, 80, 16
    bias = np.zeros(E, dtype=np.float32)
    bias[4:8] = 3.0
    bias[8:12] = -40.0
    _check_against_one_device_layer(R, T, 256, E, 3, 256, seed=52, bias=bias)


def test_expert_parallel_two_ranks_many_experts():
    _check_against_one_device_layer(2, 200, 256, 64, 6, 256, seed=53)


def test_expert_parallel_eight_ranks():
    # eight ranks (one NVL8 node's worth), 4 experts each, top-8 over 32 experts
    _check_against_one_device_layer(8, 64, 256, 32, 8, 256, seed=55)


def test_expert_parallel_wait_for_an_unpublished_step_times_out_and_recovers():
    # After a good step, rank 0's expert phase is asked for an epoch no rank published: its bounded
    # wait gives up (about 2 s), records MOE_ERR_DEVICE_TIMEOUT, and the phase's exchange kernels
    # do nothing; the next full step runs normally.
    R, T, d, E, k, I = 2, 64, 256, 8, 2, 256
    w, x = make_case(R * T, d, E, k, I, seed=54)
    bufs, ranks = _ep_layers(R, T, d, E, I, k)
    first = _ep_step(ranks, x, R, T, epoch=1)
    El = E // R
    ranks[0].fwd_experts(x["W_gate"][:El].contiguous(), x["W_up"][:El].contiguous(), x["W_down"][:El].contiguous(),
                         epoch=7)
    assert ranks[0].error() == B.MOE_ERR_DEVICE_TIMEOUT
    again = _ep_step(ranks, x, R, T, epoch=2)
    assert torch.equal(first[0].view(torch.int16), again[0].view(torch.int16))
    assert torch.equal(first[1].view(torch.int16), again[1].view(torch.int16))
