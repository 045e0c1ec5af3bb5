"""GPU parity of the whole layer (forward + backward) against the fp64 oracle.

Floating-point outputs: max |gpu - oracle| / max |oracle| <= 2e-2 per tensor (bf16 mode).
Routing table: bit-exact against the oracle's selection run on the GPU's own
fp32 logits (the argmax is decided in the kernel's precision on both sides).
Results: bit-identical across repeated runs and across workspace placements.
"""
import numpy as np
import pytest
import torch

import oracle as O
from mixture_experts_layer_27_b200 import binding as B

from _util import TOL_BF16, make_case, relerr, run_gpu, run_oracle, to64

pytestmark = pytest.mark.gpu


def _check_routing(layer, x, k, E, first, num):
    r = layer.routing()
    lg = to64(layer.logits())
    ids = O.topk_ids(lg, k)
    assert np.array_equal(r["ids"].cpu().numpy(), ids)
    s = O.schedule(ids, E, first, num or None)
    assert np.array_equal(r["counts"].cpu().numpy(), s["counts"])
    assert np.array_equal(r["offsets"].cpu().numpy(), s["offsets"])
    assert np.array_equal(r["padded_offsets"].cpu().numpy(), s["padded_offsets"])
    assert np.array_equal(r["perm"].cpu().numpy(), s["perm"])
    assert np.array_equal(r["slot_row"].cpu().numpy(), s["slot_row"])
    g = O.gates(lg, ids)
    assert np.max(np.abs(r["gates"].cpu().numpy() - g)) < 1e-6
    # the fp32 logits themselves against fp64
    X, Wr = to64(x["X"]), to64(x["W_r"])
    b = None if x["bias"] is None else to64(x["bias"])
    assert relerr(lg, O.router_logits(X, Wr, b)) < 1e-5
    return s


def _check_layer(T, d, E, k, I, first=0, num=0, bias=None, seed=0):
    w, x = make_case(T, d, E, k, I, seed=seed, bias=bias)
    layer, Y, g, st = run_gpu(x, T, d, E, k, I, first, num)
    assert st == B.MOE_OK, B.status_string(st)
    _check_routing(layer, x, k, E, first, num)
    Yo, ctx, go = run_oracle(x, k, first, num or None)
    El = num or (E - first)
    errs = {
        "Y": relerr(to64(Y), Yo),
        "dX": relerr(to64(g["dX"]), go["dX"]),
        "dW_r": relerr(to64(g["dW_r"]), go["dW_r"]),
        "dW_gate": relerr(to64(g["dW_gate"]), np.stack([go["dW_gate"][first + e] for e in range(El)])),
        "dW_up": relerr(to64(g["dW_up"]), np.stack([go["dW_up"][first + e] for e in range(El)])),
        "dW_down": relerr(to64(g["dW_down"]), np.stack([go["dW_down"][first + e] for e in range(El)])),
    }
    bad = {kk: v for kk, v in errs.items() if not v <= TOL_BF16}
    assert not bad, errs
    return layer, x, Y, g


def test_tiny_config_matches_oracle():
    """T=128, d=256, E=8, top-2, I=512 (the small workload), seed 0."""
    _check_layer(128, 256, 8, 2, 512)


def test_ragged_tokens_and_uneven_experts():
    _check_layer(77, 256, 6, 3, 256, seed=1)


def test_hot_expert_spans_many_tiles_and_empty_expert():
    bias = np.zeros(4, dtype=np.float32)
    bias[0] = 8.0    # every token picks expert 0: 600 rows -> 5 padded tiles
    bias[3] = -40.0  # expert 3 is never picked: zero gradient
    _check_layer(600, 512, 4, 2, 512, bias=bias, seed=2)


def test_k_equals_E():
    _check_layer(64, 256, 4, 4, 256, seed=3)


def test_top_k_16_the_largest_supported():
    _check_layer(96, 256, 32, 16, 256, seed=11)


def test_single_expert():
    _check_layer(100, 256, 1, 1, 256, seed=4)


def test_many_experts_mostly_empty():
    _check_layer(256, 256, 384, 8, 256, seed=5)


def test_local_expert_slice():
    _check_layer(200, 256, 16, 4, 256, first=4, num=5, seed=6)


def test_many_token_blocks_two_level_scan():
    # 4112 tokens = 257 blocks of 16: the expert scan runs in two levels (groups of 32 rows,
    # the last group holding one row); routing stays bit-exact against the oracle
    _check_layer(4112, 256, 16, 2, 256, seed=14)


def test_expert_slice_router_gradient_over_listed_tokens():
    # In a slice only the tokens with a local assignment carry router gradient; the weight
    # gradient contracts over that list (here about 120 of 700 tokens, spread over three
    # 256-token blocks and a ragged tail).
    _check_layer(700, 256, 64, 4, 256, first=10, num=3, seed=12)


def test_expert_slice_that_receives_no_tokens():
    bias = np.zeros(8, dtype=np.float32)
    bias[6:] = -40.0  # the slice's experts are never picked: no token is listed
    layer, x, Y, g = _check_layer(300, 256, 8, 2, 256, first=6, num=2, bias=bias, seed=13)
    for n in ("dW_r", "dW_gate", "dW_up", "dW_down"):
        assert torch.count_nonzero(g[n]) == 0, n
    assert torch.count_nonzero(Y) == 0 and torch.count_nonzero(g["dX"]) == 0


def test_no_tokens():
    T, d, E, k, I = 0, 256, 4, 2, 256
    layer = B.MoELayer(T, d, E, I, k)
    x = {n: torch.randn(*s, device="cuda").to(torch.bfloat16) for n, s in
         dict(X=(1, d), W_r=(d, E), W_gate=(E, d, I), W_up=(E, d, I), W_down=(E, I, d), dY=(1, d)).items()}
    X0, dY0 = x["X"][:0], x["dY"][:0]
    layer.forward(X0, x["W_r"], None, x["W_gate"], x["W_up"], x["W_down"], Y=torch.empty(0, d, device="cuda",
                                                                                         dtype=torch.bfloat16))
    g = layer.backward(X0, x["W_r"], x["W_gate"], x["W_up"], x["W_down"], dY0,
                       out=dict(dX=torch.empty(0, d, device="cuda", dtype=torch.bfloat16),
                                dW_gate=torch.full((E, d, I), 7.0, device="cuda", dtype=torch.bfloat16),
                                dW_up=torch.full((E, d, I), 7.0, device="cuda", dtype=torch.bfloat16),
                                dW_down=torch.full((E, I, d), 7.0, device="cuda", dtype=torch.bfloat16),
                                dW_r=torch.full((d, E), 7.0, device="cuda")))
    torch.cuda.synchronize()
    for n in ("dW_gate", "dW_up", "dW_down", "dW_r"):
        assert torch.count_nonzero(g[n]) == 0


def test_bit_identical_across_runs_and_workspace_placement():
    T, d, E, k, I = 300, 512, 8, 2, 512
    w, x = make_case(T, d, E, k, I, seed=7)
    _, Y1, g1, st1 = run_gpu(x, T, d, E, k, I)
    _, Y2, g2, st2 = run_gpu(x, T, d, E, k, I)
    # a second layer whose ctx / ws start 256 bytes further into larger buffers
    lay = B.MoELayer(T, d, E, I, k)
    lay.ctx = torch.empty(lay.ctx.numel() + 4096, dtype=torch.uint8, device="cuda")[256:]
    lay.ws = torch.empty(lay.ws.numel() + 4096, dtype=torch.uint8, device="cuda")[1024:]
    _, Y3, g3, st3 = run_gpu(x, T, d, E, k, I, layer=lay)
    assert st1 == st2 == st3 == B.MOE_OK
    for Ya, ga in ((Y2, g2), (Y3, g3)):
        assert torch.equal(Y1.view(torch.int16), Ya.view(torch.int16))
        for n in g1:
            assert torch.equal(g1[n].view(torch.int16) if g1[n].dtype == torch.bfloat16 else g1[n].view(torch.int32),
                               ga[n].view(torch.int16) if ga[n].dtype == torch.bfloat16 else ga[n].view(torch.int32)), n


def test_results_do_not_depend_on_stale_ctx_and_workspace_contents():
    # Pad rows of the expert segments are never written; whatever ctx / ws hold there (here
    # NaN bit patterns in both bf16 and fp32) must not reach any output.
    T, d, E, k, I = 333, 512, 12, 3, 512
    w, x = make_case(T, d, E, k, I, seed=9)
    outs = []
    for fill in (0, 255):
        lay = B.MoELayer(T, d, E, I, k)
        lay.ctx.fill_(fill)
        lay.ws.fill_(fill)
        _, Y, g, st = run_gpu(x, T, d, E, k, I, layer=lay)
        assert st == B.MOE_OK
        assert torch.isfinite(Y.float()).all()
        outs.append((Y, g))
    (Y0, g0), (Y1, g1) = outs
    assert torch.equal(Y0.view(torch.int16), Y1.view(torch.int16))
    for n in g0:
        a, b = g0[n], g1[n]
        assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32),
                           b.view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32)), n


def test_cuda_graph_replay_matches_direct_launches():
    # moe_fwd + moe_bwd only enqueue work (no host synchronisation, no allocation), so one step
    # can be captured as a CUDA graph; its replays must give the direct launches' bits.
    T, d, E, k, I = 300, 512, 8, 2, 512
    w, x = make_case(T, d, E, k, I, seed=10)
    lay = B.MoELayer(T, d, E, I, k)
    Y = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    g = dict(dX=torch.empty(T, d, dtype=torch.bfloat16, device="cuda"),
             dW_gate=torch.empty(E, d, I, dtype=torch.bfloat16, device="cuda"),
             dW_up=torch.empty(E, d, I, dtype=torch.bfloat16, device="cuda"),
             dW_down=torch.empty(E, I, d, dtype=torch.bfloat16, device="cuda"),
             dW_r=torch.empty(d, E, dtype=torch.float32, device="cuda"))

    def step():
        lay.forward(x["X"], x["W_r"], x["bias"], x["W_gate"], x["W_up"], x["W_down"], Y=Y)
        lay.backward(x["X"], x["W_r"], x["W_gate"], x["W_up"], x["W_down"], x["dY"], out=g)

    step()
    torch.cuda.synchronize()
    ref = (Y.clone(), {n: t.clone() for n, t in g.items()})
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for n in g:
        g[n].zero_()
    Y.zero_()
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    assert lay.error() == B.MOE_OK
    assert torch.equal(Y.view(torch.int16), ref[0].view(torch.int16))
    for n in g:
        a, b = g[n], ref[1][n]
        assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32),
                           b.view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32)), n


def test_bounded_wait_gives_up_records_timeout_and_the_context_stays_usable():
    # An mbarrier nothing arrives at: the GEMM roles' bounded wait gives up (about 2 s),
    # records MOE_ERR_DEVICE_TIMEOUT in ctx's status word and the kernel returns.
    T, d, E, k, I = 64, 256, 4, 2, 256
    w, x = make_case(T, d, E, k, I, seed=12)
    lay = B.MoELayer(T, d, E, I, k)
    assert B.moe_debug_bounded_wait(lay.shape, lay.ctx) == B.MOE_OK
    torch.cuda.synchronize()
    assert lay.error() == B.MOE_ERR_DEVICE_TIMEOUT
    assert lay.error() == B.MOE_OK  # reading the status clears it
    _, Y, g, st = run_gpu(x, T, d, E, k, I, layer=lay)  # the context still runs the layer
    assert st == B.MOE_OK
    Yo, ctx, go = run_oracle(x, k)
    assert relerr(to64(Y), Yo) <= TOL_BF16 and relerr(to64(g["dX"]), go["dX"]) <= TOL_BF16


def test_nonfinite_logit_sets_status():
    T, d, E, k, I = 32, 256, 8, 2, 256
    w, x = make_case(T, d, E, k, I, seed=8)
    x["X"][5, 3] = float("inf")
    layer, Y, g, st = run_gpu(x, T, d, E, k, I)
    assert st == B.MOE_ERR_NONFINITE
    assert layer.error() == B.MOE_OK  # reading the status clears it
