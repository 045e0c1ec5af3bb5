"""Ring-streamed layer (moe_fwd_stream / moe_bwd_stream) on the GPU.

* values: the layer over all M*T tokens, against the fp64 oracle on the
  concatenated batch (the ring changes where rows live, not the arithmetic);
* plan: macrobatch grouping, ring placement, residency and backward chunks,
  bit-exact against oracle.stream_plan on the same per-minibatch counts;
* small rings force replay and several backward chunks (fp32 accumulation of
  the gate/up weight gradient); a large ring keeps everything resident;
* two runs are bit-identical.
"""
import numpy as np
import pytest
import torch

import oracle as O
from mixture_experts_layer_27_b200 import binding as B

from _util import TOL_BF16, make_case, relerr, to64

pytestmark = pytest.mark.gpu


def _mb_counts(ids, T_mb, M, first, El):
    cnt = np.zeros((M, El), dtype=np.int64)
    for t in range(ids.shape[0]):
        for e in ids[t]:
            if first <= e < first + El:
                cnt[t // T_mb, e - first] += 1
    return cnt


@pytest.mark.parametrize("T_mb,M,d,E,k,I,first,num,ring_mult,seed", [
    (128, 8, 256, 16, 4, 256, 0, 0, 1.0, 31),    # smallest legal ring: replay, several chunks
    (128, 8, 256, 16, 4, 256, 0, 0, 100.0, 32),  # everything stays resident
    (64, 10, 512, 24, 6, 512, 3, 6, 1.5, 33),    # a local expert slice (6 of 24)
])
def test_streamed_layer(T_mb, M, d, E, k, I, first, num, ring_mult, seed):
    T = T_mb * M
    w, x = make_case(T, d, E, k, I, seed=seed)
    El = num or E - first
    shape = B.make_shape(T_mb, d, E, I, k, first_local_expert=first, num_local_experts=num)
    ring_bytes = int(B.moe_stream_min_ring_bytes(shape) * ring_mult) // (2 * d) * (2 * d)
    Wg = x["W_gate"][first:first + El].contiguous()
    Wu = x["W_up"][first:first + El].contiguous()
    Wd = x["W_down"][first:first + El].contiguous()
    s = B.MoEStream(T_mb, d, E, I, k, M, ring_bytes, first, num)

    def run():
        Y = s.forward(x["X"], x["W_r"], x["bias"], Wg, Wu, Wd)
        g = s.backward(x["X"], x["W_r"], Wg, Wu, Wd, x["dY"])
        torch.cuda.synchronize()
        assert s.error() == B.MOE_OK
        return Y, g

    Y, g = run()
    plan = s.plan()
    Yo, ctx, go = run_oracle_stream(x, k, first, num or None)
    errs = {"Y": relerr(to64(Y), Yo), "dX": relerr(to64(g["dX"]), go["dX"]),
            "dW_r": relerr(to64(g["dW_r"]), go["dW_r"]),
            "dW_gate": relerr(to64(g["dW_gate"]), np.stack([go["dW_gate"][first + e] for e in range(El)])),
            "dW_up": relerr(to64(g["dW_up"]), np.stack([go["dW_up"][first + e] for e in range(El)])),
            "dW_down": relerr(to64(g["dW_down"]), np.stack([go["dW_down"][first + e] for e in range(El)]))}
    assert all(v <= TOL_BF16 for v in errs.values()), errs

    # plan against the oracle's, on the oracle's per-minibatch counts
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    min_rows = 2 * sms * 128 // (I // 128)
    ring_rows = ring_bytes // (2 * d)
    op = O.stream_plan(_mb_counts(ctx["ids"], T_mb, M, first, El), ring_rows, min_rows)
    n = len(op["macro"])
    hdr = plan["plan"]
    assert hdr[0] == n and hdr[1] == len(op["chunks"]) and hdr[2] == op["rows"] and hdr[3] == op["replayed"]
    assert [tuple(plan["mb_range"][2 * m:2 * m + 2]) for m in range(n)] == op["macro"]
    assert plan["seg_poff"][:n * El].reshape(n, El).tolist() == op["seg_poff"]
    assert plan["ring_start"][:n].tolist() == op["ring_start"]
    assert [tuple(plan["chunk"][4 * c:4 * c + 2]) for c in range(len(op["chunks"]))] == op["chunks"]
    if ring_mult == 1.0:
        assert op["replayed"] > 0 and len(op["chunks"]) > 1  # the case exercises replay and accumulation
    if ring_mult >= 100:
        assert op["replayed"] == 0

    # bit-identical second run
    Y2, g2 = run()
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))
    for nme in ("dX", "dW_gate", "dW_up", "dW_down"):
        assert torch.equal(g[nme].view(torch.int16), g2[nme].view(torch.int16)), nme
    assert torch.equal(g["dW_r"].view(torch.int32), g2["dW_r"].view(torch.int32))


def run_oracle_stream(x, k, first, num):
    X, Wr, dY = to64(x["X"]), to64(x["W_r"]), to64(x["dY"])
    b = None if x["bias"] is None else to64(x["bias"])
    Y, ctx = O.forward(X, Wr, b, to64(x["W_gate"]), to64(x["W_up"]), to64(x["W_down"]), k,
                       first_local=first, num_local=num)
    return Y, ctx, O.backward(ctx, dY)


def test_stream_refuses_a_ring_below_one_minibatch():
    shape = B.make_shape(128, 256, 16, 256, 4)
    s = B.MoEStream(128, 256, 16, 256, 4, 4, B.moe_stream_min_ring_bytes(shape) - 512)
    x = {n: torch.zeros(*sz, dtype=torch.bfloat16, device="cuda") for n, sz in
         dict(X=(512, 256), W_r=(256, 16), W_gate=(16, 256, 256), W_up=(16, 256, 256), W_down=(16, 256, 256)).items()}
    st = B.moe_fwd_stream(s.shape, 4, x["X"], x["W_r"], None, x["W_gate"], x["W_up"], x["W_down"],
                          torch.empty_like(x["X"]), s.ctx, s.ring, s.ws)
    assert st == B.MOE_ERR_WORKSPACE_TOO_SMALL


def test_stream_results_do_not_depend_on_stale_ring_ctx_and_workspace():
    T_mb, M, d, E, k, I = 128, 6, 256, 16, 4, 256
    T = T_mb * M
    w, x = make_case(T, d, E, k, I, seed=34)
    shape = B.make_shape(T_mb, d, E, I, k)
    ring_bytes = int(B.moe_stream_min_ring_bytes(shape) * 1.2) // (2 * d) * (2 * d)
    outs = []
    for fill in (0, 255):
        s = B.MoEStream(T_mb, d, E, I, k, M, ring_bytes)
        for buf in (s.ctx, s.ws, s.ring):
            buf.fill_(fill)
        Y = s.forward(x["X"], x["W_r"], x["bias"], x["W_gate"], x["W_up"], x["W_down"])
        g = s.backward(x["X"], x["W_r"], x["W_gate"], x["W_up"], x["W_down"], x["dY"])
        torch.cuda.synchronize()
        assert s.error() == B.MOE_OK
        outs.append((Y, g))
    (Y0, g0), (Y1, g1) = outs
    assert torch.equal(Y0.view(torch.int16), Y1.view(torch.int16))
    for n in ("dX", "dW_gate", "dW_up", "dW_down"):
        assert torch.equal(g0[n].view(torch.int16), g1[n].view(torch.int16)), n
    assert torch.equal(g0["dW_r"].view(torch.int32), g1["dW_r"].view(torch.int32))
