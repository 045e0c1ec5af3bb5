"""moe_route_static: router GEMM + top-k gating without any allocation.

Some callers cannot allocate device memory while they run -- code inside an
allocator or memory-planner callback (cudaMalloc would re-enter the
allocator), or a service whose device memory its own pool already owns.  For
them the library keeps the step's scratch in a fixed static device array.
These tests check that entry point, through the C ABI, against the routing
table the regular moe_fwd writes, over consecutive calls whose leftover
scratch must not leak into the next result; that after the first call on the
device (the set-up, which loads the kernels and the array) further calls
leave the device's free memory and torch's reserved memory unchanged; and the
NULL-status and no-token forms of the call.
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_27_b200 import binding as B
from mixture_experts_layer_27_b200 import build as BUILD

from _util import make_case

GATE_TOL = 1e-6  # the gate tolerance of the routing parity tests


def _regular(T, d, E, k, I, x):
    layer = B.MoELayer(T, d, E, I, k)
    layer.forward(x["X"], x["W_r"], x["bias"], x["W_gate"], x["W_up"], x["W_down"])
    assert layer.error() == B.MOE_OK
    r = layer.routing()
    return r["ids"], r["gates"]


def _outputs(T, k):
    ids = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    gates = torch.full((T, k), -7.0, dtype=torch.float32, device="cuda")
    status = torch.full((1,), 99, dtype=torch.int32, device="cuda")
    return ids, gates, status


@pytest.mark.gpu
def test_static_scratch_routing_matches_moe_fwd_on_consecutive_calls():
    cases = [(2048, 7168, 256, 8, 256, None, 21),          # the DeepSeek-V3-like routing shape
             (300, 512, 40, 6, 256, np.linspace(-1, 1, 40), 22)]  # ragged T, biased router
    made = [(c, make_case(*c[:5], seed=c[6], bias=c[5])[1]) for c in cases]
    want = [_regular(*c[:5], x) for c, x in made]
    # every output buffer of the calls below exists before the first of them
    seq = made + made[:1]  # A, B, then A again over B's leftover scratch
    outs = [_outputs(c[0], c[3]) for c, _ in seq]
    st_none = _outputs(cases[1][0], cases[1][3])
    empty = torch.full((1,), 99, dtype=torch.int32, device="cuda")
    c1, x1 = made[1]

    # set-up: the first call on this device loads the kernels and the static array
    warm = _outputs(c1[0], c1[3])
    assert B.moe_route_static(B.make_shape(*c1[:3], c1[4], c1[3]), x1["X"], x1["W_r"], x1["bias"], *warm) == B.MOE_OK
    torch.cuda.synchronize()
    free0, reserved0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_reserved()

    for (c, x), (ids, gates, status) in zip(seq, outs):
        shape = B.make_shape(c[0], c[1], c[2], c[4], c[3])
        assert B.moe_route_static(shape, x["X"], x["W_r"], x["bias"], ids, gates, status) == B.MOE_OK
    # no status word: device errors are not reported, the routing is the same
    shape1 = B.make_shape(c1[0], c1[1], c1[2], c1[4], c1[3])
    assert B.moe_route_static(shape1, x1["X"], x1["W_r"], x1["bias"], st_none[0], st_none[1], None) == B.MOE_OK
    # no tokens: only the status word is touched (cleared)
    shape0 = B.make_shape(0, c1[1], c1[2], c1[4], c1[3])
    assert B.moe_route_static(shape0, None, x1["W_r"], x1["bias"], None, None, empty) == B.MOE_OK
    torch.cuda.synchronize()
    free1, reserved1 = torch.cuda.mem_get_info()[0], torch.cuda.memory_reserved()
    assert free1 == free0, (free0, free1)
    assert reserved1 == reserved0, (reserved0, reserved1)

    for (ids, gates, status), (wid, wg) in zip(outs, want + want[:1]):
        assert int(status.item()) == B.MOE_OK
        assert torch.equal(ids, wid)
        assert float((gates - wg).abs().max()) <= GATE_TOL
    assert torch.equal(st_none[0], want[1][0])
    assert float((st_none[1] - want[1][1]).abs().max()) <= GATE_TOL
    assert int(empty.item()) == B.MOE_OK


def test_shapes_beyond_the_static_scratch_are_refused():
    BUILD.build()
    big = B.make_shape(65536, 256, 512, 256, 2)  # logits alone need 128 MiB
    fake = 1 << 20  # never dereferenced: the size check comes first
    assert B.moe_route_static(big, fake, fake, None, fake, fake, None, stream=0) == B.MOE_ERR_WORKSPACE_TOO_SMALL
