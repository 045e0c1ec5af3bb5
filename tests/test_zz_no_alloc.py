"""moe_route_static: router GEMM + top-k gating without any allocation.

Some callers cannot allocate device memory while they run -- code inside an
allocator or memory-planner callback (cudaMalloc would re-enter the
allocator), or a service whose device memory its own pool already owns.  For
them the library keeps the step's scratch in a fixed static device array.
These tests check that entry point, through the C ABI, against the routing
table the regular moe_fwd writes, over consecutive calls whose leftover
scratch must not leak into the next result.
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


def _static(T, d, E, k, I, x):
    shape = B.make_shape(T, d, E, I, k)
    ids = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    gates = torch.full((T, k), -7.0, dtype=torch.float32, device="cuda")
    status = torch.full((1,), 99, dtype=torch.int32, device="cuda")
    assert B.moe_route_static(shape, x["X"], x["W_r"], x["bias"], ids, gates, status) == B.MOE_OK
    return ids, gates, status


@pytest.mark.gpu
def test_static_scratch_routing_matches_moe_fwd_on_consecutive_calls():
    cases = [(2048, 7168, 256, 8, 256, None, 21),          # the DeepSeek-V3-like routing shape
             (300, 512, 40, 6, 256, np.linspace(-1, 1, 40), 22)]  # ragged T, biased router
    made = [(c, make_case(*c[:5], seed=c[6], bias=c[5])[1]) for c in cases]
    want = [_regular(*c[:5], x) for c, x in made]
    # three calls back to back: A, B, then A again over B's leftover scratch
    got = [_static(*c[:5], x) for c, x in (made + made[:1])]
    torch.cuda.synchronize()
    for (ids, gates, status), (wid, wg) in zip(got, want + want[:1]):
        assert int(status.item()) == B.MOE_OK
        assert torch.equal(ids, wid)
        assert float((gates - wg).abs().max()) <= GATE_TOL


def test_shapes_beyond_the_static_scratch_are_refused():
    BUILD.build()
    big = B.make_shape(65536, 256, 512, 256, 2)  # logits alone need 128 MiB
    fake = 1 << 20  # never dereferenced: the size check comes first
    assert B.moe_route_static(big, fake, fake, None, fake, fake, None, stream=0) == B.MOE_ERR_WORKSPACE_TOO_SMALL
