"""The C-ABI library: it loads, exports every declared symbol, sizes buffers
from shapes alone and rejects bad arguments on the host (no GPU needed)."""
import ctypes
import os
import re

import pytest

from mixture_experts_layer_27_b200 import binding as B
from mixture_experts_layer_27_b200 import build as BUILD

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    BUILD.build()
    return B.lib()


def declared_functions():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(moe_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert {"moe_fwd", "moe_bwd", "moe_ctx_size", "moe_workspace_size", "moe_get_error"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_sizes_depend_on_shape_only_and_grow_with_it():
    s1 = B.make_shape(128, 256, 8, 512, 2)
    s2 = B.make_shape(2048, 7168, 256, 2048, 8)
    for s in (s1, s2):
        assert B.moe_ctx_size(s) > 0 and B.moe_workspace_size(s) > 0
    assert B.moe_workspace_size(s2) > B.moe_workspace_size(s1)
    # worst-case padded rows for the DeepSeek-V3-like shape: T*k + 127*E rows of X_perm (bf16)
    rp = -(-(2048 * 8 + 127 * 256) // 128) * 128
    assert B.moe_ctx_size(s2) >= rp * 7168 * 2 + 2 * rp * 2048 * 2


def test_sizes_do_not_depend_on_the_weight_gradient_dtype():
    for kw in (dict(T=128, d=256, E=8, I=512, top_k=2), dict(T=2048, d=7168, E=256, I=2048, top_k=8)):
        s16 = B.make_shape(**kw, wgrad_dtype=B.MOE_WGRAD_BF16)
        s32 = B.make_shape(**kw, wgrad_dtype=B.MOE_WGRAD_FP32)
        assert B.moe_ctx_size(s16) == B.moe_ctx_size(s32) > 0
        assert B.moe_workspace_size(s16) == B.moe_workspace_size(s32) > 0
        assert B.moe_stream_ctx_size(s16, 4) == B.moe_stream_ctx_size(s32, 4) > 0


@pytest.mark.parametrize("bad", [
    dict(T=-1), dict(d=0), dict(d=200), dict(I=100), dict(E=0), dict(E=513), dict(top_k=0), dict(top_k=17),
    dict(E=4, top_k=5), dict(first_local_expert=-1), dict(first_local_expert=6, num_local_experts=4),
    dict(wgrad_dtype=2), dict(wgrad_dtype=-1),
])
def test_invalid_shapes_size_zero(bad):
    kw = dict(T=64, d=256, E=8, I=256, top_k=2)
    kw.update(bad)
    s = B.make_shape(**kw)
    assert B.moe_ctx_size(s) == 0 and B.moe_workspace_size(s) == 0


def test_argument_errors_are_synchronous(lib):
    s = B.make_shape(64, 256, 8, 256, 2)
    nc, nw = B.moe_ctx_size(s), B.moe_workspace_size(s)
    fake = 1 << 20  # never dereferenced: validation fails first
    ok = dict(X=fake, W_r=fake, bias=None, W_gate=fake, W_up=fake, W_down=fake, Y=fake, ctx=fake, ws=fake)

    def fwd(**over):
        a = dict(ok, **over)
        return B.moe_fwd(s, a["X"], a["W_r"], a["bias"], a["W_gate"], a["W_up"], a["W_down"], a["Y"], a["ctx"],
                         a["ws"], stream=0, ctx_bytes=over.get("cb", nc), ws_bytes=over.get("wb", nw))

    assert fwd(X=None) == B.MOE_ERR_INVALID_ARG
    assert fwd(ctx=None) == B.MOE_ERR_INVALID_ARG
    assert fwd(X=fake + 2) == B.MOE_ERR_INVALID_ARG  # misaligned
    assert fwd(cb=nc - 1) == B.MOE_ERR_WORKSPACE_TOO_SMALL
    assert fwd(wb=nw - 1) == B.MOE_ERR_WORKSPACE_TOO_SMALL
    bad = B.make_shape(64, 256, 8, 256, 9)
    assert B.moe_fwd(bad, *[fake] * 2, None, *[fake] * 5, nc, fake, nw, 0) == B.MOE_ERR_UNSUPPORTED
    mx = B.make_shape(64, 256, 8, 256, 2, prec=B.MOE_MXFP8)
    assert B.moe_fwd(mx, *[fake] * 2, None, *[fake] * 5, nc, fake, nw, 0) == B.MOE_ERR_UNSUPPORTED
    r = B.moe_bwd(s, fake, fake, fake, fake, fake, None, fake, fake, fake, fake, fake, fake, fake, stream=0,
                  ctx_bytes=nc, ws_bytes=nw)
    assert r == B.MOE_ERR_INVALID_ARG  # dY missing
    for wd in (2, -1):  # a weight-gradient dtype other than bf16 (0) or fp32 (1): refused before any launch
        sw = B.make_shape(64, 256, 8, 256, 2, wgrad_dtype=wd)
        r = B.moe_bwd(sw, *[fake] * 6, fake, fake, fake, fake, fake, fake, fake, stream=0, ctx_bytes=nc, ws_bytes=nw)
        assert r == B.MOE_ERR_UNSUPPORTED
    assert B.moe_get_error(None, 0) == B.MOE_ERR_INVALID_ARG
    for code in range(7):
        assert B.status_string(code)


def test_stream_shapes_and_sizes():
    s = B.make_shape(2048, 7168, 384, 2048, 8, first_local_expert=0, num_local_experts=6)
    assert B.moe_stream_ctx_size(s, 16) > 0 and B.moe_stream_workspace_size(s, 16) > 0
    # one minibatch's worst case: T*min(k, El) rows + 127 pad rows per local expert, in 128-row tiles
    rows = -(-(2048 * 6 + 127 * 6) // 128) * 128
    assert B.moe_stream_min_ring_bytes(s) == rows * 7168 * 2
    for M in (0, -1, 257):
        assert B.moe_stream_ctx_size(s, M) == 0 and B.moe_stream_workspace_size(s, M) == 0
    ragged = B.make_shape(2050, 7168, 384, 2048, 8)  # minibatches are whole 16-token blocks
    assert B.moe_stream_ctx_size(ragged, 4) == 0 and B.moe_stream_min_ring_bytes(ragged) == 0
    # MXFP8 streams with bf16 weight gradients: the same ctx (X's codes live in the ring), a workspace
    # larger by the backward's fp8 operands; with MXFP8 weight gradients ctx also keeps X's codes
    # along the rows, and the ring holds codes only
    mx = B.make_shape(2048, 7168, 384, 2048, 8, prec=B.MOE_MXFP8)
    bf = B.make_shape(2048, 7168, 384, 2048, 8)
    assert B.moe_stream_ctx_size(mx, 4) == B.moe_stream_ctx_size(bf, 4) > 0
    assert B.moe_stream_workspace_size(mx, 4) > B.moe_stream_workspace_size(bf, 4) > 0
    rows = B.moe_stream_min_ring_bytes(bf) // (2 * 7168)
    assert B.moe_stream_min_ring_bytes(mx) == rows * (3 * 7168 + 7168 // 32)
    mxa = B.make_shape(2048, 7168, 384, 2048, 8, prec=B.MOE_MXFP8_ALL)
    assert B.moe_stream_ctx_size(mxa, 4) > B.moe_stream_ctx_size(mx, 4)
    assert B.moe_stream_min_ring_bytes(mxa) == rows * (7168 + 7168 // 32)


def test_stream_mx_argument_errors_are_synchronous(lib):
    s = B.make_shape(128, 256, 16, 256, 4, prec=B.MOE_MXFP8)
    M = 4
    nc, nw, nr = B.moe_stream_ctx_size(s, M), B.moe_stream_workspace_size(s, M), B.moe_stream_min_ring_bytes(s)
    nq = B.moe_weights_size(s)
    f = 1 << 20  # never dereferenced

    def fwd(shape=s, wq_bytes=nq, ring_bytes=nr, X=f, wq=f):
        return lib.moe_fwd_stream_mx(ctypes.byref(shape), M, X, f, None, wq, wq_bytes, f, f, nc, f, ring_bytes, f, nw,
                                     None)

    def bwd(shape=s, wq_bytes=nq):
        return lib.moe_bwd_stream_mx(ctypes.byref(shape), M, f, f, f, wq_bytes, f, f, nc, f, f, f, f, f, f, nr, f, nw,
                                     None)

    assert fwd(X=None) == B.MOE_ERR_INVALID_ARG
    assert fwd(wq=None) == B.MOE_ERR_INVALID_ARG
    assert fwd(wq_bytes=nq - 1) == B.MOE_ERR_WORKSPACE_TOO_SMALL
    assert fwd(ring_bytes=nr - 2 * 256) == B.MOE_ERR_WORKSPACE_TOO_SMALL
    assert bwd(wq_bytes=nq - 1) == B.MOE_ERR_WORKSPACE_TOO_SMALL
    bf = B.make_shape(128, 256, 16, 256, 4)  # the MX entry points take MXFP8 shapes only
    assert fwd(shape=bf) == B.MOE_ERR_UNSUPPORTED and bwd(shape=bf) == B.MOE_ERR_UNSUPPORTED
    # and the bf16 entry points refuse MXFP8 shapes
    assert lib.moe_fwd_stream(ctypes.byref(s), M, f, f, None, f, f, f, f, f, nc, f, nr, f, nw, None) == \
        B.MOE_ERR_UNSUPPORTED


def test_stream_argument_errors_are_synchronous(lib):
    s = B.make_shape(128, 256, 16, 256, 4)
    M = 4
    nc, nw, nr = B.moe_stream_ctx_size(s, M), B.moe_stream_workspace_size(s, M), B.moe_stream_min_ring_bytes(s)
    f = 1 << 20  # never dereferenced

    def fwd(ring_bytes=nr, X=f, ctx=f, M=M):
        return lib.moe_fwd_stream(ctypes.byref(s), M, X, f, None, f, f, f, f, ctx, nc, f, ring_bytes, f, nw, None)

    assert fwd(X=None) == B.MOE_ERR_INVALID_ARG
    assert fwd(X=f + 8) == B.MOE_ERR_INVALID_ARG  # misaligned
    assert fwd(M=0) == B.MOE_ERR_INVALID_ARG
    assert fwd(ring_bytes=nr - 512) == B.MOE_ERR_WORKSPACE_TOO_SMALL  # less than one minibatch
    r = lib.moe_bwd_stream(ctypes.byref(s), M, f, f, f, f, f, None, f, nc, f, f, f, f, f, f, nr, f, nw, None)
    assert r == B.MOE_ERR_INVALID_ARG  # dY missing


def test_mxfp8_sizes_and_argument_errors(lib):
    mx = B.make_shape(256, 256, 8, 512, 2, prec=B.MOE_MXFP8)
    bf = B.make_shape(256, 256, 8, 512, 2)
    nq = B.moe_weights_size(mx)
    # five prepared regions of E*d*I codes (W_gate and W_up together in the first) and 1/32 of scales
    assert nq >= 6 * 8 * 256 * 512 * 33 // 32
    assert B.moe_weights_size(bf) == 0
    nc, nw = B.moe_ctx_size(mx), B.moe_workspace_size(mx)
    assert nc > B.moe_ctx_size(bf) and nw > B.moe_workspace_size(bf)  # fp8 copies of the operands
    f = 1 << 20
    assert lib.moe_prepare_weights(ctypes.byref(mx), f, f, None, f, nq, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_prepare_weights(ctypes.byref(mx), f, f, f, f, nq - 1, None) == B.MOE_ERR_WORKSPACE_TOO_SMALL
    # the MXFP8 entry points refuse a bf16 shape, the bf16 ones an MXFP8 shape
    assert lib.moe_fwd_mx(ctypes.byref(bf), f, f, None, f, nq, f, f, nc, f, nw, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_fwd_mx(ctypes.byref(mx), f, f, None, f, nq - 1, f, f, nc, f, nw, None) == \
        B.MOE_ERR_WORKSPACE_TOO_SMALL
    r = lib.moe_bwd_mx(ctypes.byref(mx), f, f, f, nq, None, f, nc, f, f, f, f, f, f, nw, None)
    assert r == B.MOE_ERR_INVALID_ARG  # dY missing


def test_nvfp4_sizes_and_argument_errors(lib):
    nv = B.make_shape(256, 256, 8, 512, 2, prec=B.MOE_NVFP4)
    mx = B.make_shape(256, 256, 8, 512, 2, prec=B.MOE_MXFP8)
    bf = B.make_shape(256, 256, 8, 512, 2)
    nq = B.moe_weights_size(nv)
    # five prepared regions at half a byte per value and one scale byte per 16 values
    assert nq >= 6 * 8 * 256 * 512 * 9 // 16 and nq < B.moe_weights_size(mx)
    nc, nw = B.moe_ctx_size(nv), B.moe_workspace_size(nv)
    assert nc > 0 and nw > B.moe_workspace_size(bf)  # fp32 H, dA, dB and the codes
    offs = B.moe_debug_nv_offsets(nv)
    assert len(offs) == 23 and all(o % 256 == 0 for o in offs)
    assert max(offs[0:2]) < nc and max(offs[2:6] + offs[11:17]) < nw and max(offs[6:11] + offs[17:23]) < nq
    with pytest.raises(B.MoeError):
        B.moe_debug_nv_offsets(mx)
    f = 1 << 20  # never dereferenced: every check below comes before any launch
    by = ctypes.byref
    assert lib.moe_prepare_weights(by(nv), f, f, None, f, nq, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_prepare_weights(by(nv), f, f, f, f, nq - 1, None) == B.MOE_ERR_WORKSPACE_TOO_SMALL
    # the NVFP4 entry points refuse other precisions, and the MXFP8 / bf16 ones an NVFP4 shape
    for other in (bf, mx):
        assert lib.moe_fwd_nvfp4(by(other), f, f, None, f, nq, f, f, nc, f, nw, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_fwd_mx(by(nv), f, f, None, f, nq, f, f, nc, f, nw, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_fwd(by(nv), f, f, None, f, f, f, f, f, nc, f, nw, None) != B.MOE_OK
    assert lib.moe_fwd_nvfp4(by(nv), f, f, None, f, nq - 1, f, f, nc, f, nw, None) == B.MOE_ERR_WORKSPACE_TOO_SMALL
    assert lib.moe_fwd_nvfp4(by(nv), f, f, None, f, nq, f, f, nc, f, nw - 1, None) == B.MOE_ERR_WORKSPACE_TOO_SMALL
    assert lib.moe_fwd_nvfp4(by(nv), f + 8, f, None, f, nq, f, f, nc, f, nw, None) == B.MOE_ERR_INVALID_ARG
    r = lib.moe_bwd_nvfp4(by(nv), f, f, f, nq, None, f, nc, f, f, f, f, f, f, nw, None)
    assert r == B.MOE_ERR_INVALID_ARG  # dY missing
    r = lib.moe_bwd_nvfp4(by(nv), f, f, f, nq, f, f, nc - 1, f, f, f, f, f, f, nw, None)
    assert r == B.MOE_ERR_WORKSPACE_TOO_SMALL


def test_expert_parallel_sizes_and_argument_errors(lib):
    s = B.make_shape(64, 256, 8, 256, 2)
    assert B.moe_ep_buffer_size(s, 3) == 0 and B.moe_ep_ctx_size(s, 3) == 0  # E not a multiple of R
    assert B.moe_ep_buffer_size(s, 0) == 0 and B.moe_ep_buffer_size(s, 65) == 0
    nb, nc, nw = B.moe_ep_buffer_size(s, 2), B.moe_ep_ctx_size(s, 2), B.moe_ep_workspace_size(s, 2)
    assert nb > 0 and nc > 0 and nw > 0
    assert B.moe_ep_buffer_size(B.make_shape(128, 256, 8, 256, 2), 2) > nb  # more tokens, larger exchange
    mx = B.make_shape(64, 256, 8, 256, 2, prec=B.MOE_MXFP8)
    assert B.moe_ep_buffer_size(mx, 2) == 0
    fake = 1 << 20  # never dereferenced: every check below comes before any launch
    good, keep1 = B._ptr_array([fake, fake + 4096])
    misaligned, keep2 = B._ptr_array([fake, fake + 16])
    by = ctypes.byref

    def route(shape, R, rank, bufs, ctx_bytes=nc, ws_bytes=nw):
        return lib.moe_ep_fwd_route(by(shape), R, rank, bufs, fake, fake, None, fake, ctx_bytes, fake, ws_bytes, 1,
                                    None)
    assert route(s, 2, 2, good) == B.MOE_ERR_INVALID_ARG      # rank out of range
    assert route(s, 2, -1, good) == B.MOE_ERR_INVALID_ARG
    assert route(s, 3, 0, good) == B.MOE_ERR_INVALID_ARG      # E = 8 over 3 ranks
    assert route(s, 2, 0, misaligned) == B.MOE_ERR_INVALID_ARG
    assert route(s, 2, 0, None) == B.MOE_ERR_INVALID_ARG
    assert route(s, 2, 0, good, ctx_bytes=nc - 1) == B.MOE_ERR_WORKSPACE_TOO_SMALL
    assert route(s, 2, 0, good, ws_bytes=nw - 1) == B.MOE_ERR_WORKSPACE_TOO_SMALL
    assert route(mx, 2, 0, good) == B.MOE_ERR_UNSUPPORTED
    assert lib.moe_ep_fwd_combine(by(s), 2, 0, good, None, fake, nc, 1, None) == B.MOE_ERR_INVALID_ARG  # no Y
    assert lib.moe_ep_bwd_finish(by(s), 2, 0, good, fake, fake, fake, None, fake, nc, fake, nw, 1,
                                 None) == B.MOE_ERR_INVALID_ARG  # no dW_r


def test_binding_refuses_tensors_of_the_wrong_shape_before_any_call(lib):
    # The C ABI takes bare pointers; the binding checks every tensor against the layer's shape
    # (here a 2-expert slice of 8) and raises before the library sees a pointer.  Host tensors
    # suffice: nothing reaches the device.
    import torch
    T, d, E, I, k = 16, 256, 8, 256, 2
    lay = B.MoELayer(T, d, E, I, k, first_local_expert=2, num_local_experts=2, device="cpu")
    bf = torch.bfloat16
    X, W_r = torch.zeros(T, d, dtype=bf), torch.zeros(d, E, dtype=bf)
    Wg, Wu, Wd = torch.zeros(2, d, I, dtype=bf), torch.zeros(2, d, I, dtype=bf), torch.zeros(2, I, d, dtype=bf)
    full = torch.zeros(E, d, I, dtype=bf)  # every expert's weights, not the slice's
    with pytest.raises(ValueError, match="W_gate"):
        lay.forward(X, W_r, None, full, Wu, Wd)
    with pytest.raises(ValueError, match="X"):
        lay.forward(torch.zeros(T + 1, d, dtype=bf), W_r, None, Wg, Wu, Wd)
    with pytest.raises(ValueError, match="bias"):
        lay.forward(X, W_r, torch.zeros(E - 1), Wg, Wu, Wd)
    with pytest.raises(ValueError, match="contiguous"):
        lay.forward(X, W_r, None, Wg, Wu, torch.zeros(2, d, I, dtype=bf).transpose(1, 2))
    with pytest.raises(ValueError, match="dY"):
        lay.backward(X, W_r, Wg, Wu, Wd, torch.zeros(T, d + 1, dtype=bf))
    mx = B.MoELayerMX(T, d, E, I, k, 2, 2, device="cpu")
    with pytest.raises(ValueError, match="W_down"):
        mx.prepare(Wg, Wu, torch.zeros(E, I, d, dtype=bf))
