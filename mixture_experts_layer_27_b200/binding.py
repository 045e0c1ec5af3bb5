"""Thin ctypes binding of libmoe.so: the C entry points under the same names.

Only argument marshalling happens here (tensor -> device pointer, stream ->
handle).  Every step of the layer runs in the library's CUDA kernels; there
is no Python or CPU fallback: if the library is missing, loading it raises.
PyTorch is used for device memory and streams only.
"""
from __future__ import annotations

import ctypes
import os

from .build import LIB

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_WORKSPACE_TOO_SMALL = 3
MOE_ERR_CUDA = 4
MOE_ERR_DEVICE_TIMEOUT = 5
MOE_ERR_NONFINITE = 6
MOE_ERR_EXCHANGE = 7
MOE_BF16 = 0
MOE_MXFP8 = 1
MOE_MXFP8_ALL = 2  # MOE_MXFP8 with the weight-gradient GEMMs on MXFP8 too (operands along tokens)
MOE_NVFP4 = 3  # E2M1 operands, E4M3 scale per 16 along K, fp32 scale per tensor (bf16 weight gradients)
MOE_WGRAD_BF16 = 0
MOE_WGRAD_FP32 = 1


class moe_shape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d", ctypes.c_int32), ("E", ctypes.c_int32), ("I", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("prec", ctypes.c_int32), ("first_local_expert", ctypes.c_int32),
                ("num_local_experts", ctypes.c_int32), ("wgrad_dtype", ctypes.c_int32)]


def make_shape(T, d, E, I, top_k, prec=MOE_BF16, first_local_expert=0, num_local_experts=0,
               wgrad_dtype=MOE_WGRAD_BF16) -> moe_shape:
    return moe_shape(T, d, E, I, top_k, prec, first_local_expert, num_local_experts, wgrad_dtype)


def _wgrad_code(dtype) -> int:
    """moe_wgrad_dtype of a torch dtype (bfloat16 or float32)."""
    import torch
    if dtype == torch.bfloat16:
        return MOE_WGRAD_BF16
    if dtype == torch.float32:
        return MOE_WGRAD_FP32
    raise ValueError(f"expert weight gradients are bfloat16 or float32, not {dtype}")


def _expect(t, shape, name):
    """Refuses a tensor whose shape does not match the layer's: the C ABI takes bare device
    pointers and cannot see sizes, so a wrong tensor would otherwise be read or written out of
    bounds on the device.  None passes (optional arguments, empty batches)."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, this layer expects {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous (row-major)")


def _expect_layer(lay, T, X=None, W_r=None, bias=None, W_gate=None, W_up=None, W_down=None, Y=None, dY=None,
                  out=None):
    d, E, I, El = lay.d, lay.E, lay.I, lay.El
    _expect(X, (T, d), "X")
    _expect(W_r, (d, E), "W_r")
    _expect(bias, (E,), "bias")
    _expect(W_gate, (El, d, I), "W_gate")
    _expect(W_up, (El, d, I), "W_up")
    _expect(W_down, (El, I, d), "W_down")
    _expect(Y, (T, d), "Y")
    _expect(dY, (T, d), "dY")
    if out is not None:
        _expect(out["dX"], (T, d), "dX")
        _expect(out["dW_gate"], (El, d, I), "dW_gate")
        _expect(out["dW_up"], (El, d, I), "dW_up")
        _expect(out["dW_down"], (El, I, d), "dW_down")
        _expect(out["dW_r"], (d, E), "dW_r")


def _grad_buffers(T, d, E, I, El, wdt, dev) -> dict:
    import torch
    return dict(dX=torch.empty(T, d, dtype=torch.bfloat16, device=dev),
                dW_gate=torch.empty(El, d, I, dtype=wdt, device=dev),
                dW_up=torch.empty(El, d, I, dtype=wdt, device=dev),
                dW_down=torch.empty(El, I, d, dtype=wdt, device=dev),
                dW_r=torch.empty(d, E, dtype=torch.float32, device=dev))


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} ({status})")
        self.status = status


_lib = None
_P = ctypes.c_void_p
_S = ctypes.POINTER(moe_shape)
_PP = ctypes.POINTER(ctypes.c_void_p)

_SIGS = {
    "moe_ctx_size": (ctypes.c_size_t, [_S]),
    "moe_workspace_size": (ctypes.c_size_t, [_S]),
    "moe_fwd": (ctypes.c_int, [_S, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P, ctypes.c_size_t, _P]),
    "moe_fwd_persistent": (ctypes.c_int, [_S, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P, ctypes.c_size_t,
                                          _P]),
    "moe_bwd": (ctypes.c_int, [_S, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P, _P, _P, _P, _P, _P,
                               ctypes.c_size_t, _P]),
    "moe_bwd_persistent": (ctypes.c_int, [_S, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P, _P, _P, _P, _P, _P,
                                          ctypes.c_size_t, _P]),
    "moe_get_error": (ctypes.c_int, [_P, _P]),
    "moe_debug_routing": (ctypes.c_int, [_S, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_debug_logits": (ctypes.c_int, [_S, _P, _P, _P]),
    "moe_debug_router_grad": (ctypes.c_int, [_S, _P, _P, _P]),
    "moe_debug_mx_wgrad_operand": (ctypes.c_int, [_S, _P, _P, ctypes.c_int32, _P, _P, _P]),
    "moe_padded_rows": (ctypes.c_int64, [_S]),
    "moe_debug_bounded_wait": (ctypes.c_int, [_S, _P, ctypes.c_size_t, _P]),
    "moe_debug_pair_wait": (ctypes.c_int, [_S, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P, ctypes.c_size_t,
                                           _P]),
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_profile_enable": (ctypes.c_int, [ctypes.c_int]),
    "moe_profile_read": (ctypes.c_int, [ctypes.c_int, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int)]),
    "moe_kernel_name": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_kernel_launches": (ctypes.c_ulonglong, []),
    "moe_route_static": (ctypes.c_int, [_S, _P, _P, _P, _P, _P, _P, _P]),
    "moe_stream_ctx_size": (ctypes.c_size_t, [_S, ctypes.c_int32]),
    "moe_stream_workspace_size": (ctypes.c_size_t, [_S, ctypes.c_int32]),
    "moe_stream_min_ring_bytes": (ctypes.c_size_t, [_S]),
    "moe_fwd_stream": (ctypes.c_int, [_S, ctypes.c_int32, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P,
                                      ctypes.c_size_t, _P, ctypes.c_size_t, _P]),
    "moe_bwd_stream": (ctypes.c_int, [_S, ctypes.c_int32, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P, _P, _P,
                                      _P, _P, _P, ctypes.c_size_t, _P, ctypes.c_size_t, _P]),
    "moe_debug_stream_plan": (ctypes.c_int, [_S, ctypes.c_int32, _P, _P, _P]),
    "moe_weights_size": (ctypes.c_size_t, [_S]),
    "moe_prepare_weights": (ctypes.c_int, [_S, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_fwd_stream_mx": (ctypes.c_int, [_S, ctypes.c_int32, _P, _P, _P, _P, ctypes.c_size_t, _P, _P, ctypes.c_size_t,
                                         _P, ctypes.c_size_t, _P, ctypes.c_size_t, _P]),
    "moe_bwd_stream_mx": (ctypes.c_int, [_S, ctypes.c_int32, _P, _P, _P, ctypes.c_size_t, _P, _P, ctypes.c_size_t,
                                         _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P, ctypes.c_size_t, _P]),
    "moe_fwd_mx": (ctypes.c_int, [_S, _P, _P, _P, _P, ctypes.c_size_t, _P, _P, ctypes.c_size_t, _P, ctypes.c_size_t,
                                  _P]),
    "moe_bwd_mx": (ctypes.c_int, [_S, _P, _P, _P, ctypes.c_size_t, _P, _P, ctypes.c_size_t, _P, _P, _P, _P, _P, _P,
                                  ctypes.c_size_t, _P]),
    "moe_fwd_nvfp4": (ctypes.c_int, [_S, _P, _P, _P, _P, ctypes.c_size_t, _P, _P, ctypes.c_size_t, _P,
                                     ctypes.c_size_t, _P]),
    "moe_bwd_nvfp4": (ctypes.c_int, [_S, _P, _P, _P, ctypes.c_size_t, _P, _P, ctypes.c_size_t, _P, _P, _P, _P, _P,
                                     _P, ctypes.c_size_t, _P]),
    "moe_debug_nv_offsets": (ctypes.c_int, [_S, ctypes.POINTER(ctypes.c_int64)]),
    "moe_ep_buffer_size": (ctypes.c_size_t, [_S, ctypes.c_int32]),
    "moe_ep_ctx_size": (ctypes.c_size_t, [_S, ctypes.c_int32]),
    "moe_ep_workspace_size": (ctypes.c_size_t, [_S, ctypes.c_int32]),
    "moe_ep_fwd_route": (ctypes.c_int, [_S, ctypes.c_int32, ctypes.c_int32, _PP, _P, _P, _P, _P, ctypes.c_size_t, _P,
                                        ctypes.c_size_t, ctypes.c_int32, _P]),
    "moe_ep_fwd_experts": (ctypes.c_int, [_S, ctypes.c_int32, ctypes.c_int32, _PP, _P, _P, _P, _P, ctypes.c_size_t,
                                          _P, ctypes.c_size_t, ctypes.c_int32, _P]),
    "moe_ep_fwd_combine": (ctypes.c_int, [_S, ctypes.c_int32, ctypes.c_int32, _PP, _P, _P, ctypes.c_size_t,
                                          ctypes.c_int32, _P]),
    "moe_ep_bwd_publish": (ctypes.c_int, [_S, ctypes.c_int32, ctypes.c_int32, _PP, _P, _P, ctypes.c_size_t,
                                          ctypes.c_int32, _P]),
    "moe_ep_bwd_experts": (ctypes.c_int, [_S, ctypes.c_int32, ctypes.c_int32, _PP, _P, _P, _P, _P, _P, _P, _P,
                                          ctypes.c_size_t, _P, ctypes.c_size_t, ctypes.c_int32, _P]),
    "moe_ep_bwd_finish": (ctypes.c_int, [_S, ctypes.c_int32, ctypes.c_int32, _PP, _P, _P, _P, _P, _P,
                                         ctypes.c_size_t, _P, ctypes.c_size_t, ctypes.c_int32, _P]),
    "moe_ep_debug_plan": (ctypes.c_int, [_S, ctypes.c_int32, ctypes.c_int32, _P, _P, _P, _P, _P]),
}


def lib() -> ctypes.CDLL:
    """The loaded libmoe.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise RuntimeError(f"{LIB} is missing: build it with `python -m mixture_experts_layer_27_b200.build`")
        h = ctypes.CDLL(LIB)
        for name, (res, args) in _SIGS.items():
            f = getattr(h, name)
            f.restype = res
            f.argtypes = args
        _lib = h
    return _lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _nbytes(t):
    return t.numel() * t.element_size()


def status_string(status: int) -> str:
    return lib().moe_status_string(int(status)).decode()


def moe_ctx_size(shape: moe_shape) -> int:
    return int(lib().moe_ctx_size(ctypes.byref(shape)))


def moe_workspace_size(shape: moe_shape) -> int:
    return int(lib().moe_workspace_size(ctypes.byref(shape)))


def moe_fwd(shape, X, W_r, bias, W_gate, W_up, W_down, Y, ctx, ws, stream=None, ctx_bytes=None, ws_bytes=None):
    return int(lib().moe_fwd(ctypes.byref(shape), _ptr(X), _ptr(W_r), _ptr(bias), _ptr(W_gate), _ptr(W_up),
                             _ptr(W_down), _ptr(Y), _ptr(ctx), ctx_bytes if ctx_bytes is not None else _nbytes(ctx),
                             _ptr(ws), ws_bytes if ws_bytes is not None else _nbytes(ws), _stream(stream)))


def moe_fwd_persistent(shape, X, W_r, bias, W_gate, W_up, W_down, Y, ctx, ws, stream=None, ctx_bytes=None,
                       ws_bytes=None):
    return int(lib().moe_fwd_persistent(ctypes.byref(shape), _ptr(X), _ptr(W_r), _ptr(bias), _ptr(W_gate),
                                        _ptr(W_up), _ptr(W_down), _ptr(Y), _ptr(ctx),
                                        ctx_bytes if ctx_bytes is not None else _nbytes(ctx), _ptr(ws),
                                        ws_bytes if ws_bytes is not None else _nbytes(ws), _stream(stream)))


def moe_bwd(shape, X, W_r, W_gate, W_up, W_down, dY, ctx, dX, dW_gate, dW_up, dW_down, dW_r, ws, stream=None,
            ctx_bytes=None, ws_bytes=None, persistent=False):
    fn = lib().moe_bwd_persistent if persistent else lib().moe_bwd
    return int(fn(ctypes.byref(shape), _ptr(X), _ptr(W_r), _ptr(W_gate), _ptr(W_up), _ptr(W_down), _ptr(dY),
                  _ptr(ctx), ctx_bytes if ctx_bytes is not None else _nbytes(ctx), _ptr(dX), _ptr(dW_gate),
                  _ptr(dW_up), _ptr(dW_down), _ptr(dW_r), _ptr(ws), ws_bytes if ws_bytes is not None else _nbytes(ws),
                  _stream(stream)))


def moe_get_error(ctx, stream=None) -> int:
    return int(lib().moe_get_error(_ptr(ctx), _stream(stream)))


def moe_debug_routing(shape, ctx, ids=None, gates=None, counts=None, offsets=None, padded_offsets=None, perm=None,
                      slot_row=None, stream=None) -> int:
    return int(lib().moe_debug_routing(ctypes.byref(shape), _ptr(ctx), _ptr(ids), _ptr(gates), _ptr(counts),
                                       _ptr(offsets), _ptr(padded_offsets), _ptr(perm), _ptr(slot_row),
                                       _stream(stream)))


def moe_debug_logits(shape, ws, logits, stream=None) -> int:
    return int(lib().moe_debug_logits(ctypes.byref(shape), _ptr(ws), _ptr(logits), _stream(stream)))


def moe_debug_pair_wait(shape, X, W_r, bias, W_gate, W_up, W_down, Y, ctx, ws, stream=None) -> int:
    return int(lib().moe_debug_pair_wait(ctypes.byref(shape), _ptr(X), _ptr(W_r), _ptr(bias), _ptr(W_gate),
                                         _ptr(W_up), _ptr(W_down), _ptr(Y), _ptr(ctx), _nbytes(ctx), _ptr(ws),
                                         _nbytes(ws), _stream(stream)))


def moe_debug_bounded_wait(shape, ctx, stream=None) -> int:
    return int(lib().moe_debug_bounded_wait(ctypes.byref(shape), _ptr(ctx), _nbytes(ctx), _stream(stream)))


def moe_debug_mx_wgrad_operand(shape, ctx, ws, which, codes, scales, stream=None) -> int:
    return int(lib().moe_debug_mx_wgrad_operand(ctypes.byref(shape), _ptr(ctx), _ptr(ws), int(which), _ptr(codes),
                                                _ptr(scales), _stream(stream)))


def moe_padded_rows(shape) -> int:
    return int(lib().moe_padded_rows(ctypes.byref(shape)))


def moe_debug_router_grad(shape, ws, dl, stream=None) -> int:
    return int(lib().moe_debug_router_grad(ctypes.byref(shape), _ptr(ws), _ptr(dl), _stream(stream)))


def moe_profile_enable(on: bool) -> int:
    return int(lib().moe_profile_enable(1 if on else 0))


def moe_profile_read(max_kernels: int = 64) -> dict:
    """{kernel name: (total ms, launches)} since the last read (synchronises the device)."""
    ms = (ctypes.c_double * max_kernels)()
    n = (ctypes.c_int * max_kernels)()
    k = int(lib().moe_profile_read(max_kernels, ms, n))
    if k < 0:
        raise MoeError(MOE_ERR_CUDA, "moe_profile_read")
    return {moe_kernel_name(i): (ms[i], n[i]) for i in range(k) if n[i] > 0}


def moe_kernel_name(kernel_id: int) -> str:
    return lib().moe_kernel_name(int(kernel_id)).decode()


def moe_kernel_launches() -> int:
    return int(lib().moe_kernel_launches())


def moe_route_static(shape, X, W_r, bias, ids, gates, status=None, stream=None) -> int:
    """Router + top-k gating with the library's static scratch (no allocation)."""
    return int(lib().moe_route_static(ctypes.byref(shape), _ptr(X), _ptr(W_r), _ptr(bias), _ptr(ids), _ptr(gates),
                                      _ptr(status), _stream(stream)))


def moe_stream_ctx_size(shape, M) -> int:
    return int(lib().moe_stream_ctx_size(ctypes.byref(shape), int(M)))


def moe_stream_workspace_size(shape, M) -> int:
    return int(lib().moe_stream_workspace_size(ctypes.byref(shape), int(M)))


def moe_stream_min_ring_bytes(shape) -> int:
    return int(lib().moe_stream_min_ring_bytes(ctypes.byref(shape)))


def moe_fwd_stream(shape, M, X, W_r, bias, W_gate, W_up, W_down, Y, ctx, ring, ws, stream=None):
    return int(lib().moe_fwd_stream(ctypes.byref(shape), int(M), _ptr(X), _ptr(W_r), _ptr(bias), _ptr(W_gate),
                                    _ptr(W_up), _ptr(W_down), _ptr(Y), _ptr(ctx), _nbytes(ctx), _ptr(ring),
                                    _nbytes(ring), _ptr(ws), _nbytes(ws), _stream(stream)))


def moe_bwd_stream(shape, M, X, W_r, W_gate, W_up, W_down, dY, ctx, dX, dW_gate, dW_up, dW_down, dW_r, ring, ws,
                   stream=None):
    return int(lib().moe_bwd_stream(ctypes.byref(shape), int(M), _ptr(X), _ptr(W_r), _ptr(W_gate), _ptr(W_up),
                                    _ptr(W_down), _ptr(dY), _ptr(ctx), _nbytes(ctx), _ptr(dX), _ptr(dW_gate),
                                    _ptr(dW_up), _ptr(dW_down), _ptr(dW_r), _ptr(ring), _nbytes(ring), _ptr(ws),
                                    _nbytes(ws), _stream(stream)))


def moe_debug_stream_plan(shape, M, ctx, tables, stream=None) -> int:
    return int(lib().moe_debug_stream_plan(ctypes.byref(shape), int(M), _ptr(ctx), _ptr(tables), _stream(stream)))


def moe_weights_size(shape) -> int:
    return int(lib().moe_weights_size(ctypes.byref(shape)))


def moe_prepare_weights(shape, W_gate, W_up, W_down, wq, stream=None) -> int:
    return int(lib().moe_prepare_weights(ctypes.byref(shape), _ptr(W_gate), _ptr(W_up), _ptr(W_down), _ptr(wq),
                                         _nbytes(wq), _stream(stream)))


def moe_fwd_stream_mx(shape, M, X, W_r, bias, wq, Y, ctx, ring, ws, stream=None) -> int:
    return int(lib().moe_fwd_stream_mx(ctypes.byref(shape), int(M), _ptr(X), _ptr(W_r), _ptr(bias), _ptr(wq),
                                       _nbytes(wq), _ptr(Y), _ptr(ctx), _nbytes(ctx), _ptr(ring), _nbytes(ring),
                                       _ptr(ws), _nbytes(ws), _stream(stream)))


def moe_bwd_stream_mx(shape, M, X, W_r, wq, dY, ctx, dX, dW_gate, dW_up, dW_down, dW_r, ring, ws,
                      stream=None) -> int:
    return int(lib().moe_bwd_stream_mx(ctypes.byref(shape), int(M), _ptr(X), _ptr(W_r), _ptr(wq), _nbytes(wq),
                                       _ptr(dY), _ptr(ctx), _nbytes(ctx), _ptr(dX), _ptr(dW_gate), _ptr(dW_up),
                                       _ptr(dW_down), _ptr(dW_r), _ptr(ring), _nbytes(ring), _ptr(ws), _nbytes(ws),
                                       _stream(stream)))


def moe_fwd_mx(shape, X, W_r, bias, wq, Y, ctx, ws, stream=None) -> int:
    return int(lib().moe_fwd_mx(ctypes.byref(shape), _ptr(X), _ptr(W_r), _ptr(bias), _ptr(wq), _nbytes(wq), _ptr(Y),
                                _ptr(ctx), _nbytes(ctx), _ptr(ws), _nbytes(ws), _stream(stream)))


def moe_bwd_mx(shape, X, W_r, wq, dY, ctx, dX, dW_gate, dW_up, dW_down, dW_r, ws, stream=None) -> int:
    return int(lib().moe_bwd_mx(ctypes.byref(shape), _ptr(X), _ptr(W_r), _ptr(wq), _nbytes(wq), _ptr(dY), _ptr(ctx),
                                _nbytes(ctx), _ptr(dX), _ptr(dW_gate), _ptr(dW_up), _ptr(dW_down), _ptr(dW_r),
                                _ptr(ws), _nbytes(ws), _stream(stream)))


def moe_fwd_nvfp4(shape, X, W_r, bias, wq, Y, ctx, ws, stream=None) -> int:
    return int(lib().moe_fwd_nvfp4(ctypes.byref(shape), _ptr(X), _ptr(W_r), _ptr(bias), _ptr(wq), _nbytes(wq),
                                   _ptr(Y), _ptr(ctx), _nbytes(ctx), _ptr(ws), _nbytes(ws), _stream(stream)))


def moe_bwd_nvfp4(shape, X, W_r, wq, dY, ctx, dX, dW_gate, dW_up, dW_down, dW_r, ws, stream=None) -> int:
    return int(lib().moe_bwd_nvfp4(ctypes.byref(shape), _ptr(X), _ptr(W_r), _ptr(wq), _nbytes(wq), _ptr(dY),
                                   _ptr(ctx), _nbytes(ctx), _ptr(dX), _ptr(dW_gate), _ptr(dW_up), _ptr(dW_down),
                                   _ptr(dW_r), _ptr(ws), _nbytes(ws), _stream(stream)))


def moe_debug_nv_offsets(shape) -> list:
    out = (ctypes.c_int64 * 23)()
    check(int(lib().moe_debug_nv_offsets(ctypes.byref(shape), out)), "moe_debug_nv_offsets")
    return [int(v) for v in out]


def check(status: int, what: str = "moe"):
    if status != MOE_OK:
        raise MoeError(status, what)


class MoELayerMX:
    """MXFP8 layer: prepared (quantised) weights + ctx / workspace owner.

    mx_wgrad: the weight-gradient GEMMs on MXFP8 as well (MOE_MXFP8_ALL), their operands
    quantised along each expert's rows; otherwise they contract the bf16 operands."""

    def __init__(self, T, d, E, I, top_k, first_local_expert=0, num_local_experts=0, device="cuda",
                 wgrad_dtype=None, mx_wgrad=False):
        import torch
        self.wgrad_dtype = wgrad_dtype or torch.bfloat16
        self.mx_wgrad = bool(mx_wgrad)
        self.shape = make_shape(T, d, E, I, top_k, MOE_MXFP8_ALL if mx_wgrad else MOE_MXFP8, first_local_expert,
                                num_local_experts, _wgrad_code(self.wgrad_dtype))
        self.shape_bf16 = make_shape(T, d, E, I, top_k, MOE_BF16, first_local_expert, num_local_experts)
        nc, nw, nq = moe_ctx_size(self.shape), moe_workspace_size(self.shape), moe_weights_size(self.shape)
        if nc == 0 or nw == 0 or nq == 0:
            raise MoeError(MOE_ERR_UNSUPPORTED, "shape")
        self.ctx = torch.empty(nc, dtype=torch.uint8, device=device)
        self.ws = torch.empty(nw, dtype=torch.uint8, device=device)
        self.wq = torch.empty(nq, dtype=torch.uint8, device=device)
        self.T, self.d, self.E, self.I, self.k = T, d, E, I, top_k
        self.El = num_local_experts or (E - first_local_expert)

    def prepare(self, W_gate, W_up, W_down, stream=None):
        _expect_layer(self, self.T, W_gate=W_gate, W_up=W_up, W_down=W_down)
        check(moe_prepare_weights(self.shape, W_gate, W_up, W_down, self.wq, stream), "moe_prepare_weights")

    def forward(self, X, W_r, bias, Y=None, stream=None):
        import torch
        if Y is None:
            Y = torch.empty(self.T, self.d, dtype=torch.bfloat16, device=X.device)
        _expect_layer(self, self.T, X=X, W_r=W_r, bias=bias, Y=Y)
        check(moe_fwd_mx(self.shape, X, W_r, bias, self.wq, Y, self.ctx, self.ws, stream), "moe_fwd_mx")
        return Y

    def backward(self, X, W_r, dY, out=None, stream=None):
        import torch
        if out is None:
            out = _grad_buffers(self.T, self.d, self.E, self.I, self.El, self.wgrad_dtype, X.device)
        _expect_layer(self, self.T, X=X, W_r=W_r, dY=dY, out=out)
        check(moe_bwd_mx(self.shape, X, W_r, self.wq, dY, self.ctx, out["dX"], out["dW_gate"], out["dW_up"],
                         out["dW_down"], out["dW_r"], self.ws, stream), "moe_bwd_mx")
        return out

    def wgrad_operand(self, which):
        """(codes [C, RP], scale bytes [C, RP / 32]) of weight-gradient operand `which` (0 X_perm,
        1 dY_perm, 2 dA, 3 dB, 4 Hg) from the last backward, as host numpy arrays, column c's codes
        and scales along the padded rows (MOE_MXFP8_ALL only; reordered here from the device's
        128-row-tile layout)."""
        import numpy as np
        import torch
        RP = moe_padded_rows(self.shape)
        C = self.d if which < 2 else self.I
        codes = torch.empty(C * RP, dtype=torch.uint8, device=self.ws.device)
        scales = torch.empty(C * RP // 32, dtype=torch.uint8, device=self.ws.device)
        check(moe_debug_mx_wgrad_operand(self.shape, self.ctx, self.ws, which, codes, scales),
              "moe_debug_mx_wgrad_operand")
        torch.cuda.synchronize()
        q = codes.cpu().numpy().reshape(RP // 128, C, 128).transpose(1, 0, 2).reshape(C, RP)
        ch = scales.cpu().numpy()
        c = np.arange(C)[:, None]
        kb = np.arange(RP // 32)[None, :]
        idx = ((kb // 4) * (C // 128) + c // 128) * 512 + (c % 32) * 16 + ((c % 128) // 32) * 4 + kb % 4
        return q, ch[idx]

    def weight_regions(self):
        """Host numpy views (codes [R, K], scale chunks) of the five prepared weights."""
        import numpy as np
        a = self.wq.cpu().numpy()
        El, d, I = self.El, self.d, self.I
        out, o = {}, 0
        for name, R, K in (("Wgu", El * 2 * I, d), ("Wd2", El * d, I), ("Wd3", El * I, d), ("Wg4", El * d, I),
                           ("Wu4", El * d, I)):
            codes = a[o:o + R * K].reshape(R, K)
            o = (o + R * K + 255) // 256 * 256
            sc = a[o:o + R * K // 32]
            o = (o + R * K // 32 + 255) // 256 * 256
            out[name] = (codes, sc, R, K)
        return out

    def routing(self):
        return MoELayer.routing(self)

    def logits(self):
        return MoELayer.logits(self)

    def router_grad(self):
        # the ws regions before the MXFP8-only ones sit where the bf16 layout puts them
        import torch
        out = torch.empty(self.T, self.k, dtype=torch.float32, device=self.ws.device)
        check(moe_debug_router_grad(self.shape_bf16, self.ws, out), "moe_debug_router_grad")
        return out

    def error(self, stream=None) -> int:
        return moe_get_error(self.ctx, stream)


class MoELayerNVFP4:
    """NVFP4 layer: prepared (quantised) weights + ctx / workspace owner."""

    def __init__(self, T, d, E, I, top_k, first_local_expert=0, num_local_experts=0, device="cuda"):
        import torch
        self.shape = make_shape(T, d, E, I, top_k, MOE_NVFP4, first_local_expert, num_local_experts)
        self.shape_bf16 = make_shape(T, d, E, I, top_k, MOE_BF16, first_local_expert, num_local_experts)
        nc, nw, nq = moe_ctx_size(self.shape), moe_workspace_size(self.shape), moe_weights_size(self.shape)
        if nc == 0 or nw == 0 or nq == 0:
            raise MoeError(MOE_ERR_UNSUPPORTED, "shape")
        self.ctx = torch.empty(nc, dtype=torch.uint8, device=device)
        self.ws = torch.empty(nw, dtype=torch.uint8, device=device)
        self.wq = torch.empty(nq, dtype=torch.uint8, device=device)
        self.T, self.d, self.E, self.I, self.k = T, d, E, I, top_k
        self.El = num_local_experts or (E - first_local_expert)
        self.off = moe_debug_nv_offsets(self.shape)

    def prepare(self, W_gate, W_up, W_down, stream=None):
        _expect_layer(self, self.T, W_gate=W_gate, W_up=W_up, W_down=W_down)
        check(moe_prepare_weights(self.shape, W_gate, W_up, W_down, self.wq, stream), "moe_prepare_weights")

    def forward(self, X, W_r, bias, Y=None, stream=None):
        import torch
        if Y is None:
            Y = torch.empty(self.T, self.d, dtype=torch.bfloat16, device=X.device)
        _expect_layer(self, self.T, X=X, W_r=W_r, bias=bias, Y=Y)
        check(moe_fwd_nvfp4(self.shape, X, W_r, bias, self.wq, Y, self.ctx, self.ws, stream), "moe_fwd_nvfp4")
        return Y

    def backward(self, X, W_r, dY, out=None, stream=None):
        import torch
        if out is None:
            out = _grad_buffers(self.T, self.d, self.E, self.I, self.El, torch.bfloat16, X.device)
        _expect_layer(self, self.T, X=X, W_r=W_r, dY=dY, out=out)
        check(moe_bwd_nvfp4(self.shape, X, W_r, self.wq, dY, self.ctx, out["dX"], out["dW_gate"], out["dW_up"],
                            out["dW_down"], out["dW_r"], self.ws, stream), "moe_bwd_nvfp4")
        return out

    # --- test accessors (host numpy copies; unpacked codes: one 4-bit code per byte) ---
    @staticmethod
    def _unpack(packed, R, K):
        import numpy as np
        b = np.asarray(packed, dtype=np.uint8).reshape(R, K // 2)
        out = np.empty((R, K), dtype=np.uint8)
        out[:, 0::2] = b & 0xF
        out[:, 1::2] = b >> 4
        return out

    def _operand(self, buf, o_codes, o_scales, R, K):
        a = buf.cpu().numpy()
        codes = self._unpack(a[o_codes:o_codes + R * K // 2], R, K)
        return codes, unchunk_scales_nv(a[o_scales:o_scales + R * K // 16], R, K)

    def x_operand(self):
        """(codes [RP, d], scale bytes [RP, d/16]) of the dispatched X of the last forward."""
        torch_sync()
        return self._operand(self.ctx, self.off[0], self.off[1], moe_padded_rows(self.shape_bf16), self.d)

    def h_operand(self):
        """(codes [RP, I], scale bytes [RP, I/16]) of the quantised H of the last forward."""
        torch_sync()
        return self._operand(self.ws, self.off[2], self.off[3], moe_padded_rows(self.shape_bf16), self.I)

    def h_fp32(self):
        import numpy as np
        torch_sync()
        RP = moe_padded_rows(self.shape_bf16)
        a = self.ws.cpu().numpy()
        return a[self.off[4]:self.off[4] + RP * self.I * 4].view(np.float32).reshape(RP, self.I)

    def scales(self):
        """(gs_X, gs_H) of the last forward and (gs_gate, gs_up, gs_down, gs_gate_up) of the
        prepared weights."""
        import numpy as np
        torch_sync()
        w = self.ws.cpu().numpy()[self.off[5]:self.off[5] + 32].view(np.float32)
        q = self.wq.cpu().numpy()[self.off[10]:self.off[10] + 16].view(np.float32)
        return (w[2], w[3]), tuple(q)

    def bwd_scales(self):
        """(gs_dY, gs_[dA | dB]) of the last backward."""
        import numpy as np
        torch_sync()
        w = self.ws.cpu().numpy()[self.off[5]:self.off[5] + 32].view(np.float32)
        return w[6], w[7]

    def dy_operand(self):
        """(codes [RP, d], scale bytes [RP, d/16]) of the quantised dY_perm of the last backward."""
        torch_sync()
        return self._operand(self.ws, self.off[11], self.off[12], moe_padded_rows(self.shape_bf16), self.d)

    def bwd_weight_regions(self):
        """{"Wd3": W_down [El*I, d], "Wg4": W_gate [El*d, I], "Wu4": W_up [El*d, I]}: (codes, scales)."""
        El, d, I = self.El, self.d, self.I
        return {"Wd3": self._operand(self.wq, self.off[17], self.off[18], El * I, d),
                "Wg4": self._operand(self.wq, self.off[19], self.off[20], El * d, I),
                "Wu4": self._operand(self.wq, self.off[21], self.off[22], El * d, I)}

    def weight_regions(self):
        """{"Wgu": (codes [El*2I, d], scales [El*2I, d/16]), "Wd2": (codes [El*d, I], scales [El*d, I/16])}."""
        El, d, I = self.El, self.d, self.I
        return {"Wgu": self._operand(self.wq, self.off[6], self.off[7], El * 2 * I, d),
                "Wd2": self._operand(self.wq, self.off[8], self.off[9], El * d, I)}

    def routing(self):
        return MoELayer.routing(self)

    def logits(self):
        return MoELayer.logits(self)

    def error(self, stream=None) -> int:
        return moe_get_error(self.ctx, stream)


def torch_sync():
    import torch
    torch.cuda.synchronize()


def unchunk_scales_nv(chunks, R, K):
    """[R, K/16] scale bytes from the 512-byte chunk order of a K-major NVFP4 operand."""
    import numpy as np
    r = np.arange(R)[:, None]
    kb = np.arange(K // 16)[None, :]
    idx = ((r // 128) * (K // 64) + kb // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + kb % 4
    return np.asarray(chunks)[idx]


def unchunk_scales(chunks, R, K):
    """[R, K/32] scale bytes from the 512-byte chunk order of a K-major fp8 operand."""
    import numpy as np
    r = np.arange(R)[:, None]
    kb = np.arange(K // 32)[None, :]
    idx = ((r // 128) * (K // 128) + (kb * 32) // 128) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + kb % 4
    return chunks[idx]


# ---------------------------------------------------------------------------
# expert parallelism across R ranks (argument marshalling only)
# ---------------------------------------------------------------------------
def _ptr_array(bufs):
    arr = (ctypes.c_void_p * len(bufs))(*[_ptr(b) for b in bufs])
    return ctypes.cast(arr, _PP), arr


def moe_ep_buffer_size(shape, R) -> int:
    return int(lib().moe_ep_buffer_size(ctypes.byref(shape), int(R)))


def moe_ep_ctx_size(shape, R) -> int:
    return int(lib().moe_ep_ctx_size(ctypes.byref(shape), int(R)))


def moe_ep_workspace_size(shape, R) -> int:
    return int(lib().moe_ep_workspace_size(ctypes.byref(shape), int(R)))


class MoEExpertParallel:
    """One rank of the expert-parallel layer: its ctx / workspace, and the R ranks' exchange
    buffers (device memory this process can address: peer mappings across GPUs, or all on one
    device).  Each step runs three forward phases and three backward phases on every rank; a
    phase's waits are satisfied by the other ranks' earlier phases of the same step (epoch)."""

    def __init__(self, T, d, E, I, top_k, R, rank, bufs, device="cuda", wgrad_dtype=None):
        import torch
        self.wgrad_dtype = wgrad_dtype or torch.bfloat16
        self.shape = make_shape(T, d, E, I, top_k, MOE_BF16, 0, 0, _wgrad_code(self.wgrad_dtype))
        nc, nw = moe_ep_ctx_size(self.shape, R), moe_ep_workspace_size(self.shape, R)
        if nc == 0 or nw == 0:
            raise MoeError(MOE_ERR_UNSUPPORTED, "expert-parallel shape")
        self.ctx = torch.empty(nc, dtype=torch.uint8, device=device)
        self.ws = torch.empty(nw, dtype=torch.uint8, device=device)
        self.T, self.d, self.E, self.I, self.k, self.R, self.rank = T, d, E, I, top_k, R, rank
        self.El = E // R
        self._bufs, self._keep = _ptr_array(bufs)

    def _call(self, name, *args, stream=None):
        check(int(getattr(lib(), name)(ctypes.byref(self.shape), self.R, self.rank, self._bufs, *args,
                                      _stream(stream))), name)

    def fwd_route(self, X, W_r, bias, epoch, stream=None):
        self._call("moe_ep_fwd_route", _ptr(X), _ptr(W_r), _ptr(bias), _ptr(self.ctx), _nbytes(self.ctx),
                   _ptr(self.ws), _nbytes(self.ws), int(epoch), stream=stream)

    def fwd_experts(self, W_gate, W_up, W_down, epoch, stream=None):
        self._call("moe_ep_fwd_experts", _ptr(W_gate), _ptr(W_up), _ptr(W_down), _ptr(self.ctx), _nbytes(self.ctx),
                   _ptr(self.ws), _nbytes(self.ws), int(epoch), stream=stream)

    def fwd_combine(self, Y, epoch, stream=None):
        self._call("moe_ep_fwd_combine", _ptr(Y), _ptr(self.ctx), _nbytes(self.ctx), int(epoch), stream=stream)

    def bwd_publish(self, dY, epoch, stream=None):
        self._call("moe_ep_bwd_publish", _ptr(dY), _ptr(self.ctx), _nbytes(self.ctx), int(epoch), stream=stream)

    def bwd_experts(self, W_gate, W_up, W_down, dW_gate, dW_up, dW_down, epoch, stream=None):
        self._call("moe_ep_bwd_experts", _ptr(W_gate), _ptr(W_up), _ptr(W_down), _ptr(dW_gate), _ptr(dW_up),
                   _ptr(dW_down), _ptr(self.ctx), _nbytes(self.ctx), _ptr(self.ws), _nbytes(self.ws), int(epoch),
                   stream=stream)

    def bwd_finish(self, X, W_r, dX, dW_r, epoch, stream=None):
        self._call("moe_ep_bwd_finish", _ptr(X), _ptr(W_r), _ptr(dX), _ptr(dW_r), _ptr(self.ctx), _nbytes(self.ctx),
                   _ptr(self.ws), _nbytes(self.ws), int(epoch), stream=stream)

    def plan(self):
        """Owner-side plan of the last forward: rows per local expert [El], padded offsets [El+1],
        and each padded row's source (source rank * T k + assignment; -1 / -2 for pad rows)."""
        import torch
        dev = self.ctx.device
        counts = torch.empty(self.El, dtype=torch.int32, device=dev)
        poff = torch.empty(self.El + 1, dtype=torch.int32, device=dev)
        rows = torch.empty(self._rp(), dtype=torch.int32, device=dev)
        check(int(lib().moe_ep_debug_plan(ctypes.byref(self.shape), self.R, self.rank, _ptr(self.ctx), _ptr(counts),
                                          _ptr(poff), _ptr(rows), None)), "moe_ep_debug_plan")
        torch.cuda.synchronize()
        return dict(counts=counts, padded_offsets=poff, row_src=rows[:int(poff[-1].item())])

    def _rp(self):
        # padded-row capacity of the owner role: R T min(k, El) + 127 El, rounded up to 128
        A = self.R * self.T * min(self.k, self.El) + 127 * self.El
        return max((A + 127) // 128 * 128, 128)

    def error(self, stream=None):
        return moe_get_error(self.ctx, stream)


class MoEStream:
    """ctx / ring / workspace owner for the ring-streamed layer (M minibatches of T tokens)."""

    def __init__(self, T, d, E, I, top_k, M, ring_bytes, first_local_expert=0, num_local_experts=0, device="cuda",
                 wgrad_dtype=None):
        import torch
        self.wgrad_dtype = wgrad_dtype or torch.bfloat16
        self.shape = make_shape(T, d, E, I, top_k, MOE_BF16, first_local_expert, num_local_experts,
                                _wgrad_code(self.wgrad_dtype))
        nc, nw = moe_stream_ctx_size(self.shape, M), moe_stream_workspace_size(self.shape, M)
        if nc == 0 or nw == 0:
            raise MoeError(MOE_ERR_UNSUPPORTED, "stream shape")
        self.ctx = torch.empty(nc, dtype=torch.uint8, device=device)
        self.ws = torch.empty(nw, dtype=torch.uint8, device=device)
        self.ring = torch.empty(ring_bytes, dtype=torch.uint8, device=device)
        self.T, self.d, self.E, self.I, self.k, self.M = T, d, E, I, top_k, M
        self.El = num_local_experts or (E - first_local_expert)

    def forward(self, X, W_r, bias, W_gate, W_up, W_down, Y=None, stream=None):
        import torch
        if Y is None:
            Y = torch.empty(self.M * self.T, self.d, dtype=torch.bfloat16, device=X.device)
        _expect_layer(self, self.M * self.T, X=X, W_r=W_r, bias=bias, W_gate=W_gate, W_up=W_up, W_down=W_down, Y=Y)
        check(moe_fwd_stream(self.shape, self.M, X, W_r, bias, W_gate, W_up, W_down, Y, self.ctx, self.ring,
                             self.ws, stream), "moe_fwd_stream")
        return Y

    def backward(self, X, W_r, W_gate, W_up, W_down, dY, out=None, stream=None):
        import torch
        if out is None:
            out = _grad_buffers(self.M * self.T, self.d, self.E, self.I, self.El, self.wgrad_dtype, X.device)
        _expect_layer(self, self.M * self.T, X=X, W_r=W_r, W_gate=W_gate, W_up=W_up, W_down=W_down, dY=dY, out=out)
        check(moe_bwd_stream(self.shape, self.M, X, W_r, W_gate, W_up, W_down, dY, self.ctx, out["dX"],
                             out["dW_gate"], out["dW_up"], out["dW_down"], out["dW_r"], self.ring, self.ws, stream),
              "moe_bwd_stream")
        return out

    def plan(self) -> dict:
        """The device plan of the last forward, split into named tables (host numpy)."""
        return _stream_plan(self)

    def error(self, stream=None) -> int:
        return moe_get_error(self.ctx, stream)


class MoEStreamMX(MoEStream):
    """The ring-streamed layer in MXFP8 (gate/up, down and both dgrads on MXFP8 tensor cores):
    ctx / ring / workspace owner plus the prepared weights.  mx_wgrad: the weight-gradient GEMMs on
    MXFP8 too (MOE_MXFP8_ALL); otherwise bf16 (MOE_MXFP8)."""

    def __init__(self, T, d, E, I, top_k, M, ring_bytes, first_local_expert=0, num_local_experts=0, device="cuda",
                 wgrad_dtype=None, mx_wgrad=False):
        import torch
        self.wgrad_dtype = wgrad_dtype or torch.bfloat16
        self.mx_wgrad = bool(mx_wgrad)
        self.shape = make_shape(T, d, E, I, top_k, MOE_MXFP8_ALL if mx_wgrad else MOE_MXFP8, first_local_expert,
                                num_local_experts, _wgrad_code(self.wgrad_dtype))
        nc, nw = moe_stream_ctx_size(self.shape, M), moe_stream_workspace_size(self.shape, M)
        nq = moe_weights_size(self.shape)
        if nc == 0 or nw == 0 or nq == 0:
            raise MoeError(MOE_ERR_UNSUPPORTED, "stream shape")
        self.ctx = torch.empty(nc, dtype=torch.uint8, device=device)
        self.ws = torch.empty(nw, dtype=torch.uint8, device=device)
        self.wq = torch.empty(nq, dtype=torch.uint8, device=device)
        self.ring = torch.empty(ring_bytes, dtype=torch.uint8, device=device)
        self.T, self.d, self.E, self.I, self.k, self.M = T, d, E, I, top_k, M
        self.El = num_local_experts or (E - first_local_expert)

    def prepare(self, W_gate, W_up, W_down, stream=None):
        _expect_layer(self, self.M * self.T, W_gate=W_gate, W_up=W_up, W_down=W_down)
        check(moe_prepare_weights(self.shape, W_gate, W_up, W_down, self.wq, stream), "moe_prepare_weights")

    def forward(self, X, W_r, bias, Y=None, stream=None):
        import torch
        if Y is None:
            Y = torch.empty(self.M * self.T, self.d, dtype=torch.bfloat16, device=X.device)
        _expect_layer(self, self.M * self.T, X=X, W_r=W_r, bias=bias, Y=Y)
        check(moe_fwd_stream_mx(self.shape, self.M, X, W_r, bias, self.wq, Y, self.ctx, self.ring, self.ws, stream),
              "moe_fwd_stream_mx")
        return Y

    def backward(self, X, W_r, dY, out=None, stream=None):
        if out is None:
            out = _grad_buffers(self.M * self.T, self.d, self.E, self.I, self.El, self.wgrad_dtype, X.device)
        _expect_layer(self, self.M * self.T, X=X, W_r=W_r, dY=dY, out=out)
        check(moe_bwd_stream_mx(self.shape, self.M, X, W_r, self.wq, dY, self.ctx, out["dX"], out["dW_gate"],
                                out["dW_up"], out["dW_down"], out["dW_r"], self.ring, self.ws, stream),
              "moe_bwd_stream_mx")
        return out


def _stream_plan(layer) -> dict:
    """The device plan of a stream layer's last forward, split into named tables (host numpy)."""
    import torch
    M, El = layer.M, layer.El
    n = 16 + M + (M * El + 1) + M * El + 2 * M + 4 * M + 4 * M
    t = torch.empty(n, dtype=torch.int32, device=layer.ctx.device)
    check(moe_debug_stream_plan(layer.shape, M, layer.ctx, t), "moe_debug_stream_plan")
    torch.cuda.synchronize()
    a = t.cpu().numpy()
    out, o = {}, 0
    for name, size in (("plan", 16), ("mb_of", M), ("seg_poff", M * El + 1), ("cum", M * El),
                       ("mb_range", 2 * M), ("shift_fwd", M), ("shift_bwd", M), ("replay", M),
                       ("chunk", 4 * M), ("ring_start", M)):
        out[name] = a[o:o + size]
        o += size
    return out


class MoELayer:
    """Convenience owner of ctx / workspace buffers (allocated by torch) for one shape."""

    def __init__(self, T, d, E, I, top_k, prec=MOE_BF16, first_local_expert=0, num_local_experts=0,
                 device="cuda", wgrad_dtype=None):
        import torch
        self.wgrad_dtype = wgrad_dtype or torch.bfloat16
        self.shape = make_shape(T, d, E, I, top_k, prec, first_local_expert, num_local_experts,
                                _wgrad_code(self.wgrad_dtype))
        nc, nw = moe_ctx_size(self.shape), moe_workspace_size(self.shape)
        if nc == 0 or nw == 0:
            raise MoeError(MOE_ERR_UNSUPPORTED, "shape")
        self.ctx = torch.empty(nc, dtype=torch.uint8, device=device)
        self.ws = torch.empty(nw, dtype=torch.uint8, device=device)
        self.T, self.d, self.E, self.I, self.k = T, d, E, I, top_k
        self.El = num_local_experts or (E - first_local_expert)

    def forward(self, X, W_r, bias, W_gate, W_up, W_down, Y=None, stream=None, persistent=False):
        """persistent: the two GEMMs as one persistent launch (moe_fwd_persistent); same results."""
        import torch
        if Y is None:
            Y = torch.empty(self.T, self.d, dtype=torch.bfloat16, device=X.device)
        _expect_layer(self, self.T, X=X, W_r=W_r, bias=bias, W_gate=W_gate, W_up=W_up, W_down=W_down, Y=Y)
        fn, name = (moe_fwd_persistent, "moe_fwd_persistent") if persistent else (moe_fwd, "moe_fwd")
        check(fn(self.shape, X, W_r, bias, W_gate, W_up, W_down, Y, self.ctx, self.ws, stream), name)
        return Y

    def backward(self, X, W_r, W_gate, W_up, W_down, dY, out=None, stream=None, persistent=False):
        """persistent: the two dgrad GEMMs as one persistent launch (moe_bwd_persistent); same results."""
        import torch
        if out is None:
            out = _grad_buffers(self.T, self.d, self.E, self.I, self.El, self.wgrad_dtype, X.device)
        _expect_layer(self, self.T, X=X, W_r=W_r, W_gate=W_gate, W_up=W_up, W_down=W_down, dY=dY, out=out)
        check(moe_bwd(self.shape, X, W_r, W_gate, W_up, W_down, dY, self.ctx, out["dX"], out["dW_gate"],
                      out["dW_up"], out["dW_down"], out["dW_r"], self.ws, stream, persistent=persistent),
              "moe_bwd_persistent" if persistent else "moe_bwd")
        return out

    def routing(self):
        import torch
        T, k, El, dev = self.T, self.k, self.El, self.ctx.device
        r = dict(ids=torch.empty(T, k, dtype=torch.int32, device=dev),
                 gates=torch.empty(T, k, dtype=torch.float32, device=dev),
                 counts=torch.empty(El, dtype=torch.int32, device=dev),
                 offsets=torch.empty(El + 1, dtype=torch.int32, device=dev),
                 padded_offsets=torch.empty(El + 1, dtype=torch.int32, device=dev),
                 perm=torch.empty(max(T * k, 1), dtype=torch.int32, device=dev),
                 slot_row=torch.empty(T, k, dtype=torch.int32, device=dev))
        check(moe_debug_routing(getattr(self, "shape_bf16", self.shape), self.ctx, r["ids"], r["gates"], r["counts"],
                                r["offsets"],
                                r["padded_offsets"], r["perm"], r["slot_row"]), "moe_debug_routing")
        torch.cuda.synchronize()
        n = int(r["offsets"][-1].item())
        r["perm"] = r["perm"][:n]
        return r

    def logits(self):
        import torch
        out = torch.empty(self.T, self.E, dtype=torch.float32, device=self.ws.device)
        check(moe_debug_logits(getattr(self, "shape_bf16", self.shape), self.ws, out), "moe_debug_logits")
        return out

    def router_grad(self):
        import torch
        out = torch.empty(self.T, self.k, dtype=torch.float32, device=self.ws.device)
        check(moe_debug_router_grad(self.shape, self.ws, out), "moe_debug_router_grad")
        return out

    def error(self, stream=None) -> int:
        return moe_get_error(self.ctx, stream)
