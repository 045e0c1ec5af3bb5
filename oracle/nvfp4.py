"""Oracle of the NVFP4 layer, forward and backward (test infrastructure only).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this module:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
use it.  It shares no code, table or helper with the CUDA path.

What it follows
---------------
Page 1 ("Cursor open-sources Mixture-of-Kittens (MoK)...", section "MoE layer as
the bottleneck") names NVFP4 training kernels as earlier work and says nothing
of the format.  NVFP4 is taken here as NVIDIA publishes it:

* element: E2M1 (1 sign, 2 exponent bits with bias 1, 1 mantissa bit), the
  magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6;
* first level: one positive E4M3 scale per 16 consecutive values along the
  contraction dimension of the GEMM that reads them;
* second level: one fp32 scale per tensor, chosen so that the tensor's largest
  magnitude maps to the largest product of the two formats (6 x 448 = 2688).

Readings (the pages are silent, so each is the plainest one; all are listed in
the design notes):

* global scale  gs = 2688 / amax(tensor) in fp32 (amax = 0 gives gs = 1; an
  overflow is clamped to the largest fp32);
* block scale   s  = e4m3_rn_satfinite((amax_block / 6) * gs), fp32 steps;
* codes         q  = e2m1_rn_satfinite(v * (gs / s)), fp32 steps; a block whose
  scale rounds to 0 holds zeros;
* value         q * s / gs;
* every quantisation decision (scale byte, code) is taken in fp32, the
  kernels' precision, on the fp32 value of the input;
* "tensor" is the operand as the layer holds it: X [T, d] (one scale for all
  tokens), each of W_gate, W_up, W_down over the local experts, and H over all
  assigned rows of the layer; a GEMM's output is multiplied back by
  1 / (gs_A gs_B);
* H = silu(A) * B from the unrounded A, B (as in the MXFP8 oracle).

The backward (backward_nv) quantises the two dgrad GEMMs' operands the same way; the
dgrad of gate/up contracts over K = 2I, so its operands [dA | dB] and [W_gate | W_up] are each
one tensor with one global scale; the weight gradients take the unrounded operands.
"""

from __future__ import annotations

import numpy as np

from .moe_oracle import (_expert, _expert_rows, _f64, e4m3_decode, e4m3_encode, gates, router_logits,
                         schedule, silu, topk_ids)

NV_BLOCK = 16
E2M1_MAX = 6.0
NV_GS_NUM = 2688.0  # 6 * 448: the largest E2M1 magnitude times the largest E4M3 one

# E2M1 magnitudes by code (bits e1 e0 m): subnormal 0.5 at e = 0, then 1, 1.5, 2, 3, 4, 6
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_decode(codes) -> np.ndarray:
    """4-bit E2M1 codes (sign in bit 3) -> fp64."""
    c = np.asarray(codes, dtype=np.int64)
    return np.where(c & 8, -1.0, 1.0) * E2M1_GRID[c & 7]


def e2m1_encode(x) -> np.ndarray:
    """fp64 -> E2M1 code: nearest magnitude, halfway cases to the even code (mantissa bit 0),
    magnitudes above 6 saturate to 6.  The sign of a value that rounds to zero is kept."""
    x = _f64(x)
    a = np.minimum(np.abs(x), E2M1_MAX)
    # the code of a magnitude is the number of midpoints between neighbours lying below it; a
    # magnitude on a midpoint sits between codes c and c + 1 and takes the even one
    mids = (E2M1_GRID[1:] + E2M1_GRID[:-1]) / 2
    c = np.searchsorted(mids, a, side="left")
    on_mid = (c < mids.size) & (a == mids[np.minimum(c, mids.size - 1)])
    c = np.where(on_mid & (c % 2 == 1), c + 1, c)
    return (c | (np.signbit(x).astype(np.int64) << 3)).astype(np.uint8)


def nv_global_scale(v) -> np.float32:
    """fp32 second-level scale of a whole tensor: 2688 / amax (1 for an all-zero tensor)."""
    amax = np.float32(np.max(np.abs(np.asarray(v, dtype=np.float64).astype(np.float32)))) if np.size(v) else 0
    if amax == 0:
        return np.float32(1.0)
    with np.errstate(over="ignore"):
        gs = np.float32(NV_GS_NUM) / np.float32(amax)
    return np.float32(min(gs, np.finfo(np.float32).max))


def nv_quantize(v, gs, axis: int = -1):
    """NVFP4 block quantisation of v along `axis` (blocks of 16) under global scale gs.

    Returns (codes uint8 with one 4-bit code per value, same shape as v;
    scale bytes uint8 (E4M3) with the block axis shortened 16 times)."""
    v32 = np.moveaxis(np.asarray(v, dtype=np.float64).astype(np.float32), axis, -1)
    n = v32.shape[-1]
    if n % NV_BLOCK:
        raise ValueError("length along the block axis must be a multiple of 16")
    vb = v32.reshape(v32.shape[:-1] + (n // NV_BLOCK, NV_BLOCK))
    gs = np.float32(gs)
    amax = np.max(np.abs(vb), axis=-1)
    s = (amax / np.float32(6.0)).astype(np.float32) * gs  # fp32 divide, then fp32 multiply
    sbytes = e4m3_encode(s.astype(np.float32).astype(np.float64))
    sdec = e4m3_decode(sbytes).astype(np.float32)
    zero = sdec == 0
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        inv = np.where(zero, np.float32(0.0), gs / np.where(zero, np.float32(1.0), sdec)).astype(np.float32)
        x = (vb * inv[..., None]).astype(np.float32)
    codes = e2m1_encode(x.astype(np.float64))
    codes[zero] = 0
    codes = np.moveaxis(codes.reshape(v32.shape), -1, axis)
    return codes, np.moveaxis(sbytes, -1, axis)


def nv_dequantize(codes, sbytes, gs, axis: int = -1) -> np.ndarray:
    c = np.moveaxis(np.asarray(codes), axis, -1)
    s = e4m3_decode(np.moveaxis(np.asarray(sbytes), axis, -1))
    vals = e2m1_decode(c).reshape(c.shape[:-1] + (c.shape[-1] // NV_BLOCK, NV_BLOCK)) * s[..., None]
    return np.moveaxis(vals.reshape(c.shape) / np.float64(np.float32(gs)), -1, axis)


def nv_round(v, gs, axis: int) -> np.ndarray:
    """v rounded to its NVFP4 value along `axis` under global scale gs (fp64)."""
    c, s = nv_quantize(v, gs, axis=axis)
    return nv_dequantize(c, s, gs, axis=axis)


def nv_weight_scales(W_gate, W_up, W_down, first_local: int = 0, num_local: int | None = None):
    """Global scales of the three weight tensors over the local experts."""
    if num_local is None and callable(W_gate):
        raise ValueError("num_local is needed when the weights come from a callable")
    n = num_local if num_local is not None else len(W_gate) - first_local
    out = []
    for W in (W_gate, W_up, W_down):
        amax = np.float32(0.0)
        for e in range(first_local, first_local + n):
            amax = max(amax, np.float32(np.max(np.abs(_f64(_expert(W, e)).astype(np.float32)))))
        with np.errstate(over="ignore"):
            out.append(np.float32(NV_GS_NUM) / amax if amax > 0 else np.float32(1.0))
    return tuple(np.float32(min(g, np.finfo(np.float32).max)) for g in out)


def nv_weight_layouts(Wg, Wu, Wd, gs_w) -> dict:
    """One expert's weights rounded for the forward GEMMs that read them (fp64): gate and up
    along d (K of the gate/up GEMM), down along I (K of the down GEMM)."""
    return dict(gate=nv_round(_f64(Wg), gs_w[0], axis=0), up=nv_round(_f64(Wu), gs_w[1], axis=0),
                down=nv_round(_f64(Wd), gs_w[2], axis=0))


def forward_nv(X, W_r, bias, W_gate, W_up, W_down, top_k: int, first_local: int = 0,
               num_local: int | None = None, gs_w=None, rounded=None):
    """NVFP4 layer forward: the routing of `forward`, then per local expert
    A = Xq Wgq, B = Xq Wuq (K = d), H = silu(A) B, O = Hq Wdq (K = I), Y = sum_j g O.

    gs_w: optional (gs_gate, gs_up, gs_down) computed once by the caller
    (nv_weight_scales); without it they are computed here.
    rounded: optional callable e -> nv_weight_layouts of expert e under gs_w (the same values,
    computed once by the caller); without it the weights are rounded here.
    Returns (Y, info) with the routing, the five global scales and, per local expert,
    (tokens, slots, H, A, B) or None."""
    X64 = _f64(X)
    T, d = X64.shape
    E = np.asarray(W_r).shape[1]
    logits = router_logits(X64, W_r, bias)
    ids = topk_ids(logits, top_k)
    g = gates(logits, ids)
    sched = schedule(ids, E, first_local, num_local)
    nl = sched["num_local"]
    if gs_w is None:
        gs_w = nv_weight_scales(W_gate, W_up, W_down, first_local, nl)
    gs_g, gs_u, gs_d = gs_w
    gs_x = nv_global_scale(X64)
    Hs = []
    for el in range(nl):
        toks, slots = _expert_rows(ids, sched, el)
        if toks.size == 0:
            Hs.append(None)
            continue
        e = el + first_local
        Wq = rounded(e) if rounded is not None else None
        Xq = nv_round(X64[toks], gs_x, axis=1)  # K = d
        A = Xq @ (Wq["gate"] if Wq else nv_round(_expert(W_gate, e), gs_g, axis=0))
        B = Xq @ (Wq["up"] if Wq else nv_round(_expert(W_up, e), gs_u, axis=0))
        Hs.append((toks, slots, silu(A) * B, A, B))
    live = [h[2] for h in Hs if h is not None]
    gs_h = nv_global_scale(np.concatenate(live, axis=0)) if live else np.float32(1.0)
    Y = np.zeros((T, d))
    for el, h in enumerate(Hs):
        if h is None:
            continue
        toks, slots, H = h[:3]
        Wdq = rounded(el + first_local)["down"] if rounded is not None else \
            nv_round(_expert(W_down, el + first_local), gs_d, axis=0)
        O = nv_round(H, gs_h, axis=1) @ Wdq  # K = I
        Y[toks] += g[toks, slots][:, None] * O
    info = dict(ids=ids, g=g, sched=sched, gs_x=gs_x, gs_h=gs_h, gs_w=(gs_g, gs_u, gs_d), experts=Hs)
    return Y, info


def nv_weight_scales_bwd(W_gate, W_up, W_down, first_local: int = 0, num_local: int | None = None):
    """Global scales of the backward's weight operands: [W_gate | W_up] along I as one tensor (the
    dgrad of gate/up contracts over both halves into one sum), W_down as in the forward."""
    g, u, d = nv_weight_scales(W_gate, W_up, W_down, first_local, num_local)
    return np.float32(min(g, u)), d


def nv_weight_layouts_bwd(Wg, Wu, Wd, gs_bwd) -> dict:
    """One expert's weights rounded for the backward's dgrad GEMMs (fp64): gate and up along I
    under the joint [gate | up] scale, down along d."""
    return dict(gate_i=nv_round(_f64(Wg), gs_bwd[0], axis=1), up_i=nv_round(_f64(Wu), gs_bwd[0], axis=1),
                down_d=nv_round(_f64(Wd), gs_bwd[1], axis=1))


def backward_nv(info, X, W_r, W_gate, W_up, W_down, dY, gs_bwd=None, rounded=None):
    """NVFP4 layer backward after forward_nv (its info): the dgrad GEMMs on NVFP4 operands,
    the weight gradients from the unrounded operands (as the MXFP8 layer with bf16 weight
    gradients does).

    dgrad of W_down (K = d): dY rows along d under gs(dY [T, d]), W_down along d;
    dgrad of gate/up (K = 2I): [dA | dB] rows along I under one scale over every assigned row's
    dA and dB, [W_gate | W_up] along I under one scale (nv_weight_scales_bwd).
    A and B are read as bf16 (the layer keeps them in bf16), H = silu(A) B recomputed from them.
    gs_bwd: optional (gs_gate_up, gs_down) computed once by the caller; rounded: optional
    callable e -> nv_weight_layouts_bwd of expert e under gs_bwd (the same values, computed once)."""
    from .moe_oracle import bf16_round, silu_grad
    X64, dY64 = _f64(X), _f64(dY)
    ids, g, sched = info["ids"], info["g"], info["sched"]
    T, d = X64.shape
    k = ids.shape[1]
    E = np.asarray(W_r).shape[1]
    first, nl = sched["first_local"], sched["num_local"]
    if gs_bwd is None:
        gs_bwd = nv_weight_scales_bwd(W_gate, W_up, W_down, first, nl)
    gs_gu, gs_d = gs_bwd
    gs_dy = nv_global_scale(dY64)
    dX = np.zeros((T, d))
    dg = np.zeros((T, k))
    dW_gate, dW_up, dW_down, parts = {}, {}, {}, []
    for el, item in enumerate(info["experts"]):
        e = el + first
        if item is None:
            I = np.asarray(_expert(W_gate, e)).shape[1]
            dW_gate[e] = np.zeros((d, I)); dW_up[e] = np.zeros((d, I)); dW_down[e] = np.zeros((I, d))
            continue
        toks, slots, _, A, B = item
        A, B = bf16_round(A), bf16_round(B)
        ge = g[toks, slots]
        dYe = dY64[toks]
        H = silu(A) * B
        Wdq = rounded(e)["down_d"] if rounded is not None else nv_round(_expert(W_down, e), gs_d, axis=1)
        dHp = nv_round(dYe, gs_dy, axis=1) @ Wdq.T  # K = d
        dg[toks, slots] = np.sum(dHp * H, axis=1)
        dH = ge[:, None] * dHp
        dA = dH * B * silu_grad(A)
        dB = dH * silu(A)
        Xe = X64[toks]
        dW_gate[e] = Xe.T @ dA
        dW_up[e] = Xe.T @ dB
        dW_down[e] = H.T @ (ge[:, None] * dYe)
        parts.append((e, toks, dA, dB))
    live = [np.abs(p[2]).max() for p in parts] + [np.abs(p[3]).max() for p in parts]
    gs_ab = nv_global_scale(np.array(live)) if live else np.float32(1.0)
    for e, toks, dA, dB in parts:  # K = I
        if rounded is not None:
            Wgq, Wuq = rounded(e)["gate_i"], rounded(e)["up_i"]
        else:
            Wgq = nv_round(_expert(W_gate, e), gs_gu, axis=1)
            Wuq = nv_round(_expert(W_up, e), gs_gu, axis=1)
        dX[toks] += nv_round(dA, gs_ab, axis=1) @ Wgq.T + nv_round(dB, gs_ab, axis=1) @ Wuq.T
    dl = np.zeros((T, E))
    s = np.sum(g * dg, axis=1, keepdims=True)
    np.put_along_axis(dl, ids.astype(np.int64), g * (dg - s), axis=1)
    dX += dl @ _f64(W_r).T
    return dict(dX=dX, dW_gate=dW_gate, dW_up=dW_up, dW_down=dW_down, dW_r=X64.T @ dl, dl=dl, dg=dg,
                gs_dy=gs_dy, gs_ab=gs_ab)
