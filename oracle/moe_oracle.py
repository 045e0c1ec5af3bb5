"""Oracle: a plain, slow, fp64 CPU statement of the MoE layer forward and backward.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this module:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
use it.  It shares no code, table or helper with the CUDA path.

What it follows
---------------
The pages ("Cursor open-sources Mixture-of-Kittens (MoK)...", page 1) describe a
mixture-of-experts training layer:

* "MoE layer as the bottleneck" and the toknow.ai summary (page 2): every token is
  routed to a few experts (router scores -> top-k experts).
* "Three design decisions that matter", bullet 1: one schedule table drives the
  forward dispatch / combine and the backward reverse-combine / reverse-dispatch.
* "Three design decisions that matter", bullet 2: experts run as an
  expert-grouped GEMM.
* same section, closing paragraph: the experts are SwiGLU MLPs, and the router
  weight gradient is computed "SonicMoE-style" inside the SwiGLU backward; the
  layer supports BF16 and MXFP8 precision modes and is fully deterministic.

The pages print no formula.  The layer's arithmetic is therefore the plain
definition of a top-k softmax-gated SwiGLU mixture of experts:

    l   = X W_r + b                         router logits            [T, E]
    S_t = the k largest entries of l_t      (descending; ties -> lower expert id)
    g   = exp(l_t,e) / sum_{e' in S_t} exp(l_t,e')   for e in S_t     (gates)
    A   = X_t W_gate[e],  B = X_t W_up[e],  H = silu(A) * B
    O   = H W_down[e]
    Y_t = sum_{e in S_t} g_t,e O_t,e

and its exact gradient (the selection is piecewise constant, so no gradient
flows through it; the bias b is an input without gradient):

    dO  = g dY_t,  dH = dO W_down[e]^T
    dA  = dH * B * silu'(A),  dB = dH * silu(A)
    dg  = <dY_t, O_t,e>
    dl_t,e = g_t,e (dg_t,e - sum_m g_t,m dg_t,m) on S_t, 0 elsewhere
    dX_t  = sum_e (dA W_gate[e]^T + dB W_up[e]^T) + dl_t W_r^T
    dW_r  = X^T dl
    dW_gate[e] = sum_t X_t^T dA,  dW_up[e] = sum_t X_t^T dB,
    dW_down[e] = sum_t H^T dO.

Readings where the pages are silent (each is listed in the design notes):

* selection runs on the (biased) logits, ties broken by the lower expert id,
  values compared as numbers (-0 == +0), NaN ranked lowest;
* ids inside a token are ordered by descending logit (ties: ascending id);
* "softmax over E then renormalise over the top k" equals a softmax over the
  selected k logits, which is what is computed;
* the schedule: counts per expert, exclusive prefix sums (unpadded and padded
  to P = 128 rows), a stable per-expert token order (ascending token id);
* experts outside [first_local, first_local + num_local) are excluded (their
  assignments belong to another rank): they add nothing to Y, dX or dl;
* dg is computed the direct way, <dY, O>; the fused "SonicMoE-style" form
  <dY W_down^T, H> is an identity the tests check, not something shared.

Every floating-point step is fp64; inputs are the exact values the GPU gets.
"""

from __future__ import annotations

import numpy as np

P_PAD = 128  # rows per expert segment are padded to a multiple of this


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------
def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def _expert(W, e: int) -> np.ndarray:
    """Weights of expert e as fp64; W is an [E, ...] array or a callable e -> array."""
    return _f64(W(e) if callable(W) else W[e])


def silu(a: np.ndarray) -> np.ndarray:
    """silu(a) = a * sigmoid(a) = a / (1 + exp(-a)), written overflow-safely."""
    return a * _sigmoid(a)


def _sigmoid(a: np.ndarray) -> np.ndarray:
    out = np.empty_like(a)
    pos = a >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-a[pos]))
    ea = np.exp(a[~pos])
    out[~pos] = ea / (1.0 + ea)
    return out


def silu_grad(a: np.ndarray) -> np.ndarray:
    """d silu / da = s (1 + a (1 - s)), s = sigmoid(a)."""
    s = _sigmoid(a)
    return s * (1.0 + a * (1.0 - s))


# ----------------------------------------------------------------------------
# routing (page 2 "routes each input to a few of them"; page 1 closing
# paragraph of "Three design decisions": deterministic)
# ----------------------------------------------------------------------------
def router_logits(X, W_r, bias=None) -> np.ndarray:
    """l = X W_r (+ b).  X [T, d], W_r [d, E], b [E] or None -> [T, E] fp64."""
    l = _f64(X) @ _f64(W_r)
    if bias is not None:
        l = l + _f64(bias)[None, :]
    return l


def topk_ids(logits, k: int) -> np.ndarray:
    """Top-k expert ids per row, by descending logit; equal logits -> lower id first.

    Values are compared as numbers, so -0 and +0 tie; NaN ranks below everything
    (also below -inf).  Returns int32 [T, k].
    """
    l = np.asarray(logits)
    T, E = l.shape
    if not 1 <= k <= E:
        raise ValueError("top_k must be in [1, E]")
    ids = np.empty((T, k), dtype=np.int32)
    idx = np.arange(E)
    for t in range(T):
        row = l[t].astype(np.float64)
        nan = np.isnan(row)
        key = np.where(nan, 0.0, -row)  # descending value ...
        # lexsort: last key is primary.  NaN first pushed to the back, then value, then id.
        order = np.lexsort((idx, key, nan.astype(np.int8)))
        ids[t] = order[:k]
    return ids


def gates(logits, ids) -> np.ndarray:
    """Softmax over the k selected logits of each row (fp64 [T, k])."""
    l = _f64(logits)
    sel = np.take_along_axis(l, ids.astype(np.int64), axis=1)
    m = sel.max(axis=1, keepdims=True)
    ex = np.exp(sel - m)
    return ex / ex.sum(axis=1, keepdims=True)


def schedule(ids, E: int, first_local: int = 0, num_local: int | None = None, P: int = P_PAD) -> dict:
    """The routing table shared by dispatch, combine and their backward mirrors.

    counts[e]          number of (token, slot) assignments to local expert e
    offsets[E_l+1]     exclusive prefix sum of counts (unpadded rows)
    padded_offsets     exclusive prefix sum of ceil(counts / P) * P
    perm[rows]         token of each unpadded row; inside an expert, ascending token id
    slot_row[T, k]     padded row of each assignment, -1 for non-local experts
    Here e runs over the local experts only (index e - first_local).
    """
    ids = np.asarray(ids)
    T, k = ids.shape
    if num_local is None:
        num_local = E - first_local
    El = num_local
    local = (ids >= first_local) & (ids < first_local + El)
    le = np.where(local, ids - first_local, -1)
    counts = np.zeros(El, dtype=np.int64)
    for e in le[local]:
        counts[e] += 1
    offsets = np.zeros(El + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    padded = ((counts + P - 1) // P) * P
    padded_offsets = np.zeros(El + 1, dtype=np.int64)
    padded_offsets[1:] = np.cumsum(padded)
    perm = np.empty(int(offsets[-1]), dtype=np.int64)
    slot_row = np.full((T, k), -1, dtype=np.int64)
    fill = np.zeros(El, dtype=np.int64)
    for t in range(T):  # ascending token order gives the stable per-expert order
        for j in range(k):
            e = le[t, j]
            if e < 0:
                continue
            pos = fill[e]
            fill[e] += 1
            perm[offsets[e] + pos] = t
            slot_row[t, j] = padded_offsets[e] + pos
    return dict(counts=counts, offsets=offsets, padded_offsets=padded_offsets,
                perm=perm, slot_row=slot_row, first_local=first_local, num_local=El)


def _expert_rows(ids, sched, e_local: int):
    """(tokens, slots) assigned to local expert e_local, in the schedule's row order."""
    o0, o1 = sched["offsets"][e_local], sched["offsets"][e_local + 1]
    toks = sched["perm"][o0:o1]
    e = e_local + sched["first_local"]
    slots = np.array([int(np.nonzero(ids[t] == e)[0][0]) for t in toks], dtype=np.int64)
    return toks, slots


# ----------------------------------------------------------------------------
# forward / backward (page 1, "Three design decisions that matter")
# ----------------------------------------------------------------------------
def forward(X, W_r, bias, W_gate, W_up, W_down, top_k: int,
            first_local: int = 0, num_local: int | None = None, keep=True):
    """MoE layer forward in fp64.  Returns (Y [T, d], ctx for backward)."""
    X64 = _f64(X)
    T, d = X64.shape
    E = np.asarray(W_r).shape[1]
    logits = router_logits(X64, W_r, bias)
    ids = topk_ids(logits, top_k)
    g = gates(logits, ids)
    sched = schedule(ids, E, first_local, num_local)
    Y = np.zeros((T, d))
    saved = []
    for el in range(sched["num_local"]):
        toks, slots = _expert_rows(ids, sched, el)
        if toks.size == 0:
            saved.append(None)
            continue
        e = el + sched["first_local"]
        Xe = X64[toks]
        A = Xe @ _expert(W_gate, e)
        B = Xe @ _expert(W_up, e)
        H = silu(A) * B
        O = H @ _expert(W_down, e)
        ge = g[toks, slots]
        Y[toks] += ge[:, None] * O  # each token appears once per expert
        saved.append((toks, slots, A, B) if keep else None)
    ctx = dict(X=X64, W_r=_f64(W_r), W_gate=W_gate, W_up=W_up, W_down=W_down,
               logits=logits, ids=ids, g=g, sched=sched, saved=saved, E=E)
    return Y, ctx


def backward(ctx, dY):
    """Exact gradient of the forward (selection held fixed).  All fp64."""
    dY64 = _f64(dY)
    X64, ids, g, sched = ctx["X"], ctx["ids"], ctx["g"], ctx["sched"]
    T, d = X64.shape
    k = ids.shape[1]
    E = ctx["E"]
    dX = np.zeros((T, d))
    dg = np.zeros((T, k))
    dW_gate, dW_up, dW_down = {}, {}, {}
    for el in range(sched["num_local"]):
        e = el + sched["first_local"]
        item = ctx["saved"][el]
        Wg, Wu, Wd = _expert(ctx["W_gate"], e), _expert(ctx["W_up"], e), _expert(ctx["W_down"], e)
        if item is None:
            toks, slots = _expert_rows(ids, sched, el)
            if toks.size == 0:
                I = Wg.shape[1]
                dW_gate[e] = np.zeros((d, I)); dW_up[e] = np.zeros((d, I)); dW_down[e] = np.zeros((I, d))
                continue
            Xe = X64[toks]
            A, B = Xe @ Wg, Xe @ Wu
        else:
            toks, slots, A, B = item
            Xe = X64[toks]
        H = silu(A) * B
        O = H @ Wd
        dYe = dY64[toks]
        ge = g[toks, slots]
        dg[toks, slots] = np.sum(dYe * O, axis=1)  # <dY_t, O_t,e>
        dO = ge[:, None] * dYe
        dH = dO @ Wd.T
        dA = dH * B * silu_grad(A)
        dB = dH * silu(A)
        dX[toks] += dA @ Wg.T + dB @ Wu.T
        dW_gate[e] = Xe.T @ dA
        dW_up[e] = Xe.T @ dB
        dW_down[e] = H.T @ dO
    # router: softmax-over-selected Jacobian, scattered to the selected experts
    dl = np.zeros((T, E))
    s = np.sum(g * dg, axis=1, keepdims=True)
    np.put_along_axis(dl, ids.astype(np.int64), g * (dg - s), axis=1)
    dX += dl @ ctx["W_r"].T
    dW_r = X64.T @ dl
    return dict(dX=dX, dW_gate=dW_gate, dW_up=dW_up, dW_down=dW_down, dW_r=dW_r,
                dl=dl, dg=dg)


def token_forward_backward(t: int, X, W_r, bias, W_gate, W_up, W_down, top_k: int, dY,
                           first_local: int = 0, num_local: int | None = None):
    """Y_t, dX_t and dl_t for one token: each depends on that token's data alone.

    Used to check full-size GPU results at sampled tokens without running the
    whole layer on the CPU.  Same definition as forward/backward, one row.
    """
    x = _f64(X)[t:t + 1]
    E = np.asarray(W_r).shape[1]
    l = router_logits(x, W_r, bias)
    ids = topk_ids(l, top_k)
    g = gates(l, ids)[0]
    lo = first_local
    hi = E if num_local is None else first_local + num_local
    dy = _f64(dY)[t]
    y = np.zeros(x.shape[1])
    dx = np.zeros(x.shape[1])
    dg = np.zeros(top_k)
    for j, e in enumerate(ids[0]):
        if not lo <= e < hi:
            continue
        Wg, Wu, Wd = _expert(W_gate, e), _expert(W_up, e), _expert(W_down, e)
        a = x[0] @ Wg
        b = x[0] @ Wu
        h = silu(a) * b
        o = h @ Wd
        y += g[j] * o
        dg[j] = dy @ o
        dh = (g[j] * dy) @ Wd.T
        dx += (dh * b * silu_grad(a)) @ Wg.T + (dh * silu(a)) @ Wu.T
    dl = np.zeros(E)
    dl[ids[0]] = g * (dg - np.sum(g * dg))
    dx += dl @ _f64(W_r).T
    return y, dx, dl, ids[0], g


# ----------------------------------------------------------------------------
# MXFP8 (page 1, closing paragraph of "Three design decisions that matter": the layer has a
# BF16 and an MXFP8 precision mode).  The block
# format (E4M3 payload, one E8M0 power-of-two scale per 32 values along the
# contraction dimension) is the OCP Microscaling v1.0 format; the scale rule is
# that format's: shared exponent = floor(log2(amax)) - emax(E4M3) = ... - 8.
# ----------------------------------------------------------------------------
E4M3_MAX = 448.0


def e4m3_decode(codes) -> np.ndarray:
    """E4M3 (OCP 'FN': bias 7, no infinities, S.1111.111 = NaN) bytes -> fp64."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    ex = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(ex == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * 2.0 ** (ex - 7))
    val = np.where((ex == 0xF) & (m == 0x7), np.nan, val)
    return s * val


def e4m3_encode(x) -> np.ndarray:
    """fp64 -> E4M3 byte, round to nearest even, saturating to +-448 (satfinite)."""
    x = _f64(x)
    out = np.zeros(x.shape, dtype=np.uint8)
    sign = (np.signbit(x)).astype(np.int64) << 7
    a = np.abs(x)
    a = np.minimum(a, E4M3_MAX)  # satfinite (NaN input is not produced by the layer)
    nz = a > 0
    # exponent of the binade, at least the subnormal exponent -6
    e = np.full(a.shape, -6, dtype=np.int64)
    e[nz] = np.maximum(np.floor(np.log2(a[nz])).astype(np.int64), -6)
    quantum = np.ldexp(1.0, (e - 3).astype(np.int64))
    q = np.round(a / quantum) * quantum  # np.round rounds halves to even
    q = np.minimum(q, E4M3_MAX)
    # encode q exactly
    code = np.zeros(a.shape, dtype=np.int64)
    qnz = q > 0
    eq = np.full(a.shape, -6, dtype=np.int64)
    eq[qnz] = np.floor(np.log2(q[qnz])).astype(np.int64)
    normal = qnz & (eq >= -6) & (q >= 2.0 ** -6)
    sub = qnz & ~normal
    mant_n = np.rint(q / np.ldexp(1.0, eq) * 8.0 - 8.0).astype(np.int64)
    code = np.where(normal, ((eq + 7) << 3) | mant_n, code)
    code = np.where(sub, np.rint(q / 2.0 ** -9).astype(np.int64), code)
    out[...] = (code | sign).astype(np.uint8)
    return out


def mx_quantize(v, axis: int = -1, block: int = 32):
    """MX block quantisation of v along `axis` in blocks of `block` values.

    Returns (codes uint8 [same shape], scale bytes uint8 [..., n/block, ...]).
    scale byte = shared exponent + 127; a block whose amax is 0 gets byte 0 and
    all-zero codes.  Value represented: e4m3_decode(code) * 2**(byte - 127).
    """
    v = np.moveaxis(_f64(v), axis, -1)
    n = v.shape[-1]
    if n % block:
        raise ValueError("length along the block axis must be a multiple of the block")
    vb = v.reshape(v.shape[:-1] + (n // block, block))
    amax = np.max(np.abs(vb), axis=-1)
    zero = amax == 0
    se = np.zeros(amax.shape, dtype=np.int64)
    se[~zero] = np.floor(np.log2(amax[~zero])).astype(np.int64) - 8
    se = np.clip(se, -127, 127)
    scaled = vb * np.ldexp(1.0, -se)[..., None]
    codes = e4m3_encode(scaled)
    codes[zero] = 0
    sbytes = np.where(zero, 0, se + 127).astype(np.uint8)
    codes = np.moveaxis(codes.reshape(v.shape), -1, axis)
    sbytes = np.moveaxis(sbytes, -1, axis)
    return codes, sbytes


def mx_dequantize(codes, sbytes, axis: int = -1, block: int = 32) -> np.ndarray:
    c = np.moveaxis(np.asarray(codes), axis, -1)
    s = np.moveaxis(np.asarray(sbytes), axis, -1).astype(np.int64)
    vals = e4m3_decode(c).reshape(c.shape[:-1] + (c.shape[-1] // block, block))
    vals = vals * np.ldexp(1.0, s - 127)[..., None]
    return np.moveaxis(vals.reshape(c.shape), -1, axis)


# ----------------------------------------------------------------------------
# Ring-streamed layer ("Three design decisions that matter", bullets 2 and 3):
# minibatches grouped into macrobatches of at least two full waves of
# grouped-GEMM tiles, dispatched rows cycled through a fixed ring, the ring
# walked in reverse in the backward with replay of what was overwritten.
# Readings: a macrobatch also closes before a minibatch that would not fit in
# the ring with it; a segment that would run past the ring's end restarts at
# row 0; the backward reuses the macrobatches still intact (a suffix in time)
# and replays older ones in groups of consecutive macrobatches that fit in the
# ring together.  The layer's values do not depend on the plan.
# ----------------------------------------------------------------------------
def stream_plan(mb_counts, ring_rows: int, min_rows: int, P: int = P_PAD) -> dict:
    """mb_counts[b][el]: assignments of local expert el in minibatch b."""
    mb_counts = np.asarray(mb_counts, dtype=np.int64)
    M, El = mb_counts.shape

    def padded(c):
        return int(np.sum((np.asarray(c) + P - 1) // P * P))

    macro, cur, b0 = [], np.zeros(El, dtype=np.int64), 0
    for b in range(M):
        if b > b0 and padded(cur + mb_counts[b]) > ring_rows:
            macro.append((b0, b, cur.copy()))
            cur[:] = 0
            b0 = b
        cur += mb_counts[b]
        if padded(cur) >= min_rows:
            macro.append((b0, b + 1, cur.copy()))
            cur[:] = 0
            b0 = b + 1
    if b0 < M:
        macro.append((b0, M, cur.copy()))
    seg_poff, rows, ring_start, sizes, wp, row = [], [], [], [], 0, 0
    for (_, _, cnt) in macro:
        starts = []
        for el in range(El):
            starts.append(row)
            row += (int(cnt[el]) + P - 1) // P * P
        seg_poff.append(starts)
        size = row - starts[0]
        if wp + size > ring_rows:
            wp = 0
        ring_start.append(wp)
        sizes.append(size)
        wp += size
    n = len(macro)
    resident = []
    for m in range(n):
        a0, a1 = ring_start[m], ring_start[m] + sizes[m]
        resident.append(all(not (sizes[m] > 0 and sizes[q] > 0 and ring_start[q] < a1 and a0 < ring_start[q] + sizes[q])
                            for q in range(m + 1, n)))
    chunks, m = [], n - 1
    while m >= 0 and resident[m]:
        m -= 1
    if m + 1 < n:
        chunks.append((m + 1, n))
    replayed = 0
    while m >= 0:
        hi, rows_c = m + 1, 0
        while True:
            rows_c += sizes[m]
            m -= 1
            if m < 0 or rows_c + sizes[m] > ring_rows:
                break
        chunks.append((m + 1, hi))
        replayed += rows_c
    if not chunks:
        chunks = [(0, 0)]
    return dict(macro=[(a, b) for a, b, _ in macro], seg_poff=seg_poff, rows=row, ring_start=ring_start,
                sizes=sizes, resident=resident, chunks=chunks, replayed=replayed)


# ----------------------------------------------------------------------------
# MXFP8 layer: every operand of the gate/up, down and dgrad GEMMs rounded to MX
# (E4M3 + E8M0 per 32 along that GEMM's contraction dimension) before the
# product.  The weight-gradient GEMMs contract over tokens: unquantised by
# default; with mx_wgrad their operands (X, dA, dB, Hg = g H and dY of one
# expert) are rounded along the expert's rows, in blocks of 32 rows from its
# first row, the rows zero-padded to a multiple of 32.
# fp64 everywhere else.  The router gradient takes dg = <dH', H> with dH' the
# quantised dgrad of W_down (the fused form; the identity with <dY, O> holds only
# without quantisation).
# ----------------------------------------------------------------------------
def mx_round(v, axis: int):
    """v rounded to its MXFP8 value along `axis` (fp64)."""
    c, s = mx_quantize(v, axis=axis)
    return mx_dequantize(c, s, axis=axis)


def bf16_round(v):
    """v rounded to bfloat16 through float32 (round to nearest even at each step), as fp64."""
    x = np.asarray(v, dtype=np.float64).astype(np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def mx_round_rows(v, groups=None):
    """v [rows, n] (one expert's rows in order) rounded to MXFP8 along the rows, in blocks
    of 32 rows from the first; rows past the last multiple of 32 are padded with zeros.
    groups: lengths of consecutive runs of rows (summing to rows), each rounded on its own in
    blocks of 32 from its first row (a ring-streamed layer's (macrobatch, expert) segments);
    None: one run."""
    v = _f64(v)
    if groups is not None:
        out, r = [], 0
        for n in groups:
            out.append(mx_round_rows(v[r:r + n]))
            r += n
        if r != v.shape[0]:
            raise ValueError("row groups must cover the rows")
        return np.concatenate(out, axis=0) if out else v
    pad = (-v.shape[0]) % 32
    vp = np.concatenate([v, np.zeros((pad,) + v.shape[1:])], axis=0) if pad else v
    return mx_round(vp, axis=0)[:v.shape[0]]


def mx_weight_layouts(Wg, Wu, Wd) -> dict:
    """One expert's weights rounded for each GEMM that reads them, along its contraction:

    gate_d, up_d   W_gate, W_up [d, I] along d   (forward gate/up GEMM, K = d)
    down_i         W_down [I, d] along I         (forward down GEMM, K = I)
    down_d         W_down [I, d] along d         (dgrad of W_down, K = d)
    gate_i, up_i   W_gate, W_up [d, I] along I   (dgrad of gate/up, K = I)
    """
    Wg, Wu, Wd = _f64(Wg), _f64(Wu), _f64(Wd)
    return dict(gate_d=mx_round(Wg, axis=0), up_d=mx_round(Wu, axis=0), down_i=mx_round(Wd, axis=0),
                down_d=mx_round(Wd, axis=1), gate_i=mx_round(Wg, axis=1), up_i=mx_round(Wu, axis=1))


def _layouts(rounded, W_gate, W_up, W_down, e: int) -> dict:
    """Rounded weights of expert e: from the caller's `rounded(e)` (e.g. a cache), else computed."""
    if rounded is not None:
        return {k: _f64(v) for k, v in rounded(e).items()}
    return mx_weight_layouts(_expert(W_gate, e), _expert(W_up, e), _expert(W_down, e))


def forward_mx(X, W_r, bias, W_gate, W_up, W_down, top_k: int, first_local: int = 0, num_local: int | None = None,
               rounded=None):
    """MXFP8 layer forward (experts [first_local, first_local + num_local) as in forward).

    rounded: optional callable e -> mx_weight_layouts of expert e (the same values, computed
    once by the caller); without it the weights are rounded here."""
    X64 = _f64(X)
    T, d = X64.shape
    E = np.asarray(W_r).shape[1]
    logits = router_logits(X64, W_r, bias)
    ids = topk_ids(logits, top_k)
    g = gates(logits, ids)
    sched = schedule(ids, E, first_local, num_local)
    Y = np.zeros((T, d))
    saved = []
    for el in range(sched["num_local"]):
        toks, slots = _expert_rows(ids, sched, el)
        if toks.size == 0:
            saved.append(None)
            continue
        Wq = _layouts(rounded, W_gate, W_up, W_down, el + sched["first_local"])
        Xq = mx_round(X64[toks], axis=1)  # K = d
        A = Xq @ Wq["gate_d"]
        B = Xq @ Wq["up_d"]
        H = silu(A) * B
        O = mx_round(H, axis=1) @ Wq["down_i"]  # K = I
        ge = g[toks, slots]
        Y[toks] += ge[:, None] * O
        saved.append((toks, slots, A, B))
    ctx = dict(X=X64, W_r=_f64(W_r), W_gate=W_gate, W_up=W_up, W_down=W_down, logits=logits, ids=ids, g=g,
               sched=sched, saved=saved, E=E, rounded=rounded)
    return Y, ctx


def backward_mx(ctx, dY, mx_wgrad: bool = False, row_groups=None):
    """MXFP8 layer backward.  mx_wgrad: the weight-gradient GEMMs on MXFP8 as well, each
    operand rounded along the expert's rows (mx_round_rows); otherwise they take the
    unrounded operands.  row_groups: optional callable e_local -> run lengths of the expert's
    rows (the segments of a ring-streamed layer), each run rounded on its own.

    The forward's saved pre-activations A and B are read as bf16 (bf16_round), the type the
    layer keeps them in: every operand quantised here (dA, dB along I; with mx_wgrad dA, dB and
    Hg along the rows) is computed from the values a kernel has, so both sides take each
    rounding decision from the same inputs up to the order of fp32 sums."""
    dY64 = _f64(dY)
    X64, ids, g, sched = ctx["X"], ctx["ids"], ctx["g"], ctx["sched"]
    T, d = X64.shape
    k = ids.shape[1]
    E = ctx["E"]
    dX = np.zeros((T, d))
    dg = np.zeros((T, k))
    dW_gate, dW_up, dW_down = {}, {}, {}
    for el in range(sched["num_local"]):
        e = el + sched["first_local"]
        item = ctx["saved"][el]
        if item is None:
            I = np.asarray(_expert(ctx["W_gate"], e)).shape[1]
            dW_gate[e] = np.zeros((d, I)); dW_up[e] = np.zeros((d, I)); dW_down[e] = np.zeros((I, d))
            continue
        Wq = _layouts(ctx.get("rounded"), ctx["W_gate"], ctx["W_up"], ctx["W_down"], e)
        toks, slots, A, B = item
        A, B = bf16_round(A), bf16_round(B)
        Xe = X64[toks]
        ge = g[toks, slots]
        dYe = dY64[toks]
        H = silu(A) * B
        dHp = mx_round(dYe, axis=1) @ Wq["down_d"].T  # K = d
        dg[toks, slots] = np.sum(dHp * H, axis=1)
        dH = ge[:, None] * dHp
        dA = dH * B * silu_grad(A)
        dB = dH * silu(A)
        dX[toks] += mx_round(dA, axis=1) @ Wq["gate_i"].T + mx_round(dB, axis=1) @ Wq["up_i"].T  # K = I
        if mx_wgrad:  # K = the expert's rows
            grp = None if row_groups is None else row_groups(el)
            Xr = mx_round_rows(Xe, grp)
            dW_gate[e] = Xr.T @ mx_round_rows(dA, grp)
            dW_up[e] = Xr.T @ mx_round_rows(dB, grp)
            dW_down[e] = mx_round_rows(ge[:, None] * H, grp).T @ mx_round_rows(dYe, grp)
        else:
            dW_gate[e] = Xe.T @ dA
            dW_up[e] = Xe.T @ dB
            dW_down[e] = H.T @ (ge[:, None] * dYe)
    dl = np.zeros((T, E))
    s = np.sum(g * dg, axis=1, keepdims=True)
    np.put_along_axis(dl, ids.astype(np.int64), g * (dg - s), axis=1)
    dX += dl @ ctx["W_r"].T
    return dict(dX=dX, dW_gate=dW_gate, dW_up=dW_up, dW_down=dW_down, dW_r=X64.T @ dl, dl=dl, dg=dg)


def token_forward_backward_mx(t: int, X, W_r, bias, rounded, top_k: int, dY):
    """Y_t, dX_t and dl_t of the MXFP8 layer for one token (all experts local).

    The same steps as forward_mx / backward_mx on one row: every activation is rounded
    along its own row (d or I), so a token's results depend on its data alone.
    rounded: callable e -> mx_weight_layouts of expert e."""
    x = _f64(X)[t:t + 1]
    E = np.asarray(W_r).shape[1]
    l = router_logits(x, W_r, bias)
    ids = topk_ids(l, top_k)
    g = gates(l, ids)[0]
    dy = _f64(dY)[t:t + 1]
    y = np.zeros(x.shape[1])
    dx = np.zeros(x.shape[1])
    dg = np.zeros(top_k)
    xq = mx_round(x, axis=1)
    dyq = mx_round(dy, axis=1)
    for j, e in enumerate(ids[0]):
        Wq = {k: _f64(v) for k, v in rounded(int(e)).items()}
        a = xq @ Wq["gate_d"]
        b = xq @ Wq["up_d"]
        h = silu(a) * b
        y += g[j] * (mx_round(h, axis=1) @ Wq["down_i"])[0]
        a, b = bf16_round(a), bf16_round(b)  # the backward reads the saved bf16 A, B
        h = silu(a) * b
        dhp = dyq @ Wq["down_d"].T
        dg[j] = float(np.sum(dhp * h))
        dh = g[j] * dhp
        da = dh * b * silu_grad(a)
        db = dh * silu(a)
        dx += (mx_round(da, axis=1) @ Wq["gate_i"].T + mx_round(db, axis=1) @ Wq["up_i"].T)[0]
    dl = np.zeros(E)
    dl[ids[0]] = g * (dg - np.sum(g * dg))
    dx += dl @ _f64(W_r).T
    return y, dx, dl, ids[0], g


# ----------------------------------------------------------------------------
# Expert parallelism ("Three design decisions that matter", bullet 1: pull-based
# dispatch and push-based combine, the backward mirrored, one schedule table for
# all four phases).  Readings: R ranks each hold their own tokens; rank q owns the
# contiguous experts [q E/R, (q+1) E/R); an owner pulls, for each local expert,
# the rows of every source rank in source-rank order, each source's tokens in
# ascending order; it pushes each output row back to the source's slot of that
# assignment (token t, slot j), where the source combines its k slots in slot order.
# ----------------------------------------------------------------------------
def ep_plan(ids_ranks, E: int, P: int = P_PAD) -> dict:
    """ids_ranks[r]: [T_r, k] expert ids of rank r's tokens.  Returns, per owner q:
    counts [El] (rows per local expert), padded_offsets [El+1], base [El][R+1] (first row of each
    source inside the expert's rows), rows: for every real row in order, (source, token, slot);
    and per source r: dest[r] [T_r, k] = (owner, padded row) of each assignment."""
    R = len(ids_ranks)
    if E % R:
        raise ValueError("E must be a multiple of the number of ranks")
    El = E // R
    k = np.asarray(ids_ranks[0]).shape[1]
    owners = []
    dest = [np.full(np.asarray(ids).shape + (2,), -1, dtype=np.int64) for ids in ids_ranks]
    for q in range(R):
        counts = np.zeros(El, dtype=np.int64)
        base = np.zeros((El, R + 1), dtype=np.int64)
        per = [[[] for _ in range(R)] for _ in range(El)]  # per[el][src] = [(token, slot)]
        for src, ids in enumerate(ids_ranks):
            ids = np.asarray(ids)
            for t in range(ids.shape[0]):  # ascending token
                for j in range(k):
                    el = int(ids[t, j]) - q * El
                    if 0 <= el < El:
                        per[el][src].append((t, j))
        padded_offsets = np.zeros(El + 1, dtype=np.int64)
        rows = []
        for el in range(El):
            for src in range(R):
                base[el, src + 1] = base[el, src] + len(per[el][src])
            counts[el] = base[el, R]
            padded_offsets[el + 1] = padded_offsets[el] + (counts[el] + P - 1) // P * P
            i = 0
            for src in range(R):
                for (t, j) in per[el][src]:
                    rows.append((src, t, j))
                    dest[src][t, j] = (q, padded_offsets[el] + i)
                    i += 1
        owners.append(dict(counts=counts, padded_offsets=padded_offsets, base=base, rows=rows))
    return dict(owners=owners, dest=dest, El=El, R=R)
