"""Full-size parity: the bench workloads, in the launch configuration bench.py times.

The oracle cannot run the whole layer at these sizes in seconds, so it checks
what it can compute one piece at a time:

* routing table: bit-exact against the oracle's selection on the GPU's fp32
  logits (all T tokens); against the oracle's own fp64 logits, every token
  whose ids differ must be a near-tie in fp64;
* Y, dX and the router gradient dl at sampled tokens (each depends on that
  token's data alone);
* dW_gate, dW_up, dW_down of sampled experts (each depends on that expert's
  tokens alone);
* dW_r in full against X^T dl computed in fp64 from the GPU's own dl, whose
  sampled rows were checked against the oracle; and, independent of the GPU's dl, the
  invariant that every row of dW_r sums to zero over the experts (each token's gates sum to
  one, so its dl sums to zero over its slots);
* a second run is bit-identical.
"""
import numpy as np
import pytest
import torch

import oracle as O
from mixture_experts_layer_27_b200 import binding as B
from mixture_experts_layer_27_b200 import inputs as IN

from _util import TOL_BF16, mx_layout_cache, relerr, to64

pytestmark = pytest.mark.gpu


class ExpertCache:
    """fp64 host copies of single experts' weights, fetched on demand (last few kept)."""

    def __init__(self, W, keep=2):
        self.W, self.keep, self.cache = W, keep, {}

    def __call__(self, e):
        e = int(e)
        if e not in self.cache:
            if len(self.cache) >= self.keep:
                self.cache.pop(next(iter(self.cache)))
            self.cache[e] = to64(self.W[e])
        return self.cache[e]


def _run(w, x):
    layer = B.MoELayer(w.T, w.d, w.E, w.I, w.k)
    Y = layer.forward(x["X"], x["W_r"], x["bias"], x["W_gate"], x["W_up"], x["W_down"])
    g = layer.backward(x["X"], x["W_r"], x["W_gate"], x["W_up"], x["W_down"], x["dY"])
    torch.cuda.synchronize()
    assert layer.error() == B.MOE_OK
    return layer, Y, g


@pytest.mark.parametrize("name", ["dsv3", "kimi"])
def test_full_size_workload(name):
    w = IN.WORKLOADS[name]
    x = IN.make_inputs(w, device="cuda")
    layer, Y, g = _run(w, x)
    r = layer.routing()
    lg_gpu = to64(layer.logits())
    X, Wr = to64(x["X"]), to64(x["W_r"])
    b = None if x["bias"] is None else to64(x["bias"])

    # -- routing table, bit-exact on the GPU's logits
    ids = O.topk_ids(lg_gpu, w.k)
    s = O.schedule(ids, w.E)
    gids = r["ids"].cpu().numpy()
    assert np.array_equal(gids, ids)
    for key in ("counts", "offsets", "padded_offsets", "perm", "slot_row"):
        assert np.array_equal(r[key].cpu().numpy(), s[key]), key
    assert np.max(np.abs(r["gates"].cpu().numpy() - O.gates(lg_gpu, ids))) < 1e-6

    # -- against fp64 logits: differences only at near-ties
    lg64 = O.router_logits(X, Wr, b)
    ids64 = O.topk_ids(lg64, w.k)
    srt = -np.sort(-lg64, axis=1)
    gap = srt[:, w.k - 1] - srt[:, w.k]
    differ = np.nonzero(np.any(np.sort(ids64, 1) != np.sort(gids, 1), axis=1))[0]
    near = gap < 1e-3
    assert np.all(near[differ]), (differ, gap[differ])
    tie_tokens = set(differ.tolist())

    # -- Y, dX at sampled tokens
    Wg, Wu, Wd = ExpertCache(x["W_gate"]), ExpertCache(x["W_up"]), ExpertCache(x["W_down"])
    dY = to64(x["dY"])
    rng = np.random.default_rng(1234)
    toks = [t for t in rng.choice(w.T, size=24, replace=False).tolist() if t not in tie_tokens][:16]
    Yg, dXg = to64(Y), to64(g["dX"])
    dl_gpu = to64(layer.router_grad())  # [T, k], slot order of the GPU's ids
    ys, yo, dxs, dxo, dls, dlo = [], [], [], [], [], []
    for t in toks:
        y, dx, dl, tid, gt = O.token_forward_backward(t, X, Wr, b, Wg, Wu, Wd, w.k, dY)
        ys.append(Yg[t]); yo.append(y); dxs.append(dXg[t]); dxo.append(dx)
        dls.append(dl_gpu[t]); dlo.append(dl[gids[t]])
    assert relerr(np.array(ys), np.array(yo)) <= TOL_BF16
    assert relerr(np.array(dxs), np.array(dxo)) <= TOL_BF16
    assert relerr(np.array(dls), np.array(dlo)) <= TOL_BF16

    # -- dW_r in full: X^T dl in fp64 from the GPU's (sampled-checked) dl
    dl_dense = np.zeros((w.T, w.E))
    np.put_along_axis(dl_dense, gids.astype(np.int64), dl_gpu, axis=1)
    assert relerr(to64(g["dW_r"]), X.T @ dl_dense) <= 1e-4
    # dl_t = g_t (dg_t - sum_m g_m dg_m) with sum_m g_m = 1 sums to zero over a token's slots,
    # so dW_r 1_E = X^T DL 1_E = 0 (up to the fp32 rounding of dl and of the GEMM)
    dWr64 = to64(g["dW_r"])
    assert np.max(np.abs(dl_gpu.sum(axis=1))) <= 1e-4 * max(np.max(np.abs(dl_gpu)), 1e-30)
    assert np.max(np.abs(dWr64.sum(axis=1))) <= 3e-3 * np.max(np.abs(dWr64))

    # -- expert weight gradients for the hottest and the coldest non-empty expert
    counts = r["counts"].cpu().numpy()
    nz = np.nonzero(counts)[0]
    hot, cold = int(nz[np.argmax(counts[nz])]), int(nz[np.argmin(counts[nz])])
    for e in sorted({hot, cold}):
        _, ctx = O.forward(X, Wr, b, Wg, Wu, Wd, w.k, first_local=e, num_local=1)
        ctx_tokens = set(ctx["sched"]["perm"].tolist())
        if ctx_tokens & tie_tokens:
            continue  # a near-tie token changes this expert's token set between fp32 and fp64
        go = O.backward(ctx, dY)
        assert relerr(to64(g["dW_gate"][e]), go["dW_gate"][e]) <= TOL_BF16, e
        assert relerr(to64(g["dW_up"][e]), go["dW_up"][e]) <= TOL_BF16, e
        assert relerr(to64(g["dW_down"][e]), go["dW_down"][e]) <= TOL_BF16, e

    # -- bit-identical second run
    _, Y2, g2 = _run(w, x)
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))
    for n in ("dX", "dW_gate", "dW_up", "dW_down"):
        assert torch.equal(g[n].view(torch.int16), g2[n].view(torch.int16)), n
    assert torch.equal(g["dW_r"].view(torch.int32), g2["dW_r"].view(torch.int32))
    del layer, Y, g, Y2, g2, x
    torch.cuda.empty_cache()


# MXFP8 at full size (kimi_mx).  The primary check is against the MXFP8 oracle (every GEMM
# operand MX-rounded along its contraction, fp64 otherwise) at the 6e-2 MXFP8 tolerance: Y, dX
# and the router gradient at three sampled tokens, and the hottest and coldest experts' weight
# gradients.  Only the experts those touch are rounded (six layouts each, in a spawned pool), so
# the tokens are picked to share experts.  The comparison with the unquantised fp64 oracle stays
# as a diagnostic, bounded by the format's own error (at most 9% at the tested shapes) plus 2e-2.
TOL_MX = 6e-2
TOL_MX_VS_EXACT = 0.11


def _tokens_sharing_experts(ids, candidates, counts, n=3):
    """n candidate tokens whose expert sets overlap most (greedy, starting from the token on
    the hottest experts); returns (tokens, union of their experts)."""
    first = max(candidates, key=lambda t: sum(int(counts[e]) for e in ids[t]))
    pick, union = [first], set(int(e) for e in ids[first])
    while len(pick) < n:
        rest = [t for t in candidates if t not in pick]
        t = min(rest, key=lambda t: (len(set(int(e) for e in ids[t]) - union), t))
        pick.append(t)
        union |= set(int(e) for e in ids[t])
    return pick, union


def test_full_size_mxfp8_kimi():
    w = IN.WORKLOADS["kimi_mx"]
    x = IN.make_inputs(w, device="cuda")

    def run():
        lay = B.MoELayerMX(w.T, w.d, w.E, w.I, w.k)
        lay.prepare(x["W_gate"], x["W_up"], x["W_down"])
        Y = lay.forward(x["X"], x["W_r"], x["bias"])
        g = lay.backward(x["X"], x["W_r"], x["dY"])
        torch.cuda.synchronize()
        assert lay.error() == B.MOE_OK
        return lay, Y, g

    lay, Y, g = run()
    r = lay.routing()
    lg_gpu = to64(lay.logits())
    X, Wr = to64(x["X"]), to64(x["W_r"])
    b = None if x["bias"] is None else to64(x["bias"])

    # routing: the router stays bf16, so the table is bit-exact on the GPU's logits
    ids = O.topk_ids(lg_gpu, w.k)
    s = O.schedule(ids, w.E)
    gids = r["ids"].cpu().numpy()
    assert np.array_equal(gids, ids)
    for key in ("counts", "offsets", "padded_offsets", "perm", "slot_row"):
        assert np.array_equal(r[key].cpu().numpy(), s[key]), key
    lg64 = O.router_logits(X, Wr, b)
    srt = -np.sort(-lg64, axis=1)
    gap = srt[:, w.k - 1] - srt[:, w.k]
    differ = np.nonzero(np.any(np.sort(O.topk_ids(lg64, w.k), 1) != np.sort(gids, 1), axis=1))[0]
    assert np.all(gap[differ] < 1e-3)
    tie_tokens = set(differ.tolist())

    # Y, dX, dl at sampled tokens against the fp64 (unquantised) oracle, within the format bound
    Wg, Wu, Wd = ExpertCache(x["W_gate"]), ExpertCache(x["W_up"]), ExpertCache(x["W_down"])
    dY = to64(x["dY"])
    rng = np.random.default_rng(4321)
    toks = [t for t in rng.choice(w.T, size=10, replace=False).tolist() if t not in tie_tokens][:6]
    Yg, dXg, dl_gpu = to64(Y), to64(g["dX"]), to64(lay.router_grad())
    ys, yo, dxs, dxo, dls, dlo = [], [], [], [], [], []
    for t in toks:
        y, dx, dl, tid, gt = O.token_forward_backward(t, X, Wr, b, Wg, Wu, Wd, w.k, dY)
        ys.append(Yg[t]); yo.append(y); dxs.append(dXg[t]); dxo.append(dx)
        dls.append(dl_gpu[t]); dlo.append(dl[gids[t]])
    assert relerr(np.array(ys), np.array(yo)) <= TOL_MX_VS_EXACT
    assert relerr(np.array(dxs), np.array(dxo)) <= TOL_MX_VS_EXACT
    assert relerr(np.array(dls), np.array(dlo)) <= TOL_MX_VS_EXACT

    # expert weight gradients (bf16 GEMMs over MXFP8-path activations) of the hottest and the
    # coldest non-empty expert, within the same bound
    counts = r["counts"].cpu().numpy()
    nz = np.nonzero(counts)[0]
    hot, cold = int(nz[np.argmax(counts[nz])]), int(nz[np.argmin(counts[nz])])
    for e in sorted({hot, cold}):
        _, ctx = O.forward(X, Wr, b, Wg, Wu, Wd, w.k, first_local=e, num_local=1)
        if set(ctx["sched"]["perm"].tolist()) & tie_tokens:
            continue
        go = O.backward(ctx, dY)
        for n in ("dW_gate", "dW_up", "dW_down"):
            assert relerr(to64(g[n][e]), go[n][e]) <= TOL_MX_VS_EXACT, (n, e)

    # -- against the MXFP8 oracle at 6e-2: three tokens sharing experts, the hot and cold experts
    cands = [t for t in range(w.T) if t not in tie_tokens]
    mtoks, union = _tokens_sharing_experts(gids, cands[:512], counts)
    experts = sorted(union | {e for e in (hot, cold)})
    weights = {n: ExpertCache(x[n], keep=1) for n in ("W_gate", "W_up", "W_down")}
    cache = mx_layout_cache(experts, weights)
    rounded = cache.__getitem__
    ys, yo, dxs, dxo, dls, dlo = [], [], [], [], [], []
    for t in mtoks:
        y, dx, dl, tid, gt = O.token_forward_backward_mx(t, X, Wr, b, rounded, w.k, dY)
        assert np.array_equal(tid, gids[t])
        ys.append(Yg[t]); yo.append(y); dxs.append(dXg[t]); dxo.append(dx)
        dls.append(dl_gpu[t]); dlo.append(dl[gids[t]])
    assert relerr(np.array(ys), np.array(yo)) <= TOL_MX
    assert relerr(np.array(dxs), np.array(dxo)) <= TOL_MX
    assert relerr(np.array(dls), np.array(dlo)) <= TOL_MX
    for e in sorted({hot, cold}):
        _, ctx = O.forward_mx(X, Wr, b, Wg, Wu, Wd, w.k, first_local=e, num_local=1, rounded=rounded)
        if set(ctx["sched"]["perm"].tolist()) & tie_tokens:
            continue
        go = O.backward_mx(ctx, dY)
        for n in ("dW_gate", "dW_up", "dW_down"):
            assert relerr(to64(g[n][e]), go[n][e]) <= TOL_MX, (n, e)
    del cache

    # a second run is bit-identical (the first layer's buffers are freed first; the gradients
    # are compared 32 experts at a time to keep the comparison's temporaries small)
    del lay
    torch.cuda.empty_cache()
    lay2, Y2, g2 = run()
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))
    assert torch.equal(g["dX"].view(torch.int16), g2["dX"].view(torch.int16))
    for n in ("dW_gate", "dW_up", "dW_down"):
        for e0 in range(0, w.E, 32):
            assert torch.equal(g[n][e0:e0 + 32].view(torch.int16), g2[n][e0:e0 + 32].view(torch.int16)), (n, e0)
    assert torch.equal(g["dW_r"].view(torch.int32), g2["dW_r"].view(torch.int32))
    del lay2, Y, Y2, g, g2, x
    torch.cuda.empty_cache()


def test_full_size_mxfp8_weight_gradients_kimi():
    # kimi_mx with the weight-gradient GEMMs on MXFP8 too (MOE_MXFP8_ALL): Y, dX and dW_r are the
    # plain MXFP8 mode's bits; the hottest and coldest experts' weight gradients equal the product
    # of the operands the device quantised, and are within 6e-2 of the MXFP8 oracle with MX
    # weight gradients; a rerun is bit-identical.
    w = IN.WORKLOADS["kimi_mx"]
    x = IN.make_inputs(w, device="cuda")

    def run(mx_wgrad):
        lay = B.MoELayerMX(w.T, w.d, w.E, w.I, w.k, mx_wgrad=mx_wgrad)
        lay.prepare(x["W_gate"], x["W_up"], x["W_down"])
        Y = lay.forward(x["X"], x["W_r"], x["bias"])
        g = lay.backward(x["X"], x["W_r"], x["dY"])
        torch.cuda.synchronize()
        assert lay.error() == B.MOE_OK
        return lay, Y, g

    lay0, Y0, g0 = run(False)
    del lay0
    keep = {"Y": Y0, "dX": g0["dX"], "dW_r": g0["dW_r"]}
    del g0
    torch.cuda.empty_cache()
    lay, Y, g = run(True)
    assert torch.equal(Y.view(torch.int16), keep["Y"].view(torch.int16))
    assert torch.equal(g["dX"].view(torch.int16), keep["dX"].view(torch.int16))
    assert torch.equal(g["dW_r"].view(torch.int32), keep["dW_r"].view(torch.int32))
    del keep, Y0

    r = lay.routing()
    counts = r["counts"].cpu().numpy()
    poff = r["padded_offsets"].cpu().numpy()
    gids = r["ids"].cpu().numpy()
    nz = np.nonzero(counts)[0]
    hot, cold = int(nz[np.argmax(counts[nz])]), int(nz[np.argmin(counts[nz])])
    # the GEMMs on the device's own operands (dequantised here)
    vals = {}
    for which, name in enumerate(("X", "dY", "dA", "dB", "Hg")):
        codes, sc = lay.wgrad_operand(which)
        vals[name] = {e: O.mx_dequantize(codes[:, poff[e]:poff[e] + (int(counts[e]) + 31) // 32 * 32],
                                         sc[:, poff[e] // 32:(poff[e] + (int(counts[e]) + 31) // 32 * 32) // 32],
                                         axis=1)[:, :int(counts[e])] for e in (hot, cold)}
        del codes, sc
    for e in (hot, cold):
        want = {"dW_gate": vals["X"][e] @ vals["dA"][e].T, "dW_up": vals["X"][e] @ vals["dB"][e].T,
                "dW_down": vals["Hg"][e] @ vals["dY"][e].T}
        for n in want:
            assert relerr(to64(g[n][e]), want[n]) <= 8e-3, (n, e)
    # against the MXFP8 oracle with MX weight gradients (tokens whose selection is a near tie in
    # fp64 are left out, as above)
    X, Wr, dY = to64(x["X"]), to64(x["W_r"]), to64(x["dY"])
    b = None if x["bias"] is None else to64(x["bias"])
    lg64 = O.router_logits(X, Wr, b)
    differ = np.nonzero(np.any(np.sort(O.topk_ids(lg64, w.k), 1) != np.sort(gids, 1), axis=1))[0]
    tie_tokens = set(differ.tolist())
    Wg, Wu, Wd = ExpertCache(x["W_gate"]), ExpertCache(x["W_up"]), ExpertCache(x["W_down"])
    weights = {n: ExpertCache(x[n], keep=1) for n in ("W_gate", "W_up", "W_down")}
    cache = mx_layout_cache(sorted({hot, cold}), weights)
    for e in sorted({hot, cold}):
        _, ctx = O.forward_mx(X, Wr, b, Wg, Wu, Wd, w.k, first_local=e, num_local=1, rounded=cache.__getitem__)
        if set(ctx["sched"]["perm"].tolist()) & tie_tokens:
            continue
        go = O.backward_mx(ctx, dY, mx_wgrad=True)
        for n in ("dW_gate", "dW_up", "dW_down"):
            assert relerr(to64(g[n][e]), go[n][e]) <= TOL_MX, (n, e)
    del cache
    # a second run over fresh buffers is bit-identical
    del lay
    torch.cuda.empty_cache()
    lay2, Y2, g2 = run(True)
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))
    for n in ("dW_gate", "dW_up", "dW_down"):
        for e0 in range(0, w.E, 32):
            assert torch.equal(g[n][e0:e0 + 32].view(torch.int16), g2[n][e0:e0 + 32].view(torch.int16)), (n, e0)
    del lay2, Y, Y2, g, g2, x
    torch.cuda.empty_cache()


def test_full_size_ep64_ring_stream_mx():
    # Config 5 at n = 4096 in MXFP8: the ring replays part of the stream and the gate/up weight
    # gradient accumulates over two chunks.  Y, dX and dW_r equal the one-batch MXFP8 layer's over
    # the same 32768 tokens bit for bit; the weight gradients equal them to fp32 summation order.
    w = IN.WORKLOADS["ep64mx_n4096"]
    x = IN.make_inputs(w, device="cuda")
    first, El = w.first_local, w.El

    def run():
        s = B.MoEStreamMX(w.T, w.d, w.E, w.I, w.k, w.stream_M, w.ring_bytes, first, w.num_local)
        s.prepare(x["W_gate"], x["W_up"], x["W_down"])
        Y = s.forward(x["X"], x["W_r"], x["bias"])
        g = s.backward(x["X"], x["W_r"], x["dY"])
        torch.cuda.synchronize()
        assert s.error() == B.MOE_OK
        return s, Y, g

    s, Y, g = run()
    hdr = s.plan()["plan"]
    assert hdr[1] > 1 and hdr[3] > 0  # several backward chunks, replayed rows
    del s
    torch.cuda.empty_cache()
    lay = B.MoELayerMX(w.tokens, w.d, w.E, w.I, w.k, first, w.num_local)
    lay.prepare(x["W_gate"], x["W_up"], x["W_down"])
    Y1 = lay.forward(x["X"], x["W_r"], x["bias"])
    g1 = lay.backward(x["X"], x["W_r"], x["dY"])
    torch.cuda.synchronize()
    assert lay.error() == B.MOE_OK
    del lay
    torch.cuda.empty_cache()
    assert torch.equal(Y.view(torch.int16), Y1.view(torch.int16))
    assert torch.equal(g["dX"].view(torch.int16), g1["dX"].view(torch.int16))
    assert torch.equal(g["dW_r"].view(torch.int32), g1["dW_r"].view(torch.int32))
    for n in ("dW_gate", "dW_up", "dW_down"):
        assert relerr(to64(g[n]), to64(g1[n])) <= 1e-2, n
    del Y1, g1
    # a second run is bit-identical
    _, Y2, g2 = run()
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))
    for n in ("dX", "dW_gate", "dW_up", "dW_down"):
        assert torch.equal(g[n].view(torch.int16), g2[n].view(torch.int16)), n
    del Y, Y2, g, g2, x
    torch.cuda.empty_cache()


def test_full_size_ep64_ring_stream_mx_weight_gradients():
    # Config 5 at n = 4096 in MXFP8 with MXFP8 weight gradients: eight macrobatches, each
    # (macrobatch, expert) segment quantised along its rows on its own.  Y, dX and dW_r equal the
    # one-batch layer's bits; two local experts' weight gradients are within 6e-2 of the MX oracle
    # with the device plan's segments as row groups; a rerun is bit-identical.
    w = IN.WORKLOADS["ep64mx_n4096"]
    x = IN.make_inputs(w, device="cuda")
    first, El = w.first_local, w.El

    def run():
        s = B.MoEStreamMX(w.T, w.d, w.E, w.I, w.k, w.stream_M, w.ring_bytes, first, w.num_local, mx_wgrad=True)
        s.prepare(x["W_gate"], x["W_up"], x["W_down"])
        Y = s.forward(x["X"], x["W_r"], x["bias"])
        g = s.backward(x["X"], x["W_r"], x["dY"])
        torch.cuda.synchronize()
        assert s.error() == B.MOE_OK
        return s, Y, g

    s, Y, g = run()
    plan = s.plan()
    nm = int(plan["plan"][0])
    assert nm > 1
    cum = plan["cum"].copy()
    del s
    torch.cuda.empty_cache()
    lay = B.MoELayerMX(w.tokens, w.d, w.E, w.I, w.k, first, w.num_local, mx_wgrad=True)
    lay.prepare(x["W_gate"], x["W_up"], x["W_down"])
    Y1 = lay.forward(x["X"], x["W_r"], x["bias"])
    g1 = lay.backward(x["X"], x["W_r"], x["dY"])
    torch.cuda.synchronize()
    assert lay.error() == B.MOE_OK
    counts = lay.routing()["counts"].cpu().numpy()
    gids = lay.routing()["ids"].cpu().numpy()
    del lay
    torch.cuda.empty_cache()
    assert torch.equal(Y.view(torch.int16), Y1.view(torch.int16))
    assert torch.equal(g["dX"].view(torch.int16), g1["dX"].view(torch.int16))
    assert torch.equal(g["dW_r"].view(torch.int32), g1["dW_r"].view(torch.int32))
    del Y1, g1

    def groups(el):
        return [(int(cum[(m + 1) * El + el]) if m + 1 < nm else int(counts[el])) - int(cum[m * El + el])
                for m in range(nm)]

    X, Wr, dY = to64(x["X"]), to64(x["W_r"]), to64(x["dY"])
    b = None if x["bias"] is None else to64(x["bias"])
    lg64 = O.router_logits(X, Wr, b)
    differ = np.nonzero(np.any(np.sort(O.topk_ids(lg64, w.k), 1) != np.sort(gids, 1), axis=1))[0]
    tie_tokens = set(differ.tolist())
    caches = {n: ExpertCache(x[n]) for n in ("W_gate", "W_up", "W_down")}
    Wg, Wu, Wd = (lambda e, c=caches[n]: c(e - first) for n in ("W_gate", "W_up", "W_down"))
    weights = {n: ExpertCache(x[n], keep=1) for n in ("W_gate", "W_up", "W_down")}
    cache = mx_layout_cache([0, El - 1], weights)
    for el in (0, El - 1):
        e = first + el
        _, ctx = O.forward_mx(X, Wr, b, Wg, Wu, Wd, w.k, first_local=e, num_local=1,
                              rounded=lambda q: cache[q - first])
        if set(ctx["sched"]["perm"].tolist()) & tie_tokens:
            continue
        go = O.backward_mx(ctx, dY, mx_wgrad=True, row_groups=lambda _l, el=el: groups(el))
        for n in ("dW_gate", "dW_up", "dW_down"):
            assert relerr(to64(g[n][el]), go[n][e]) <= TOL_MX, (n, e)
    del cache
    _, Y2, g2 = run()
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))
    for n in ("dX", "dW_gate", "dW_up", "dW_down"):
        assert torch.equal(g[n].view(torch.int16), g2[n].view(torch.int16)), n
    del Y, Y2, g, g2, x
    torch.cuda.empty_cache()


def test_full_size_ep64_ring_stream():
    # Config 5 at n = 4096 tokens per local expert: 16 minibatches of 2048 tokens through the
    # 256 MiB ring, 6 local experts of 384; the backward replays part of the stream into the
    # ring and accumulates the gate/up weight gradient over two chunks.
    w = IN.WORKLOADS["ep64_n4096"]
    x = IN.make_inputs(w, device="cuda")
    first, El = w.first_local, w.El

    def run():
        s = B.MoEStream(w.T, w.d, w.E, w.I, w.k, w.stream_M, w.ring_bytes, first, w.num_local)
        Y = s.forward(x["X"], x["W_r"], x["bias"], x["W_gate"], x["W_up"], x["W_down"])
        g = s.backward(x["X"], x["W_r"], x["W_gate"], x["W_up"], x["W_down"], x["dY"])
        torch.cuda.synchronize()
        assert s.error() == B.MOE_OK
        return s, Y, g

    s, Y, g = run()
    hdr = s.plan()["plan"]
    assert hdr[1] > 1 and hdr[3] > 0  # several backward chunks, replayed rows

    X, Wr, b, dY = to64(x["X"]), to64(x["W_r"]), to64(x["bias"]), to64(x["dY"])
    caches = {n: ExpertCache(x[n]) for n in ("W_gate", "W_up", "W_down")}
    Wg, Wu, Wd = (lambda e, c=caches[n]: c(e - first) for n in ("W_gate", "W_up", "W_down"))

    # Y and dX at sampled tokens, some with local experts and some without; near-ties in the
    # fp64 logits are skipped (their selection may differ between fp32 and fp64)
    rng = np.random.default_rng(99)
    cand = rng.choice(w.tokens, size=64, replace=False)
    lg = O.router_logits(X[cand], Wr, b)
    srt = -np.sort(-lg, axis=1)
    ok = (srt[:, w.k - 1] - srt[:, w.k]) > 1e-3
    ids = O.topk_ids(lg, w.k)
    has_local = np.any((ids >= first) & (ids < first + El), axis=1)
    pick = [int(t) for t, o, h in zip(cand, ok, has_local) if o and h][:5] + \
           [int(t) for t, o, h in zip(cand, ok, has_local) if o and not h][:2]
    assert len(pick) >= 5
    Yg, dXg = to64(Y), to64(g["dX"])
    ys, yo, dxs, dxo = [], [], [], []
    for t in pick:
        y, dx, _, _, _ = O.token_forward_backward(t, X, Wr, b, Wg, Wu, Wd, w.k, dY, first_local=first,
                                                  num_local=El)
        ys.append(Yg[t]); yo.append(y); dxs.append(dXg[t]); dxo.append(dx)
    assert relerr(np.array(ys), np.array(yo)) <= TOL_BF16
    assert relerr(np.array(dxs), np.array(dxo)) <= TOL_BF16

    # weight gradients of two local experts over the whole stream (the gate/up one accumulated
    # over the backward chunks in fp32)
    for el in (0, El - 1):
        e = first + el
        _, ctx = O.forward(X, Wr, b, Wg, Wu, Wd, w.k, first_local=e, num_local=1)
        go = O.backward(ctx, dY)
        for n in ("dW_gate", "dW_up", "dW_down"):
            assert relerr(to64(g[n][el]), go[n][e]) <= TOL_BF16, (n, e)

    # a second run is bit-identical
    _, Y2, g2 = run()
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))
    for n in ("dX", "dW_gate", "dW_up", "dW_down"):
        assert torch.equal(g[n].view(torch.int16), g2[n].view(torch.int16)), n
    assert torch.equal(g["dW_r"].view(torch.int32), g2["dW_r"].view(torch.int32))
