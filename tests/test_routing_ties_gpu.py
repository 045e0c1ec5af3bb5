"""GPU routing under exact ties (the deterministic tie-break: the lower expert id wins).

Random bf16 inputs almost never give two fp32 logits of one token the same value,
so these cases build logits that tie exactly and are exact in fp32:

* W_r = 0: every logit is its expert's bias, and the bias repeats values (a run
  of equal values across the top-k boundary), holds +0 and -0 (equal as numbers)
  and negative values;
* X with small integer entries and W_r with entries in {0, +-1/2, +-1} whose
  columns repeat (duplicated experts), plus a dyadic bias: every product and
  partial sum is exact in fp32, so the GPU's logits equal the fp64 logits bit
  for bit and ties are frequent, both between duplicated columns and by value.

The routing table (ids, counts, offsets, padded offsets, perm, slot_row) must
equal the oracle's, computed on the exact fp64 logits, bit for bit; the gates
equal the oracle's within 1e-6; the layer stays within the bf16 tolerance of the
oracle.
"""
import numpy as np
import pytest
import torch

import oracle as O

from _util import TOL_BF16, make_case, relerr, run_gpu, run_oracle, to64

pytestmark = pytest.mark.gpu


def _exact_routing(layer, x, k, E):
    """Routing table of the GPU against the oracle on the fp64 logits, bit for bit."""
    X, Wr = to64(x["X"]), to64(x["W_r"])
    b = None if x["bias"] is None else to64(x["bias"])
    lg64 = O.router_logits(X, Wr, b)
    lg_gpu = to64(layer.logits())
    assert np.array_equal(lg_gpu, lg64)  # the inputs make the fp32 logits exact (-0 == +0 here)
    ids = O.topk_ids(lg64, k)
    s = O.schedule(ids, E)
    r = layer.routing()
    assert np.array_equal(r["ids"].cpu().numpy(), ids)
    for key in ("counts", "offsets", "padded_offsets", "perm", "slot_row"):
        assert np.array_equal(r[key].cpu().numpy(), s[key]), key
    assert np.max(np.abs(r["gates"].cpu().numpy() - O.gates(lg64, ids))) < 1e-6
    return lg64, ids


def _ties_across_boundary(lg, k):
    """Tokens whose k-th and (k+1)-th largest logits are equal (the tie decides membership)."""
    srt = -np.sort(-lg, axis=1)
    return int(np.sum(srt[:, k - 1] == srt[:, k]))


def _layer_parity(x, T, d, E, k, I, layer, Y, g):
    Yo, ctx, go = run_oracle(x, k)
    errs = {"Y": relerr(to64(Y), Yo), "dX": relerr(to64(g["dX"]), go["dX"]),
            "dW_r": relerr(to64(g["dW_r"]), go["dW_r"])}
    for n in ("dW_gate", "dW_up", "dW_down"):
        errs[n] = relerr(to64(g[n]), np.stack([go[n][e] for e in range(E)]))
    assert all(v <= TOL_BF16 for v in errs.values()), errs


def test_zero_router_weight_bias_ties_and_signed_zeros():
    T, d, E, k, I = 200, 256, 40, 6, 256
    bias = np.full(E, -3.0, dtype=np.float32)
    bias[[7, 2]] = 5.0                       # a tie at the top: expert 2 before 7
    bias[[33, 4, 19, 11, 25]] = 1.5          # a run of five equal values across the k = 6 boundary
    bias[[9]] = 0.0
    bias[[30]] = -0.0                        # +0 and -0 compare equal: 9 before 30
    w, x = make_case(T, d, E, k, I, seed=31, bias=bias)
    x["W_r"] = torch.zeros_like(x["W_r"])
    layer, Y, g, st = run_gpu(x, T, d, E, k, I)
    assert st == 0
    lg, ids = _exact_routing(layer, x, k, E)
    # every token: 2, 7, then the four lowest ids of the 1.5-run
    assert np.array_equal(ids, np.tile(np.array([2, 7, 4, 11, 19, 25], dtype=np.int32), (T, 1)))
    assert _ties_across_boundary(lg, k) == T

    # the same with the bias run at 0 and -0 across the boundary: the signed zeros tie
    bias2 = np.full(E, -2.0, dtype=np.float32)
    bias2[[1, 5]] = 1.0
    bias2[[12, 3, 38]] = -0.0
    bias2[[20, 8]] = 0.0
    x["bias"] = torch.as_tensor(bias2, device="cuda")
    layer, Y, g, st = run_gpu(x, T, d, E, k, I)
    assert st == 0
    lg, ids = _exact_routing(layer, x, k, E)
    assert np.array_equal(ids, np.tile(np.array([1, 5, 3, 8, 12, 20], dtype=np.int32), (T, 1)))


@pytest.mark.parametrize("T,E,k,dups", [
    (333, 24, 5, [(3, 17), (5, 6, 20), (0, 23), (9, 10, 11, 12)]),
    # E = 384 runs the router GEMM as two 192-wide n-tiles: duplicates inside one tile and across
    (160, 384, 8, [(0, 191, 192, 383), (7, 200), (100, 101), (250, 251, 252)]),
])
def test_duplicated_router_columns_tie_exactly(T, E, k, dups):
    d, I = 256, 256
    rng = np.random.default_rng(1000 + E)
    X = rng.integers(-2, 3, size=(T, d)).astype(np.float32)
    Wr = rng.choice(np.array([-1.0, -0.5, 0.0, 0.5, 1.0], dtype=np.float32), size=(d, E))
    for grp in dups:
        for e in grp[1:]:
            Wr[:, e] = Wr[:, grp[0]]
    bias = (rng.integers(-4, 5, size=E) * 0.5).astype(np.float32)
    for grp in dups:
        # the duplicated experts share one bias, raised by about two standard deviations of the
        # logits (16) so that the top-k cut often falls inside a group
        bias[list(grp)] = bias[grp[0]] + 36.0
    bias[np.nonzero(bias == 0.0)[0][:1]] = -0.0
    w, x = make_case(T, d, E, k, I, seed=32)
    x["X"] = torch.as_tensor(X, device="cuda").to(torch.bfloat16)
    x["W_r"] = torch.as_tensor(Wr, device="cuda").to(torch.bfloat16)
    x["bias"] = torch.as_tensor(bias, device="cuda")
    layer, Y, g, st = run_gpu(x, T, d, E, k, I)
    assert st == 0
    lg, ids = _exact_routing(layer, x, k, E)
    # the duplicated experts tie on every token; where such a tie decides membership, the
    # lower id is in and the higher is out
    dup_ties = 0
    for grp in dups:
        sel = np.isin(ids, list(grp))
        for t in range(T):
            picked = sorted(int(e) for e in ids[t][sel[t]])
            if 0 < len(picked) < len(grp):
                assert picked == sorted(grp)[:len(picked)], (t, grp, picked)
                dup_ties += 1
    assert dup_ties > 0
    assert _ties_across_boundary(lg, k) > 0
    _layer_parity(x, T, d, E, k, I, layer, Y, g)
