"""Expert parallelism across ranks, the protocol on CPU: gloo ranks on 127.0.0.1, fp64 oracle math.

Each rank holds its own tokens and the experts [rank E/R, (rank+1) E/R).  One step runs the
exchange the expert-parallel layer runs on GPUs ("Three design decisions that matter", bullet
1): each rank routes its own tokens and publishes its routing table; each owner pulls, for its
experts, every source's rows in source-rank order (ascending token inside a source) and their
gates; it runs its experts and pushes each output row back to the source's slot of that
assignment; the sources combine their k slots in slot order.  The backward mirrors it (dY rows
pulled, router-gate gradients and dX rows pushed back; each rank's dW_r is its tokens' part).
Rows move as point-to-point messages here (peer loads and stores on GPUs).  Every result must
equal the one-process oracle layer on the rank-major concatenation of the ranks' tokens.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(R, T, d, E, I):
    rng = np.random.default_rng(70 + R)
    return dict(X=rng.standard_normal((R * T, d)), W_r=rng.standard_normal((d, E)) * 0.5,
                Wg=rng.standard_normal((E, d, I)) / np.sqrt(d), Wu=rng.standard_normal((E, d, I)) / np.sqrt(d),
                Wd=rng.standard_normal((E, I, d)) / np.sqrt(I), dY=rng.standard_normal((R * T, d)))


def _ep_worker(rank, R, port, q, shape):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    import torch.distributed as dist
    import oracle as O
    dist.init_process_group("gloo", rank=rank, world_size=R, timeout=datetime.timedelta(seconds=60))
    try:
        T, d, E, k, I = shape
        inp = _inputs(R, T, d, E, I)
        El, lo = E // R, rank * (E // R)
        X, dY = inp["X"][rank * T:(rank + 1) * T], inp["dY"][rank * T:(rank + 1) * T]
        W_r = inp["W_r"]
        Wg, Wu, Wd = inp["Wg"][lo:lo + El], inp["Wu"][lo:lo + El], inp["Wd"][lo:lo + El]  # local experts only

        # source: route the own tokens, publish the routing table
        l = O.router_logits(X, W_r, None)
        ids = O.topk_ids(l, k)
        g = O.gates(l, ids)
        tabs = [torch.empty((T, k), dtype=torch.int64) for _ in range(R)]
        dist.all_gather(tabs, torch.from_numpy(ids.astype(np.int64)))
        plan = O.ep_plan([t.numpy() for t in tabs], E)
        own = plan["owners"][rank]

        def exchange(make_rows, width, owner_side_order):
            """Moves rows between ranks.  make_rows(peer) -> this rank's rows for `peer`, in the order
            owner_side_order(peer) lists them; returns {peer: rows received from peer}."""
            recv, reqs = {}, []
            for peer in range(R):
                n = len(owner_side_order(rank, peer))
                recv[peer] = torch.empty((n, width), dtype=torch.float64)
                if peer != rank and n:
                    reqs.append(dist.irecv(recv[peer], peer))
            for peer in range(R):
                rows = make_rows(peer)
                if peer == rank:
                    if len(rows):
                        recv[rank].copy_(torch.from_numpy(np.asarray(rows).reshape(-1, width)))
                elif len(rows):
                    reqs.append(dist.isend(torch.from_numpy(np.ascontiguousarray(np.asarray(rows).reshape(-1, width))),
                                           peer))
            for r in reqs:
                r.wait()
            return {p: v.numpy() for p, v in recv.items()}

        # rows of owner `owner` that come from source `src`, in the owner's row order
        def owner_rows(owner, src):
            return [(t, j) for (s, t, j) in plan["owners"][owner]["rows"] if s == src]

        def pull(values):
            """Owner pulls values[t, j-or-token] of its rows from every source; returns rows in order."""
            got = exchange(lambda owner: [values(t, j) for (t, j) in owner_rows(owner, rank)],
                           width=values(0, 0).size if T else 1, owner_side_order=lambda me, src: owner_rows(me, src))
            it = {s: iter(v) for s, v in got.items()}
            return np.array([next(it[s]) for (s, t, j) in own["rows"]]).reshape(len(own["rows"]), -1)

        def push(rows_vals):
            """Owner pushes one value row per own row back to its source; returns [T, k, width] at the source."""
            width = rows_vals.shape[1]
            by_src = {s: [rows_vals[i] for i, (ss, t, j) in enumerate(own["rows"]) if ss == s] for s in range(R)}
            got = exchange(lambda src: by_src[src], width, owner_side_order=lambda me, owner: owner_rows(owner, me))
            out = np.zeros((T, k, width))
            for owner in range(R):
                for (t, j), v in zip(owner_rows(owner, rank), got[owner]):
                    out[t, j] = v
            return out

        # ---- forward: pull dispatch (X row and gate), experts, push combine
        xg = pull(lambda t, j: np.concatenate([X[t], [g[t, j]]]))
        Xp, gp = xg[:, :d], xg[:, d]
        Op = np.zeros((len(own["rows"]), d))
        saved = []
        for el in range(El):
            r0 = int(own["base"][el, 0]) + sum(int(own["counts"][e]) for e in range(el))
            r1 = r0 + int(own["counts"][el])
            A = Xp[r0:r1] @ Wg[el]
            B = Xp[r0:r1] @ Wu[el]
            H = O.silu(A) * B
            Op[r0:r1] = gp[r0:r1, None] * (H @ Wd[el])
            saved.append((r0, r1, A, B, H))
        Y = push(Op).sum(axis=1)  # slot order

        # ---- backward: pull reverse-combine (dY rows), experts, push dg and dX rows back
        dYp = pull(lambda t, j: dY[t])
        dXp = np.zeros((len(own["rows"]), d))
        dgp = np.zeros((len(own["rows"]), 1))
        dW = {}
        for el, (r0, r1, A, B, H) in enumerate(saved):
            dO = gp[r0:r1, None] * dYp[r0:r1]
            dH = dO @ Wd[el].T
            dA = dH * B * O.silu_grad(A)
            dB = dH * O.silu(A)
            dgp[r0:r1, 0] = np.sum(dYp[r0:r1] * (H @ Wd[el]), axis=1)
            dXp[r0:r1] = dA @ Wg[el].T + dB @ Wu[el].T
            dW[lo + el] = (Xp[r0:r1].T @ dA, Xp[r0:r1].T @ dB, H.T @ dO)
        dg = push(dgp)[:, :, 0]
        dl = np.zeros((T, E))
        np.put_along_axis(dl, ids.astype(np.int64), g * (dg - np.sum(g * dg, axis=1, keepdims=True)), axis=1)
        dX = push(dXp).sum(axis=1) + dl @ W_r.T
        dWr = torch.from_numpy(X.T @ dl)
        dist.all_reduce(dWr)  # the router is replicated: its gradient is the sum of the ranks' parts

        # ---- the one-process oracle layer on the rank-major batch
        Yo, ctx = O.forward(inp["X"], W_r, None, inp["Wg"], inp["Wu"], inp["Wd"], k)
        go = O.backward(ctx, inp["dY"])
        sl = slice(rank * T, (rank + 1) * T)

        def rel(a, b):
            return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)) if b.size else 0.0
        errs = dict(Y=rel(Y, Yo[sl]), dX=rel(dX, go["dX"][sl]), dW_r=rel(dWr.numpy(), go["dW_r"]),
                    dW=max(max(rel(dW[e][0], go["dW_gate"][e]), rel(dW[e][1], go["dW_up"][e]),
                               rel(dW[e][2], go["dW_down"][e])) for e in dW))
        q.put((rank, errs, int(own["counts"].sum())))
    finally:
        dist.destroy_process_group()


def _run(R, shape):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ep_worker, args=(r, R, port, q, shape)) for r in range(R)]
    for p in procs:
        p.start()
    out = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(out)


@pytest.mark.parametrize("R", [2, 4])
def test_expert_parallel_exchange_equals_the_one_process_layer(R):
    T, d, E, k, I = 24, 32, 8, 3, 16
    out = _run(R, (T, d, E, k, I))
    assert [r for r, _, _ in out] == list(range(R))
    assert sum(n for _, _, n in out) == R * T * k  # every assignment ran on exactly one owner
    for rank, errs, _ in out:
        assert all(v < 1e-10 for v in errs.values()), (rank, errs)
