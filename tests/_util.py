"""Shared helpers of the test suite (not collected as tests)."""
import numpy as np
import torch

import oracle as O
from mixture_experts_layer_27_b200 import binding as B
from mixture_experts_layer_27_b200 import inputs as IN

TOL_BF16 = 2e-2  # max |gpu - ref| / max |ref| per tensor, bf16 mode


def to64(t) -> np.ndarray:
    """bf16 / fp32 tensor -> fp64 numpy (exact: every bf16 and fp32 value is an fp64 value)."""
    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


def relerr(gpu, ref) -> float:
    gpu, ref = np.asarray(gpu, dtype=np.float64), np.asarray(ref, dtype=np.float64)
    scale = np.max(np.abs(ref)) if ref.size else 0.0
    if scale == 0.0:
        return float(np.max(np.abs(gpu))) if gpu.size else 0.0
    return float(np.max(np.abs(gpu - ref)) / scale)


def make_case(T, d, E, k, I, seed=0, bias=None, device="cuda"):
    w = IN.Workload(f"case_{T}_{d}_{E}_{k}_{I}", T, d, E, k, I, seed=seed)
    x = IN.make_inputs(w, device=device)
    if bias is not None:
        x["bias"] = torch.as_tensor(bias, dtype=torch.float32, device=device)
    return w, x


def run_gpu(x, T, d, E, k, I, first=0, num=0, layer=None):
    layer = layer or B.MoELayer(T, d, E, I, k, first_local_expert=first, num_local_experts=num)
    El = num or (E - first)
    Wg, Wu, Wd = x["W_gate"][first:first + El], x["W_up"][first:first + El], x["W_down"][first:first + El]
    Y = layer.forward(x["X"], x["W_r"], x["bias"], Wg.contiguous(), Wu.contiguous(), Wd.contiguous())
    g = layer.backward(x["X"], x["W_r"], Wg.contiguous(), Wu.contiguous(), Wd.contiguous(), x["dY"])
    torch.cuda.synchronize()
    st = layer.error()
    return layer, Y, g, st


def run_oracle(x, k, first=0, num=None):
    X, Wr, dY = to64(x["X"]), to64(x["W_r"]), to64(x["dY"])
    b = None if x["bias"] is None else to64(x["bias"])
    Wg, Wu, Wd = to64(x["W_gate"]), to64(x["W_up"]), to64(x["W_down"])
    Y, ctx = O.forward(X, Wr, b, Wg, Wu, Wd, k, first_local=first, num_local=num)
    return Y, ctx, O.backward(ctx, dY)


def mx_layout_job(args):
    """Worker of a spawned process pool: one MX-rounded weight layout of one expert.

    args = (expert, layout name, float32 weight, axis); returns (expert, name, float32 layout).
    The rounded values (E4M3 times a power of two) are exact in float32."""
    e, name, W, axis = args
    return e, name, O.mx_round(np.asarray(W, dtype=np.float64), axis).astype(np.float32)


# the six layouts of oracle.mx_weight_layouts: (name, weight, axis)
MX_LAYOUTS = (("gate_d", "W_gate", 0), ("up_d", "W_up", 0), ("down_i", "W_down", 0),
              ("down_d", "W_down", 1), ("gate_i", "W_gate", 1), ("up_i", "W_up", 1))


def mx_layout_cache(experts, weights, processes=8) -> dict:
    """{expert: {layout: float32 array}} for `experts`, rounded in a spawned pool.

    weights: dict name -> callable e -> fp64 weight (host).  The pool is started with
    'spawn', so it is safe after CUDA has been initialised in this process."""
    import multiprocessing as mp
    from concurrent.futures import ProcessPoolExecutor
    out = {int(e): {} for e in experts}
    # a worker that dies raises BrokenProcessPool here (no silent respawning)
    with ProcessPoolExecutor(max_workers=processes, mp_context=mp.get_context("spawn")) as pool:
        futs = [pool.submit(mx_layout_job, (int(e), ln, weights[wn](e).astype(np.float32), ax))
                for e in experts for ln, wn, ax in MX_LAYOUTS]
        for f in futs:
            e, ln, arr = f.result(timeout=600)
            out[e][ln] = arr
    return out
