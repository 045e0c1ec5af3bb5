"""bench.py's own accounting on CPU: algorithmic bytes and FLOPs per kernel, and when an ncu
traffic figure may be attached to the roofline."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from mixture_experts_layer_27_b200 import inputs as IN  # noqa: E402


def test_dsv3_weight_gradient_bytes():
    w = IN.WORKLOADS["dsv3"]
    rows, d, I, El = w.T * w.k, w.d, w.I, w.El
    b = bench.algorithmic_bytes(w)
    # dW_gate + dW_up written once (bf16) + X_perm and dA, dB read once
    assert b["gemm_wgrad_gateup"] == 2 * El * d * I * 2 + rows * d * 2 + 2 * rows * I * 2
    assert abs(b["gemm_wgrad_gateup"] / 1e9 - 15.401484288) < 1e-9
    assert b["gemm_wgrad_down"] == El * I * d * 2 + rows * I * 2 + rows * d * 2


def test_fp32_weight_gradients_double_only_the_gradient_writes():
    for name in ("dsv3", "kimi_mx", "ep64_n2368"):
        w = IN.WORKLOADS[name]
        g1 = w.El * w.d * w.I * 2  # one family's bf16 gradient bytes
        b2, b4 = bench.algorithmic_bytes(w, 2), bench.algorithmic_bytes(w, 4)
        assert b4["gemm_wgrad_gateup"] - b2["gemm_wgrad_gateup"] == 2 * g1
        assert b4["gemm_wgrad_down"] - b2["gemm_wgrad_down"] == g1
        for k in b2:
            if not k.startswith("gemm_wgrad"):
                assert b4[k] == b2[k], k


def test_router_weight_gradient_flops():
    w = IN.WORKLOADS["dsv3"]
    f = bench.algorithmic_flops(w)
    assert f["router_wgrad"] == 2 * w.T * w.d * w.E == f["router_logits"]
    rows, dI = w.T * w.k, w.d * w.I
    assert f["gemm_gateup_swiglu"] + f["gemm_down_combw"] == 6 * dI * rows
    # the persistent kernel runs gate/up and down in one launch: an alternative, not an extra GEMM
    assert f["gemm_gateup_down_persistent"] == f["gemm_gateup_swiglu"] + f["gemm_down_combw"]
    assert f["gemm_dgrads_persistent"] == f["gemm_dgrad_down_swiglu_bwd"] + f["gemm_dgrad_gateup"]
    # the MXFP8 weight-gradient GEMMs replace the bf16 ones (MOE_MXFP8_ALL): alternatives as well
    assert f["gemm_wgrad_gateup_mx"] == f["gemm_wgrad_gateup"] and f["gemm_wgrad_down_mx"] == f["gemm_wgrad_down"]
    assert sum(v for k, v in f.items()
               if k.startswith("gemm_") and "persistent" not in k and not k.endswith("_mx")) == 18 * dI * rows


def test_traffic_figure_only_for_the_captured_sources():
    key = next(iter(bench.NCU_TRAFFIC))
    value, src = bench.NCU_TRAFFIC[key]
    t = bench.ncu_traffic(*key)
    assert t is None or (t == value and src == bench.gemm_source_hash())
    assert bench.ncu_traffic(key[0], key[1] + "+wgrad_fp32") is None
    assert bench.ncu_traffic("no_such_kernel", key[1]) is None


def test_nvfp4_step_accounting():
    # the NVFP4 step's four expert GEMMs carry the layer's forward and dgrad FLOPs (6 + 6 d I per
    # assignment), the bf16 weight gradients the other 6; their weights stream at 9/16 byte per value
    for name in ("dsv3_nv", "epnv_n2368"):
        w = IN.WORKLOADS[name]
        by, fl = bench.nv_algorithmic(w)
        rows, d, I, El = bench.local_rows(w), w.d, w.I, w.El
        nv = [fl[k] for k in bench.NV_GEMMS]
        assert sum(nv) == 12 * d * I * rows
        assert fl["gemm_wgrad_gateup"] + fl["gemm_wgrad_down"] == 6 * d * I * rows
        assert sum(nv) + fl["gemm_wgrad_gateup"] + fl["gemm_wgrad_down"] == 18 * d * I * rows
        W = El * d * I * 9 / 16
        assert by["gemm_down_combw_nvfp4"] == W + rows * I * 9 / 16 + rows * d * 2
        assert by["gemm_dgrad_gateup_nvfp4"] == 2 * W + 2 * rows * I * 9 / 16 + rows * d * 2
        # the weight gradients are the bf16 layer's
        assert by["gemm_wgrad_gateup"] == bench.algorithmic_bytes(w)["gemm_wgrad_gateup"]
        cfg = bench.nv_config(w)
        assert cfg["precision"] == "nvfp4" and cfg["wgrad_dtype"] == "bf16" and " nvfp4," in cfg["workload"]
    assert IN.WORKLOADS["dsv3_nv"].model_flops() == IN.WORKLOADS["dsv3"].model_flops()
