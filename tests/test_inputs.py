"""The seeded input recipe on CPU: Zipf target shares, router-bias load calibration,
per-tensor seeding, dtype and the fan-in scales of the weights."""
import dataclasses
import math

import torch

from mixture_experts_layer_27_b200 import inputs as IN


def test_zipf_shares_put_ten_times_the_mean_on_the_hottest_expert():
    for E in (64, 256, 384):
        q = IN.zipf_target_shares(E)
        assert abs(float(q.sum()) - 1.0) < 1e-12
        assert abs(float(q[0] / q.mean()) - 10.0) < 1e-6
        assert torch.all(q[1:] < q[:-1])
        # a power law of exponent 1.2 in (r + r0): log-ratios of consecutive shares match it
        r = torch.arange(1, E + 1, dtype=torch.float64)
        r0 = float(q[0] ** (-1 / 1.2) / (q[1] ** (-1 / 1.2) - q[0] ** (-1 / 1.2))) - 1.0
        assert torch.allclose(q / q[0], ((r + r0) / (1 + r0)) ** -1.2, rtol=1e-9)


def test_pure_zipf_would_overload_the_hottest_expert():
    # why the recipe offsets the ranks: plain Zipf(1.2) over 384 experts gives ~94x the mean
    q = torch.arange(1, 385, dtype=torch.float64) ** -1.2
    assert 90.0 < float(q[0] / q.mean()) < 100.0


def test_inputs_are_seeded_per_tensor_and_rounded_to_bf16():
    w = IN.Workload("t_inputs", 64, 256, 8, 2, 256, seed=3)
    a, b = IN.make_inputs(w), IN.make_inputs(w)
    for n in ("X", "W_r", "dY", "W_gate", "W_up", "W_down"):
        assert a[n].dtype == torch.bfloat16 and torch.equal(a[n], b[n]), n
    assert not torch.equal(a["X"], a["dY"]) and not torch.equal(a["W_gate"], a["W_up"])
    # an expert slice regenerates exactly the same expert weights
    s = IN.make_inputs(dataclasses.replace(w, first_local=3, num_local=2))
    for n in ("W_gate", "W_up", "W_down"):
        assert torch.equal(s[n], a[n][3:5]), n
    assert torch.equal(s["X"], a["X"])
    c = IN.make_inputs(dataclasses.replace(w, seed=4))
    assert not torch.equal(c["X"], a["X"])


def test_weight_scales_follow_fan_in():
    w = IN.Workload("t_scale", 512, 1024, 4, 2, 512, seed=4)
    x = IN.make_inputs(w)

    def std(t):
        return float(t.float().std())

    assert abs(std(x["X"]) - 1.0) < 0.02
    assert abs(std(x["dY"]) - 1.0) < 0.02
    assert abs(std(x["W_gate"]) * math.sqrt(1024) - 1.0) < 0.02
    assert abs(std(x["W_up"]) * math.sqrt(1024) - 1.0) < 0.02
    assert abs(std(x["W_down"]) * math.sqrt(512) - 1.0) < 0.02
    assert abs(std(x["W_r"]) / 0.02 - 1.0) < 0.03


def _loads(x, k, E):
    logits = x["X"].float() @ x["W_r"].float() + x["bias"]
    idx = torch.topk(logits, k, dim=1).indices
    return torch.bincount(idx.flatten(), minlength=E).double()


# The calibrations run at the model width d = 7168 (router logits with std ~1.7, as in the
# workloads); I = 8 keeps the unused expert weights small.
def test_zipf_bias_skews_the_load_to_the_target():
    w = IN.Workload("t_zipf", 4096, 7168, 64, 2, 8, zipf=True, seed=5)
    obs = _loads(IN.make_inputs(w), w.k, w.E)
    assert obs.sum() == w.T * w.k
    assert 9.5 < float(obs.max() / obs.mean()) < 10.5  # target 10x the mean
    q = IN.zipf_target_shares(w.E)
    srt = torch.sort(obs, descending=True).values / obs.sum()
    assert float(torch.max(torch.abs(srt - q))) < 0.005


def test_local_load_bias_gives_each_local_expert_its_token_count():
    w = IN.Workload("t_local", 4096, 7168, 64, 2, 8, first_local=8, num_local=4, local_tokens=300, seed=6)
    obs = _loads(IN.make_inputs(w), w.k, w.E)
    local = obs[8:12]
    assert torch.all(torch.abs(local - 300) <= 10), local
