"""Seeded synthetic inputs for the MoE layer (shared by tests, bench and smoke).

This module holds no arithmetic of the layer itself: it only draws tensors.
Both the CUDA path and the CPU oracle consume the exact bits it produces.

Workloads (the pages name model families and print no shapes; these stand in):

* ``tiny``      T=128,  d=256,  E=8,   k=2, I=512
* ``dsv3``      T=2048, d=7168, E=256, k=8, I=2048   (DeepSeek-V3-like, near-uniform routing)
* ``kimi``      T=4096, d=7168, E=384, k=8, I=2048   (Kimi-K2-like, Zipf(1.2)-skewed load)
* ``kimi_mx``   ``kimi`` in MXFP8 mode
* ``ep64``      6 local experts of 384, 16 minibatches x 2048 tokens, ring buffer
* ``ep64mx``  the ring-streamed slice in MXFP8
* ``epmx``, ``epbf``  the same slice as one batch of 32768 tokens (MXFP8 / bf16), no ring
* ``dsv3_e16``  the dsv3 expert shape with 16 experts and 128 tokens (profiler captures)
* ``kimi_mx_e24`` the kimi expert shape in MXFP8, 24 experts, 256 tokens (profiler captures)
* ``epmx_t8192_n2368`` epmx_n2368's dispatched rows over 8192 tokens, 96 experts (profiler captures)

Distributions: X, dY ~ N(0, 1); W_gate, W_up ~ N(0, 1/d) (std 1/sqrt(fan_in));
W_down ~ N(0, 1/I); W_r ~ N(0, 0.02^2); every tensor rounded once to bf16 (RNE).
Every tensor (and every expert's slice) has its own seed derived from the
workload seed and the tensor name, so tensors can be regenerated one by one.
"""

from __future__ import annotations

import dataclasses
import hashlib
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    E: int
    k: int
    I: int
    mxfp8: bool = False
    zipf: bool = False          # per-expert router bias giving a Zipf(1.2)-shaped load
    first_local: int = 0
    num_local: int = 0          # 0 = all experts are local
    seed: int = 0
    stream_M: int = 0           # > 0: M minibatches of T tokens through a ring of ring_bytes
    ring_bytes: int = 0
    local_tokens: int = 0       # streamed slice: assignments each local expert receives over the stream
    nvfp4: bool = False         # NVFP4 layer (moe_fwd_nvfp4 / moe_bwd_nvfp4)

    @property
    def El(self) -> int:
        return self.num_local or self.E

    @property
    def tokens(self) -> int:
        """Tokens per step (all minibatches of a streamed workload)."""
        return self.T * max(self.stream_M, 1)

    def model_flops(self) -> float:
        """fwd+bwd model FLOPs: 18 d I per local assignment (6 fwd, 12 bwd) + 6 T d E router."""
        assign = self.El * self.local_tokens if self.local_tokens else self.tokens * self.k
        return 18.0 * self.d * self.I * assign + 6.0 * self.tokens * self.d * self.E

    def forward_flops(self) -> float:
        """forward model FLOPs: 6 d I per local assignment + 2 T d E router."""
        assign = self.El * self.local_tokens if self.local_tokens else self.tokens * self.k
        return 6.0 * self.d * self.I * assign + 2.0 * self.tokens * self.d * self.E


WORKLOADS = {
    "tiny": Workload("tiny", 128, 256, 8, 2, 512),
    "dsv3": Workload("dsv3", 2048, 7168, 256, 8, 2048),
    "kimi": Workload("kimi", 4096, 7168, 384, 8, 2048, zipf=True),
    "kimi_mx": Workload("kimi_mx", 4096, 7168, 384, 8, 2048, mxfp8=True, zipf=True),
    # the 256-expert top-8 configuration in MXFP8 (the precision north of the bf16 dsv3 line)
    "dsv3_mx": Workload("dsv3_mx", 2048, 7168, 256, 8, 2048, mxfp8=True),
    # the dsv3 expert shape and load (64 tokens per expert) with 16 experts: a
    # ~3 GB case for profiler captures (weights still exceed the 126 MB L2)
    "dsv3_e16": Workload("dsv3_e16", 128, 7168, 16, 8, 2048),
    # the kimi expert shape in MXFP8 with 24 experts and 256 tokens (~85 per expert, near-uniform):
    # a few-GB case for profiler captures of the block-scaled GEMMs
    "kimi_mx_e24": Workload("kimi_mx_e24", 256, 7168, 24, 8, 2048, mxfp8=True),
    # dsv3_e16 in MXFP8 (64 tokens per expert): profiler captures of the MXFP8 weight gradients
    "dsv3_mx_e16": Workload("dsv3_mx_e16", 128, 7168, 16, 8, 2048, mxfp8=True),
}
# Per-rank expert slice as at EP64: 6 local experts of 384, 16 minibatches of 2048
# tokens streamed through a 256 MiB ring; n = tokens each local expert receives.
for _n in (512, 1024, 2048, 2368, 4096, 8192, 16384):
    WORKLOADS[f"ep64_n{_n}"] = Workload(f"ep64_n{_n}", 2048, 7168, 384, 8, 2048, first_local=0, num_local=6,
                                        stream_M=16, ring_bytes=256 << 20, local_tokens=_n)
# The same ring-streamed slice in MXFP8 (gate/up, down and both dgrads on MXFP8, bf16 weight gradients).
# A ring row holds the bf16 row and its fp8 codes (1.52x the bytes): 384 MiB hold 18,432 rows, about
# the 18,724 of the bf16 stream's 256 MiB ring.
for _n in (512, 2368, 4096):
    WORKLOADS[f"ep64mx_n{_n}"] = Workload(f"ep64mx_n{_n}", 2048, 7168, 384, 8, 2048, mxfp8=True, first_local=0,
                                          num_local=6, stream_M=16, ring_bytes=384 << 20, local_tokens=_n)
# The same per-rank slice (6 of 384 experts, 32768 tokens, n per local expert) as one batch, the
# dispatched rows held whole instead of in a ring: MXFP8 (epmx) and bf16 (epbf), the regime
# where the grouped GEMMs are bound by the tensor cores rather than by the weight stream.
for _n in (512, 2368, 4096, 8192):
    WORKLOADS[f"epmx_n{_n}"] = Workload(f"epmx_n{_n}", 32768, 7168, 384, 8, 2048, mxfp8=True, first_local=0,
                                        num_local=6, local_tokens=_n)
    WORKLOADS[f"epbf_n{_n}"] = Workload(f"epbf_n{_n}", 32768, 7168, 384, 8, 2048, first_local=0, num_local=6,
                                        local_tokens=_n)
# epmx_n2368's expert work (6 local experts x 2368 rows, MXFP8) over 8192 tokens and 96 experts: the
# same dispatched rows and GEMM tiles with a padded-row capacity (and workspace) a quarter of the
# size, for profiler captures (a few GB on the device)
# NVFP4 layer (forward and backward, bf16 weight gradients): the dsv3 and kimi configurations, the EP64 slice as one batch (where the
# grouped GEMMs are tensor-bound), and two few-GB cases for profiler captures
WORKLOADS["dsv3_nv"] = Workload("dsv3_nv", 2048, 7168, 256, 8, 2048, nvfp4=True)
WORKLOADS["kimi_nv"] = Workload("kimi_nv", 4096, 7168, 384, 8, 2048, zipf=True, nvfp4=True)
WORKLOADS["dsv3_nv_e16"] = Workload("dsv3_nv_e16", 128, 7168, 16, 8, 2048, nvfp4=True)
for _n in (512, 2368, 4096, 8192):
    WORKLOADS[f"epnv_n{_n}"] = Workload(f"epnv_n{_n}", 32768, 7168, 384, 8, 2048, first_local=0, num_local=6,
                                        local_tokens=_n, nvfp4=True)
WORKLOADS["epnv_t8192_n2368"] = Workload("epnv_t8192_n2368", 8192, 7168, 96, 8, 2048, first_local=0, num_local=6,
                                         local_tokens=2368, nvfp4=True)
WORKLOADS["epmx_t8192_n2368"] = Workload("epmx_t8192_n2368", 8192, 7168, 96, 8, 2048, mxfp8=True, first_local=0,
                                         num_local=6, local_tokens=2368)


def _seed(base: int, *names) -> int:
    h = hashlib.sha256(("%d/" % base + "/".join(str(n) for n in names)).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _normal(shape, std, seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def expert_weights(w: Workload, name: str, e: int, device="cpu") -> torch.Tensor:
    """One expert's slice of W_gate / W_up ([d, I]) or W_down ([I, d]), bf16."""
    if name in ("W_gate", "W_up"):
        return _normal((w.d, w.I), 1.0 / math.sqrt(w.d), _seed(w.seed, w.name, name, e), device)
    if name == "W_down":
        return _normal((w.I, w.d), 1.0 / math.sqrt(w.I), _seed(w.seed, w.name, name, e), device)
    raise KeyError(name)


def make_inputs(w: Workload, device="cpu", T: int | None = None) -> dict:
    """All layer inputs for workload w (T may be overridden to sub-sample tokens).

    Streamed workloads get all M * T tokens; only the local experts' weights."""
    T = T or w.tokens
    out = {
        "X": _normal((T, w.d), 1.0, _seed(w.seed, w.name, "X"), device),
        "W_r": _normal((w.d, w.E), 0.02, _seed(w.seed, w.name, "W_r"), device),
        "dY": _normal((T, w.d), 1.0, _seed(w.seed, w.name, "dY"), device),
    }
    El = w.El
    for name in ("W_gate", "W_up", "W_down"):
        shape = (El, w.d, w.I) if name != "W_down" else (El, w.I, w.d)
        t = torch.empty(shape, dtype=torch.bfloat16, device=device)
        for el in range(El):
            t[el] = expert_weights(w, name, w.first_local + el, device)
        out[name] = t
    if w.zipf:
        out["bias"] = zipf_bias(w, out["X"], out["W_r"])
    elif w.local_tokens:
        out["bias"] = local_load_bias(w, out["X"], out["W_r"])
    else:
        out["bias"] = None
    return out


def local_load_bias(w: Workload, X: torch.Tensor, W_r: torch.Tensor, iters: int = 60) -> torch.Tensor:
    """Router bias giving each local expert about w.local_tokens assignments over the
    stream, the other experts sharing the rest evenly (same fixed-count calibration
    as zipf_bias; torch.topk only measures the load)."""
    dev = X.device
    logits = X.float() @ W_r.float()
    total = X.shape[0] * w.k
    target = torch.full((w.E,), (total - w.El * w.local_tokens) / (w.E - w.El), dtype=torch.float64, device=dev)
    target[w.first_local:w.first_local + w.El] = float(w.local_tokens)
    b = torch.zeros(w.E, dtype=torch.float64, device=dev)
    for _ in range(iters):
        idx = torch.topk(logits + b.float(), w.k, dim=1).indices
        obs = torch.bincount(idx.flatten(), minlength=w.E).double()
        b += 0.5 * (torch.log(target) - torch.log(torch.clamp(obs, min=0.5)))
        b -= b.mean()
    return b.float()


def zipf_target_shares(E: int, s: float = 1.2, hot_over_mean: float = 10.0) -> torch.Tensor:
    """Shares q_r proportional to (r + r0)^-s, r = 1..E, with r0 chosen so max/mean = hot_over_mean.

    Pure Zipf(1.2) at E = 384 would put ~94x the mean load on the hottest
    expert, more than one expert can take (T tokens = 48x the mean at k = 8),
    and the workload asks for ~10x; the offset r0 reconciles the two.
    """
    r = torch.arange(1, E + 1, dtype=torch.float64)

    def ratio(r0):
        q = (r + r0) ** (-s)
        return float(q[0] / q.mean())

    lo, hi = 0.0, 1e4
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if ratio(mid) > hot_over_mean:
            lo = mid
        else:
            hi = mid
    q = (r + 0.5 * (lo + hi)) ** (-s)
    return q / q.sum()


def zipf_bias(w: Workload, X: torch.Tensor, W_r: torch.Tensor, iters: int = 60) -> torch.Tensor:
    """Per-expert router bias (fp32 [E]) that skews top-k load toward Zipf shares.

    Fixed-count calibration on the seeded logits: b_e += 0.5 (log target_e -
    log max(observed_e, 0.5)).  The rank -> expert map is a seeded permutation.
    torch.topk only measures load here; the layer's own selection rule is not used.
    """
    dev = X.device
    logits = X.float() @ W_r.float()
    q = zipf_target_shares(w.E)
    g = torch.Generator(device="cpu")
    g.manual_seed(_seed(w.seed, w.name, "zipf_perm"))
    perm = torch.randperm(w.E, generator=g)
    target = torch.empty(w.E, dtype=torch.float64)
    target[perm] = q * X.shape[0] * w.k
    target = target.to(dev)
    b = torch.zeros(w.E, dtype=torch.float64, device=dev)
    for _ in range(iters):
        idx = torch.topk(logits + b.float(), w.k, dim=1).indices
        obs = torch.bincount(idx.flatten(), minlength=w.E).double()
        b += 0.5 * (torch.log(target) - torch.log(torch.clamp(obs, min=0.5)))
        b -= b.mean()
    return b.float()
