"""Seeded synthetic inputs for the MoE layer -- shared by the tests, the bench
and the CPU oracle's callers.  Holds no arithmetic of the method itself: only
shapes, distributions and seeds.

Workloads (the pages publish no dataset for this path; every tensor is drawn
from the stated distributions):

  tiny_fp32    T=128,   d=256,  E=256, k=8, 1 shared, I=Is=64,     fp32
               x~N(0,1), W~N(0,0.02), bias~U(-0.05,0.05), 1 bias step
  small_bf16   T=4096,  d=2048, E=64,  k=6, 2 shared, I=Is=1408,   bf16
               x~N(0,1), W~N(0,0.02), bias=0, 10 bias steps
  v3_prefill   T=8192,  d=7168, E=256, k=8, 1 shared, I=Is=2048,   bf16
               x~N(0,1), W~N(0,0.006), bias~U(-0.01,0.01)
  v3_decode    T=64 per call, V3 shape and distributions, fresh x per call
  *_fp8        small_fp8, v3_prefill_fp8, v3_decode_fp8: the same tensors,
               expert GEMMs in E4M3 (weights, tokens and h quantized in
               1x32 tiles along the contraction, power-of-two scales)
  skew_stress  T=32768, V3 shape; x[:,0]=1 and W_g[i][0]=o_i, a per-expert
               logit offset that ranks expert popularity by a seeded
               permutation with Zipf exponent 1.2 (see ``zipf_offsets``);
               200 bias steps with fresh x per step

The DeepSeek-V3 shape (256 routed experts, top-8, one shared expert) is the
one "DeepSeek V3 From Scratch" ("The idea") and the crackai.dev DeepSeek-V3
page ("How It Works") describe; d=7168 and I=2048 are the layer sizes the
workload fixes.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int
    d: int
    E: int
    k: int
    I: int
    S: int
    Is: int
    dtype: str            # "f32", "bf16" or "fp8" (bf16 tokens, E4M3 expert GEMMs)
    w_std: float
    bias_kind: str        # "uniform" or "zero"
    bias_range: float
    seed: int
    steps: int = 0        # bias-update steps the workload runs
    step_size: float = 1e-3
    zipf_s: float = 0.0   # > 0: skewed popularity through a logit offset

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def scaled(self, **kw) -> "MoEConfig":
        return dataclasses.replace(self, **kw)

    # algorithmic work per forward (real assignment rows only, no padding)
    def flops(self) -> int:
        return self.T * (2 * self.d * self.E + 6 * self.d * self.I * self.k + 6 * self.d * self.Is * self.S)


CONFIGS = {
    "tiny_fp32": MoEConfig("tiny_fp32", 128, 256, 256, 8, 64, 1, 64, "f32", 0.02, "uniform", 0.05, 0, steps=1),
    "small_bf16": MoEConfig("small_bf16", 4096, 2048, 64, 6, 1408, 2, 1408, "bf16", 0.02, "zero", 0.0, 1, steps=10),
    "v3_prefill": MoEConfig("v3_prefill", 8192, 7168, 256, 8, 2048, 1, 2048, "bf16", 0.006, "uniform", 0.01, 2),
    "v3_decode": MoEConfig("v3_decode", 64, 7168, 256, 8, 2048, 1, 2048, "bf16", 0.006, "uniform", 0.01, 3, steps=1000),
    "skew_stress": MoEConfig("skew_stress", 32768, 7168, 256, 8, 2048, 1, 2048, "bf16", 0.006, "uniform", 0.01, 4,
                             steps=200, zipf_s=1.2),
}
# The same workloads with E4M3 expert GEMMs (same seeds, so the same bf16
# tensors before quantization).
for _n in ("small_bf16", "v3_prefill", "v3_decode"):
    _c = CONFIGS[_n]
    _fp8 = _n.replace("_bf16", "") + "_fp8"
    CONFIGS[_fp8] = _c.scaled(name=_fp8, dtype="fp8")


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal(shape, std, g, device, dtype):
    return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(dtype)


def zipf_offsets(cfg: MoEConfig, device) -> torch.Tensor:
    """Per-expert logit offsets o_i = -s * sigma_z * ln(r_i).

    r_i = 1 + pi(i) is expert i's popularity rank under a permutation pi
    seeded by the workload seed, and sigma_z = w_std * sqrt(d) is the standard
    deviation of a raw gate logit for x~N(0,1).  The most popular expert gets
    offset 0 and the least popular -s * sigma_z * ln(E)."""
    g = _gen("cpu", cfg.seed * 7 + 3)
    perm = torch.randperm(cfg.E, generator=g)
    ranks = (perm + 1).to(torch.float64)
    sigma_z = cfg.w_std * math.sqrt(cfg.d)
    return (-cfg.zipf_s * sigma_z * torch.log(ranks)).to(torch.float32).to(device)


def make_layer(cfg: MoEConfig, device="cpu") -> dict:
    """Layer parameters in natural (nn.Linear [out][in]) layouts:
    w_gate [E][d]; w1, w3 [E][I][d]; w2 [E][d][I]; ws1, ws3 [S][Is][d];
    ws2 [S][d][Is]; bias fp32 [E]."""
    dt = cfg.torch_dtype
    g = _gen(device, cfg.seed * 1_000_003 + 11)
    p = {}
    p["w_gate"] = _normal((cfg.E, cfg.d), cfg.w_std, g, device, dt)
    if cfg.zipf_s > 0:
        wg = p["w_gate"].float()
        wg[:, 0] = zipf_offsets(cfg, device)
        p["w_gate"] = wg.to(dt)
    # experts are drawn one at a time to bound the fp32 staging memory
    for name, rows, cols, n in (("w1", cfg.I, cfg.d, cfg.E), ("w3", cfg.I, cfg.d, cfg.E), ("w2", cfg.d, cfg.I, cfg.E),
                                ("ws1", cfg.Is, cfg.d, cfg.S), ("ws3", cfg.Is, cfg.d, cfg.S),
                                ("ws2", cfg.d, cfg.Is, cfg.S)):
        t = torch.empty((n, rows, cols), dtype=dt, device=device)
        for e in range(n):
            t[e] = _normal((rows, cols), cfg.w_std, g, device, dt)
        p[name] = t
    gb = _gen("cpu", cfg.seed * 1_000_003 + 17)
    if cfg.bias_kind == "uniform":
        b = (torch.rand(cfg.E, generator=gb, dtype=torch.float64) * 2 - 1) * cfg.bias_range
        p["bias"] = b.to(torch.float32).to(device)
    else:
        p["bias"] = torch.zeros(cfg.E, dtype=torch.float32, device=device)
    return p


def make_tokens(cfg: MoEConfig, device="cpu", step: int = 0, T: int | None = None) -> torch.Tensor:
    """x [T][d] ~ N(0,1) for step/call ``step`` (fresh draw per step)."""
    T = cfg.T if T is None else T
    g = _gen(device, cfg.seed * 1_000_003 + 7919 * (step + 1))
    x = torch.randn((T, cfg.d), generator=g, device=device, dtype=torch.float32)
    if cfg.zipf_s > 0:
        x[:, 0] = 1.0
    return x.to(cfg.torch_dtype)


def to_numpy(t: torch.Tensor):
    """CPU numpy view for the oracle: fp32 stays fp32, bf16 becomes its raw
    uint16 bits."""
    import numpy as np
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    return t.numpy()


def from_numpy(a, like: torch.dtype) -> torch.Tensor:
    import numpy as np
    if like == torch.bfloat16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a))
