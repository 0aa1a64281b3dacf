"""Seeded synthetic inputs for the MoE layer workloads.

This module only draws random tensors of the right shapes; it holds none of the layer's
arithmetic. The same tensors feed both the CUDA path and the CPU oracle.

Recipe (per tensor its own seed, derived from the run seed and a tensor id):
  x     [T, H]        ~ N(0, 1)
  W_g   [H, E]        ~ N(0, 1/sqrt(H))   (the Phi-3.5-shaped layer: N(0, 1) unscaled)
  W1    [E, H, 2F]    ~ N(0, 1/sqrt(H))   (SwiGLU: columns [0,F) gate, [F,2F) up)
        [E, H, F]     for non-gated activations
  W2    [E, F, H]     ~ N(0, 1/sqrt(F))
  bias  [E] fp32 or None; the skewed layer uses b[e] = ln p_e with p a Zipf(s=1.2) prior
        over expert ids (expert 0 hottest), which makes many experts get 0-1 tokens and a
        few get more than 10% of the tokens.
Values are drawn in fp32 with torch's seeded generator and rounded to bf16 (RNE).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

ACT_SWIGLU, ACT_GELU_TANH, ACT_RELU, ACT_IDENTITY = 0, 1, 2, 3
GATE_SOFTMAX_TOPK, GATE_SOFTMAX_ALL = 0, 1


@dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int
    H: int
    F: int
    E: int
    k: int
    act: int = ACT_SWIGLU
    gate: int = GATE_SOFTMAX_TOPK
    gate_std_unscaled: bool = False   # W_g ~ N(0,1) instead of N(0,1/sqrt(H))
    zipf_s: float = 0.0               # > 0: add ln(Zipf(s)) expert prior to the logits

    def with_tokens(self, T: int) -> "LayerConfig":
        return replace(self, T=T, name=f"{self.name}_T{T}")

    @property
    def useful_flops(self) -> float:
        """Algorithmic FLOPs of one forward: 2THE router + 6THFk (SwiGLU) or 4THFk."""
        ffn = (6 if self.act == ACT_SWIGLU else 4) * self.T * self.k * self.H * self.F
        return float(ffn + 2 * self.T * self.H * self.E)


CONFIGS = {
    "tiny": LayerConfig("tiny", T=256, H=256, F=512, E=8, k=2),
    "mixtral": LayerConfig("mixtral", T=8192, H=4096, F=14336, E=8, k=2),
    "phi35": LayerConfig("phi35", T=16384, H=4096, F=6400, E=16, k=2, gate_std_unscaled=True),
    "qwen2": LayerConfig("qwen2", T=8192, H=3584, F=2560, E=64, k=8),
    "skew": LayerConfig("skew", T=4096, H=7168, F=2048, E=256, k=8, zipf_s=1.2),
    "skew_decode": LayerConfig("skew_decode", T=64, H=7168, F=2048, E=256, k=8, zipf_s=1.2),
}

_TENSOR_IDS = {"x": 1, "Wg": 2, "W1": 3, "W2": 4, "W1s": 5, "W2s": 6, "w_sg": 7}


def tensor_seed(seed: int, name: str) -> int:
    return int(seed) * 1000 + _TENSOR_IDS[name]


def _randn_bf16(shape, seed, std, device):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


def _randn_bf16_chunked(shape, seed, std, device):
    """Large weight tensors: draw one expert at a time (same generator stream) to bound
    the fp32 temporary."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    for e in range(shape[0]):
        t = torch.randn(shape[1:], generator=g, device=device, dtype=torch.float32)
        if std != 1.0:
            t.mul_(std)
        out[e].copy_(t)
    return out


def zipf_log_prior(E: int, s: float) -> torch.Tensor:
    """b[e] = ln p_e, p_e = (e+1)^-s / sum_i i^-s (expert 0 is the hottest)."""
    ranks = torch.arange(1, E + 1, dtype=torch.float64)
    p = ranks.pow(-s)
    p = p / p.sum()
    return p.log().to(torch.float32)


def make_inputs(cfg: LayerConfig, seed: int = 0, device="cpu", x_seed: int | None = None,
                experts: bool = True):
    """Return dict(x, Wg, W1, W2, bias) on ``device`` (bias is None unless cfg.zipf_s > 0).

    ``x_seed`` overrides the seed of x only (data-parallel replicas draw their own batch
    while sharing the weights). ``experts=False`` leaves W1 and W2 out (None), for the router
    alone; the other tensors are the same draws."""
    T, H, F, E = cfg.T, cfg.H, cfg.F, cfg.E
    w1_cols = 2 * F if cfg.act == ACT_SWIGLU else F
    xs = tensor_seed(seed if x_seed is None else x_seed, "x")
    x = _randn_bf16((T, H), xs, 1.0, device)
    Wg = _randn_bf16((H, E), tensor_seed(seed, "Wg"),
                     1.0 if cfg.gate_std_unscaled else 1.0 / math.sqrt(H), device)
    W1 = W2 = None
    if experts:
        W1 = _randn_bf16_chunked((E, H, w1_cols), tensor_seed(seed, "W1"), 1.0 / math.sqrt(H), device)
        W2 = _randn_bf16_chunked((E, F, H), tensor_seed(seed, "W2"), 1.0 / math.sqrt(F), device)
    bias = zipf_log_prior(E, cfg.zipf_s).to(device) if cfg.zipf_s > 0 else None
    return dict(x=x, Wg=Wg, W1=W1, W2=W2, bias=bias)


def make_shared_weights(H: int, Fs: int, seed: int = 0, device="cpu", gate: bool = True):
    """Shared-expert weights (W1s [H, 2Fs], W2s [Fs, H], w_sg [H] or None), drawn with the
    same scaling as the routed experts' (std 1/sqrt(fan-in))."""
    W1s = _randn_bf16((H, 2 * Fs), tensor_seed(seed, "W1s"), 1.0 / math.sqrt(H), device)
    W2s = _randn_bf16((Fs, H), tensor_seed(seed, "W2s"), 1.0 / math.sqrt(Fs), device)
    w_sg = _randn_bf16((H,), tensor_seed(seed, "w_sg"), 1.0 / math.sqrt(H), device) if gate else None
    return W1s, W2s, w_sg


def bf16_bits(t: torch.Tensor):
    """A bf16 tensor's bit patterns as a contiguous numpy uint16 array (host copy)."""
    import numpy as np

    assert t.dtype == torch.bfloat16
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def from_bf16_bits(a) -> torch.Tensor:
    """numpy uint16 bit patterns -> torch bf16 tensor (host)."""
    import numpy as np

    a = np.ascontiguousarray(a, dtype=np.uint16)
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
