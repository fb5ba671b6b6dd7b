"""Seeded synthetic inputs for the MoE layer.

This module only draws random numbers; it holds none of the layer's
arithmetic, so both the CUDA path and the fp64 oracle can be fed from it.

Recipe (every tensor has its own generator, seeded ``base_seed*1000 + j``,
drawn in the fixed order j = 0..6):

    j=0  x        [T, d]     N(0, 1)
    j=1  w_router [E, d]     N(0, w_std)          (nn.Linear layout: out x in)
    j=2  w1       [N, I, d]  N(0, w_std)  gate projection, drawn expert by expert
    j=3  w3       [N, I, d]  N(0, w_std)  up projection, drawn expert by expert
    j=4  w2       [N, d, I]  N(0, w_std)  down projection, drawn expert by expert
    j=5  bias     [E] fp32   0, or U(-bias_amp, bias_amp)
    j=6  skew permutation of the FFN experts (skewed-routing workload only)

Draws are fp32; bf16 workloads round them to bf16 with round-to-nearest-even
(torch's conversion).  The expert bias is always fp32.
"""
import torch

from .configs import MoEConfig


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def draw_device(cfg: MoEConfig, device) -> torch.device:
    """fp32 workloads are drawn on the CPU, bf16 ones on ``device``."""
    return torch.device("cpu") if cfg.dtype == "f32" else torch.device(device)


def storage_dtype(cfg: MoEConfig) -> torch.dtype:
    return torch.float32 if cfg.dtype == "f32" else torch.bfloat16


def _normal(shape, std, g, dev, out_dtype):
    t = torch.randn(shape, generator=g, device=dev, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(out_dtype)


def make_x(cfg: MoEConfig, device, seed: int) -> torch.Tensor:
    dev = draw_device(cfg, device)
    return _normal((cfg.T, cfg.d), 1.0, _gen(dev, seed), dev,
                   storage_dtype(cfg)).to(device)


def make_layer_inputs(cfg: MoEConfig, device="cpu", base_seed: int = 0,
                      with_x: bool = True, with_experts: bool = True) -> dict:
    """All tensors of one layer instance, placed on ``device`` (without the
    expert weights when ``with_experts`` is False; the other draws are the
    same either way, each tensor having its own generator)."""
    dev = draw_device(cfg, device)
    sd = storage_dtype(cfg)
    s = base_seed * 1000
    out = {}
    if with_x:
        out["x"] = _normal((cfg.T, cfg.d), 1.0, _gen(dev, s + 0), dev, sd).to(device)
    out["w_router"] = _normal((cfg.E, cfg.d), cfg.w_std, _gen(dev, s + 1), dev, sd).to(device)
    for j, name, shape in ((2, "w1", (cfg.I, cfg.d)), (3, "w3", (cfg.I, cfg.d)),
                           (4, "w2", (cfg.d, cfg.I))) if with_experts else ():
        g = _gen(dev, s + j)
        w = torch.empty((cfg.N,) + shape, dtype=sd, device=device)
        for e in range(cfg.N):
            w[e].copy_(_normal(shape, cfg.w_std, g, dev, sd))
        out[name] = w
    g = _gen(dev, s + 5)
    if cfg.bias_kind == "zero":
        b = torch.zeros(cfg.E, dtype=torch.float32, device=dev)
    elif cfg.bias_kind == "uniform":
        b = (torch.rand(cfg.E, generator=g, device=dev, dtype=torch.float32) * 2.0 - 1.0) \
            * cfg.bias_amp
    else:
        raise ValueError(cfg.bias_kind)
    out["bias"] = b.to(device)
    return out


def skew_permutation(cfg: MoEConfig, base_seed: int = 0) -> torch.Tensor:
    """Seeded global permutation of the N FFN experts (j=6)."""
    return torch.randperm(cfg.N, generator=_gen("cpu", base_seed * 1000 + 6))


def make_skewed_step(cfg: MoEConfig, step: int, device="cpu", base_seed: int = 0,
                     zipf_s: float = 1.1, hot_boost: float = 3.0,
                     zero_boost: float = 2.0) -> tuple:
    """x and the additive logit offset of one step of the skewed-routing workload.

    Step ``step`` draws x from seed 1000 + step.  Each token draws a rank r from
    a Zipf(zipf_s) law truncated to 1..N and gets ``hot_boost`` on the logit of
    FFN expert perm[r-1]; a Bernoulli(1/2) half of the tokens gets
    ``zero_boost`` on every zero-expert logit.  Returns (x [T,d] fp32,
    offset [T,E] fp32) on ``device``.
    """
    g = _gen("cpu", 1000 + step + base_seed * 1000)
    x = torch.randn((cfg.T, cfg.d), generator=g, dtype=torch.float32)
    ranks = torch.arange(1, cfg.N + 1, dtype=torch.float64)
    p = ranks.pow(-zipf_s)
    r = torch.multinomial(p / p.sum(), cfg.T, replacement=True, generator=g)
    perm = skew_permutation(cfg, base_seed)
    hot = perm[r]
    to_zero = torch.rand(cfg.T, generator=g) < 0.5
    off = torch.zeros((cfg.T, cfg.E), dtype=torch.float32)
    off[torch.arange(cfg.T), hot] += hot_boost
    off[to_zero, cfg.N:] += zero_boost
    return x.to(device), off.to(device)
