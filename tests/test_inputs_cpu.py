"""The seeded input generators: every tensor has its own generator, so leaving
the expert weights out (the route-only timing driver) draws the same x, W_r and
bias as the full layer."""
import torch

from mixture_experts_layer_30_b200 import configs as C
from mixture_experts_layer_30_b200 import inputs as IN


def test_route_only_inputs_match_the_full_layer():
    for cfg in (C.TINY_F32, C.DECODE_T16):
        full = IN.make_layer_inputs(cfg, device="cpu")
        part = IN.make_layer_inputs(cfg, device="cpu", with_experts=False)
        assert set(part) == {"x", "w_router", "bias"}
        for k in part:
            assert torch.equal(full[k], part[k]), (cfg.name, k)
