"""LongCat-shaped prefill layer at full size (T=8192, d=6144, N=512, Z=256, K=12,
I=2048; 38.7 GB of bf16 expert weights), in the launch configuration of the
benchmark.  Routing, counts and the dispatch layout are checked on every token;
the expert FFN on a seeded sample of experts (the oracle recomputes their rows
one by one); the combine stage on every token from the GPU's expert outputs."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_30_b200 import binding as B
from mixture_experts_layer_30_b200 import configs as C
from mixture_experts_layer_30_b200 import inputs as IN
from oracle import moe_oracle as orc
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def longcat():
    cfg = C.LONGCAT_PREFILL
    free, _ = torch.cuda.mem_get_info()
    if free < 48 * 2 ** 30:
        pytest.skip(f"needs ~48 GB of free device memory, {free / 2**30:.1f} GB free")
    L = IN.make_layer_inputs(cfg, device="cuda")
    # the benchmark's launch configuration: expert weights repacked to the tiled
    # order, route, dispatch with the x_perm copy, gate/up and down as two calls,
    # combine
    run = P.GpuRun(B.shape_of(cfg, weight_layout=B.WEIGHTS_TILED), L["x"], L["w_router"],
                   L["w1"], L["w3"], L["w2"], L["bias"], split_ffn=True)
    yield cfg, L, run
    del L, run
    torch.cuda.empty_cache()


def test_longcat_routing_dispatch_and_counts(longcat):
    cfg, L, run = longcat
    assert run.status == 0, hex(run.status)
    g = run.host()
    x64 = P.to_f64(L["x"])
    idx_ref, probs, nties = P.check_routing_and_dispatch(g, x64, P.to_f64(L["w_router"]),
                                                         L["bias"], cfg.N, cfg.K)
    # b = 0 and iid weights give a mean of K*N/E = 8 FFN experts per token
    assert abs(g["n_ffn"].mean() - cfg.K_e) < 0.1
    assert g["counts"].sum() == cfg.T * cfg.K


def test_longcat_expert_ffn_sampled(longcat):
    cfg, L, run = longcat
    g = run.host()
    rng = np.random.default_rng(0)
    sizes = np.diff(g["offsets"])
    experts = sorted(set(rng.choice(cfg.N, size=6, replace=False).tolist())
                     | {int(sizes.argmax()), int(sizes.argmin())})
    x64 = P.to_f64(L["x"])
    for e in experts:
        lo, hi = int(g["offsets"][e]), int(g["offsets"][e + 1])
        if hi == lo:
            continue
        rows = x64[g["row_token"][lo:hi]]
        y = orc.expert_ffn(rows, P.to_f64(L["w1"][e]), P.to_f64(L["w3"][e]), P.to_f64(L["w2"][e]))
        P.assert_close(g["y_perm"][lo:hi], y, "bf16", f"y_perm of expert {e}")


def test_longcat_combine_all_tokens(longcat):
    cfg, L, run = longcat
    g = run.host()
    x64 = P.to_f64(L["x"])
    probs = g["probs"]
    gate = g["gate"]
    out = orc.combine(x64, g["y_perm"], g["idx"], gate, g["slot_pos"], cfg.N)
    P.assert_close(g["out"], out, "bf16", "combine stage")
