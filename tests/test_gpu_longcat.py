"""LongCat-shaped prefill layer at full size (T=8192, d=6144, N=512, Z=256, K=12,
I=2048; 38.7 GB of bf16 expert weights), in the launch configuration of the
benchmark.  Routing, counts and the dispatch layout are checked on every token;
the expert FFN on a seeded sample of experts (the oracle recomputes their rows
one by one); the layer output end to end on a seeded sample of tokens (the
oracle computes those tokens' FFN rows and combines them itself); the combine
stage on every token from the GPU's expert outputs."""
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


@pytest.fixture(scope="module")
def routed_ref(longcat):
    """Routing, counts and dispatch checked on every token; the oracle's
    probabilities and its selection (tie-band rows as the GPU chose)."""
    cfg, L, run = longcat
    assert run.status == 0, hex(run.status)
    g = run.host()
    x64 = P.to_f64(L["x"])
    idx_ref, probs, nties = P.check_routing_and_dispatch(g, x64, P.to_f64(L["w_router"]),
                                                         L["bias"], cfg.N, cfg.K)
    return g, x64, idx_ref, probs


def test_longcat_routing_dispatch_and_counts(longcat, routed_ref):
    cfg, L, run = longcat
    g, x64, idx_ref, probs = routed_ref
    # b = 0 and iid weights give a mean of K*N/E = 8 FFN experts per token
    assert abs(g["n_ffn"].mean() - cfg.K_e) < 0.1
    assert g["counts"].sum() == cfg.T * cfg.K


def test_longcat_output_on_a_token_sample(longcat, routed_ref):
    """out[t] for 64 seeded tokens against Eq. (1) computed by the oracle alone:
    its own FFN_e(x_t) for each token's selected experts and its own gates."""
    cfg, L, run = longcat
    g, x64, idx_ref, probs = routed_ref
    toks = np.sort(np.random.default_rng(7).choice(cfg.T, size=64, replace=False))
    idx_s = idx_ref[toks]
    gate_s = orc.gates(probs[toks], idx_s)
    off, rt, sp = orc.canonical_permutation(idx_s, cfg.N)
    y_s = orc.grouped_ffn(x64[toks][rt], off, L["w1"], L["w3"], L["w2"], decode=P.to_f64)
    out_s = orc.combine(x64[toks], y_s, idx_s, gate_s, sp, cfg.N, cfg.gamma)
    P.assert_close(g["out"][toks], out_s, "bf16", "out on the token sample")
    zm = orc.zero_mass(idx_s, gate_s, cfg.N)
    P.assert_ffn_part_close(g["out"][toks], out_s, cfg.gamma * zm[:, None] * x64[toks], "bf16",
                            "out minus identity term on the token sample")


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
