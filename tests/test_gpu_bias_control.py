"""Skewed routing with budget control (Eq. (2)): 200 closed-loop steps on the GPU
against the oracle, plus an exact open-loop check of every step."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_30_b200 import binding as B
from mixture_experts_layer_30_b200 import configs as C
from mixture_experts_layer_30_b200 import inputs as IN
from oracle import moe_oracle as orc
from tests import parity as P

pytestmark = pytest.mark.gpu


def test_skewed_bias_control_trajectory():
    cfg = C.SKEWED_BIAS_CONTROL
    L = IN.make_layer_inputs(cfg, device="cuda", with_x=False)
    shape = B.shape_of(cfg)
    wr64 = P.to_f64(L["w_router"])
    N, K, E, T = cfg.N, cfg.K, cfg.E, cfg.T
    K_e, mu = float(np.float32(cfg.K_e)), float(np.float32(cfg.mu))
    ws = B.new_workspace(shape)
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    gate = torch.empty((T, K), dtype=torch.float32, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    nffn = torch.empty(T, dtype=torch.uint8, device="cuda")
    bias = L["bias"].clone()
    gpu_stats, ties_total = [], 0
    for s in range(cfg.steps):
        x, off = IN.make_skewed_step(cfg, s, device="cuda")
        b_before = bias.cpu().numpy().copy()
        B.route(shape, x, L["w_router"], bias, ws, idx, gate, counts, nffn, logit_offset=off)
        B.bias_update(N, cfg.Z, counts, T, K, K_e, mu, bias)
        torch.cuda.synchronize()
        g_idx, g_counts = idx.cpu().numpy(), counts.cpu().numpy()
        g_nffn = nffn.cpu().numpy()
        # open loop, exact: the oracle routes with the GPU's bias of this step ...
        probs = orc.softmax_rows(orc.router_logits(P.to_f64(x), wr64,
                                                   off.cpu().numpy().astype(np.float64)))
        oidx, _ = orc.biased_topk(probs, b_before.astype(np.float64), K)
        ties = P.check_selection(g_idx, probs + b_before[None, :], oidx, K)
        ties_total += len(ties)
        idx_ref = oidx.copy()
        idx_ref[ties] = g_idx[ties]
        np.testing.assert_array_equal(g_counts, orc.expert_counts(idx_ref, E))
        np.testing.assert_array_equal(g_nffn, orc.ffn_experts_per_token(idx_ref, N))
        # ... and applies Eq. (2) to the GPU's counts: identical fp32 bias
        want = orc.bias_update(b_before.astype(np.float64), g_counts, N, K, K_e, mu, T)
        assert bias.cpu().numpy().tobytes() == want.astype(np.float32).tobytes(), s
        load = g_counts[:N].astype(np.float64)
        gpu_stats.append((g_nffn.mean(), g_nffn.std(), load.max() / load.mean()))
    # closed loop: the oracle's own trajectory from b_0
    hist, b_final = orc.bias_control_trajectory(
        cfg.steps, lambda s: tuple(t.cpu().numpy().astype(np.float64)
                                   for t in IN.make_skewed_step(cfg, s, device="cpu")),
        wr64, L["bias"].cpu().numpy(), N, K, K_e, mu)
    for s, (h, gs) in enumerate(zip(hist, gpu_stats)):
        assert abs(gs[0] - h["n_ffn_mean"]) <= 1e-3, (s, gs, h["n_ffn_mean"])
        assert abs(gs[1] - h["n_ffn_std"]) <= 1e-2, (s, gs, h["n_ffn_std"])
        assert abs(gs[2] / h["max_over_mean_load"] - 1.0) <= 1e-2, (s, gs)
    assert np.abs(bias.cpu().numpy() - b_final).max() <= 1e-5
    # the controller does its job: the mean FFN count approaches K_e and load evens out
    assert abs(hist[-1]["n_ffn_mean"] - K_e) < 0.05
    assert hist[-1]["max_over_mean_load"] < hist[0]["max_over_mean_load"]
    print(f"tie-band rows over {cfg.steps} steps: {ties_total}; "
          f"mean FFN experts {hist[0]['n_ffn_mean']:.3f} -> {hist[-1]['n_ffn_mean']:.3f} "
          f"(target {K_e:.3f}); max/mean load {hist[0]['max_over_mean_load']:.3f} -> "
          f"{hist[-1]['max_over_mean_load']:.3f}")


def test_bias_checkpoint_resume_is_bit_exact(tmp_path):
    """The expert bias is the layer's only state: a checkpoint is a host copy of
    it (saved to a file here), and resuming from it reproduces the rest of the
    closed-loop trajectory bit for bit."""
    cfg = C.SKEWED_BIAS_CONTROL
    L = IN.make_layer_inputs(cfg, device="cuda", with_x=False)
    shape = B.shape_of(cfg)
    N, K, E, T = cfg.N, cfg.K, cfg.E, cfg.T
    K_e, mu = float(np.float32(cfg.K_e)), float(np.float32(cfg.mu))
    ws = B.new_workspace(shape)
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    gate = torch.empty((T, K), dtype=torch.float32, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    nffn = torch.empty(T, dtype=torch.uint8, device="cuda")

    def run(bias, steps):
        trail = []
        for s in steps:
            x, off = IN.make_skewed_step(cfg, s, device="cuda")
            B.route(shape, x, L["w_router"], bias, ws, idx, gate, counts, nffn, logit_offset=off)
            B.bias_update(N, cfg.Z, counts, T, K, K_e, mu, bias)
            trail.append((idx.cpu().clone(), bias.cpu().clone()))
        return trail

    bias = L["bias"].clone()
    run(bias, range(0, 5))
    ckpt = tmp_path / "bias.pt"
    torch.save(bias.cpu(), ckpt)                      # checkpoint: device -> host -> file
    first = run(bias, range(5, 10))
    resumed = torch.load(ckpt).to("cuda")             # resume: file -> host -> device
    second = run(resumed, range(5, 10))
    for (i1, b1), (i2, b2) in zip(first, second):
        assert torch.equal(i1, i2) and torch.equal(b1, b2)
