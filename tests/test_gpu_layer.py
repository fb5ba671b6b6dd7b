"""Parity of the CUDA path (through the C ABI) with the fp64 oracle, stage by stage."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_30_b200 import binding as B
from mixture_experts_layer_30_b200 import configs as C
from mixture_experts_layer_30_b200 import inputs as IN
from oracle import moe_oracle as orc
from tests import parity as P

pytestmark = pytest.mark.gpu


def _run_and_check(shape, dtype, L, N, K, gamma=1.0, logit_offset=None, split_ffn=False,
                   experts=None, fused_gather=False):
    run = P.GpuRun(shape, L["x"], L["w_router"], L["w1"], L["w3"], L["w2"], L["bias"],
                   gamma=gamma, logit_offset=logit_offset, split_ffn=split_ffn,
                   fused_gather=fused_gather)
    assert run.status == 0, hex(run.status)
    g = run.host()
    x64 = P.to_f64(L["x"])
    wr64 = P.to_f64(L["w_router"])
    idx_ref, probs, nties = P.check_routing_and_dispatch(g, x64, wr64, L["bias"], N, K,
                                                         logit_offset)
    gate = orc.gates(probs, idx_ref)
    off, rt, sp = orc.canonical_permutation(idx_ref, N)
    y_o = orc.grouped_ffn(x64[rt], off, L["w1"], L["w3"], L["w2"], experts=experts,
                          decode=P.to_f64)
    rows = ~np.isnan(y_o[:, 0]) if len(y_o) else np.zeros(0, bool)
    P.assert_close(g["y_perm"][rows], y_o[rows], dtype, "y_perm")
    zm = orc.zero_mass(idx_ref, gate, N)
    if experts is None:
        out_o = orc.combine(x64, y_o, idx_ref, gate, sp, N, gamma)
        P.assert_close(g["out"], out_o, dtype, "out")
        # FFN part alone (the identity term would hide FFN errors)
        P.assert_ffn_part_close(g["out"], out_o, gamma * zm[:, None] * x64, dtype,
                                "out minus identity term")
    # combine stage on the GPU's own expert outputs
    out_stage = orc.combine(x64, g["y_perm"], idx_ref, gate, sp, N, gamma)
    P.assert_close(g["out"], out_stage, dtype, "combine stage")
    return run, g, nties


def _cfg_inputs(cfg, device="cuda", **over):
    L = IN.make_layer_inputs(cfg, device=device)
    L.update(over)
    return L


def test_tiny_f32_layer():
    cfg = C.TINY_F32
    L = _cfg_inputs(cfg)
    _run_and_check(B.shape_of(cfg), "f32", L, cfg.N, cfg.K)


def test_tiny_f32_layer_split_ffn_and_gamma():
    cfg = C.TINY_F32
    L = _cfg_inputs(cfg)
    _run_and_check(B.shape_of(cfg), "f32", L, cfg.N, cfg.K, gamma=2.5, split_ffn=True)


def test_mid_bf16_layer():
    cfg = C.MID_BF16
    L = _cfg_inputs(cfg)
    _, g, nties = _run_and_check(B.shape_of(cfg), "bf16", L, cfg.N, cfg.K, split_ffn=True)
    # the U(-0.05, 0.05) bias sends roughly a third of the slots to zero experts
    frac_zero = 1.0 - g["n_ffn"].mean() / cfg.K
    assert 0.15 < frac_zero < 0.6


@pytest.mark.parametrize("cfg", [C.DECODE_T16, C.DECODE_T64, C.DECODE_T256],
                         ids=lambda c: c.name)
def test_decode_bf16(cfg):
    L = _cfg_inputs(cfg)
    _run_and_check(B.shape_of(cfg), "bf16", L, cfg.N, cfg.K, split_ffn=True)


def test_pack_weights_layout():
    """Tiled order: tile (m, rb, cb) = rows rb*128.., columns cb*64.. of matrix m,
    stored contiguously at tile index (m*rows/128 + rb)*cols/64 + cb."""
    g = torch.Generator(device="cpu").manual_seed(9)
    for (n, rows, cols) in ((3, 256, 192), (1, 128, 64), (2, 384, 1024)):
        w = torch.randn((n, rows, cols), generator=g).to(torch.bfloat16).cuda()
        got = B.pack_weights(w)
        want = w.view(n, rows // 128, 128, cols // 64, 64).permute(0, 1, 3, 2, 4).contiguous()
        assert torch.equal(got.view(-1), want.view(-1))


@pytest.mark.parametrize("cfg", [C.MID_BF16, C.DECODE_T16, C.DECODE_T64, C.DECODE_T256],
                         ids=lambda c: c.name)
@pytest.mark.parametrize("mode", ["split", "ffn", "gather"])
def test_tiled_weights_layer(cfg, mode):
    """The expert GEMMs on weights repacked by moe_pack_weights."""
    L = _cfg_inputs(cfg)
    _run_and_check(B.shape_of(cfg, weight_layout=B.WEIGHTS_TILED), "bf16", L, cfg.N, cfg.K,
                   split_ffn=mode == "split", fused_gather=mode == "gather")


@pytest.mark.parametrize("T", [1, 200, 777])
def test_tiled_weights_ragged(T):
    shape, L = _small(T, 256, 12, 4, 3, 128, "bf16", seed=300 + T)
    shape.weight_layout = B.WEIGHTS_TILED
    _run_and_check(shape, "bf16", L, 12, 3, split_ffn=True)


@pytest.mark.parametrize("cfg", [C.TINY_F32, C.MID_BF16, C.DECODE_T16, C.DECODE_T256],
                         ids=lambda c: c.name)
def test_fused_gather_layer(cfg):
    """Dispatch without the x_perm copy: the gate/up GEMM reads x through row_token."""
    L = _cfg_inputs(cfg)
    _run_and_check(B.shape_of(cfg), cfg.dtype, L, cfg.N, cfg.K, fused_gather=True)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T", [1, 13, 700])
def test_fused_gather_ragged(dtype, T):
    shape, L = _small(T, 128, 12, 4, 3, 64, dtype, seed=100 + T)
    _run_and_check(shape, dtype, L, 12, 3, fused_gather=True)


def _small(T, d, N, Z, K, I, dtype, seed=0, bias=None, w_std=0.05):
    g = torch.Generator(device="cpu").manual_seed(seed)
    E = N + Z
    dt = torch.float32 if dtype == "f32" else torch.bfloat16

    def rn(*shape, std=1.0):
        return (torch.randn(shape, generator=g) * std).to(dt).cuda()
    L = dict(x=rn(T, d), w_router=rn(E, d, std=0.1), w1=rn(N, I, d, std=w_std),
             w3=rn(N, I, d, std=w_std), w2=rn(N, d, I, std=w_std),
             bias=(torch.zeros(E) if bias is None else torch.as_tensor(bias, dtype=torch.float32)).cuda())
    return B.make_shape(T, d, N, Z, K, I, dtype), L


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T", [1, 7, 300, 513])
def test_ragged_token_counts(dtype, T):
    shape, L = _small(T, 128, 12, 4, 3, 64, dtype, seed=T)
    _run_and_check(shape, dtype, L, 12, 3)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_k_equals_e(dtype):
    N, Z = 5, 3
    shape, L = _small(40, 64, N, Z, N + Z, 64, dtype, seed=11)
    _, g, _ = _run_and_check(shape, dtype, L, N, N + Z)
    np.testing.assert_allclose(g["gate"].sum(axis=1), 1.0, atol=1e-5)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_all_slots_to_zero_experts(dtype):
    N, Z, K = 6, 4, 3
    bias = [0.0] * N + [10.0] * Z
    shape, L = _small(70, 64, N, Z, K, 64, dtype, seed=5, bias=bias)
    run, g, _ = _run_and_check(shape, dtype, L, N, K)
    assert g["R"] == 0 and (g["slot_pos"] == -1).all()
    # bit-exact fixed point: out = fl32(sum of the GPU's gates) * x, rounded to dtype
    zs = torch.zeros(70, dtype=torch.float32)
    gate = run.buf.topk_gate.cpu()
    for k in range(K):
        zs = zs + gate[:, k]
    want = (zs[:, None] * L["x"].float().cpu()).to(L["x"].dtype)
    assert torch.equal(run.buf.out.cpu(), want)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_one_hot_expert_long_segment(dtype):
    N, Z, K = 8, 4, 2
    bias = [0.0] * (N + Z)
    bias[3] = 10.0
    shape, L = _small(700, 128, N, Z, K, 64, dtype, seed=7, bias=bias)
    _, g, _ = _run_and_check(shape, dtype, L, N, K)
    assert g["offsets"][4] - g["offsets"][3] == 700


@pytest.mark.parametrize("mode", ["fused", "split", "gather"])
def test_decode_tile_long_segment(mode):
    """A decode-sized batch (16.7 routed rows per expert on average: the 64-row
    token tiles) whose expert 5 takes every token: 200 rows, three full tiles and
    an 8-row tail of one segment."""
    N, Z, K = 32, 16, 4
    bias = [0.0] * (N + Z)
    bias[5] = 10.0
    shape, L = _small(200, 128, N, Z, K, 128, "bf16", seed=8, bias=bias)
    _, g, _ = _run_and_check(shape, "bf16", L, N, K, split_ffn=mode == "split",
                             fused_gather=mode == "gather")
    assert g["offsets"][6] - g["offsets"][5] == 200


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_no_zero_experts(dtype):
    shape, L = _small(200, 64, 10, 0, 3, 64, dtype, seed=3)
    _run_and_check(shape, dtype, L, 10, 3)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_max_experts_large_k(dtype):
    """E = N + Z = 1024, the library's limit (32 scores per lane in the top-K
    kernel), with K = 40 slots per token (more than one 32-lane pass)."""
    N, Z, K = 640, 384, 40
    shape, L = _small(150, 128, N, Z, K, 128, dtype, seed=21)
    _run_and_check(shape, dtype, L, N, K)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_single_ffn_expert_top1(dtype):
    shape, L = _small(90, 64, 1, 2, 1, 64, dtype, seed=22)
    _run_and_check(shape, dtype, L, 1, 1)


@pytest.mark.parametrize("mode", ["split", "ffn", "gather"])
def test_bf16_cuda_core_fallback(mode):
    """bf16 shapes the tensor-core kernels do not take (d = 72, I = 40: not
    multiples of 64) run the CUDA-core router and grouped GEMMs."""
    shape, L = _small(130, 72, 9, 3, 3, 40, "bf16", seed=23)
    _run_and_check(shape, "bf16", L, 9, 3, split_ffn=mode == "split",
                   fused_gather=mode == "gather")


def test_bf16_router_fallback_odd_expert_count():
    """E = 13 (not a multiple of 8): the CUDA-core router, tensor-core experts."""
    shape, L = _small(200, 128, 9, 4, 3, 64, "bf16", seed=24)
    _run_and_check(shape, "bf16", L, 9, 3, split_ffn=True)


def test_empty_batch():
    shape, L = _small(0, 64, 6, 2, 2, 64, "f32", seed=1)
    L["x"] = torch.empty((0, 64), device="cuda")
    buf = B.LayerBuffers(shape, with_probs=True)
    buf.counts.fill_(-1)
    buf.offsets.fill_(-1)
    B.forward(buf, L["x"], L["w_router"], L["w1"], L["w3"], L["w2"], L["bias"])
    torch.cuda.synchronize()
    assert (buf.counts == 0).all() and (buf.offsets == 0).all()
    assert B.device_status(buf.ws) == 0
    # the same through the route call that builds the dispatch layout
    buf.counts.fill_(-1)
    buf.offsets.fill_(-1)
    B.forward(buf, L["x"], L["w_router"], L["w1"], L["w3"], L["w2"], L["bias"],
              fused_gather=True)
    torch.cuda.synchronize()
    assert (buf.counts == 0).all() and (buf.offsets == 0).all()
    assert B.device_status(buf.ws) == 0


def test_deterministic_bitwise():
    cfg = C.MID_BF16
    L = _cfg_inputs(cfg)
    s = B.shape_of(cfg)
    outs = []
    for _ in range(2):
        buf = B.LayerBuffers(s)
        B.forward(buf, L["x"], L["w_router"], L["w1"], L["w3"], L["w2"], L["bias"],
                  split_ffn=True)
        outs.append((buf.out.clone(), buf.y_perm.clone(), buf.topk_idx.clone(),
                     buf.slot_pos.clone()))
    torch.cuda.synchronize()
    R = int(buf.offsets[-1])
    assert torch.equal(outs[0][0], outs[1][0])
    assert torch.equal(outs[0][1][:R], outs[1][1][:R])
    assert torch.equal(outs[0][2], outs[1][2]) and torch.equal(outs[0][3], outs[1][3])


def test_bad_expert_index_sets_status_without_fault():
    shape, L = _small(64, 64, 6, 2, 2, 64, "f32", seed=2)
    buf = B.LayerBuffers(shape)
    B.route(shape, L["x"], L["w_router"], L["bias"], buf.ws, buf.topk_idx, buf.topk_gate,
            buf.counts, buf.n_ffn)
    bad = buf.topk_idx.clone()
    t, k = [int(v) for v in (bad < shape.N).nonzero()[0]]   # an FFN slot
    bad[t, k] = 99
    B.permute(shape, L["x"], bad, buf.counts, buf.offsets, buf.row_token, buf.slot_pos,
              buf.x_perm, buf.ws)
    st = B.device_status(buf.ws)
    assert st & B.DEV_BAD_EXPERT_INDEX and st & B.DEV_COUNT_MISMATCH
    assert B.device_status(buf.ws) == 0  # cleared by the read


def test_bias_update_open_loop_bit_exact():
    rng = np.random.default_rng(0)
    for (N, Z, K, T) in ((16, 8, 4, 16384), (512, 256, 12, 8192), (64, 32, 6, 4096)):
        E = N + Z
        counts = rng.multinomial(K * T, np.ones(E) / E).astype(np.int32)
        b0 = rng.normal(scale=0.05, size=E).astype(np.float32)
        K_e = np.float32(K * N / E)
        mu = np.float32(0.1)
        bias = torch.from_numpy(b0).cuda()
        B.bias_update(N, Z, torch.from_numpy(counts).cuda(), T, K, float(K_e), float(mu), bias)
        got = bias.cpu().numpy()
        want = orc.bias_update(b0.astype(np.float64), counts, N, K, float(K_e), float(mu),
                               T).astype(np.float32)
        assert got.tobytes() == want.tobytes()
        assert got[N:].tobytes() == b0[N:].tobytes()


@pytest.mark.parametrize("cfg,D", [(C.TINY_F32, 4), (C.MID_BF16, 8), (C.DECODE_T16, 8),
                                   (C.SKEWED_BIAS_CONTROL, 2)], ids=lambda v: str(v))
def test_lb_statistics(cfg, D):
    """Eq. (3)-(5): probability column sums from the route kernel, then f_j, P_j, L."""
    if cfg.skewed:
        x, off = IN.make_skewed_step(cfg, 3, device="cuda")
        L = IN.make_layer_inputs(cfg, device="cuda", with_x=False)
        L["x"] = x
    else:
        L, off = _cfg_inputs(cfg), None
    shape = B.shape_of(cfg)
    buf = B.LayerBuffers(shape, with_probs=True)
    prob_sum = torch.empty(cfg.E, dtype=torch.float32, device="cuda")
    B.route(shape, L["x"], L["w_router"], L["bias"], buf.ws, buf.topk_idx, buf.topk_gate,
            buf.counts, buf.n_ffn, logit_offset=off, probs_out=buf.probs, prob_sum=prob_sum)
    f = torch.empty(D + 1, dtype=torch.float32, device="cuda")
    Pg = torch.empty_like(f)
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    K_e, alpha = float(np.float32(cfg.K_e)), 0.01
    B.lb_stats(cfg.N, cfg.Z, D, buf.counts, prob_sum, cfg.T, cfg.K, K_e, alpha, f, Pg, loss)
    torch.cuda.synchronize()
    assert B.device_status(buf.ws) == 0
    x64, wr64 = P.to_f64(L["x"]), P.to_f64(L["w_router"])
    g = dict(probs=buf.probs.cpu().numpy().astype(np.float64), idx=buf.topk_idx.cpu().numpy(),
             gate=buf.topk_gate.cpu().numpy().astype(np.float64), counts=buf.counts.cpu().numpy(),
             n_ffn=buf.n_ffn.cpu().numpy())
    probs = orc.softmax_rows(orc.router_logits(x64, wr64, None if off is None else
                                               off.cpu().numpy().astype(np.float64)))
    b64 = L["bias"].cpu().numpy().astype(np.float64)
    oidx, _ = orc.biased_topk(probs, b64, cfg.K)
    ties = P.check_selection(g["idx"], probs + b64[None, :], oidx, cfg.K)
    idx_ref = oidx.copy()
    idx_ref[ties] = g["idx"][ties]
    np.testing.assert_allclose(prob_sum.cpu().numpy(), probs.sum(axis=0), rtol=2e-5, atol=1e-6)
    f_o, P_o = orc.lb_statistics(probs, idx_ref, cfg.N, D, cfg.K, K_e)
    np.testing.assert_allclose(f.cpu().numpy(), f_o, rtol=1e-6, atol=0)
    np.testing.assert_allclose(Pg.cpu().numpy(), P_o, rtol=2e-5, atol=1e-7)
    np.testing.assert_allclose(loss.item(), orc.lb_loss(f_o, P_o, alpha), rtol=2e-5)
    # the groups partition all experts
    assert abs(Pg.sum().item() - 1.0) < 1e-4


@pytest.mark.parametrize("cfg", [C.DECODE_T64, C.MID_BF16], ids=lambda c: c.name)
def test_cuda_graph_replay_matches_eager(cfg):
    """The layer captured once in a CUDA graph (programmatic dependent launches
    become graph edges) and replayed on new inputs gives the eager results bit
    for bit, bias update included."""
    L = _cfg_inputs(cfg)
    s = B.shape_of(cfg)
    K_e, mu = float(np.float32(cfg.K_e)), float(np.float32(cfg.mu))
    x_in = L["x"].clone()
    bias_g = L["bias"].clone()
    gbuf = B.LayerBuffers(s)

    def step(buf, x, bias):
        B.forward(buf, x, L["w_router"], L["w1"], L["w3"], L["w2"], bias, split_ffn=True)
        B.bias_update(cfg.N, cfg.Z, buf.counts, cfg.T, cfg.K, K_e, mu, bias)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step(gbuf, x_in, bias_g)  # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    bias_g.copy_(L["bias"])
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(gbuf, x_in, bias_g)
    ebuf = B.LayerBuffers(s)
    bias_e = L["bias"].clone()
    gen = torch.Generator(device="cuda").manual_seed(77)
    for it in range(3):
        x_new = torch.randn(x_in.shape, generator=gen, device="cuda").to(x_in.dtype)
        x_in.copy_(x_new)
        graph.replay()
        step(ebuf, x_new, bias_e)
        torch.cuda.synchronize()
        R = int(ebuf.offsets[-1].item())
        assert torch.equal(gbuf.topk_idx, ebuf.topk_idx), it
        assert torch.equal(gbuf.offsets, ebuf.offsets), it
        assert torch.equal(gbuf.y_perm[:R], ebuf.y_perm[:R]), it
        assert torch.equal(gbuf.out, ebuf.out), it
        assert torch.equal(bias_g, bias_e), it
    assert B.device_status(gbuf.ws) == 0 and B.device_status(ebuf.ws) == 0
    del graph
