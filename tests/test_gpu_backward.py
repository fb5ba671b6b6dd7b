"""Parity of the backward pass (through the C ABI) with the fp64 oracle's backward.

One training step runs forward_train (route, dispatch, gate/up keeping the
pre-activations, down, combine) and backward (combine backward, router
backward, expert backward, token-gradient gather).  The routing stages are
checked as in the forward tests; the oracle's backward then takes the GPU's
validated selection (tie-band rows included) and every gradient is compared.

Tolerances: the benchmark spec's bounds of the layer output (bf16: max-abs 2e-2
and rel-L2 1e-2; fp32: 1e-4) scaled by the gradient's largest magnitude,
since gradients are not O(1) quantities: a bf16 gradient rounded once from
an exact fp32 sum is already off by up to 2^-9 of its own size.
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_30_b200 import binding as B
from mixture_experts_layer_30_b200 import configs as C
from mixture_experts_layer_30_b200 import inputs as IN
from oracle import moe_oracle as orc
from tests import parity as P

pytestmark = pytest.mark.gpu


def assert_grad_close(got, want, dtype, what):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    if got.size == 0:
        return
    assert np.isfinite(got).all(), what
    scale = max(float(np.abs(want).max()), 1e-30)
    err = float(np.abs(got - want).max())
    if dtype == "bf16":
        r = P.rel_l2(got, want)
        assert err <= P.BF16_MAX_ABS * scale and r <= P.BF16_REL_L2, \
            f"{what}: max-abs {err:.3g} (scale {scale:.3g}), rel-L2 {r:.3g}"
    else:
        assert err <= P.F32_MAX_ABS * max(1.0, scale), f"{what}: max-abs {err:.3g}"


def _dout(shape, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    dt = B.torch_dtype(shape)
    return torch.randn((shape.T, shape.d), generator=g).to(dt).cuda()


def train_step(shape, L, dout, gamma=1.0, lb=None):
    """forward_train + backward through the C ABI; returns (buf, bb).
    lb = (D, K_e, alpha): the load-balance loss joins the backward, with f from
    moe_lb_stats on this step's counts and probability sums."""
    buf = B.LayerBuffers(shape, with_probs=True)
    bb = B.BackwardBuffers(shape)
    w1, w3, w2 = L["w1"], L["w3"], L["w2"]
    if shape.weight_layout == B.WEIGHTS_TILED:
        w1, w3, w2 = B.pack_weights(w1), B.pack_weights(w3), B.pack_weights(w2)
    E = shape.N + shape.Z
    prob_sum = torch.empty(E, dtype=torch.float32, device="cuda") if lb else None
    B.forward_train(buf, bb, L["x"], L["w_router"], w1, w3, w2, L["bias"], gamma=gamma,
                    prob_sum=prob_sum)
    lb_arg = None
    if lb:
        D, K_e, alpha = lb
        f = torch.empty(D + 1, dtype=torch.float32, device="cuda")
        P = torch.empty(D + 1, dtype=torch.float32, device="cuda")
        B.lb_stats(shape.N, shape.Z, D, buf.counts, prob_sum, shape.T, shape.K, K_e, alpha, f, P)
        lb_arg = (f, D, alpha, shape.T)
    B.backward(buf, bb, L["x"], L["w_router"], w1, w3, w2, dout, gamma=gamma, lb=lb_arg)
    torch.cuda.synchronize()
    assert B.device_status(buf.ws) == 0
    assert B.device_status(bb.bws) == 0
    return buf, bb


def _host_forward(buf):
    b = buf
    R = int(b.offsets[-1].item())
    return dict(probs=b.probs.cpu().numpy().astype(np.float64), idx=b.topk_idx.cpu().numpy(),
                gate=b.topk_gate.cpu().numpy().astype(np.float64),
                counts=b.counts.cpu().numpy(), n_ffn=b.n_ffn.cpu().numpy(),
                offsets=b.offsets.cpu().numpy(), row_token=b.row_token[:R].cpu().numpy(),
                slot_pos=b.slot_pos.cpu().numpy(), x_perm=P.to_f64(b.x_perm[:R]),
                y_perm=P.to_f64(b.y_perm[:R]), out=P.to_f64(b.out), R=R)


def check_backward(shape, dtype, L, N, K, gamma=1.0, seed=0, lb=None):
    dout = _dout(shape, 5000 + seed)
    buf, bb = train_step(shape, L, dout, gamma, lb=lb)
    g = _host_forward(buf)
    x64, wr64 = P.to_f64(L["x"]), P.to_f64(L["w_router"])
    idx_ref, _, _ = P.check_routing_and_dispatch(g, x64, wr64, L["bias"], N, K)
    ref = orc.moe_layer_backward(x64, wr64, L["w1"], L["w3"], L["w2"],
                                 L["bias"].cpu().numpy().astype(np.float64), N, K,
                                 P.to_f64(dout), gamma=gamma, decode=P.to_f64,
                                 selection=idx_ref, lb=lb)
    R = g["R"]
    P.assert_close(g["y_perm"], ref["y_perm"], dtype, "y_perm")
    # the kept pre-activations a | u
    I = shape.I
    au = P.to_f64(bb.au[:R])
    a_ref = np.zeros((R, I))
    u_ref = np.zeros((R, I))
    off = ref["offsets"]
    for e in range(N):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi > lo:
            a_ref[lo:hi] = ref["x_perm"][lo:hi] @ P.to_f64(L["w1"][e]).T
            u_ref[lo:hi] = ref["x_perm"][lo:hi] @ P.to_f64(L["w3"][e]).T
    assert_grad_close(au[:, :I], a_ref, dtype, "a")
    assert_grad_close(au[:, I:], u_ref, dtype, "u")
    assert_grad_close(bb.dgate.cpu().numpy(), ref["dgate"], dtype, "dgate")
    assert_grad_close(P.to_f64(bb.dy_perm[:R]), ref["dy_perm"], dtype, "dy_perm")
    assert_grad_close(P.to_f64(bb.dx_perm[:R]), ref["dx_perm"], dtype, "dx_perm")
    assert_grad_close(P.to_f64(bb.dw1), ref["dw1"], dtype, "dw1")
    assert_grad_close(P.to_f64(bb.dw3), ref["dw3"], dtype, "dw3")
    assert_grad_close(P.to_f64(bb.dw2), ref["dw2"], dtype, "dw2")
    assert_grad_close(P.to_f64(bb.dw_router), ref["dw_router"], dtype, "dw_router")
    assert_grad_close(P.to_f64(bb.dx), ref["dx"], dtype, "dx")
    # experts that received no rows get exactly zero weight gradients
    cnt = g["counts"][:N]
    for e in np.nonzero(cnt == 0)[0]:
        assert not bb.dw1[e].any() and not bb.dw3[e].any() and not bb.dw2[e].any(), e
    return buf, bb, ref


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


def test_backward_tiny_f32():
    cfg = C.TINY_F32
    L = IN.make_layer_inputs(cfg, device="cuda")
    check_backward(B.shape_of(cfg), "f32", L, cfg.N, cfg.K)


@pytest.mark.parametrize("T", [1, 37, 300])
def test_backward_f32_ragged_gamma_empty_expert(T):
    bias = np.zeros(12)
    bias[3] = -10.0  # expert 3 is never selected: its weight gradients are zero
    shape, L = _small(T, 128, 8, 4, 3, 64, "f32", seed=T, bias=bias)
    check_backward(shape, "f32", L, 8, 3, gamma=1.7, seed=T)


@pytest.mark.parametrize("layout", [B.WEIGHTS_ROW_MAJOR, B.WEIGHTS_TILED], ids=["rowmajor", "tiled"])
@pytest.mark.parametrize("T", [512, 77])
def test_backward_bf16_multitile(T, layout):
    """d = 640 and I = 384: partial 256-feature blocks on both expert axes;
    ~170 rows per expert: three 64-row K blocks with a ragged tail in the
    weight gradients; E = 16: the router's K tail past E; one empty expert."""
    bias = np.zeros(16)
    bias[3] = -10.0
    shape, L = _small(T, 640, 12, 4, 4, 384, "bf16", seed=40 + T, bias=bias, w_std=0.03)
    shape.weight_layout = layout
    check_backward(shape, "bf16", L, 12, 4, gamma=1.3, seed=T)


def test_backward_mid_bf16():
    cfg = C.MID_BF16
    L = IN.make_layer_inputs(cfg, device="cuda")
    check_backward(B.shape_of(cfg), "bf16", L, cfg.N, cfg.K)


def test_backward_decode_bf16_tiled():
    cfg = C.DECODE_T16
    L = IN.make_layer_inputs(cfg, device="cuda")
    check_backward(B.shape_of(cfg, weight_layout=B.WEIGHTS_TILED), "bf16", L, cfg.N, cfg.K)


def test_backward_longcat_slice_bf16():
    cfg = C.LONGCAT_SLICE
    L = IN.make_layer_inputs(cfg, device="cuda")
    check_backward(B.shape_of(cfg, weight_layout=B.WEIGHTS_TILED), "bf16", L, cfg.N, cfg.K)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_backward_is_deterministic_and_forward_unchanged(dtype):
    """Two training steps give bit-identical gradients (fixed-order reductions,
    no atomics), and the training forward's h, y_perm and out equal the
    inference forward's bit for bit."""
    shape, L = _small(300, 256, 12, 4, 4, 128, dtype, seed=7)
    dout = _dout(shape, 99)
    buf1, bb1 = train_step(shape, L, dout)
    buf2, bb2 = train_step(shape, L, dout)
    for name in ("dgate", "dy_perm", "dx_perm", "dx_router", "dx", "dw_router", "dw1", "dw3",
                 "dw2"):
        a, b = getattr(bb1, name), getattr(bb2, name)
        if name in ("dy_perm", "dx_perm"):
            R = int(buf1.offsets[-1].item())
            a, b = a[:R], b[:R]
        assert torch.equal(a, b), name
    ref = B.LayerBuffers(shape, with_probs=True)
    B.forward(ref, L["x"], L["w_router"], L["w1"], L["w3"], L["w2"], L["bias"], split_ffn=True)
    torch.cuda.synchronize()
    R = int(ref.offsets[-1].item())
    assert torch.equal(ref.h[:R], buf1.h[:R])
    assert torch.equal(ref.y_perm[:R], buf1.y_perm[:R])
    assert torch.equal(ref.out, buf1.out)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_backward_k_equals_e(dtype):
    """Every expert selected: the gates sum to 1 and dlogits covers all E."""
    N, Z = 12, 4
    shape, L = _small(60, 256, N, Z, N + Z, 128, dtype, seed=61)
    check_backward(shape, dtype, L, N, N + Z, seed=61)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_backward_all_slots_to_zero_experts(dtype):
    """No routed rows: the expert weight gradients are exactly zero and dx is
    the identity term plus the router term."""
    N, Z, K = 8, 8, 3
    bias = [0.0] * N + [10.0] * Z
    shape, L = _small(70, 256, N, Z, K, 128, dtype, seed=62, bias=bias)
    buf, bb, _ = check_backward(shape, dtype, L, N, K, gamma=0.8, seed=62)
    assert int(buf.offsets[-1].item()) == 0
    assert not bb.dw1.any() and not bb.dw3.any() and not bb.dw2.any()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_backward_no_zero_experts(dtype):
    shape, L = _small(150, 256, 16, 0, 3, 128, dtype, seed=63)
    check_backward(shape, dtype, L, 16, 3, seed=63)


def test_backward_max_experts_bf16():
    """E = 1024 experts and K = 40 slots per token."""
    N, Z, K = 640, 384, 40
    shape, L = _small(150, 128, N, Z, K, 128, "bf16", seed=64)
    check_backward(shape, "bf16", L, N, K, seed=64)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_backward_empty_batch(dtype):
    """T = 0: every call is a no-op except that the weight gradients are zero."""
    shape, L = _small(0, 256, 8, 8, 2, 128, dtype, seed=65)
    L["x"] = torch.empty((0, 256), dtype=L["x"].dtype, device="cuda")
    dout = torch.empty((0, 256), dtype=L["x"].dtype, device="cuda")
    buf = B.LayerBuffers(shape, with_probs=True)
    bb = B.BackwardBuffers(shape)
    for t in (bb.dw1, bb.dw3, bb.dw2, bb.dw_router):
        t.fill_(1.0)
    B.forward_train(buf, bb, L["x"], L["w_router"], L["w1"], L["w3"], L["w2"], L["bias"])
    B.backward(buf, bb, L["x"], L["w_router"], L["w1"], L["w3"], L["w2"], dout)
    torch.cuda.synchronize()
    assert B.device_status(buf.ws) == 0 and B.device_status(bb.bws) == 0
    for t in (bb.dw1, bb.dw3, bb.dw2, bb.dw_router):
        assert not t.any()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_backward_with_load_balance_loss(dtype):
    """The load-balance loss alpha sum_j f_j P_j (Eq. (3)-(5)) in the router's
    gradient: f from moe_lb_stats on the GPU, the oracle's own f from the same
    selection; alpha is large enough that the term moves dW_r and dx."""
    N, Z, K, D = 16, 8, 4, 4
    K_e = float(np.float32(K * N / (N + Z)))
    shape, L = _small(300, 256, N, Z, K, 128, dtype, seed=66)
    check_backward(shape, dtype, L, N, K, seed=66, lb=(D, K_e, 5.0))


def test_backward_load_balance_term_changes_only_the_router_gradients():
    N, Z, K, D = 16, 8, 4, 4
    K_e = float(np.float32(K * N / (N + Z)))
    shape, L = _small(200, 256, N, Z, K, 128, "bf16", seed=67)
    dout = _dout(shape, 67)
    buf0, b0 = train_step(shape, L, dout)
    _, b1 = train_step(shape, L, dout, lb=(D, K_e, 5.0))
    R = int(buf0.offsets[-1].item())  # rows past R are not written
    for name in ("dw1", "dw3", "dw2", "dgate"):
        assert torch.equal(getattr(b0, name), getattr(b1, name)), name
    assert torch.equal(b0.dy_perm[:R], b1.dy_perm[:R])
    assert not torch.equal(b0.dw_router, b1.dw_router)
    assert not torch.equal(b0.dx, b1.dx)


def test_weight_gradients_isolated_from_a_nonfinite_neighbour():
    """Each expert's weight gradients depend on its own rows only.  The wgrad
    GEMMs read whole 16-row steps: the gradient operand (dy, da|du) is zeroed
    past every segment end, so the next expert's gradient rows -- even
    infinite ones -- never enter; the activation operand (x_perm, h) past the
    last segment was never written by the forward pass and is cleared, so
    garbage there (here: infinities) never enters either."""
    shape, L = _small(96, 256, 8, 0, 2, 128, "bf16", seed=11)
    buf = B.LayerBuffers(shape, with_probs=True)
    bb = B.BackwardBuffers(shape)
    B.forward_train(buf, bb, L["x"], L["w_router"], L["w1"], L["w3"], L["w2"], L["bias"])
    dout = _dout(shape, 77)
    B.combine_backward(shape, L["x"], buf.y_perm, buf.topk_idx, buf.topk_gate, buf.slot_pos,
                       dout, 1.0, bb.dy_perm, bb.dgate)
    torch.cuda.synchronize()
    off = buf.offsets.cpu().numpy()
    cnt = np.diff(off)
    R = int(off[-1])
    nbr = [e for e in range(shape.N - 1) if cnt[e] % 16 and cnt[e + 1] > 0]
    assert nbr, cnt  # a segment end inside a 16-row step, followed by rows of another expert

    def expert_bwd(dy):
        B.expert_ffn_backward(shape, buf.x_perm, L["w1"], L["w3"], L["w2"], buf.offsets, buf.h,
                              bb.au, dy, bb.dx_perm, bb.dw1, bb.dw3, bb.dw2, bb.bws)
        torch.cuda.synchronize()
        assert B.device_status(bb.bws) == 0
        return bb.dw1.clone(), bb.dw3.clone(), bb.dw2.clone()

    def same(a, b, skip=()):
        for c, d in zip(a, b):
            for j in range(shape.N):
                if j in skip:
                    continue
                assert torch.isfinite(d[j]).all(), j
                assert torch.equal(c[j], d[j]), j

    buf.x_perm[R:] = 0
    buf.h[R:] = 0
    clean = expert_bwd(bb.dy_perm)
    # rows never written by the forward pass hold garbage
    buf.x_perm[R:] = float("inf")
    buf.h[R:] = float("inf")
    same(clean, expert_bwd(bb.dy_perm))
    # infinite gradient rows in the next expert's segment
    for e in nbr:
        dy = bb.dy_perm.clone()
        dy[int(off[e + 1]):int(off[e + 2])] = float("inf")
        same(clean, expert_bwd(dy), skip=(e + 1,))
