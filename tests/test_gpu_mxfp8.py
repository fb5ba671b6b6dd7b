"""MXFP8 expert path against the oracle: quantised weights and dispatch codes
bit for bit, expert outputs and the layer output within the bf16 tolerance of
the oracle's own MXFP8 FFN."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_30_b200 import binding as B
from mixture_experts_layer_30_b200 import configs as C
from mixture_experts_layer_30_b200 import inputs as IN
from oracle import moe_oracle as orc
from tests import parity as P

pytestmark = pytest.mark.gpu


def untile_codes(q, n, rows, cols):
    """[n*rows*cols] in 128x128 tiles -> [n, rows, cols]."""
    return q.view(n, rows // 128, cols // 128, 128, 128).permute(0, 1, 3, 2, 4).reshape(
        n, rows, cols)


def untile_scales(sf, n, rows, cols):
    """512-byte atoms (byte 16*(r%32) + 4*(r//32) + b) -> [n, rows, cols//32]."""
    a = sf.view(n, rows // 128, cols // 128, 32, 4, 4)        # (l, c, b): row 32c + l
    a = a.permute(0, 1, 4, 3, 2, 5)                            # n, rb, c, l, cb, b
    return a.reshape(n, rows, cols // 32)


def test_weight_quantisation_bit_exact():
    g = torch.Generator(device="cpu").manual_seed(21)
    n, rows, cols = 2, 256, 384
    w = (torch.randn((n, rows, cols), generator=g) * torch.exp(torch.randn((n, rows, 1),
                                                                           generator=g) * 2))
    w[0, 5, 64:96] = 0.0
    w = w.to(torch.bfloat16).cuda()
    q, sf = B.quantize_weights_mxfp8(w)
    torch.cuda.synchronize()
    codes = untile_codes(q, n, rows, cols).cpu().numpy()
    scales = untile_scales(sf, n, rows, cols).cpu().numpy().astype(np.int64)
    oc, os_, _ = orc.mxfp8_quantize(P.to_f64(w))
    np.testing.assert_array_equal(codes, oc)
    np.testing.assert_array_equal(scales, os_ + 127)


def _fp8_layer(cfg, T=None):
    L = IN.make_layer_inputs(cfg if T is None else cfg.with_T(T, cfg.name), device="cuda")
    shape = B.shape_of(cfg, T=T)
    W = {k: B.quantize_weights_mxfp8(L[k]) for k in ("w1", "w3", "w2")}
    buf = B.LayerBuffers(shape, with_probs=True)
    fb = B.Mxfp8Buffers(shape)
    B.forward_mxfp8(buf, fb, L["x"], L["w_router"], W["w1"], W["w3"], W["w2"], L["bias"])
    torch.cuda.synchronize()
    assert B.device_status(buf.ws) == 0
    return L, shape, buf, fb


@pytest.mark.parametrize("cfg", [C.MID_BF16, C.DECODE_T16, C.DECODE_T256, C.LONGCAT_SLICE],
                         ids=lambda c: c.name)
def test_mxfp8_layer(cfg):
    L, shape, buf, fb = _fp8_layer(cfg)
    x64, wr64 = P.to_f64(L["x"]), P.to_f64(L["w_router"])
    R = int(buf.offsets[-1])
    g = dict(probs=buf.probs.cpu().numpy().astype(np.float64), idx=buf.topk_idx.cpu().numpy(),
             gate=buf.topk_gate.cpu().numpy().astype(np.float64), counts=buf.counts.cpu().numpy(),
             n_ffn=buf.n_ffn.cpu().numpy(), offsets=buf.offsets.cpu().numpy(),
             row_token=buf.row_token[:R].cpu().numpy(), slot_pos=buf.slot_pos.cpu().numpy(),
             x_perm=None, R=R)
    idx_ref, probs, _ = P.check_routing_and_dispatch(g, x64, wr64, L["bias"], cfg.N, cfg.K)
    off, rt, sp = orc.canonical_permutation(idx_ref, cfg.N)
    # the quantising dispatch: codes and scales bit for bit
    xc, xs, _ = orc.mxfp8_quantize(x64[rt])
    np.testing.assert_array_equal(fb.x_perm_q[:R].cpu().numpy(), xc)
    np.testing.assert_array_equal(fb.x_perm_sf[:R].cpu().numpy().astype(np.int64), xs + 127)
    # expert outputs against the oracle's MXFP8 FFN
    y_o = np.zeros((R, cfg.d))
    h_codes_o = np.zeros((R, cfg.I), dtype=np.uint8)
    for e in range(cfg.N):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi > lo:
            y_o[lo:hi], h = orc.expert_ffn_mxfp8(x64[rt[lo:hi]], P.to_f64(L["w1"][e]),
                                                 P.to_f64(L["w3"][e]), P.to_f64(L["w2"][e]))
            h_codes_o[lo:hi] = orc.mxfp8_quantize(h)[0]
    y_g = P.to_f64(buf.y_perm[:R])
    P.assert_close(y_g, y_o, "bf16", "y_perm (mxfp8)")
    # h codes agree except where the fp32 and fp64 h fall on different sides
    # of a rounding or scale boundary
    mism = (fb.h_q[:R].cpu().numpy() != h_codes_o).mean()
    assert mism < 2e-3, mism
    gate = orc.gates(probs, idx_ref)
    P.assert_close(P.to_f64(buf.out), orc.combine(x64, y_o, idx_ref, gate, sp, cfg.N), "bf16",
                   "out (mxfp8)")
    # and the quantised layer stays close to the bf16 one (the cost of MXFP8)
    y_bf = orc.grouped_ffn(x64[rt], off, L["w1"], L["w3"], L["w2"], decode=P.to_f64)
    assert P.rel_l2(y_g, y_bf) < 0.08


def test_mxfp8_shape_guard():
    import ctypes
    s = B.make_shape(16, 128, 4, 2, 2, 128, "bf16")   # d % 256 != 0
    fake = ctypes.c_void_p(256)
    ws = ctypes.c_void_p(1 << 20)
    code = B.lib().moe_expert_down_mxfp8(ctypes.byref(s), fake, fake, fake, fake, fake, fake,
                                         ws, 1 << 30, None)
    assert code == 2 and b"MXFP8" in B.lib().moe_last_error()
