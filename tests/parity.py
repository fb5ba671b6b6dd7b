"""GPU-vs-oracle comparison helpers (used by the -m gpu tests).

Stage-by-stage checks of one forward pass, in the order the method computes:
probabilities, top-K selection (bit-exact except inside the tie band), gates,
counts, dispatch layout (bit-exact), routed copies (bit-exact), expert
outputs, combined output.  Where the oracle's top-K margin is below the tie
band the GPU may legitimately pick another ordering; such rows are checked for
validity and then the oracle's downstream stages are re-derived from the GPU's
selection so the integer comparisons stay exact everywhere.
"""
import numpy as np
import torch

from mixture_experts_layer_30_b200 import binding as B
from oracle import moe_oracle as orc

TIE_BAND = 1e-6
# Router probabilities.  fp32 layers: |p_gpu - p| <= 1e-6 (the logits are
# fp32 FMA chains over d <= 2048 products, rounded to nearest).  bf16 layers:
# the large-batch router accumulates d bf16 products in fp32 on the tensor
# cores, whose alignment inside each K = 16 step truncates; a logit error delta
# moves p by about p * delta, so the bound there is relative as well:
# |p_gpu - p| <= 1e-6 + 3e-5 p.  The selection check does not rest on either
# bound: outside the 1e-6 tie band it is exact, and the error of the GPU's
# scores at each token's decision boundary is recorded (ROUTER_ERRORS) and
# must stay below half the band, so that no selection with an oracle margin
# above the band can flip.
PROB_ATOL = 1e-6
PROB_RTOL = {"f32": 0.0, "bf16": 3e-5}
BF16_MAX_ABS, BF16_REL_L2 = 2e-2, 1e-2
F32_MAX_ABS = 1e-4
# measured router errors, one entry per checked forward pass (printed at the
# end of the session): label -> (max |dp|, max |dp| near the decision boundary)
ROUTER_ERRORS = {}


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a device tensor (bf16 decoded by the oracle's decoder)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return orc.bf16_bits_to_f64(t.view(torch.int16).numpy().view(np.uint16))
    return t.numpy().astype(np.float64)


def rel_l2(a, b):
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / den) if den > 0 else float(np.linalg.norm(a - b))


def assert_close(got, want, dtype, what):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    if got.size == 0:
        return
    err = np.abs(got - want).max()
    if dtype == "bf16":
        r = rel_l2(got, want)
        assert err <= BF16_MAX_ABS and r <= BF16_REL_L2, f"{what}: max-abs {err:.3g}, rel-L2 {r:.3g}"
    else:
        assert err <= F32_MAX_ABS, f"{what}: max-abs {err:.3g}"


def assert_ffn_part_close(got_out, want_out, identity_term, dtype, what):
    """Compare out with the identity term subtracted (the FFN part).

    In bf16 the stored out carries a rounding error of up to 2^-8 |out| that
    comes from the (large) identity term; that budget is removed element by
    element before the FFN-part tolerance is applied."""
    got_out, want_out = np.asarray(got_out), np.asarray(want_out)
    if got_out.size == 0:
        return
    ffn_want = want_out - identity_term
    if dtype != "bf16":
        assert_close(got_out - identity_term, ffn_want, dtype, what)
        return
    excess = np.maximum(0.0, np.abs(got_out - want_out) - 2.0 ** -8 * np.abs(got_out))
    err = excess.max()
    den = np.linalg.norm(ffn_want)
    r = float(np.linalg.norm(excess) / den) if den > 0 else float(np.linalg.norm(excess))
    assert err <= BF16_MAX_ABS and r <= BF16_REL_L2, f"{what}: max-abs {err:.3g}, rel-L2 {r:.3g}"


def decision_boundary_error(p_gpu, p_orc, bias, K, window=1e-4):
    """Largest |p_gpu - p| over the experts that could take part in a selection
    decision: those whose oracle biased score lies within ``window`` of the
    token's K-th or (K+1)-th largest score.  (The bias is exact on both sides,
    so this is the error of the biased scores there.)"""
    T, E = p_orc.shape
    if T == 0 or K >= E:
        return 0.0
    s = p_orc + bias[None, :]
    srt = -np.sort(-s, axis=1)
    lo = srt[:, K][:, None] - window
    hi = srt[:, K - 1][:, None] + window
    near = (s >= lo) & (s <= hi)
    err = np.abs(p_gpu - p_orc)
    return float(err[near].max()) if near.any() else 0.0


def check_selection(gpu_idx, s_orc, orc_idx, K, band=TIE_BAND):
    """Rows where the GPU's ordered top-K differs from the oracle's must be a
    valid ordered top-K of the oracle's biased scores within ``band``.
    Returns the indices of those rows."""
    T, E = s_orc.shape
    diff = np.nonzero((gpu_idx != orc_idx).any(axis=1))[0]
    for t in diff:
        L = [int(v) for v in gpu_idx[t]]
        assert len(set(L)) == K and all(0 <= v < E for v in L), (t, L)
        s = s_orc[t]
        chosen = np.zeros(E, bool)
        chosen[L] = True
        if K < E:
            assert s[chosen].min() >= s[~chosen].max() - band, (t, L, "not a top-K within band")
        for a, b in zip(L[:-1], L[1:]):
            assert s[a] >= s[b] - band, (t, L, "order outside band")
    return diff


class GpuRun:
    """Runs the layer through the C ABI and keeps every intermediate."""

    def __init__(self, shape, x, w_router, w1, w3, w2, bias, gamma=1.0, logit_offset=None,
                 split_ffn=False, fused_gather=False):
        self.buf = B.LayerBuffers(shape, device=x.device, with_probs=True)
        self.fused_gather = fused_gather
        if shape.weight_layout == B.WEIGHTS_TILED:
            # the library repacks; the oracle keeps the row-major originals
            w1, w3, w2 = B.pack_weights(w1), B.pack_weights(w3), B.pack_weights(w2)
        B.forward(self.buf, x, w_router, w1, w3, w2, bias, gamma=gamma,
                  logit_offset=logit_offset, split_ffn=split_ffn, fused_gather=fused_gather)
        del w1, w3, w2
        torch.cuda.synchronize()
        self.status = B.device_status(self.buf.ws)

    def host(self):
        b, s = self.buf, self.buf.shape
        R = int(b.offsets[-1].item())
        return dict(dtype="bf16" if s.dtype == B.MOE_BF16 else "f32",
                    label=f"{'bf16' if s.dtype == B.MOE_BF16 else 'f32'} T={s.T} d={s.d} "
                          f"E={s.N + s.Z} K={s.K}",
                    probs=b.probs.cpu().numpy().astype(np.float64),
                    idx=b.topk_idx.cpu().numpy(), gate=b.topk_gate.cpu().numpy().astype(np.float64),
                    counts=b.counts.cpu().numpy(), n_ffn=b.n_ffn.cpu().numpy(),
                    offsets=b.offsets.cpu().numpy(), row_token=b.row_token[:R].cpu().numpy(),
                    slot_pos=b.slot_pos.cpu().numpy(),
                    x_perm=None if self.fused_gather else to_f64(b.x_perm[:R]),
                    y_perm=to_f64(b.y_perm[:R]), out=to_f64(b.out), R=R)


def check_routing_and_dispatch(g, x64, wr64, bias, N, K, logit_offset=None):
    """Stages 1-3 on every token.  Returns (idx_ref, probs_orc) where idx_ref is
    the oracle's selection with tie-band rows replaced by the GPU's."""
    E = wr64.shape[0]
    dtype = g.get("dtype", "bf16")
    off = None if logit_offset is None else logit_offset.detach().cpu().numpy().astype(np.float64)
    probs = orc.softmax_rows(orc.router_logits(x64, wr64, off))
    np.testing.assert_allclose(g["probs"], probs, rtol=PROB_RTOL[dtype], atol=PROB_ATOL)
    b64 = bias.detach().cpu().numpy().astype(np.float64)
    oidx, margin = orc.biased_topk(probs, b64, K)
    boundary_err = decision_boundary_error(g["probs"], probs, b64, K)
    ROUTER_ERRORS[g.get("label", f"T={x64.shape[0]} E={E}")] = (
        float(np.abs(g["probs"] - probs).max()) if probs.size else 0.0, boundary_err)
    assert 2 * boundary_err < TIE_BAND, (
        f"router error {boundary_err:.3g} at the decision boundary could flip a selection "
        f"whose margin exceeds the {TIE_BAND} band")
    ties = check_selection(g["idx"], probs + b64[None, :], oidx, K)
    idx_ref = oidx.copy()
    idx_ref[ties] = g["idx"][ties]
    np.testing.assert_array_equal(g["idx"], idx_ref)
    np.testing.assert_allclose(g["gate"], orc.gates(probs, idx_ref), rtol=PROB_RTOL[dtype],
                               atol=PROB_ATOL)
    np.testing.assert_array_equal(g["counts"], orc.expert_counts(idx_ref, E))
    np.testing.assert_array_equal(g["n_ffn"], orc.ffn_experts_per_token(idx_ref, N))
    off_o, rt_o, sp_o = orc.canonical_permutation(idx_ref, N)
    np.testing.assert_array_equal(g["offsets"], off_o)
    np.testing.assert_array_equal(g["row_token"], rt_o)
    np.testing.assert_array_equal(g["slot_pos"], sp_o)
    assert g["R"] == off_o[-1]
    # the copies are exact (absent when the dispatch copy is fused into the GEMM)
    if g["x_perm"] is not None:
        assert np.array_equal(g["x_perm"], x64[rt_o])
    return idx_ref, probs, len(ties)


def weights_f64(w, e):
    return to_f64(w[e])
