"""Plant plausible mistakes in the CPU oracle and check that the pins catch each one.

Every mutation patches one function of the oracle module (on the CPU only)
and the test passes when at least one pin of ``oracle_pins`` fails.
"""
import numpy as np
import pytest

from oracle import moe_oracle as orc
from tests import oracle_pins


def _mut_gate_renormalised(mp):
    real = orc.gates

    def gates(probs, idx):
        g = real(probs, idx)
        return g / g.sum(axis=1, keepdims=True)
    mp.setattr(orc, "gates", gates)


def _mut_combine_drops_zero_term(mp):
    real = orc.combine

    def combine(x, y_perm, idx, g, slot_pos, N, gamma=1.0):
        g2 = np.where(idx >= N, 0.0, g)
        return real(x, y_perm, idx, g2, slot_pos, N, gamma)
    mp.setattr(orc, "combine", combine)


def _mut_bias_sign(mp):
    real = orc.bias_update

    def bias_update(bias, counts, N, K, K_e, mu, T_all):
        return real(bias, counts, N, K, K_e, -mu, T_all)
    mp.setattr(orc, "bias_update", bias_update)


def _mut_bias_updates_zero_experts(mp):
    def bias_update(bias, counts, N, K, K_e, mu, T_all):
        b = np.asarray(bias, dtype=np.float64).copy()
        E = len(b)
        b += mu * (K_e / (K * N) - np.asarray(counts[:E], dtype=np.float64) / (K * T_all))
        return b
    mp.setattr(orc, "bias_update", bias_update)


def _mut_tie_to_high_index(mp):
    def biased_topk(probs, bias, K):
        T, E = probs.shape
        s = probs + np.asarray(bias)[None, :]
        order = np.argsort(-s[:, ::-1], axis=1, kind="stable")
        order = E - 1 - order
        idx = order[:, :K].astype(np.int32)
        rows = np.arange(T)
        margin = (s[rows, order[:, K - 1]] - s[rows, order[:, K]]) if K < E else np.full(T, np.inf)
        return idx, margin
    mp.setattr(orc, "biased_topk", biased_topk)


def _mut_select_by_unbiased(mp):
    real = orc.biased_topk

    def biased_topk(probs, bias, K):
        return real(probs, np.zeros_like(np.asarray(bias, dtype=np.float64)), K)
    mp.setattr(orc, "biased_topk", biased_topk)


def _mut_no_silu(mp):
    mp.setattr(orc, "silu", lambda a: a)


def _mut_swapped_gate_up(mp):
    def expert_ffn(x_rows, w1, w3, w2):
        a = x_rows @ np.asarray(w3, dtype=np.float64).T
        u = x_rows @ np.asarray(w1, dtype=np.float64).T
        return (orc.silu(a) * u) @ np.asarray(w2, dtype=np.float64).T

    def expert_hidden(x_rows, w1, w3):
        return orc.silu(x_rows @ np.asarray(w3).T) * (x_rows @ np.asarray(w1).T)
    mp.setattr(orc, "expert_ffn", expert_ffn)
    mp.setattr(orc, "expert_hidden", expert_hidden)


def _mut_descending_tokens(mp):
    real = orc.canonical_permutation

    def canonical_permutation(idx, N):
        off, row_token, slot_pos = real(idx, N)
        rt = row_token.copy()
        sp = slot_pos.copy()
        for e in range(N):
            lo, hi = off[e], off[e + 1]
            rt[lo:hi] = row_token[lo:hi][::-1]
            mask = (idx == e)
            sp[mask] = lo + hi - 1 - slot_pos[mask]
        return off, rt, sp
    mp.setattr(orc, "canonical_permutation", canonical_permutation)


def _mut_softmax_no_max_shift_wrong_axis(mp):
    def softmax_rows(logits):
        e = np.exp(logits)
        return e / e.sum(axis=0, keepdims=True)
    mp.setattr(orc, "softmax_rows", softmax_rows)


def _mut_gamma_only_ffn(mp):
    real = orc.combine

    def combine(x, y_perm, idx, g, slot_pos, N, gamma=1.0):
        full = real(x, y_perm, idx, g, slot_pos, N, gamma)
        zm = np.where(idx >= N, g, 0.0).sum(axis=1)
        return full - (gamma - 1.0) * zm[:, None] * np.asarray(x, dtype=np.float64)
    mp.setattr(orc, "combine", combine)


def _mut_lb_indicator_per_token(mp):
    """'selects group j' as a 0/1 indicator per token instead of a count."""
    def lb_statistics(probs, idx, N, D, K, K_e):
        T, E = probs.shape
        G = N // D
        f, P = np.zeros(D + 1), np.zeros(D + 1)
        for j in range(D):
            hit = ((idx >= j * G) & (idx < (j + 1) * G)).any(axis=1)
            f[j] = D / (K_e * T) * hit.sum()
            P[j] = probs[:, j * G:(j + 1) * G].sum() / T
        f[D] = (idx >= N).any(axis=1).sum() / ((K - K_e) * T)
        P[D] = probs[:, N:].sum() / T
        return f, P
    mp.setattr(orc, "lb_statistics", lb_statistics)


def _mut_lb_zero_group_normaliser(mp):
    real = orc.lb_statistics

    def lb_statistics(probs, idx, N, D, K, K_e):
        f, P = real(probs, idx, N, D, K, K_e)
        f[D] *= (K - K_e) / K_e  # K_e in place of K - K_e
        return f, P
    mp.setattr(orc, "lb_statistics", lb_statistics)


def _mut_e4m3_ties_away(mp):
    real = orc.round_to_e4m3

    def round_to_e4m3(v):
        v = np.asarray(v, dtype=np.float64)
        codes, vals = real(v * (1 + 1e-15))     # nudges exact ties upward
        return codes, vals
    mp.setattr(orc, "round_to_e4m3", round_to_e4m3)


def _mut_mx_scale_off_by_one(mp):
    real = orc.mx_scale_exponent
    mp.setattr(orc, "mx_scale_exponent", lambda amax: real(amax) - 1)


def _mut_silu_derivative_sigma_only(mp):
    """SiLU'(a) taken as sigma(a), the derivative of SiLU mistaken for the gate."""
    def expert_backward(x_rows, w1, w3, w2, dy):
        w1, w3, w2 = (np.asarray(w, dtype=np.float64) for w in (w1, w3, w2))
        a, u = x_rows @ w1.T, x_rows @ w3.T
        sg = orc.sigmoid(a)
        h = a * sg * u
        dh = dy @ w2
        da, du = dh * u * sg, dh * a * sg
        return da @ w1 + du @ w3, da.T @ x_rows, du.T @ x_rows, dy.T @ h
    mp.setattr(orc, "expert_backward", expert_backward)


def _mut_lb_gradient_without_frequency(mp):
    """The aux-loss gradient taken as alpha/T, dropping the f_j weight."""
    def lb_prob_gradient(f, N, D, E, T, alpha):
        return np.full(E, float(alpha) / T)
    mp.setattr(orc, "lb_prob_gradient", lb_prob_gradient)


def _mut_softmax_backward_no_centering(mp):
    mp.setattr(orc, "softmax_backward", lambda probs, dR: probs * dR)


def _mut_mxfp8_h_unquantised(mp):
    """The SwiGLU hidden h fed to the down projection without its MXFP8 rounding."""
    q = orc.mxfp8_quantize

    def expert_ffn_mxfp8(x_rows, w1, w3, w2):
        xq = q(x_rows)[2]
        h = orc.silu(xq @ q(w1)[2].T) * (xq @ q(w3)[2].T)
        return h @ q(w2)[2].T, h
    mp.setattr(orc, "expert_ffn_mxfp8", expert_ffn_mxfp8)


def _mut_mxfp8_h_wrong_axis(mp):
    """h blocked along the token axis instead of along I (its reduction axis)."""
    q = orc.mxfp8_quantize

    def expert_ffn_mxfp8(x_rows, w1, w3, w2):
        xq = q(x_rows)[2]
        h = orc.silu(xq @ q(w1)[2].T) * (xq @ q(w3)[2].T)
        return q(h.T)[2].T @ q(w2)[2].T, h
    mp.setattr(orc, "expert_ffn_mxfp8", expert_ffn_mxfp8)


def _mut_mxfp8_x_unquantised(mp):
    """The routed token rows used at full precision."""
    q = orc.mxfp8_quantize

    def expert_ffn_mxfp8(x_rows, w1, w3, w2):
        x = np.asarray(x_rows, dtype=np.float64)
        h = orc.silu(x @ q(w1)[2].T) * (x @ q(w3)[2].T)
        return q(h)[2] @ q(w2)[2].T, h
    mp.setattr(orc, "expert_ffn_mxfp8", expert_ffn_mxfp8)


def _trajectory_record(b, idx, probs, margin, N, E):
    counts = orc.expert_counts(idx, E)
    nf = orc.ffn_experts_per_token(idx, N)
    load = counts[:N].astype(np.float64)
    return counts, dict(bias=b.copy(), counts=counts, n_ffn_mean=float(nf.mean()),
                        n_ffn_std=float(nf.std()),
                        max_over_mean_load=float(load.max() / load.mean()),
                        min_margin=float(margin.min()))


def _mut_trajectory_routes_with_next_bias(mp):
    """Step s reported (and its counts fed forward) from a routing with b_{s+1}."""
    def bias_control_trajectory(steps, route_inputs, w_router, bias0, N, K, K_e, mu):
        b = np.asarray(bias0, dtype=np.float64).copy()
        hist = []
        for s in range(steps):
            x, off = route_inputs(s)
            probs = orc.softmax_rows(orc.router_logits(x, w_router, off))
            E = probs.shape[1]
            idx, _ = orc.biased_topk(probs, b, K)
            b_next = orc.bias_update(b, orc.expert_counts(idx, E), N, K, K_e, mu, x.shape[0])
            idx, margin = orc.biased_topk(probs, b_next, K)
            counts, rec = _trajectory_record(b_next, idx, probs, margin, N, E)
            hist.append(rec)
            b = orc.bias_update(b, counts, N, K, K_e, mu, x.shape[0])
        return hist, b
    mp.setattr(orc, "bias_control_trajectory", bias_control_trajectory)


def _mut_trajectory_lagged_update(mp):
    """The update of step s applied only after step s+1 has routed (one step late)."""
    def bias_control_trajectory(steps, route_inputs, w_router, bias0, N, K, K_e, mu):
        b = np.asarray(bias0, dtype=np.float64).copy()
        hist, pending = [], None
        for s in range(steps):
            x, off = route_inputs(s)
            probs = orc.softmax_rows(orc.router_logits(x, w_router, off))
            E = probs.shape[1]
            idx, margin = orc.biased_topk(probs, b, K)
            counts, rec = _trajectory_record(b, idx, probs, margin, N, E)
            hist.append(rec)
            if pending is not None:
                b = orc.bias_update(b, pending, N, K, K_e, mu, x.shape[0])
            pending = counts
        return hist, b
    mp.setattr(orc, "bias_control_trajectory", bias_control_trajectory)


MUTATIONS = [_mut_mxfp8_h_unquantised, _mut_mxfp8_h_wrong_axis, _mut_mxfp8_x_unquantised,
             _mut_trajectory_routes_with_next_bias, _mut_trajectory_lagged_update,
             _mut_lb_gradient_without_frequency, _mut_silu_derivative_sigma_only,
             _mut_softmax_backward_no_centering,
             _mut_e4m3_ties_away, _mut_mx_scale_off_by_one, _mut_lb_indicator_per_token, _mut_lb_zero_group_normaliser, _mut_gate_renormalised, _mut_combine_drops_zero_term, _mut_bias_sign,
             _mut_bias_updates_zero_experts, _mut_tie_to_high_index, _mut_select_by_unbiased,
             _mut_no_silu, _mut_swapped_gate_up, _mut_descending_tokens,
             _mut_softmax_no_max_shift_wrong_axis, _mut_gamma_only_ffn]


@pytest.mark.parametrize("mutate", MUTATIONS, ids=lambda m: m.__name__)
def test_pins_catch_planted_mistake(mutate, monkeypatch):
    mutate(monkeypatch)
    failed = []
    for check in oracle_pins.ALL_CHECKS:
        try:
            check(orc)
        except Exception:  # an assertion or a shape error both expose the mistake
            failed.append(check.__name__)
    assert failed, f"no pin caught {mutate.__name__}"
