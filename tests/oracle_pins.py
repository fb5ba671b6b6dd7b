"""Checks that pin the fp64 oracle to facts that do not come from the oracle.

Each ``check_*`` takes the oracle module and raises AssertionError on a
mismatch, so the same checks run against the real oracle (test_oracle_pins)
and against copies with a planted mistake (test_oracle_mutations).

Sources of truth used here, none of them the oracle's own code:
  * hand derivations of tiny layers stored under tests/golden/ (closed forms);
  * brute-force enumeration of expert subsets with exact rational sums;
  * the Z = 0 reduction to a textbook dense top-K MoE, written with torch's
    float64 CPU linear layer and SiLU;
  * closed forms of softmax (E = 2 is a logistic sigmoid) and of Eq. (2);
  * permutation invariants (bijection, sortedness, segment sizes).
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------
# worked examples (hand derivations)
# ---------------------------------------------------------------------------

def check_worked_tiny_layer(orc):
    g = load_golden("worked_example_tiny_layer.json")
    sh, ex = g["shape"], g["expected"]
    r = orc.moe_layer(np.array(g["x"]), np.array(g["w_router"]), np.array(g["w1"]),
                      np.array(g["w3"]), np.array(g["w2"]), np.array(g["bias"]),
                      N=sh["N"], K=sh["K"])
    np.testing.assert_allclose(r["probs"], ex["probs"], rtol=0, atol=1e-15)
    np.testing.assert_array_equal(r["idx"], ex["topk_idx"])
    np.testing.assert_allclose(r["gate"], ex["gate"], rtol=0, atol=1e-15)
    np.testing.assert_array_equal(r["counts"], ex["counts"])
    np.testing.assert_array_equal(r["n_ffn"], ex["n_ffn"])
    np.testing.assert_allclose(r["y_perm"][0, 0], ex["y_expert0"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(r["out"], ex["out"], rtol=0, atol=1e-15)


def check_worked_swiglu(orc):
    g = load_golden("worked_example_swiglu.json")
    ex = g["expected"]
    y = orc.expert_ffn(np.array([[g["x"]]]), np.array([[g["w1"]]]), np.array([[g["w3"]]]),
                       np.array([[g["w2"]]]))
    h = orc.expert_hidden(np.array([[g["x"]]]), np.array([[g["w1"]]]), np.array([[g["w3"]]]))
    np.testing.assert_allclose(orc.silu(np.array([1.0]))[0], ex["silu_a"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(h[0, 0], ex["h"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(y[0, 0], ex["y"], rtol=0, atol=1e-14)


def check_worked_bias_update(orc):
    g = load_golden("worked_example_bias_update.json")
    b = orc.bias_update(np.array(g["bias"]), np.array(g["counts"]), g["N"], g["K"],
                        g["K_e"], g["mu"], g["T_all"])
    np.testing.assert_allclose(b, g["expected_bias"], rtol=0, atol=1e-16)
    # zero experts unchanged bit for bit
    assert b[g["N"]:].tobytes() == np.array(g["bias"][g["N"]:]).tobytes()


def check_worked_zero_experts(orc):
    g = load_golden("worked_example_zero_experts.json")
    sh, ex = g["shape"], g["expected"]
    probs = orc.softmax_rows(np.array(g["router_logits"]))
    np.testing.assert_allclose(probs, ex["probs"], rtol=0, atol=1e-15)
    idx, _ = orc.biased_topk(probs, np.array(g["bias"]), sh["K"])
    np.testing.assert_array_equal(idx, ex["topk_idx"])
    gate = orc.gates(probs, idx)
    _, _, slot_pos = orc.canonical_permutation(idx, sh["N"])
    out = orc.combine(np.array(g["x"]), np.zeros((0, sh["d"])), idx, gate, slot_pos, sh["N"])
    np.testing.assert_allclose(orc.zero_mass(idx, gate, sh["N"]), [ex["zero_mass"]],
                               rtol=0, atol=1e-15)
    np.testing.assert_allclose(out, ex["out"], rtol=0, atol=1e-15)


# ---------------------------------------------------------------------------
# softmax closed forms
# ---------------------------------------------------------------------------

def check_softmax_closed_forms(orc, seed=0):
    rng = np.random.default_rng(seed)
    lg = rng.normal(size=(64, 2)) * 3
    p = orc.softmax_rows(lg)
    sig = np.array([1.0 / (1.0 + math.exp(-(a - b))) for a, b in lg])
    np.testing.assert_allclose(p[:, 0], sig, rtol=0, atol=1e-15)
    lg = rng.normal(size=(32, 17))
    p = orc.softmax_rows(lg)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-15)
    p2 = orc.softmax_rows(lg + rng.normal(size=(32, 1)) * 50)
    np.testing.assert_allclose(p2, p, rtol=1e-12, atol=0)
    # ratio of two entries is exp of the logit gap
    np.testing.assert_allclose(p[:, 3] / p[:, 5], np.exp(lg[:, 3] - lg[:, 5]), rtol=1e-12)


# ---------------------------------------------------------------------------
# top-K against brute force with exact sums
# ---------------------------------------------------------------------------

def brute_force_topk(s_row, K):
    """The K-subset with the largest exact sum, ties to the smallest sorted index tuple;
    returned in (score desc, index asc) order."""
    E = len(s_row)
    fr = [Fraction(v) for v in s_row]
    best, best_sum = None, None
    for sub in itertools.combinations(range(E), K):
        sm = sum(fr[i] for i in sub)
        if best is None or sm > best_sum or (sm == best_sum and sub < best):
            best, best_sum = sub, sm
    return sorted(best, key=lambda i: (-fr[i], i))


def check_topk_brute_force(orc, cases=300, seed=1):
    rng = np.random.default_rng(seed)
    for c in range(cases):
        E = int(rng.integers(2, 11))
        K = int(rng.integers(1, min(4, E) + 1))
        if c % 3 == 0:
            # forced ties: few distinct dyadic values so sums are exact and equal
            probs = rng.integers(0, 4, size=(1, E)) / 8.0
            bias = rng.integers(-1, 2, size=E) / 16.0
        else:
            probs = orc.softmax_rows(rng.normal(size=(1, E)))
            bias = rng.uniform(-0.1, 0.1, size=E)
        idx, margin = orc.biased_topk(probs, bias, K)
        s = probs[0] + bias
        want = brute_force_topk(s, K)
        assert list(idx[0]) == want, (probs, bias, K, idx, want)
        srt = sorted(s, reverse=True)
        m_want = srt[K - 1] - srt[K] if K < E else math.inf
        assert margin[0] == m_want


# ---------------------------------------------------------------------------
# Z = 0: textbook dense top-K MoE; general Z: dense masked formulation
# ---------------------------------------------------------------------------

def dense_moe_torch(x, w_router, w1, w3, w2, bias, N, K, gamma=1.0):
    """Run every expert on every token (zero experts as identity) and mask by
    the top-K of (p + b); torch float64 CPU ops only."""
    F = torch.nn.functional
    x = torch.as_tensor(x, dtype=torch.float64)
    p = torch.softmax(F.linear(x, torch.as_tensor(w_router, dtype=torch.float64)), dim=1)
    T, E = p.shape
    s = p + torch.as_tensor(bias, dtype=torch.float64)[None, :]
    out = torch.zeros_like(x)
    for t in range(T):
        chosen = sorted(range(E), key=lambda i: (-float(s[t, i]), i))[:K]
        for i in chosen:
            if i < N:
                w1e = torch.as_tensor(w1[i], dtype=torch.float64)
                w3e = torch.as_tensor(w3[i], dtype=torch.float64)
                w2e = torch.as_tensor(w2[i], dtype=torch.float64)
                y = F.linear(F.silu(F.linear(x[t], w1e)) * F.linear(x[t], w3e), w2e)
            else:
                y = x[t]
            out[t] += p[t, i] * y
    return (gamma * out).numpy()


def _rand_layer(rng, T, d, N, Z, I, bias_amp):
    E = N + Z
    return dict(x=rng.normal(size=(T, d)), w_router=rng.normal(size=(E, d)) * 0.5,
                w1=rng.normal(size=(N, I, d)) * 0.3, w3=rng.normal(size=(N, I, d)) * 0.3,
                w2=rng.normal(size=(N, d, I)) * 0.3, bias=rng.uniform(-bias_amp, bias_amp, E))


def check_dense_reduction(orc, seed=2):
    rng = np.random.default_rng(seed)
    for (T, d, N, Z, K, I, amp, gamma) in ((9, 5, 6, 0, 2, 3, 0.0, 1.0),
                                           (9, 5, 6, 0, 3, 3, 0.2, 1.0),
                                           (11, 4, 5, 3, 3, 7, 0.1, 1.0),
                                           (7, 6, 4, 4, 8, 2, 0.3, 2.5)):
        L = _rand_layer(rng, T, d, N, Z, I, amp)
        r = orc.moe_layer(L["x"], L["w_router"], L["w1"], L["w3"], L["w2"], L["bias"],
                          N=N, K=K, gamma=gamma)
        want = dense_moe_torch(L["x"], L["w_router"], L["w1"], L["w3"], L["w2"], L["bias"],
                               N, K, gamma)
        np.testing.assert_allclose(r["out"], want, rtol=1e-12, atol=1e-12)


def check_all_zero_experts_fixed_point(orc, seed=3):
    """b_zero = +10 routes every slot to zero experts: out = (sum g) x exactly."""
    rng = np.random.default_rng(seed)
    T, d, N, Z, K, I = 13, 6, 5, 4, 3, 4
    L = _rand_layer(rng, T, d, N, Z, I, 0.0)
    L["bias"][N:] = 10.0
    r = orc.moe_layer(L["x"], L["w_router"], L["w1"], L["w3"], L["w2"], L["bias"], N=N, K=K)
    assert (r["idx"] >= N).all()
    assert r["offsets"][-1] == 0 and (r["slot_pos"] == -1).all()
    g_sum = r["gate"].sum(axis=1)
    assert (r["out"] == g_sum[:, None] * L["x"]).all()


def check_k_equals_e_fixed_point(orc, seed=4):
    """K = E selects every expert: the gates sum to 1 and out = sum_i R_i E_i(x)."""
    rng = np.random.default_rng(seed)
    T, d, N, Z, I = 6, 4, 3, 2, 5
    E = N + Z
    L = _rand_layer(rng, T, d, N, Z, I, 0.1)
    r = orc.moe_layer(L["x"], L["w_router"], L["w1"], L["w3"], L["w2"], L["bias"], N=N, K=E)
    np.testing.assert_allclose(r["gate"].sum(axis=1), 1.0, rtol=0, atol=1e-15)
    want = dense_moe_torch(L["x"], L["w_router"], L["w1"], L["w3"], L["w2"], L["bias"], N, E)
    np.testing.assert_allclose(r["out"], want, rtol=1e-12, atol=1e-12)
    # for K < E the selected gates sum to at most 1
    r2 = orc.moe_layer(L["x"], L["w_router"], L["w1"], L["w3"], L["w2"], L["bias"], N=N, K=2)
    assert (r2["gate"].sum(axis=1) <= 1.0 + 1e-15).all() and (r2["gate"] > 0).all()


# ---------------------------------------------------------------------------
# permutation invariants
# ---------------------------------------------------------------------------

def check_permutation_invariants(orc, seed=5):
    rng = np.random.default_rng(seed)
    for _ in range(20):
        T, N, Z = int(rng.integers(1, 60)), int(rng.integers(1, 12)), int(rng.integers(0, 6))
        E = N + Z
        K = int(rng.integers(1, E + 1))
        idx = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int32)
        counts = orc.expert_counts(idx, E)
        assert counts.sum() == K * T
        off, row_token, slot_pos = orc.canonical_permutation(idx, N)
        R = int((idx < N).sum())
        assert off[0] == 0 and off[N] == R and len(row_token) == R
        np.testing.assert_array_equal(np.diff(off), counts[:N])
        seen = np.zeros(R, dtype=bool)
        for t in range(T):
            for k in range(K):
                e, p = idx[t, k], slot_pos[t, k]
                if e < N:
                    assert off[e] <= p < off[e + 1] and row_token[p] == t and not seen[p]
                    seen[p] = True
                else:
                    assert p == -1
        assert seen.all()
        for e in range(N):
            seg = row_token[off[e]:off[e + 1]]
            assert (np.diff(seg) > 0).all()


# ---------------------------------------------------------------------------
# Eq. (2) closed forms
# ---------------------------------------------------------------------------

def check_bias_update_closed_form(orc, seed=6):
    rng = np.random.default_rng(seed)
    for _ in range(50):
        N, Z = int(rng.integers(1, 40)), int(rng.integers(0, 20))
        E = N + Z
        K = int(rng.integers(1, E + 1))
        T = int(rng.integers(1, 500))
        K_e = float(rng.uniform(0.5, K))
        mu = float(rng.uniform(0.001, 1.0))
        idx = np.stack([rng.permutation(E)[:K] for _ in range(T)])
        counts = np.bincount(idx.reshape(-1), minlength=E)
        b0 = rng.normal(size=E)
        b1 = orc.bias_update(b0, counts, N, K, K_e, mu, T)
        F = counts[:N].sum()
        # sum of increments over FFN experts: mu (K_e - F/T) / K
        np.testing.assert_allclose((b1 - b0)[:N].sum(), mu * (K_e - F / T) / K,
                                   rtol=1e-9, atol=1e-12)
        assert b1[N:].tobytes() == b0[N:].tobytes()
        # experts above their share move down, below it move up
        share = counts[:N] / (K * T)
        tgt = K_e / (K * N)
        assert ((b1 - b0)[:N][share > tgt + 1e-12] < 0).all()
        assert ((b1 - b0)[:N][share < tgt - 1e-12] > 0).all()
    # at rest exactly when every FFN expert sits at its target share
    N, K, T, K_e = 4, 2, 8, 1.0
    counts = np.array([2, 2, 2, 2, 5, 3])
    b1 = orc.bias_update(np.zeros(6), counts, N, K, K_e, 0.3, T)
    assert (b1 == 0).all()


def check_worked_lb_statistics(orc):
    g = load_golden("worked_example_lb_statistics.json")
    ex = g["expected"]
    f, P = orc.lb_statistics(np.array(g["probs"]), np.array(g["topk_idx"]), g["N"], g["D"],
                             g["K"], g["K_e"])
    np.testing.assert_allclose(f, ex["f"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(P, ex["P"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(orc.lb_loss(f, P, g["alpha"]), ex["loss"], rtol=0, atol=1e-15)


def check_lb_statistics_closed_forms(orc, seed=7):
    rng = np.random.default_rng(seed)
    for _ in range(30):
        D = int(rng.integers(1, 5))
        G = int(rng.integers(1, 4))
        N, Z = D * G, int(rng.integers(1, 5))
        E = N + Z
        K = int(rng.integers(2, E + 1))
        K_e = float(rng.uniform(0.5, K - 0.5))
        T = int(rng.integers(1, 40))
        probs = orc.softmax_rows(rng.normal(size=(T, E)))
        idx = np.stack([rng.permutation(E)[:K] for _ in range(T)])
        f, P = orc.lb_statistics(probs, idx, N, D, K, K_e)
        # the groups partition all experts: the P_j sum to 1
        np.testing.assert_allclose(P.sum(), 1.0, rtol=0, atol=1e-12)
        # every selection is counted once: sum_j f_j * (its normaliser) = K T
        total = f[:D].sum() * K_e * T / D + f[D] * (K - K_e) * T
        np.testing.assert_allclose(total, K * T, rtol=1e-12)
        # brute force over tokens and slots
        sel = np.zeros(D + 1)
        for t in range(T):
            for k in range(K):
                e = int(idx[t, k])
                sel[D if e >= N else e // G] += 1
        want_f = np.concatenate([sel[:D] * D / (K_e * T), [sel[D] / ((K - K_e) * T)]])
        np.testing.assert_allclose(f, want_f, rtol=1e-14)
    # balance point: every token picks one expert per FFN group and K - D zero experts
    D, G, Z, T = 3, 2, 4, 5
    N, K = D * G, D + 2
    idx = np.array([[j * G + (t % G) for j in range(D)] + [N + (t % Z), N + ((t + 1) % Z)]
                    for t in range(T)])
    f, _ = orc.lb_statistics(np.full((T, N + Z), 1.0 / (N + Z)), idx, N, D, K, float(D))
    np.testing.assert_allclose(f, 1.0, rtol=0, atol=1e-15)


def check_bf16_decode(orc):
    bits = np.array([0x3F80, 0xC000, 0x3F81, 0x7F7F, 0x0001, 0x8000, 0x4049], dtype=np.uint16)
    want = [1.0, -2.0, 1.0 + 2.0 ** -7, (2 - 2.0 ** -7) * 2.0 ** 127, 2.0 ** -133, -0.0,
            3.140625]
    got = orc.bf16_bits_to_f64(bits)
    assert list(got) == want
    assert math.copysign(1.0, got[5]) == -1.0


def check_e4m3_table(orc):
    """Values fixed by the E4M3 definition (sign, 4-bit exponent with bias 7,
    3-bit mantissa, subnormals, 0x7F/0xFF NaN, no infinity)."""
    t = orc.e4m3_values()
    assert t[0x7E] == 448.0 and t[0x08] == 2.0 ** -6 and t[0x01] == 2.0 ** -9
    assert t[0x38] == 1.0 and t[0x40] == 2.0 and t[0x3F] == 1.875 and t[0x07] == 7 * 2.0 ** -9
    assert t[0xB8] == -1.0 and t[0x80] == 0.0 and np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    finite = t[~np.isnan(t)]
    assert len(np.unique(finite)) == 253  # +-0 coincide


def brute_force_e4m3(v):
    """Nearest finite E4M3 code by exhaustive search; ties to the even code."""
    t = e4m3_table_cache()
    a = min(abs(v), 448.0)
    best = None
    for c in range(0x7F):
        d = abs(t[c] - a)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c)
    c = best[1]
    if math.copysign(1.0, v) < 0:
        c |= 0x80
    return c


_E4M3 = None


def e4m3_table_cache():
    global _E4M3
    if _E4M3 is None:
        vals = []
        for c in range(256):
            e, m = (c >> 3) & 0xF, c & 7
            mag = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
            vals.append(-mag if c & 0x80 else mag)
        _E4M3 = vals
    return _E4M3


def check_e4m3_rounding_brute_force(orc, seed=8):
    rng = np.random.default_rng(seed)
    t = e4m3_table_cache()
    mids = [(t[c] + t[c + 1]) / 2 for c in range(0x7E)]           # exact ties
    vals = list(rng.normal(size=300) * 50) + list(rng.uniform(-1e-3, 1e-3, 100)) + mids + \
        [-m for m in mids] + [0.0, -0.0, 500.0, -1e6, 448.0, 2.0 ** -10]
    codes, deq = orc.round_to_e4m3(np.array(vals))
    for v, c, dv in zip(vals, codes, deq):
        want = brute_force_e4m3(v)
        assert int(c) == want, (v, int(c), want)
        assert dv == t[want & 0x7F] * (-1 if want & 0x80 else 1)


def check_mxfp8_block_quantization(orc, seed=9):
    rng = np.random.default_rng(seed)
    a = rng.normal(size=(7, 96)) * np.exp(rng.normal(size=(7, 1)) * 3)
    a[3, 32:64] = 0.0                                               # an all-zero block
    codes, s, deq = orc.mxfp8_quantize(a)
    blocks = np.abs(a).reshape(7, 3, 32)
    amax = blocks.max(axis=-1)
    nz = amax > 0
    # the scale puts every block's largest magnitude in (224, 448] before rounding:
    # the smallest power of two that avoids saturation
    assert ((amax[nz] / 2.0 ** s[nz] > 224) & (amax[nz] / 2.0 ** s[nz] <= 448)).all()
    assert (s[~nz] == 0).all() and (deq[3, 32:64] == 0).all()
    # exact powers-of-two boundaries: 448 * 2^k maps to s = k, just above it to k + 1
    sb = orc.mx_scale_exponent(np.array([448.0, 448.0 * 2 ** -5, 448.0 * 2 ** 3 * (1 + 2 ** -40),
                                         1.0, 0.0]))
    assert list(sb) == [0, -5, 4, -8, 0]
    # normal-range elements are within half an E4M3 step (2^-4 relative)
    big = np.abs(a) >= (2.0 ** np.repeat(s, 32, axis=1)) * 2.0 ** -6
    rel = np.abs(deq - a)[big] / np.abs(a)[big]
    assert rel.max() <= 2.0 ** -4 + 1e-12
    # quantising a quantised array changes nothing
    _, s2, deq2 = orc.mxfp8_quantize(deq)
    assert np.array_equal(deq2, deq)


def _golden_mxfp8_weights(g):
    d, I = g["shape"]["d"], g["shape"]["I"]
    w = {"w1": np.zeros((I, d)), "w3": np.zeros((I, d)), "w2": np.zeros((d, I))}
    for name, entries in g["weights"].items():
        if name in w:
            for key, v in entries.items():
                r, c = (int(t) for t in key.split(","))
                w[name][r, c] = v
    return w


def check_worked_mxfp8_ffn(orc):
    """One MXFP8 expert derived by hand: exact weights, x exact or rounded, h rounded."""
    g = load_golden("worked_example_mxfp8_ffn.json")
    d = g["shape"]["d"]
    w = _golden_mxfp8_weights(g)
    for case in g["cases"]:
        x = np.zeros((1, d))
        x[0, 0] = case["x0"]
        y, h = orc.expert_ffn_mxfp8(x, w["w1"], w["w3"], w["w2"])
        want_y = np.zeros(d)
        want_y[:2] = case["expected_y"]
        np.testing.assert_allclose(h[0, :2], case["expected_h"], rtol=0, atol=1e-14,
                                   err_msg=case["name"])
        assert (h[0, 2:] == 0).all()
        np.testing.assert_allclose(y[0], want_y, rtol=0, atol=1e-14, err_msg=case["name"])


def brute_force_mx_quantize(a):
    """MXFP8 of a [m, K] array along its rows by exhaustive search: for each block
    of 32 values the scale 2^s with s found by counting up to the first integer
    with amax <= 448 * 2^s, and each scaled value by a search over all 127
    non-negative E4M3 codes (nearest, ties to the even code).  Returns the
    dequantised values."""
    t = np.array(e4m3_table_cache()[:0x7F])
    even = (np.arange(0x7F) % 2) == 0
    a = np.asarray(a, dtype=np.float64)
    out = np.zeros_like(a)
    m, K = a.shape
    for r in range(m):
        for b0 in range(0, K, 32):
            blk = a[r, b0:b0 + 32]
            amax = np.abs(blk).max()
            s = 0
            if amax > 0:
                s = -160
                while 448.0 * 2.0 ** s < amax:
                    s += 1
            mag = np.minimum(np.abs(blk) / 2.0 ** s, 448.0)
            dist = np.abs(t[None, :] - mag[:, None])
            best = dist == dist.min(axis=1, keepdims=True)
            pick = np.where((best & even).any(axis=1), np.argmax(best & even, axis=1),
                            np.argmax(best, axis=1))
            out[r, b0:b0 + 32] = np.where(np.signbit(blk), -t[pick], t[pick]) * 2.0 ** s
    return out


def check_mxfp8_ffn_brute_force(orc, seed=13):
    """The MXFP8 expert against a plain restatement built on the exhaustive
    quantiser above: x, W1, W3 quantised along d, h = SiLU(a) u along I, W2
    along I, products in float64.  32 token rows, so h also has whole blocks
    along the token axis and a quantiser applied along the wrong axis differs."""
    rng = np.random.default_rng(seed)
    m, d, I = 32, 64, 32
    x = rng.normal(size=(m, d)) * np.exp(rng.normal(size=(m, 1)))
    w1 = rng.normal(size=(I, d)) * 0.2
    w3 = rng.normal(size=(I, d)) * 0.2
    w2 = rng.normal(size=(d, I)) * 0.2
    xq = brute_force_mx_quantize(x)
    a = xq @ brute_force_mx_quantize(w1).T
    u = xq @ brute_force_mx_quantize(w3).T
    h = np.array([[ai / (1.0 + math.exp(-ai)) for ai in row] for row in a]) * u
    want = brute_force_mx_quantize(h) @ brute_force_mx_quantize(w2).T
    y, h_got = orc.expert_ffn_mxfp8(x, w1, w3, w2)
    np.testing.assert_allclose(h_got, h, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-13)


def check_worked_bias_trajectory(orc):
    """Three closed-loop steps of Eq. (2) derived by hand (route with b_s, then update)."""
    g = load_golden("worked_example_bias_trajectory.json")
    sh = g["shape"]
    E = sh["N"] + sh["Z"]
    logits = np.log(np.array(g["router_probs"]))

    def route_inputs(s):
        return np.zeros((sh["T"], 1)), logits

    steps = len(g["expected_steps"])
    hist, b = orc.bias_control_trajectory(steps, route_inputs, np.zeros((E, 1)),
                                          np.array(g["bias0"]), sh["N"], sh["K"], g["K_e"],
                                          g["mu"])
    assert len(hist) == steps
    for s, (got, want) in enumerate(zip(hist, g["expected_steps"])):
        np.testing.assert_allclose(got["bias"], want["bias"], rtol=0, atol=1e-15,
                                   err_msg=f"bias used by step {s}")
        np.testing.assert_array_equal(got["counts"], want["counts"], err_msg=f"step {s}")
        for key in ("n_ffn_mean", "n_ffn_std", "max_over_mean_load", "min_margin"):
            np.testing.assert_allclose(got[key], want[key], rtol=0, atol=1e-12,
                                       err_msg=f"{key} at step {s}")
        assert (got["bias"][sh["N"]:] == 0).all()
    np.testing.assert_allclose(b, g["expected_final_bias"], rtol=0, atol=1e-15)


def _loss_and_grads(orc, L, N, K, gamma, dout):
    r = orc.moe_layer_backward(L["x"], L["w_router"], L["w1"], L["w3"], L["w2"], L["bias"],
                               N=N, K=K, dout=dout, gamma=gamma)
    return r


def check_backward_finite_differences(orc, seed=10):
    """Central differences of L = <dout, out> in float64 against every gradient
    (inputs drawn so that no small step changes the top-K selection)."""
    rng = np.random.default_rng(seed)
    T, d, N, Z, K, I, gamma = 5, 4, 3, 2, 3, 3, 1.5
    L = _rand_layer(rng, T, d, N, Z, I, 0.2)
    dout = rng.normal(size=(T, d))
    r = _loss_and_grads(orc, L, N, K, gamma, dout)
    assert r["margin"].min() > 1e-4

    def loss(LL):
        o = orc.moe_layer(LL["x"], LL["w_router"], LL["w1"], LL["w3"], LL["w2"], LL["bias"],
                          N=N, K=K, gamma=gamma)["out"]
        return float((o * dout).sum())
    eps = 1e-6
    for name, grad in (("x", "dx"), ("w_router", "dw_router"), ("w1", "dw1"), ("w3", "dw3"),
                       ("w2", "dw2")):
        base = L[name]
        fd = np.zeros_like(base)
        for ix in np.ndindex(base.shape):
            Lp = dict(L); Lm = dict(L)
            Lp[name] = base.copy(); Lp[name][ix] += eps
            Lm[name] = base.copy(); Lm[name][ix] -= eps
            fd[ix] = (loss(Lp) - loss(Lm)) / (2 * eps)
        np.testing.assert_allclose(r[grad], fd, rtol=1e-5, atol=1e-7, err_msg=name)


def check_backward_against_autograd(orc, seed=11):
    """The dense top-K MoE written with torch float64 ops, differentiated by
    torch autograd, against the oracle's hand-written backward."""
    rng = np.random.default_rng(seed)
    T, d, N, Z, K, I, gamma = 9, 6, 5, 3, 4, 7, 0.7
    L = _rand_layer(rng, T, d, N, Z, I, 0.1)
    dout = rng.normal(size=(T, d))
    r = _loss_and_grads(orc, L, N, K, gamma, dout)
    tens = {k: torch.tensor(L[k], dtype=torch.float64, requires_grad=True)
            for k in ("x", "w_router", "w1", "w3", "w2")}
    F = torch.nn.functional
    p = torch.softmax(F.linear(tens["x"], tens["w_router"]), dim=1)
    s_ = p.detach() + torch.tensor(L["bias"])[None, :]
    out = torch.zeros_like(tens["x"])
    rows = []
    for t in range(T):
        chosen = sorted(range(N + Z), key=lambda i: (-float(s_[t, i]), i))[:K]
        acc = torch.zeros(d, dtype=torch.float64)
        for i in chosen:
            if i < N:
                y = F.linear(F.silu(F.linear(tens["x"][t], tens["w1"][i])) *
                             F.linear(tens["x"][t], tens["w3"][i]), tens["w2"][i])
            else:
                y = tens["x"][t]
            acc = acc + p[t, i] * y
        rows.append(gamma * acc)
    out = torch.stack(rows)
    (out * torch.tensor(dout)).sum().backward()
    for name, grad in (("x", "dx"), ("w_router", "dw_router"), ("w1", "dw1"), ("w3", "dw3"),
                       ("w2", "dw2")):
        np.testing.assert_allclose(r[grad], tens[name].grad.numpy(), rtol=1e-10, atol=1e-12,
                                   err_msg=name)


def check_lb_backward_finite_differences(orc, seed=12):
    """With the load-balance loss: central differences of
    <dout, out> + alpha sum_j f_j P_j (f from the selection, which no small step
    changes) against dx and dW_r; the expert weights do not enter L_LB."""
    rng = np.random.default_rng(seed)
    T, d, N, Z, K, I, gamma = 6, 4, 4, 2, 3, 3, 1.0
    D, K_e, alpha = 2, 2.0, 0.7
    L = _rand_layer(rng, T, d, N, Z, I, 0.2)
    dout = rng.normal(size=(T, d))
    r = orc.moe_layer_backward(L["x"], L["w_router"], L["w1"], L["w3"], L["w2"], L["bias"],
                               N=N, K=K, dout=dout, gamma=gamma, lb=(D, K_e, alpha))
    assert r["margin"].min() > 1e-4
    base = orc.moe_layer_backward(L["x"], L["w_router"], L["w1"], L["w3"], L["w2"],
                                  L["bias"], N=N, K=K, dout=dout, gamma=gamma)
    # the aux loss moves the router's gradients and leaves the expert weights' alone
    assert not np.allclose(r["dw_router"], base["dw_router"])
    np.testing.assert_array_equal(r["dw1"], base["dw1"])

    def total(LL):
        f = orc.moe_layer(LL["x"], LL["w_router"], LL["w1"], LL["w3"], LL["w2"], LL["bias"],
                          N=N, K=K, gamma=gamma)
        lf, lP = orc.lb_statistics(f["probs"], f["idx"], N, D, K, K_e)
        return float((f["out"] * dout).sum()) + orc.lb_loss(lf, lP, alpha)
    eps = 1e-6
    for name, grad in (("x", "dx"), ("w_router", "dw_router")):
        b0 = L[name]
        fd = np.zeros_like(b0)
        for ix in np.ndindex(b0.shape):
            Lp = dict(L); Lm = dict(L)
            Lp[name] = b0.copy(); Lp[name][ix] += eps
            Lm[name] = b0.copy(); Lm[name][ix] -= eps
            fd[ix] = (total(Lp) - total(Lm)) / (2 * eps)
        np.testing.assert_allclose(r[grad], fd, rtol=1e-5, atol=1e-7, err_msg=name)


ALL_CHECKS = [check_worked_mxfp8_ffn, check_mxfp8_ffn_brute_force,
              check_worked_bias_trajectory, check_lb_backward_finite_differences, check_backward_finite_differences, check_backward_against_autograd, check_e4m3_table, check_e4m3_rounding_brute_force,
              check_mxfp8_block_quantization, check_worked_tiny_layer, check_worked_swiglu, check_worked_bias_update,
              check_worked_zero_experts, check_softmax_closed_forms, check_topk_brute_force,
              check_dense_reduction, check_all_zero_experts_fixed_point,
              check_k_equals_e_fixed_point, check_permutation_invariants,
              check_bias_update_closed_form, check_bf16_decode, check_worked_lb_statistics,
              check_lb_statistics_closed_forms]
