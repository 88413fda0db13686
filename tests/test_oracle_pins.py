"""Pins of the float64 oracle to facts that do not come from the oracle itself.

Each test checks ``oracle.ref`` against something the pages or plain
mathematics fix: a hand-worked example, closed forms, invariants of the delta
rule, special cases that reduce to simpler recurrences, and a brute force built
from a different view of the operator (products of per-token DPLR transitions).
``test_planted_mistakes_are_caught`` shows that a set of plausible mistakes in
a recurrence of this kind each fail at least one of these pins.
"""
import json
import os

import numpy as np
import pytest

from oracle import brute, chunk_mirror, epilogue, prologue, ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_problem(seed, T, H, dk, dv, N=1, s0=0.5, cu=None):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, H, dk))
    k = rng.standard_normal((T, H, dk))
    v = rng.standard_normal((T, H, dv))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, H))))
    z = rng.standard_normal((T, H, dk))
    A = rng.standard_normal(H)
    S0 = None if s0 is None else rng.standard_normal((N, H, dk, dv)) * s0
    return dict(q=q, k=k, v=v, beta=beta, z=z, A=A, S0=S0, cu=cu)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


# ----------------------------------------------------------------- golden ---

def test_hand_worked_two_tokens():
    """Kimi Linear summary §3: decay first, then delta correction, o from S_t."""
    d = json.load(open(os.path.join(GOLDEN, "kda_hand_two_tokens.json")))
    q = np.array(d["q"])[:, None, :]
    k = np.array(d["k"])[:, None, :]
    v = np.array(d["v"])[:, None, :]
    beta = np.array(d["beta"])[:, None]
    g = np.log(np.array(d["alpha"]))[:, None, :]
    S0 = np.array(d["S0"])[None, None]
    o, Sf, St = ref.forward(q, k, v, beta, g=g, S0=S0, trace=True)
    tol = d["tolerance_abs"]
    np.testing.assert_allclose(o[:, 0], d["expected_o"], atol=tol, rtol=0)
    np.testing.assert_allclose(St[0, 0], d["expected_S1"], atol=tol, rtol=0)
    np.testing.assert_allclose(St[1, 0], d["expected_S2"], atol=tol, rtol=0)
    np.testing.assert_allclose(Sf[0, 0], d["expected_S2"], atol=tol, rtol=0)


def test_gate_closed_values():
    """Kimi K3 architecture summary: g = -5 sigmoid(e^A z)."""
    d = json.load(open(os.path.join(GOLDEN, "kda_gate_values.json")))
    for c in d["cases"]:
        z = np.full((1, 1, 4), c["z"])
        g = ref.gate(z, np.array([c["A"]]))
        np.testing.assert_allclose(g, c["g"], atol=d["tolerance_abs"], rtol=0)


# ------------------------------------------------------------- brute force ---

@pytest.mark.parametrize("seed", [0, 1, 2])
def test_brute_force_transition_products(seed):
    """Kimi Linear summary §6.1/§6.2: materialised products of the DPLR
    transitions Diag(a) - b k k^T Diag(a) give the same o and S_final."""
    cu = np.array([0, 9, 9, 23, 30])
    p = _rand_problem(seed, 30, 2, 6, 5, N=4, cu=cu)
    o, Sf = ref.forward(p["q"], p["k"], p["v"], p["beta"], z=p["z"], A=p["A"],
                        S0=p["S0"], cu_seqlens=cu)
    ob, Sb = brute.forward(p["q"], p["k"], p["v"], p["beta"], z=p["z"], A=p["A"],
                           S0=p["S0"], cu_seqlens=cu)
    assert np.abs(o - ob).max() < 1e-12
    assert np.abs(Sf - Sb).max() < 1e-12


def test_state_trace_matches_brute_force_prefixes():
    """The state after token t (what intermediate-state checkpoints store) is the
    final state of the sequence cut after t, here from the transition-product
    view, for every t of two packed sequences."""
    cu = np.array([0, 7, 16])
    p = _rand_problem(3, 16, 2, 5, 4, N=2, cu=cu)
    _, _, St = ref.forward(p["q"], p["k"], p["v"], p["beta"], z=p["z"], A=p["A"],
                           S0=p["S0"], cu_seqlens=cu, trace=True)
    for n in range(2):
        for t in range(cu[n], cu[n + 1]):
            sl = slice(cu[n], t + 1)
            _, Sb = brute.forward(p["q"][sl], p["k"][sl], p["v"][sl], p["beta"][sl],
                                  z=p["z"][sl], A=p["A"], S0=p["S0"][n:n + 1],
                                  cu_seqlens=np.array([0, t + 1 - cu[n]]))
            assert np.abs(St[t] - Sb[0]).max() < 1e-12


def test_brute_force_attention_matrix_is_causal():
    p = _rand_problem(5, 12, 1, 4, 3)
    g = brute.lower_bounded_gate(p["z"], p["A"])
    _, _, attn = brute.single_head(p["q"][:, 0], p["k"][:, 0], p["v"][:, 0], g[:, 0],
                                   p["beta"][:, 0])
    assert np.all(np.triu(attn, 1) == 0.0)
    assert np.all(np.abs(np.diag(attn)) > 0.0)


# ------------------------------------------------------------ closed forms ---

def test_beta_zero_is_pure_channel_decay():
    """beta = 0 switches off erase and write: S_t = Diag(e^{G_t}) S0 with G_t the
    sequence-level cumulative log-decay; o_t = S_t^T q^_t."""
    p = _rand_problem(3, 40, 2, 8, 7, N=1)
    beta = np.zeros_like(p["beta"])
    o, Sf = ref.forward(p["q"], p["k"], p["v"], beta, z=p["z"], A=p["A"], S0=p["S0"])
    g = brute.lower_bounded_gate(p["z"], p["A"])
    G = np.cumsum(g, axis=0)  # [T,H,dk]
    qh = p["q"] / np.sqrt(np.sum(p["q"] ** 2, -1, keepdims=True) + 1e-6)
    St = np.exp(G)[..., None] * p["S0"][0][None]  # [T,H,dk,dv]
    o_cf = np.einsum("thkv,thk->thv", St, qh)
    assert np.abs(o - o_cf).max() < 1e-12
    assert np.abs(Sf[0] - St[-1]).max() < 1e-12


@pytest.mark.parametrize("decay", [False, True])
def test_orthonormal_keys_reduce_to_linear_attention(decay):
    """Distinct basis keys, S0 = 0: the erase term only meets rows that are still
    zero, so KDA is channel-decayed linear attention; with g = 0, beta = 1 it is
    plain causal linear attention o_t = sum_{i<=t} (q_t . k_i) v_i."""
    rng = np.random.default_rng(11)
    T, dk, dv = 10, 12, 5
    perm = rng.permutation(dk)[:T]
    k = np.eye(dk)[perm][:, None, :]
    q = _unit(rng.standard_normal((T, 1, dk)))
    v = rng.standard_normal((T, 1, dv))
    if decay:
        g = -5.0 * rng.random((T, 1, dk))
        beta = rng.random((T, 1))
    else:
        g = np.zeros((T, 1, dk))
        beta = np.ones((T, 1))
    o, _ = ref.forward(q, k, v, beta, g=g)
    G = np.cumsum(g[:, 0], axis=0)
    c = 1.0 / np.sqrt(1.0 + 1e-6)  # a basis key after the operator's normalisation
    qh = q[:, 0] / np.sqrt(np.sum(q[:, 0] ** 2, -1, keepdims=True) + 1e-6)
    o_la = np.zeros((T, dv))
    for t in range(T):
        for i in range(t + 1):
            w = beta[i, 0] * np.sum(qh[t] * np.exp(G[t] - G[i]) * k[i, 0] * c)
            o_la[t] += w * v[i, 0]
    assert np.abs(o[:, 0] - o_la).max() < 1e-12


def test_single_token_from_zero_state():
    """S_1 = beta k^ v^T and o_1 = beta (q^ . k^) v for S0 = 0."""
    p = _rand_problem(4, 1, 3, 8, 6, s0=None)
    o, Sf = ref.forward(p["q"], p["k"], p["v"], p["beta"], z=p["z"], A=p["A"])
    n = lambda x: x / np.sqrt(np.sum(x * x, -1, keepdims=True) + 1e-6)
    qh, kh = n(p["q"][0]), n(p["k"][0])
    for h in range(3):
        b = p["beta"][0, h]
        np.testing.assert_allclose(Sf[0, h], b * np.outer(kh[h], p["v"][0, h]), atol=1e-14)
        np.testing.assert_allclose(o[0, h], b * (qh[h] @ kh[h]) * p["v"][0, h], atol=1e-14)


# -------------------------------------------------------------- invariants ---

def _trace_problem(seed=7, T=25, H=2, dk=8, dv=6):
    p = _rand_problem(seed, T, H, dk, dv)
    o, Sf, St = ref.forward(p["q"], p["k"], p["v"], p["beta"], z=p["z"], A=p["A"],
                            S0=p["S0"], trace=True)
    g = brute.lower_bounded_gate(p["z"], p["A"])
    kh = p["k"] / np.sqrt(np.sum(p["k"] ** 2, -1, keepdims=True) + 1e-6)
    prev = np.concatenate([p["S0"], St[:-1]], axis=0)  # S_{t-1} [T,H,dk,dv]
    Sp = np.exp(g)[..., None] * prev                    # Diag(alpha_t) S_{t-1}
    return p, St, Sp, kh, prev


def test_delta_rule_invariant():
    """S_t^T k_t = (1 - b|k|^2) (Diag(a)S_{t-1})^T k_t + b|k|^2 v_t."""
    p, St, Sp, kh, _ = _trace_problem()
    kk = np.sum(kh * kh, -1)[..., None]
    lhs = np.einsum("thkv,thk->thv", St, kh)
    rhs = (1 - p["beta"][..., None] * kk) * np.einsum("thkv,thk->thv", Sp, kh) \
        + p["beta"][..., None] * kk * p["v"]
    assert np.abs(lhs - rhs).max() < 1e-12


def test_online_gradient_step_form():
    """Kimi Linear summary §2.2: DeltaNet is online gradient descent on
    1/2 |S^T k - v|^2, i.e. S_t = S' - b k (S'^T k - v)^T with S' the decayed state."""
    p, St, Sp, kh, _ = _trace_problem(seed=8)
    grad = np.einsum("thk,thv->thkv", kh,
                     np.einsum("thkv,thk->thv", Sp, kh) - p["v"])
    S_gd = Sp - p["beta"][..., None, None] * grad
    assert np.abs(St - S_gd).max() < 1e-12


def test_deltanet_special_case_stores_value_exactly():
    """alpha = 1 (g = 0) and beta = 1: the stored association is exact,
    S_t^T k^_t = |k^|^2 v_t + (1-|k^|^2)(...) -> v_t up to the 1e-6 epsilon."""
    p = _rand_problem(9, 20, 2, 8, 5)
    g = np.zeros_like(p["z"])
    beta = np.ones_like(p["beta"])
    _, _, St = ref.forward(p["q"], p["k"], p["v"], beta, g=g, S0=p["S0"], trace=True)
    kh = p["k"] / np.sqrt(np.sum(p["k"] ** 2, -1, keepdims=True) + 1e-6)
    got = np.einsum("thkv,thk->thv", St, kh)
    assert np.abs(got - p["v"]).max() < 1e-5


def test_scalar_gate_factorises_like_gated_deltanet():
    """Kimi Linear summary §2.2: with one gate per head (GDN), the decay commutes
    with the delta step, so S_t = c_t * S~_t where S~ is DeltaNet (alpha = 1)
    run on v_t / c_t, c_t = prod_{s<=t} alpha_s (S0 = 0)."""
    rng = np.random.default_rng(12)
    T, H, dk, dv = 18, 2, 6, 4
    p = _rand_problem(12, T, H, dk, dv, s0=None)
    gs = -0.3 * rng.random((T, H))
    g = np.repeat(gs[..., None], dk, axis=-1)
    o, Sf = ref.forward(p["q"], p["k"], p["v"], p["beta"], g=g)
    c = np.exp(np.cumsum(gs, axis=0))  # [T,H]
    o2, Sf2 = ref.forward(p["q"], p["k"], p["v"] / c[..., None], p["beta"], g=np.zeros_like(g))
    assert np.abs(o - c[..., None] * o2).max() < 1e-12
    assert np.abs(Sf[0] - c[-1][:, None, None] * Sf2[0]).max() < 1e-12


def test_non_expansive():
    """|(I - b k k^T) Diag(a)|_2 <= 1 for b in [0,1], a in (0,1], unit k:
    |S_t|_F <= |S_{t-1}|_F + b |v_t|."""
    p, St, _, _, prev = _trace_problem(seed=10, T=40)
    lhs = np.linalg.norm(St.reshape(*St.shape[:2], -1), axis=-1)
    rhs = np.linalg.norm(prev.reshape(*prev.shape[:2], -1), axis=-1) \
        + p["beta"] * np.linalg.norm(p["v"], axis=-1)
    assert np.all(lhs <= rhs + 1e-12)


def test_gate_bounds_and_tile_range():
    """g in [-5, 0]; the 16-token partial sums stay in [-80, 0] (Kimi K3
    architecture summary: range argument for the 16-token tiles)."""
    rng = np.random.default_rng(13)
    z = rng.standard_normal((256, 4, 32)) * 4
    A = rng.standard_normal(4) * 2
    g = ref.gate(z, A)
    assert g.min() >= -5.0 and g.max() <= 0.0
    tiles = g.reshape(16, 16, 4, 32).sum(axis=1)
    assert tiles.min() >= -80.0 and tiles.max() <= 0.0


def test_gate_entry_matches_gate_inputs():
    p = _rand_problem(14, 33, 2, 8, 8)
    o1, S1 = ref.forward(p["q"], p["k"], p["v"], p["beta"], z=p["z"], A=p["A"], S0=p["S0"])
    o2, S2 = ref.forward(p["q"], p["k"], p["v"], p["beta"], g=ref.gate(p["z"], p["A"]),
                         S0=p["S0"])
    assert np.array_equal(o1, o2) and np.array_equal(S1, S2)


def test_normalisation_scale_invariance():
    """q and k enter only through their unit directions (Kimi Linear summary §4)."""
    p = _rand_problem(15, 20, 2, 8, 4)
    rng = np.random.default_rng(16)
    sq = rng.uniform(0.5, 3.0, (20, 2, 1))
    sk = rng.uniform(0.5, 3.0, (20, 2, 1))
    o1, S1 = ref.forward(p["q"], p["k"], p["v"], p["beta"], z=p["z"], A=p["A"], S0=p["S0"])
    o2, S2 = ref.forward(p["q"] * sq, p["k"] * sk, p["v"], p["beta"], z=p["z"], A=p["A"],
                         S0=p["S0"])
    assert np.abs(o1 - o2).max() < 1e-5 and np.abs(S1 - S2).max() < 1e-5


# --------------------------------------------------- structure / plumbing ---

def test_state_passing_equals_one_call():
    p = _rand_problem(17, 30, 2, 8, 6)
    o, Sf = ref.forward(p["q"], p["k"], p["v"], p["beta"], z=p["z"], A=p["A"], S0=p["S0"])
    o1, S1 = ref.forward(p["q"][:13], p["k"][:13], p["v"][:13], p["beta"][:13],
                         z=p["z"][:13], A=p["A"], S0=p["S0"])
    o2, S2 = ref.forward(p["q"][13:], p["k"][13:], p["v"][13:], p["beta"][13:],
                         z=p["z"][13:], A=p["A"], S0=S1)
    assert np.abs(np.concatenate([o1, o2]) - o).max() < 1e-14
    assert np.abs(S2 - Sf).max() < 1e-14


def test_decode_steps_equal_forward():
    p = _rand_problem(18, 6, 3, 8, 6, N=1)
    o, Sf = ref.forward(p["q"], p["k"], p["v"], p["beta"], z=p["z"], A=p["A"], S0=p["S0"])
    S = p["S0"]
    for t in range(6):
        ot, S = ref.decode_step(p["q"][t:t + 1], p["k"][t:t + 1], p["v"][t:t + 1],
                                p["beta"][t:t + 1], S, z=p["z"][t:t + 1], A=p["A"])
        assert np.abs(ot[0] - o[t]).max() < 1e-14
    assert np.abs(S - Sf).max() < 1e-14


def test_empty_sequence_keeps_state():
    p = _rand_problem(19, 10, 2, 4, 4, N=3)
    cu = np.array([0, 0, 10, 10])
    _, Sf = ref.forward(p["q"], p["k"], p["v"], p["beta"], z=p["z"], A=p["A"], S0=p["S0"],
                        cu_seqlens=cu)
    assert np.array_equal(Sf[0], p["S0"][0]) and np.array_equal(Sf[2], p["S0"][2])


def test_invalid_arguments_rejected():
    p = _rand_problem(20, 10, 1, 4, 4, N=2)
    with pytest.raises(ValueError):
        ref.forward(p["q"], p["k"], p["v"], p["beta"], z=p["z"], A=p["A"], S0=p["S0"],
                    cu_seqlens=np.array([0, 6, 5]))
    with pytest.raises(ValueError):
        ref.forward(p["q"], p["k"], p["v"], p["beta"], z=p["z"], A=p["A"], S0=p["S0"],
                    cu_seqlens=np.array([0, 6, 9]))


# ------------------------------------------------------------ chunk mirror ---

@pytest.mark.parametrize("chunk", [16, 64])
def test_chunk_mirror_matches_oracle(chunk):
    """The derived chunkwise algebra (WY/UT, sub-tile references, blocked
    forward substitution) reproduces the sequential recurrence."""
    cu = np.array([0, 70, 70, 75, 150])
    p = _rand_problem(21, 150, 2, 8, 6, N=4, cu=cu)
    o, Sf = ref.forward(p["q"], p["k"], p["v"], p["beta"], z=p["z"], A=p["A"], S0=p["S0"],
                        cu_seqlens=cu)
    oc, Sc = chunk_mirror.forward(p["q"], p["k"], p["v"], p["beta"], z=p["z"], A=p["A"],
                                  S0=p["S0"], cu_seqlens=cu, chunk=chunk)
    assert np.abs(o - oc).max() < 1e-12
    assert np.abs(Sf - Sc).max() < 1e-12


def test_chunk_mirror_strong_decay_stays_finite():
    """g at the -5 floor everywhere: cumulative log-decay reaches -320 in a
    64-token chunk; the sub-tile references keep every factor finite."""
    p = _rand_problem(22, 128, 1, 8, 4)
    g = np.full_like(p["z"], -5.0)
    o, Sf = ref.forward(p["q"], p["k"], p["v"], p["beta"], g=g, S0=p["S0"])
    oc, Sc = chunk_mirror.forward(p["q"], p["k"], p["v"], p["beta"], g=g, S0=p["S0"], chunk=64)
    assert np.all(np.isfinite(oc))
    assert np.abs(o - oc).max() < 1e-12 and np.abs(Sf - Sc).max() < 1e-12


def test_unit_lower_inverse():
    rng = np.random.default_rng(23)
    L = np.tril(rng.standard_normal((64, 64)) * 0.2, -1)
    T = chunk_mirror.blocked_unit_lower_inverse(L)
    assert np.abs(T @ (np.eye(64) + L) - np.eye(64)).max() < 1e-12


# -------------------------------------------------------- pin sensitivity ---

def _planted(q, k, v, beta, g, S0, mistake):
    """A small sequential KDA with one planted mistake (CPU only)."""
    T, H, dk = q.shape
    n = lambda x: x / np.sqrt(np.sum(x * x) + 1e-6)
    o = np.zeros((T, H, v.shape[-1]))
    Sf = np.zeros_like(S0)
    for h in range(H):
        S = S0[0, h].copy()
        for t in range(T):
            kh = k[t, h] if mistake == "no_norm" else n(k[t, h])
            qh = n(q[t, h])
            a = np.exp(-g[t, h] if mistake == "gate_sign" else g[t, h])
            b = beta[t, h]
            S_prev = S.copy()
            if mistake == "decay_on_value_axis":  # needs dk == dv
                Sd = S * a[None, :]
            else:
                Sd = a[:, None] * S
            if mistake == "delta_first":
                S = S - b * np.outer(kh, kh @ S)
                S = a[:, None] * S + b * np.outer(kh, v[t, h])
            else:
                w = 1.0 if mistake == "no_beta_write" else b
                S = Sd - b * np.outer(kh, kh @ Sd) + w * np.outer(kh, v[t, h])
            Sout = S_prev if mistake == "o_from_previous" else S
            o[t, h] = Sout.T @ qh
        Sf[0, h] = S
    return o, Sf


@pytest.mark.parametrize("mistake", ["delta_first", "o_from_previous", "no_beta_write",
                                     "gate_sign", "no_norm", "decay_on_value_axis"])
def test_planted_mistakes_are_caught(mistake):
    d = json.load(open(os.path.join(GOLDEN, "kda_hand_two_tokens.json")))
    q = np.array(d["q"])[:, None, :]
    k = np.array(d["k"])[:, None, :]
    v = np.array(d["v"])[:, None, :]
    beta = np.array(d["beta"])[:, None]
    g = np.log(np.array(d["alpha"]))[:, None, :]
    S0 = np.array(d["S0"])[None, None]
    caught = False
    o, Sf = _planted(q, k, v, beta, g, S0, mistake)
    if np.abs(o[:, 0] - np.array(d["expected_o"])).max() > d["tolerance_abs"]:
        caught = True
    # a random problem against the brute force catches what the unit-vector
    # hand example cannot (e.g. a missing normalisation)
    p = _rand_problem(24, 8, 1, 4, 4)
    gg = brute.lower_bounded_gate(p["z"], p["A"])
    ob, Sb = brute.forward(p["q"], p["k"], p["v"], p["beta"], g=gg, S0=p["S0"])
    o2, S2 = _planted(p["q"], p["k"], p["v"], p["beta"], gg, p["S0"], mistake)
    if np.abs(o2 - ob).max() > 1e-9 or np.abs(S2 - Sb).max() > 1e-9:
        caught = True
    assert caught, f"planted mistake '{mistake}' passed every pin"
    # and the unmodified recurrence passes the same checks
    o3, S3 = _planted(p["q"], p["k"], p["v"], p["beta"], gg, p["S0"], None)
    assert np.abs(o3 - ob).max() < 1e-12 and np.abs(S3 - Sb).max() < 1e-12


# --------------------------------------------------------- output epilogue ---

def _golden_epilogue():
    with open(os.path.join(GOLDEN, "kda_output_norm_gate.json")) as f:
        return json.load(f)


def test_output_norm_gate_hand_worked():
    d = _golden_epilogue()
    o = np.array(d["o"])[None]           # [T=1, H=2, dv=4]
    y = epilogue.norm_gate(o, np.array(d["r"])[None], np.array(d["w"]), eps=d["eps"])
    assert np.abs(y[0] - np.array(d["expected_y"])).max() < d["tolerance_abs"]


def test_output_norm_gate_invariants():
    rng = np.random.default_rng(31)
    o = rng.standard_normal((5, 3, 16)) * rng.uniform(0.1, 10, (5, 3, 1))
    r = rng.standard_normal((5, 3, 16))
    y = epilogue.norm_gate(o, r, eps=0.0)
    # per-head scale invariance: each (token, head) row may carry its own scale
    c = rng.uniform(0.01, 100, (5, 3, 1))
    assert np.abs(epilogue.norm_gate(c * o, r, eps=0.0) - y).max() < 1e-12
    # a gate wide open and unit gain leave rows of unit root mean square
    y1 = epilogue.norm_gate(o, np.full_like(r, 60.0), eps=0.0)
    assert np.abs(np.sqrt(np.mean(y1 * y1, axis=-1)) - 1.0).max() < 1e-12
    # a closed gate zeroes the output; sigmoid(0) halves it
    assert np.abs(epilogue.norm_gate(o, np.full_like(r, -60.0), eps=0.0)).max() < 1e-20
    half = epilogue.norm_gate(o, np.zeros_like(r), eps=0.0)
    assert np.abs(2 * half - y1).max() < 1e-12
    # eps only matters against the row's mean square
    tiny = 1e-4 * o[:1, :1]
    assert np.abs(epilogue.norm_gate(tiny, r[:1, :1], eps=1.0) -
                  tiny / np.sqrt(np.mean(tiny ** 2) + 1.0) * epilogue.sigmoid(r[:1, :1])).max() < 1e-15


@pytest.mark.parametrize("mistake", ["sum", "no_sqrt", "swish", "both_heads", "no_gain",
                                     "gate_first", "one_minus"])
def test_output_epilogue_mistakes_are_caught(mistake):
    """Plausible mistakes in the epilogue, each restated here on the CPU, fail
    the hand-worked pin."""
    d = _golden_epilogue()
    o, r, w = np.array(d["o"]), np.array(d["r"]), np.array(d["w"])
    sig = epilogue.sigmoid
    ms = np.mean(o * o, axis=-1, keepdims=True)
    if mistake == "sum":
        y = o / np.sqrt(np.sum(o * o, axis=-1, keepdims=True)) * w * sig(r)
    elif mistake == "no_sqrt":
        y = o / ms * w * sig(r)
    elif mistake == "swish":
        y = o / np.sqrt(ms) * w * r * sig(r)
    elif mistake == "both_heads":
        y = o / np.sqrt(np.mean(o * o)) * w * sig(r)
    elif mistake == "no_gain":
        y = o / np.sqrt(ms) * sig(r)
    elif mistake == "gate_first":
        og = o * sig(r)
        y = og / np.sqrt(np.mean(og * og, axis=-1, keepdims=True)) * w
    else:
        y = o / np.sqrt(ms) * w * (1 - sig(r))
    assert np.abs(y - np.array(d["expected_y"])).max() > 1e-3


# ---------------------------------------------------------- input prologue ---

def _golden_prologue():
    with open(os.path.join(GOLDEN, "kda_short_conv_swish.json")) as f:
        return json.load(f)


def test_short_conv_swish_hand_worked():
    d = _golden_prologue()
    x, w, cu = np.array(d["x"]), np.array(d["w"]), np.array(d["cu_seqlens"])
    u = prologue.causal_conv(x, w, cu_seqlens=cu)
    assert np.abs(u - np.array(d["expected_u"])).max() < d["tolerance_abs"]
    y = prologue.short_conv_swish(x, w, cu_seqlens=cu)
    assert np.abs(y - np.array(d["expected_y"])).max() < d["tolerance_abs"]


def test_short_conv_matches_numpy_convolve():
    """Per sequence and channel the convolution is numpy's full convolution with
    the taps reversed, cut to the sequence length (a library routine)."""
    rng = np.random.default_rng(33)
    lens = [7, 0, 1, 3, 12]
    cu = np.concatenate([[0], np.cumsum(lens)])
    x = rng.standard_normal((cu[-1], 2, 5))
    w = rng.standard_normal((10, 4))
    u = prologue.causal_conv(x, w, cu_seqlens=cu).reshape(cu[-1], 10)
    xf = x.reshape(cu[-1], 10)
    for n in range(len(lens)):
        a, b = cu[n], cu[n + 1]
        if a == b:
            continue
        for c in range(10):
            want = np.convolve(xf[a:b, c], w[c, ::-1])[:b - a]
            assert np.abs(u[a:b, c] - want).max() < 1e-12


def test_short_conv_identity_filter_and_swish_values():
    rng = np.random.default_rng(34)
    x = rng.standard_normal((9, 3))
    w = np.zeros((3, 4))
    w[:, 3] = 1.0                      # only the current token
    y = prologue.short_conv_swish(x, w, num_seqs=1)
    assert np.abs(y - x / (1 + np.exp(-x))).max() < 1e-15
    assert prologue.swish(np.array([0.0]))[0] == 0.0
    assert abs(prologue.swish(np.array([40.0]))[0] - 40.0) < 1e-12
    assert abs(prologue.swish(np.array([-40.0]))[0]) < 1e-15


@pytest.mark.parametrize("mistake", ["flipped", "crosses_boundary", "anti_causal", "sigmoid",
                                     "no_swish"])
def test_short_conv_mistakes_are_caught(mistake):
    """Plausible mistakes in the prologue, restated here on the CPU, fail the
    hand-worked pin."""
    d = _golden_prologue()
    x, w, cu = np.array(d["x"]), np.array(d["w"]), np.array(d["cu_seqlens"])
    T, W = x.shape[0], w.shape[1]
    if mistake == "flipped":
        y = prologue.short_conv_swish(x, w[:, ::-1], cu_seqlens=cu)
    elif mistake == "crosses_boundary":
        y = prologue.short_conv_swish(x, w, num_seqs=1)
    elif mistake == "anti_causal":
        u = np.zeros_like(x)
        for t in range(T):
            for i in range(W):
                s = t + i
                if s < T:
                    u[t] += w[:, i] * x[s]
        y = prologue.swish(u)
    elif mistake == "sigmoid":
        y = 1 / (1 + np.exp(-prologue.causal_conv(x, w, cu_seqlens=cu)))
    else:
        y = prologue.causal_conv(x, w, cu_seqlens=cu)
    assert np.abs(y - np.array(d["expected_y"])).max() > 1e-3
