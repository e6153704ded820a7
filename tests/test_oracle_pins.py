"""Pins for the fp64 oracle (CPU only).

Each test checks the oracle against something that does not come from the
oracle itself: a hand-worked example, a closed form, a reduction to an older
rule written separately in matrix form, a brute-force operator product, an
invariant of the rule, or a second derivation (the chunkwise form).  Between
them a dropped term, a wrong sign, a swapped decay/erase order, a transposed
state or a read-before-write output each fail at least one test (see
``test_pins_catch_planted_mistakes``).
"""
import json
import os

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def rand_case(rng, B=1, T=12, H=2, dk=5, dv=3, mu=1.0, unit=True, init=True, beta_lo=0.0):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    if unit:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    beta = rng.uniform(beta_lo, 1.0, (B, T, H))
    la = -np.log1p(np.exp(-(rng.standard_normal((B, T, H, dk)) + mu)))  # logsigmoid
    s0 = rng.standard_normal((B, H, dk, dv)) if init else None
    return q, k, v, la, beta, s0


# ---- hand-worked example ---------------------------------------------------------------------

def test_hand_worked_example():
    """Two steps computed by hand (tests/golden/hand_worked_d2.json)."""
    with open(os.path.join(HERE, "golden", "hand_worked_d2.json")) as f:
        g = json.load(f)
    S = np.array(g["init_state"])[None, None]
    for st in g["steps"]:
        q = np.array(st["q"])[None, None]
        k = np.array(st["k"])[None, None]
        v = np.array(st["v"])[None, None]
        la = np.log(np.array(st["alpha"]))[None, None]
        b = np.array([[st["beta"]]])
        out, S = oracle.decode_step(q, k, v, la, b, S)
        np.testing.assert_allclose(S[0, 0], np.array(st["state"]), atol=1e-12, rtol=0)
        np.testing.assert_allclose(out[0, 0], np.array(st["out"]), atol=1e-12, rtol=0)


# ---- 1. alpha = 1 reduces to DeltaNet --------------------------------------------------------

def deltanet_matrix_form(q, k, v, beta, s0):
    """DeltaNet, written with the explicit d_k x d_k erase matrix (Stage 1 rule)."""
    T, dk = k.shape
    S = s0.copy()
    outs = []
    for t in range(T):
        E = np.eye(dk) - beta[t] * np.outer(k[t], k[t])
        S = E @ S + beta[t] * np.outer(k[t], v[t])
        outs.append(S.T @ q[t])
    return np.array(outs), S


def test_alpha_one_is_deltanet():
    rng = np.random.default_rng(1)
    q, k, v, la, beta, s0 = rand_case(rng, T=20, H=3, dk=6, dv=4)
    la[:] = 0.0
    out, fs = oracle.recurrent(q, k, v, la, beta, s0)
    for h in range(3):
        o_ref, s_ref = deltanet_matrix_form(q[0, :, h], k[0, :, h], v[0, :, h], beta[0, :, h], s0[0, h])
        np.testing.assert_allclose(out[0, :, h], o_ref, atol=1e-12, rtol=1e-12)
        np.testing.assert_allclose(fs[0, h], s_ref, atol=1e-12, rtol=1e-12)


def test_orthonormal_keys_replace_rows():
    """alpha = 1, beta = 1, k_t = e_{p(t)} distinct: S_T is S_0 with rows p(t) replaced by v_t."""
    rng = np.random.default_rng(2)
    dk, dv, T = 7, 3, 5
    perm = rng.permutation(dk)[:T]
    k = np.zeros((1, T, 1, dk))
    for t in range(T):
        k[0, t, 0, perm[t]] = 1.0
    v = rng.standard_normal((1, T, 1, dv))
    q = rng.standard_normal((1, T, 1, dk))
    s0 = rng.standard_normal((1, 1, dk, dv))
    _, fs = oracle.recurrent(q, k, v, np.zeros_like(k), np.ones((1, T, 1)), s0)
    expect = s0[0, 0].copy()
    for t in range(T):
        expect[perm[t]] = v[0, t, 0]
    np.testing.assert_allclose(fs[0, 0], expect, atol=1e-14, rtol=0)


# ---- 2. unit key with beta = 1 overwrites exactly ---------------------------------------------

def test_unit_key_exact_overwrite():
    rng = np.random.default_rng(3)
    q, k, v, la, beta, s0 = rand_case(rng, T=16, H=1, dk=8, dv=5, mu=0.0)
    S = s0[:, :, :, :]
    for t in range(16):
        _, S = oracle.decode_step(q[:, t], k[:, t], v[:, t], la[:, t], np.ones((1, 1)), S)
        recalled = S[0, 0].T @ k[0, t, 0]
        np.testing.assert_allclose(recalled, v[0, t, 0], atol=1e-13, rtol=0)


# ---- 3. brute-force unrolled operator product -------------------------------------------------

def test_bruteforce_operator_product():
    rng = np.random.default_rng(4)
    T, dk, dv = 14, 5, 3
    q, k, v, la, beta, s0 = rand_case(rng, T=T, H=1, dk=dk, dv=dv, mu=0.5)
    out, fs = oracle.recurrent(q, k, v, la, beta, s0)
    kk, vv, qq, bb = k[0, :, 0], v[0, :, 0], q[0, :, 0], beta[0, :, 0]
    M = [(np.eye(dk) - bb[t] * np.outer(kk[t], kk[t])) @ np.diag(np.exp(la[0, t, 0])) for t in range(T)]

    def prod(a, b):  # M_{b-1} ... M_a  (empty product = I)
        P = np.eye(dk)
        for t in range(a, b):
            P = M[t] @ P
        return P

    for t in range(T):
        St = prod(0, t + 1) @ s0[0, 0]
        for s in range(t + 1):
            St = St + prod(s + 1, t + 1) @ (bb[s] * np.outer(kk[s], vv[s]))
        np.testing.assert_allclose(out[0, t, 0], St.T @ qq[t], atol=1e-12, rtol=1e-12)
        if t == T - 1:
            np.testing.assert_allclose(fs[0, 0], St, atol=1e-12, rtol=1e-12)


# ---- 4. beta = 0: decay only -----------------------------------------------------------------

def test_beta_zero_closed_form():
    rng = np.random.default_rng(5)
    q, k, v, la, beta, s0 = rand_case(rng, T=9, H=2, dk=4, dv=6)
    beta[:] = 0.0
    out, fs = oracle.recurrent(q, k, v, la, beta, s0)
    for h in range(2):
        G = np.cumsum(la[0, :, h], axis=0)
        for t in range(9):
            St = np.exp(G[t])[:, None] * s0[0, h]
            np.testing.assert_allclose(out[0, t, h], St.T @ q[0, t, h], atol=1e-13, rtol=1e-12)
        np.testing.assert_allclose(fs[0, h], np.exp(G[-1])[:, None] * s0[0, h], atol=1e-13, rtol=1e-12)


# ---- 5. scalar gate = Gated DeltaNet ---------------------------------------------------------

def test_scalar_gate_is_gated_deltanet():
    rng = np.random.default_rng(6)
    q, k, v, la, beta, s0 = rand_case(rng, T=15, H=1, dk=6, dv=4)
    a = rng.uniform(0.3, 1.0, 15)
    la[0, :, 0, :] = np.log(a)[:, None]
    out, fs = oracle.recurrent(q, k, v, la, beta, s0)
    S = s0[0, 0].copy()
    for t in range(15):
        kt = k[0, t, 0]
        S = a[t] * (np.eye(6) - beta[0, t, 0] * np.outer(kt, kt)) @ S + beta[0, t, 0] * np.outer(kt, v[0, t, 0])
        np.testing.assert_allclose(out[0, t, 0], S.T @ q[0, t, 0], atol=1e-12, rtol=1e-12)
    np.testing.assert_allclose(fs[0, 0], S, atol=1e-12, rtol=1e-12)


def test_gdn_oracle_matches_matrix_forms():
    """The Gated DeltaNet / DeltaNet entry points against the Stage 2 and Stage 1 matrix forms,
    written here with the scalar outside the erase (g (I - b k k^T) S), over two heads and a
    packed pair of sequences."""
    rng = np.random.default_rng(61)
    q, k, v, _, beta, s0 = rand_case(rng, T=13, H=2, dk=5, dv=3)
    log_g = np.log(rng.uniform(0.2, 1.0, (1, 13, 2)))
    cu = np.array([0, 6, 13])
    s0 = rng.standard_normal((2, 2, 5, 3))
    for gate in (log_g, None):
        out, fs = oracle.gdn_recurrent(q, k, v, gate, beta, s0, cu_seqlens=cu)
        for n in range(2):
            for h in range(2):
                S = s0[n, h].copy()
                for t in range(cu[n], cu[n + 1]):
                    kt, g = k[0, t, h], 1.0 if gate is None else np.exp(gate[0, t, h])
                    S = g * (np.eye(5) - beta[0, t, h] * np.outer(kt, kt)) @ S + beta[0, t, h] * np.outer(kt, v[0, t, h])
                    np.testing.assert_allclose(out[0, t, h], S.T @ q[0, t, h], atol=1e-12, rtol=1e-12)
                np.testing.assert_allclose(fs[n, h], S, atol=1e-12, rtol=1e-12)
        # one decode step from the final state, the same form again
        qd, kd, vd = (rng.standard_normal((2, 2, d)) for d in (5, 5, 3))
        kd /= np.linalg.norm(kd, axis=-1, keepdims=True)
        bd = rng.uniform(0, 1, (2, 2))
        gd = None if gate is None else np.log(rng.uniform(0.2, 1.0, (2, 2)))
        od, Sd = oracle.gdn_decode_step(qd, kd, vd, gd, bd, fs)
        for n in range(2):
            for h in range(2):
                g = 1.0 if gd is None else np.exp(gd[n, h])
                S = g * (np.eye(5) - bd[n, h] * np.outer(kd[n, h], kd[n, h])) @ fs[n, h] + \
                    bd[n, h] * np.outer(kd[n, h], vd[n, h])
                np.testing.assert_allclose(Sd[n, h], S, atol=1e-12, rtol=1e-12)
                np.testing.assert_allclose(od[n, h], S.T @ qd[n, h], atol=1e-12, rtol=1e-12)


def test_prologue_closed_forms():
    """The raw-projection prologue: unit rows (up to the 1e-6 under the root), sigmoid(0) = 1/2,
    logsigmoid(0) = -log 2, logsigmoid = log(sigmoid) computed the other way, its asymptotes
    (x for x -> -inf, -exp(-x) for x -> +inf), and 1 - sigmoid(x) = sigmoid(-x)."""
    rng = np.random.default_rng(71)
    qr, kr = rng.standard_normal((2, 3, 4, 16)) * 5.0
    g = np.array([0.0, -40.0, 40.0, 3.0, -3.0])
    b = np.array([0.0, 2.0, -2.0, 30.0, -30.0])
    q, k, la, beta = oracle.prologue(qr, kr, g, b)
    for x, xr in ((q, qr), (k, kr)):
        n2 = np.sum(xr * xr, axis=-1)
        np.testing.assert_allclose(np.sum(x * x, axis=-1), n2 / (n2 + 1e-6), rtol=1e-14)
        np.testing.assert_allclose(x / np.linalg.norm(x, axis=-1, keepdims=True),
                                   xr / np.linalg.norm(xr, axis=-1, keepdims=True), rtol=1e-14)
    assert la[0] == -np.log(2.0) and beta[0] == 0.5
    np.testing.assert_allclose(la[3:], np.log(1.0 / (1.0 + np.exp(-g[3:]))), rtol=1e-14)
    np.testing.assert_allclose(la[1], -40.0, rtol=1e-15)            # logsigmoid(x) ~ x - exp(x)
    np.testing.assert_allclose(la[2], -np.exp(-40.0), rtol=1e-12)   # ~ -exp(-x)
    np.testing.assert_allclose(beta[1] + beta[2], 1.0, rtol=1e-15)
    np.testing.assert_allclose(beta[4], np.exp(-30.0) / (1 + np.exp(-30.0)), rtol=1e-12)
    # a zero row stays zero
    z = oracle.prologue(np.zeros((1, 4)), np.zeros((1, 4)), np.zeros(1), np.zeros(1))
    assert np.all(z[0] == 0.0) and np.all(z[1] == 0.0)


# ---- 6. linearity in (V, S_0) ----------------------------------------------------------------

def test_linearity_in_values_and_state():
    rng = np.random.default_rng(7)
    q, k, v1, la, beta, s1 = rand_case(rng, T=11, H=2, dk=5, dv=3)
    v2 = rng.standard_normal(v1.shape)
    s2 = rng.standard_normal(s1.shape)
    a, b = 0.7, -1.3
    o1, f1 = oracle.recurrent(q, k, v1, la, beta, s1)
    o2, f2 = oracle.recurrent(q, k, v2, la, beta, s2)
    o3, f3 = oracle.recurrent(q, k, a * v1 + b * v2, la, beta, a * s1 + b * s2)
    np.testing.assert_allclose(o3, a * o1 + b * o2, atol=1e-12, rtol=1e-12)
    np.testing.assert_allclose(f3, a * f1 + b * f2, atol=1e-12, rtol=1e-12)


# ---- 7. non-expansion ------------------------------------------------------------------------

def test_non_expansion():
    rng = np.random.default_rng(8)
    q, k, v, la, beta, s0 = rand_case(rng, T=40, H=1, dk=6, dv=4, mu=0.0)
    S = s0
    for t in range(40):
        prev = np.linalg.norm(S[0, 0])
        _, S = oracle.decode_step(q[:, t], k[:, t], v[:, t], la[:, t], beta[:, t], S)
        assert np.linalg.norm(S[0, 0]) <= prev + beta[0, t, 0] * np.linalg.norm(v[0, t, 0]) + 1e-12


# ---- 8. chunkwise derivation equals the recurrence -------------------------------------------

@pytest.mark.parametrize("C", [1, 2, 8, 16, 64])
def test_chunkwise_equals_recurrence(C):
    rng = np.random.default_rng(9)
    q, k, v, la, beta, s0 = rand_case(rng, B=2, T=150, H=2, dk=8, dv=6, mu=2.0)
    out, fs = oracle.recurrent(q, k, v, la, beta, s0)
    oc, fc = oracle.chunkwise(q, k, v, la, beta, s0, chunk_size=C)
    np.testing.assert_allclose(oc, out, atol=1e-11, rtol=0)
    np.testing.assert_allclose(fc, fs, atol=1e-11, rtol=0)


def test_chunkwise_varlen_equals_recurrence():
    rng = np.random.default_rng(10)
    lens = [1, 63, 64, 65, 130]
    cu = np.concatenate([[0], np.cumsum(lens)])
    q, k, v, la, beta, _ = rand_case(rng, B=1, T=int(cu[-1]), H=2, dk=8, dv=6, mu=2.0)
    s0 = rng.standard_normal((len(lens), 2, 8, 6))
    out, fs = oracle.recurrent(q, k, v, la, beta, s0, cu_seqlens=cu)
    oc, fc = oracle.chunkwise(q, k, v, la, beta, s0, cu_seqlens=cu, chunk_size=64)
    np.testing.assert_allclose(oc, out, atol=1e-11, rtol=0)
    np.testing.assert_allclose(fc, fs, atol=1e-11, rtol=0)


# ---- 9. composition --------------------------------------------------------------------------

def test_split_prefill_equals_whole():
    rng = np.random.default_rng(11)
    q, k, v, la, beta, s0 = rand_case(rng, T=50, H=2)
    out, fs = oracle.recurrent(q, k, v, la, beta, s0)
    o1, f1 = oracle.recurrent(q[:, :23], k[:, :23], v[:, :23], la[:, :23], beta[:, :23], s0)
    o2, f2 = oracle.recurrent(q[:, 23:], k[:, 23:], v[:, 23:], la[:, 23:], beta[:, 23:], f1)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=1), out, atol=1e-13, rtol=0)
    np.testing.assert_allclose(f2, fs, atol=1e-13, rtol=0)


def test_prefill_then_decode_equals_longer_prefill():
    rng = np.random.default_rng(12)
    q, k, v, la, beta, s0 = rand_case(rng, B=3, T=20, H=2)
    out, fs = oracle.recurrent(q, k, v, la, beta, s0)
    _, f19 = oracle.recurrent(q[:, :19], k[:, :19], v[:, :19], la[:, :19], beta[:, :19], s0)
    od, sd = oracle.decode_step(q[:, 19], k[:, 19], v[:, 19], la[:, 19], beta[:, 19], f19)
    np.testing.assert_allclose(od, out[:, 19], atol=1e-13, rtol=0)
    np.testing.assert_allclose(sd, fs, atol=1e-13, rtol=0)


def test_varlen_equals_per_sequence():
    rng = np.random.default_rng(13)
    lens = [5, 1, 17, 9]
    cu = np.concatenate([[0], np.cumsum(lens)])
    q, k, v, la, beta, _ = rand_case(rng, T=int(cu[-1]), H=2)
    s0 = rng.standard_normal((4, 2, 5, 3))
    out, fs = oracle.recurrent(q, k, v, la, beta, s0, cu_seqlens=cu)
    for n in range(4):
        a, b = cu[n], cu[n + 1]
        o, f = oracle.recurrent(q[:, a:b], k[:, a:b], v[:, a:b], la[:, a:b], beta[:, a:b], s0[n:n + 1])
        np.testing.assert_allclose(out[:, a:b], o, atol=1e-14, rtol=0)
        np.testing.assert_allclose(fs[n], f[0], atol=1e-14, rtol=0)


def test_threads_do_not_change_results():
    rng = np.random.default_rng(14)
    q, k, v, la, beta, s0 = rand_case(rng, B=2, T=33, H=5)
    o1, f1 = oracle.recurrent(q, k, v, la, beta, s0, nthreads=1)
    o4, f4 = oracle.recurrent(q, k, v, la, beta, s0, nthreads=4)
    assert np.array_equal(o1, o4) and np.array_equal(f1, f4)


def test_zero_length_sequences():
    """Empty sequences inside a packed batch keep their initial state and emit nothing."""
    rng = np.random.default_rng(15)
    cu = np.array([0, 0, 4, 4, 7])
    q, k, v, la, beta, _ = rand_case(rng, T=7, H=1)
    s0 = rng.standard_normal((4, 1, 5, 3))
    _, fs = oracle.recurrent(q, k, v, la, beta, s0, cu_seqlens=cu)
    np.testing.assert_array_equal(fs[0], s0[0])
    np.testing.assert_array_equal(fs[2], s0[2])


# ---- the pins fail on plausible mistakes -----------------------------------------------------
#
# The pins above are re-run as plain checks against an implementation passed in: the oracle
# passes all of them, and each plausible mistake (planted on the CPU in a copy of the rule,
# never in the oracle itself) fails at least one.

def _oracle_single(q, k, v, la, b, s0):
    out, fs = oracle.recurrent(q[None, :, None], k[None, :, None], v[None, :, None],
                               la[None, :, None], b[None, :, None], s0[None, None])
    return out[0, :, 0], fs[0, 0]


def _mutant(kind):
    def run(q, k, v, la, b, s0):
        S = s0.copy()
        outs = []
        for t in range(q.shape[0]):
            a = np.exp(la[t])
            if kind == "erase_then_decay":
                S = a[:, None] * (S - b[t] * np.outer(k[t], k[t]) @ S) + b[t] * np.outer(k[t], v[t])
            elif kind == "no_beta_on_write":
                Sd = a[:, None] * S
                S = Sd - b[t] * np.outer(k[t], k[t]) @ Sd + np.outer(k[t], v[t])
            elif kind == "read_before_write":
                Sd = a[:, None] * S
                outs.append(Sd.T @ q[t])
                S = Sd - b[t] * np.outer(k[t], k[t]) @ Sd + b[t] * np.outer(k[t], v[t])
                continue
            elif kind == "decay_on_value_side":
                Sd = S * a[None, : S.shape[1]]
                S = Sd - b[t] * np.outer(k[t], k[t]) @ Sd + b[t] * np.outer(k[t], v[t])
            elif kind == "erase_sign_flip":
                Sd = a[:, None] * S
                S = Sd + b[t] * np.outer(k[t], k[t]) @ Sd + b[t] * np.outer(k[t], v[t])
            elif kind == "decay_dropped":
                S = S - b[t] * np.outer(k[t], k[t]) @ S + b[t] * np.outer(k[t], v[t])
            outs.append(S.T @ q[t])
        return np.array(outs), S
    return run


def _check_bruteforce(impl, rng):
    T, dk, dv = 8, 5, 5
    q, k, v, la, beta, s0 = rand_case(rng, T=T, H=1, dk=dk, dv=dv, mu=0.5)
    q, k, v, la, beta, s0 = q[0, :, 0], k[0, :, 0], v[0, :, 0], la[0, :, 0], beta[0, :, 0], s0[0, 0]
    out, fs = impl(q, k, v, la, beta, s0)
    S = s0.copy()
    for t in range(T):
        M = (np.eye(dk) - beta[t] * np.outer(k[t], k[t])) @ np.diag(np.exp(la[t]))
        S = M @ S + beta[t] * np.outer(k[t], v[t])
        if not np.allclose(out[t], S.T @ q[t], atol=1e-10):
            return False
    return np.allclose(fs, S, atol=1e-10)


def _check_overwrite(impl, rng):
    q, k, v, la, beta, s0 = rand_case(rng, T=1, H=1, dk=6, dv=6, mu=0.0)
    _, fs = impl(q[0, :, 0], k[0, :, 0], v[0, :, 0], la[0, :, 0], np.ones(1), s0[0, 0])
    return np.allclose(fs.T @ k[0, 0, 0], v[0, 0, 0], atol=1e-12)


def _check_beta_zero(impl, rng):
    q, k, v, la, beta, s0 = rand_case(rng, T=6, H=1, dk=4, dv=4)
    out, fs = impl(q[0, :, 0], k[0, :, 0], v[0, :, 0], la[0, :, 0], np.zeros(6), s0[0, 0])
    G = np.cumsum(la[0, :, 0], axis=0)
    ok = np.allclose(fs, np.exp(G[-1])[:, None] * s0[0, 0], atol=1e-12)
    return ok and all(np.allclose(out[t], (np.exp(G[t])[:, None] * s0[0, 0]).T @ q[0, t, 0], atol=1e-12)
                      for t in range(6))


PIN_CHECKS = [_check_bruteforce, _check_overwrite, _check_beta_zero]


def test_oracle_passes_all_pin_checks():
    for chk in PIN_CHECKS:
        assert chk(_oracle_single, np.random.default_rng(16)), chk.__name__


@pytest.mark.parametrize("kind", ["erase_then_decay", "no_beta_on_write", "read_before_write",
                                  "decay_on_value_side", "erase_sign_flip", "decay_dropped"])
def test_pins_catch_planted_mistakes(kind):
    failed = [chk.__name__ for chk in PIN_CHECKS if not chk(_mutant(kind), np.random.default_rng(16))]
    assert failed, f"planted mistake {kind} passed every pin"
