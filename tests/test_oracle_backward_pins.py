"""Pins of the backward oracle (oracle.backward, the reverse-mode gradient of the token
recurrence), on CPU.  None of them reuses the oracle's arithmetic:

1. torch autograd of an independently written fp64 forward in the explicit matrix form
   S_t = (I - beta k k^T) Diag(alpha) S_{t-1} + beta k v^T, o_t = S_t^T q_t ("Hybrid Linear
   Attention Architectures: Breaking Through the Long-Context Engineering Bottleneck in LLMs",
   section "Core Module Design", Stage 3), with d_k x d_k operator matrices instead of the
   oracle's rank-1 updates;
2. central finite differences of the forward C oracle (oracle.recurrent);
3. the exact adjoint identity of the map (V, S_0) -> (O, S_T), which is linear for fixed q, k,
   alpha, beta: <dO, O> + <dS_T, S_T> = <dV, V> + <dS_0, S_0>;
4. planted mistakes: copies of the C oracle with one term of the backward changed must fail
   pin 1.
"""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest
import torch

import oracle

SHAPE_CASES = [
    dict(B=2, T=7, H=2, dk=5, dv=3, s0=True, dfin=True),
    dict(B=1, T=1, H=1, dk=4, dv=4, s0=False, dfin=False),
    dict(B=1, T=9, H=3, dk=3, dv=6, s0=True, dfin=False),
]


def rand_inputs(B, T, H, dk, dv, s0, dfin, seed=0, N=None):
    rng = np.random.default_rng(seed)
    N = B if N is None else N
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    la = np.log(rng.uniform(0.3, 1.0, (B, T, H, dk)))
    beta = rng.uniform(0.1, 1.0, (B, T, H))
    init = rng.standard_normal((N, H, dk, dv)) * 0.5 if s0 else None
    do = rng.standard_normal((B, T, H, dv))
    dfinal = rng.standard_normal((N, H, dk, dv)) if dfin else None
    return q, k, v, la, beta, init, do, dfinal


def torch_forward_matrix_form(q, k, v, la, beta, init, cu=None):
    """fp64 forward with explicit (I - beta k k^T) Diag(alpha) operators, differentiable."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    segs = [(b, 0, T) for b in range(B)] if cu is None else [(0, int(cu[n]), int(cu[n + 1])) for n in
                                                            range(len(cu) - 1)]
    outs = torch.zeros(B, T, H, dv, dtype=torch.float64)
    finals = []
    eye = torch.eye(dk, dtype=torch.float64)
    out_rows = {}
    for n, (b, t0, t1) in enumerate(segs):
        fin_h = []
        for h in range(H):
            S = init[n, h] if init is not None else torch.zeros(dk, dv, dtype=torch.float64)
            for t in range(t0, t1):
                kt = k[b, t, h]
                M = (eye - beta[b, t, h] * torch.outer(kt, kt)) @ torch.diag(torch.exp(la[b, t, h]))
                S = M @ S + beta[b, t, h] * torch.outer(kt, v[b, t, h])
                out_rows[(b, t, h)] = S.T @ q[b, t, h]
            fin_h.append(S)
        finals.append(torch.stack(fin_h))
    rows = [out_rows.get((b, t, h), torch.zeros(dv, dtype=torch.float64)) for b in range(B) for t in range(T)
            for h in range(H)]
    outs = torch.stack(rows).reshape(B, T, H, dv)
    return outs, torch.stack(finals)


def autograd_grads(q, k, v, la, beta, init, do, dfinal, cu=None):
    ts = [torch.tensor(x, requires_grad=True) for x in (q, k, v, la, beta)]
    s0 = torch.tensor(init, requires_grad=True) if init is not None else None
    out, fin = torch_forward_matrix_form(*ts, s0, cu)
    loss = (out * torch.tensor(do)).sum()
    if dfinal is not None:
        loss = loss + (fin * torch.tensor(dfinal)).sum()
    loss.backward()
    grads = [t.grad.numpy() for t in ts]
    grads.append(s0.grad.numpy() if s0 is not None else None)
    return grads


def assert_close(a, b, tol, name):
    scale = max(np.max(np.abs(b)), 1e-300)
    err = np.max(np.abs(a - b)) / scale
    assert err <= tol, f"{name}: {err:.3e}"


NAMES = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "d_init_state")


@pytest.mark.parametrize("case", SHAPE_CASES)
def test_backward_matches_autograd_of_matrix_form(case):
    q, k, v, la, beta, init, do, dfinal = rand_inputs(**case)
    got = oracle.backward(q, k, v, la, beta, do, init_state=init, d_final_state=dfinal)
    ref = autograd_grads(q, k, v, la, beta, init, do, dfinal)
    for name, g, r in zip(NAMES, got, ref):
        if r is None:
            continue
        assert_close(g, r, 1e-11, name)


def test_backward_matches_autograd_varlen():
    lens = [3, 0, 5, 1]
    cu = np.concatenate([[0], np.cumsum(lens)])
    q, k, v, la, beta, init, do, dfinal = rand_inputs(1, int(cu[-1]), 2, 4, 3, True, True, seed=3, N=len(lens))
    got = oracle.backward(q, k, v, la, beta, do, init_state=init, d_final_state=dfinal, cu_seqlens=cu)
    ref = autograd_grads(q, k, v, la, beta, init, do, dfinal, cu=cu)
    for name, g, r in zip(NAMES, got, ref):
        assert_close(g, r, 1e-11, name)
    # an empty sequence passes the gradient of its final state straight to its initial state
    assert np.array_equal(got[5][1], dfinal[1])


def test_backward_matches_central_differences():
    q, k, v, la, beta, init, do, dfinal = rand_inputs(B=1, T=4, H=1, dk=3, dv=2, s0=True, dfin=True, seed=7)
    args = [q, k, v, la, beta, init]
    got = oracle.backward(q, k, v, la, beta, do, init_state=init, d_final_state=dfinal)

    def loss(xs):
        o, f = oracle.recurrent(*xs[:5], init_state=xs[5])
        return float(np.sum(o * do) + np.sum(f * dfinal))

    h = 1e-6
    for ai, name in enumerate(NAMES):
        g = got[ai]
        for idx in np.ndindex(args[ai].shape):
            xp = [a.copy() for a in args]
            xm = [a.copy() for a in args]
            xp[ai][idx] += h
            xm[ai][idx] -= h
            fd = (loss(xp) - loss(xm)) / (2 * h)
            assert abs(fd - g[idx]) <= 1e-7 * max(1.0, abs(fd)), f"{name}{idx}: fd {fd} vs {g[idx]}"


def test_adjoint_identity_in_v_and_initial_state():
    """For fixed q, k, alpha, beta the output and final state are linear in (V, S_0); the
    backward of a linear map is its transpose, exactly (to rounding)."""
    q, k, v, la, beta, init, do, dfinal = rand_inputs(B=2, T=11, H=2, dk=6, dv=5, s0=True, dfin=True, seed=11)
    rng = np.random.default_rng(12)
    V = rng.standard_normal(v.shape)
    S0 = rng.standard_normal(init.shape)
    o, f = oracle.recurrent(q, k, V, la, beta, init_state=S0)
    # the gradient is evaluated at another point: for a linear map it does not depend on it
    g = oracle.backward(q, k, np.zeros_like(v), la, beta, do, init_state=None, d_final_state=dfinal)
    lhs = np.sum(do * o) + np.sum(dfinal * f)
    rhs = np.sum(g[2] * V) + np.sum(g[5] * S0)
    assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(lhs))


# ---- planted mistakes: mutated copies of the C oracle must fail the autograd pin ------------------

MUTATIONS = {
    "erase term of dk dropped": ("dkr[i] -= beta * acc;", "dkr[i] -= 0.0 * acc;"),
    "sign of the erase in dS'": ("dS[i * dv + j] -= beta * k[i] * du[j];", "dS[i * dv + j] += beta * k[i] * du[j];"),
    "decay missing from dS_prev": ("dS[i * dv + j] *= a[i]; /* now dS_prev */", "/* no decay */"),
    "output read before the write": ("dq[i] += Snew[i * dv + j] * dout[j];", "dq[i] += Sprev[i * dv + j] * dout[j];"),
    "beta missing from dv": ("dvr[j] = beta * du[j];", "dvr[j] = du[j];"),
}


def _mutant(tmp_path, name):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "kda_oracle.c")).read()
    old, new = MUTATIONS[name]
    assert src.count(old) == 1, name
    path = tmp_path / (re.sub(r"\W+", "_", name) + ".c")
    path.write_text(src.replace(old, new))
    so = str(path) + ".so"
    subprocess.check_call(["gcc", "-O1", "-fPIC", "-shared", "-o", so, str(path), "-lm", "-lpthread"])
    lib = ctypes.CDLL(so)
    lib.kda_oracle_backward.argtypes = oracle._load().kda_oracle_backward.argtypes
    lib.kda_oracle_backward.restype = ctypes.c_int
    return lib


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_backward_mistakes_fail_the_pin(tmp_path, monkeypatch, name):
    lib = _mutant(tmp_path, name)
    monkeypatch.setattr(oracle, "_lib", lib)
    q, k, v, la, beta, init, do, dfinal = rand_inputs(**SHAPE_CASES[0])
    got = oracle.backward(q, k, v, la, beta, do, init_state=init, d_final_state=dfinal)
    ref = autograd_grads(q, k, v, la, beta, init, do, dfinal)
    worst = max(np.max(np.abs(g - r)) / max(np.max(np.abs(r)), 1e-300) for g, r in zip(got, ref))
    assert worst > 1e-3, f"mutation '{name}' went unnoticed ({worst:.2e})"
