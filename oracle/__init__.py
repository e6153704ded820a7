"""fp64 CPU oracle for the KDA operator -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library
(``gated_delta_rule_86_b200``) never imports it, and the two share no code:
the only module both sides use is the seeded input generator, which holds none
of the method's arithmetic.

Contents
  * :func:`recurrent` -- the token-by-token recurrence of the "Stage 3: KDA's
    fused design" equation ("Hybrid Linear Attention Architectures: Breaking
    Through the Long-Context Engineering Bottleneck in LLMs"), in plain C
    (``kda_oracle.c``), fp64, threaded over (sequence, head) pairs.
  * :func:`decode_step` -- one iteration of the same loop body, in place.
  * :func:`backward` -- the gradient of :func:`recurrent` with respect to every
    input (reverse mode through the same token steps, fp64 C).
  * :func:`gdn_recurrent`, :func:`gdn_decode_step` -- Gated DeltaNet (one
    decay per head and token) and DeltaNet (no decay): the same recurrence
    with every key channel sharing the head's decay, the scalar-gate and
    alpha = 1 reductions that ``test_scalar_gate_is_gated_deltanet`` and
    ``test_alpha_one_is_deltanet`` pin against the matrix forms of Stages 1
    and 2 of section "Core Module Design" on the same page.
  * :func:`prologue` -- the raw projections to the recurrence's inputs (the
    fused entry points): q, k L2-normalised over d_k with eps 1e-6 under the
    root, log_alpha = logsigmoid(g), beta = sigmoid(b); fp64 NumPy.
  * :func:`chunkwise` (``chunkwise.py``) -- an independent fp64 NumPy
    restatement of the chunkwise formulas ("Hardware-Aware Chunkwise
    Parallelism" on the same page; section 3 of "Linear Attention KDA Gating in
    a 3:1 Hybrid Architecture").  It is not the oracle; the tests use it to pin
    the garbled chunk formulas against the recurrence.

Pins: every function here is checked by ``tests/test_oracle_pins.py`` against
closed forms and brute-force constructions that share no code with it
(DeltaNet reduction, exact overwrite with a unit key, the unrolled operator
product for short sequences, beta = 0 decay-only closed form, scalar-gate
reduction, linearity, non-expansion, chunkwise equivalence, composition).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "libkda_oracle.so")
_lib = None


def build_oracle(force: bool = False) -> str:
    """Compile ``kda_oracle.c`` into ``libkda_oracle.so`` with gcc (plain C)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build_oracle()
        lib = ctypes.CDLL(_LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        i64p = ctypes.POINTER(ctypes.c_int64)
        i64 = ctypes.c_int64
        lib.kda_oracle_recurrent.argtypes = [dp, dp, dp, dp, dp, dp, i64p, i64, i64, i64, i64,
                                             i64, i64, dp, dp, ctypes.c_int]
        lib.kda_oracle_recurrent.restype = ctypes.c_int
        lib.kda_oracle_decode_step.argtypes = [dp, dp, dp, dp, dp, dp, dp, i64, i64, i64, i64]
        lib.kda_oracle_decode_step.restype = ctypes.c_int
        lib.kda_oracle_backward.argtypes = [dp, dp, dp, dp, dp, dp, i64p, i64, i64, i64, i64, i64, i64,
                                            dp, dp, dp, dp, dp, dp, dp, dp, ctypes.c_int]
        lib.kda_oracle_backward.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a, ctype=ctypes.c_double):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def recurrent(q, k, v, log_alpha, beta, init_state=None, cu_seqlens=None, nthreads=None):
    """Token recurrence over [B, T, H, d] inputs; returns ``(out, final_state)`` in fp64.

    ``q, k, log_alpha``: [B, T, H, d_k]; ``v``: [B, T, H, d_v]; ``beta``: [B, T, H];
    ``init_state``: [N, H, d_k, d_v] or None (zeros); ``cu_seqlens``: int [N+1]
    with B == 1, or None (N = B).  Inputs of any float dtype are widened to fp64
    exactly (bf16 values are taken as the bf16 numbers they are).
    """
    q, k, v, log_alpha, beta = (_f64(x) for x in (q, k, v, log_alpha, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == q.shape and log_alpha.shape == q.shape
    assert v.shape == (B, T, H, dv) and beta.shape == (B, T, H)
    cu = None
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
        N = cu.shape[0] - 1
        assert B == 1
    else:
        N = B
    s0 = None if init_state is None else _f64(init_state)
    if s0 is not None:
        assert s0.shape == (N, H, dk, dv)
    out = np.zeros((B, T, H, dv), dtype=np.float64)
    fs = np.zeros((N, H, dk, dv), dtype=np.float64)
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    rc = _load().kda_oracle_recurrent(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                      _ptr(s0), _ptr(cu, ctypes.c_int64), N, B, T, H, dk, dv,
                                      _ptr(out), _ptr(fs), int(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return out, fs


def decode_step(q, k, v, log_alpha, beta, state):
    """One recurrence step for [B, H, d] inputs; returns ``(out, new_state)`` (fp64 copies)."""
    q, k, v, log_alpha, beta = (_f64(x) for x in (q, k, v, log_alpha, beta))
    S = _f64(state).copy()
    B, H, dk = q.shape
    dv = v.shape[-1]
    assert S.shape == (B, H, dk, dv) and beta.shape == (B, H)
    out = np.zeros((B, H, dv), dtype=np.float64)
    rc = _load().kda_oracle_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                        _ptr(S), _ptr(out), B, H, dk, dv)
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return out, S


def backward(q, k, v, log_alpha, beta, d_out, init_state=None, d_final_state=None, cu_seqlens=None,
             nthreads=None):
    """Gradients of :func:`recurrent` (reverse mode, fp64): given ``d_out`` = dLoss/dout
    [B, T, H, d_v] and ``d_final_state`` = dLoss/dfinal_state [N, H, d_k, d_v] (None: zero),
    returns ``(dq, dk, dv, dlog_alpha, dbeta, d_init_state)`` with the shapes of q, k, v,
    log_alpha, beta and the initial state.  The adjoint of each token step is written out in
    ``kda_oracle.c``; the forward states are kept for the whole sequence."""
    q, k, v, log_alpha, beta, d_out = (_f64(x) for x in (q, k, v, log_alpha, beta, d_out))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == q.shape and log_alpha.shape == q.shape and d_out.shape == v.shape
    cu = None
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
        N = cu.shape[0] - 1
    else:
        N = B
    s0 = None if init_state is None else _f64(init_state)
    dfin = None if d_final_state is None else _f64(d_final_state)
    for x in (s0, dfin):
        if x is not None:
            assert x.shape == (N, H, dk, dv)
    grads = [np.zeros(q.shape), np.zeros(q.shape), np.zeros(v.shape), np.zeros(q.shape), np.zeros(beta.shape),
             np.zeros((N, H, dk, dv))]
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    rc = _load().kda_oracle_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(s0),
                                     _ptr(cu, ctypes.c_int64), N, B, T, H, dk, dv, _ptr(d_out), _ptr(dfin),
                                     *(_ptr(g) for g in grads), int(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected its arguments" if rc == -1 else "oracle ran out of memory")
    return tuple(grads)


NORM_EPS = 1e-6


def prologue(q_raw, k_raw, g_raw, b_raw):
    """Raw projections -> (q, k, log_alpha, beta), fp64.

    ``q = q_raw / sqrt(sum(q_raw**2) + 1e-6)`` over the last axis (k likewise),
    ``log_alpha = logsigmoid(g_raw) = -log(1 + exp(-g_raw))``, ``beta = sigmoid(b_raw)``.
    """
    q_raw, k_raw, g_raw, b_raw = (_f64(x) for x in (q_raw, k_raw, g_raw, b_raw))
    q = q_raw / np.sqrt(np.sum(q_raw * q_raw, axis=-1, keepdims=True) + NORM_EPS)
    k = k_raw / np.sqrt(np.sum(k_raw * k_raw, axis=-1, keepdims=True) + NORM_EPS)
    log_alpha = -np.logaddexp(0.0, -g_raw)
    beta = 1.0 / (1.0 + np.exp(-b_raw))
    return q, k, log_alpha, beta


def _channel_gate(log_g, shape):
    """A per-head log-decay (or None: none) as the per-channel gate of the same recurrence."""
    if log_g is None:
        return np.zeros(shape, dtype=np.float64)
    return np.ascontiguousarray(np.broadcast_to(_f64(log_g)[..., None], shape))


def gdn_recurrent(q, k, v, log_g, beta, init_state=None, cu_seqlens=None, nthreads=None):
    """Gated DeltaNet over [B, T, H, d] inputs with ``log_g`` [B, T, H] (None: DeltaNet);
    returns ``(out, final_state)`` in fp64."""
    q = _f64(q)
    return recurrent(q, k, v, _channel_gate(log_g, q.shape), beta, init_state, cu_seqlens, nthreads)


def gdn_decode_step(q, k, v, log_g, beta, state):
    """One Gated DeltaNet / DeltaNet step for [B, H, d] inputs, ``log_g`` [B, H] or None."""
    q = _f64(q)
    return decode_step(q, k, v, _channel_gate(log_g, q.shape), beta, state)


from .chunkwise import chunkwise  # noqa: E402  (NumPy restatement, see module docstring)

__all__ = ["build_oracle", "recurrent", "decode_step", "backward", "gdn_recurrent", "gdn_decode_step", "prologue",
           "chunkwise"]
