"""Independent fp64 NumPy restatement of the chunkwise KDA formulas -- TEST ONLY.

This is not the oracle (the oracle is the token recurrence in ``kda_oracle.c``).
It restates, in the pages' order and notation, the chunkwise scheme of
"Hybrid Linear Attention Architectures: Breaking Through the Long-Context
Engineering Bottleneck in LLMs" (section "Hardware-Aware Chunkwise Parallelism:
Notation, Steps, and Implementation": the inter-chunk state update and the
intra-chunk output), which section 3 of "Linear Attention KDA Gating in a 3:1
Hybrid Architecture" repeats (3.1 inter-chunk transition, 3.2 intra-chunk
output, 3.3 the per-chunk loop).  The printed formulas are partly garbled; the
readings taken here are:

* gamma^C = prod_{i<=C} alpha_i and Gamma are per channel (C x d_k), Gamma_r =
  prod_{s<=r} alpha_s counted from the chunk start, inclusive (the loop's
  ``cumprod``); the "remaining decay" in the state update is
  Gamma^{i->C}_s = gamma^C / Gamma_s (the loop's ``cumprod_reverse``).
* W and U are not sums of outer products (those would be d_k x d_k and could
  not be multiplied as U - W S into a C x d_v term); they are the chunk's WY
  factors from the UT transform:
      T = (I + strict_tril(diag(beta) (K*Gamma) (K/Gamma)^T))^{-1},
      W = T diag(beta) (K*Gamma),   U = T diag(beta) V,
  so that U - W S is the C x d_v matrix of effective writes.
* Tril keeps the diagonal (token i sees j <= i).
* Chunks never cross sequence boundaries; the last chunk may be short.

Each chunk then performs (with S the state entering the chunk)
      Ut = U - W S
      O  = (Q*Gamma) S + tril((Q*Gamma) (K/Gamma)^T) Ut
      S  = Diag(gamma^C) S + (K * gamma^C/Gamma)^T Ut
exactly as the two printed equations read under the readings above.
"""
from __future__ import annotations

import numpy as np


def _chunk_pass(q, k, v, g, beta, S, C):
    """Run one sequence of one head through the chunk loop.

    q, k, g: [T, d_k]; v: [T, d_v]; beta: [T]; S: [d_k, d_v].  Returns (out, S).
    """
    T = q.shape[0]
    out = np.zeros((T, v.shape[1]), dtype=np.float64)
    for c0 in range(0, T, C):
        c1 = min(c0 + C, T)
        Q, K, V, b = q[c0:c1], k[c0:c1], v[c0:c1], beta[c0:c1]
        Gam = np.exp(np.cumsum(g[c0:c1], axis=0))          # Gamma_r, inclusive, [L, d_k]
        gam = Gam[-1]                                        # gamma^C, [d_k]
        L = c1 - c0
        A = np.tril(b[:, None] * ((K * Gam) @ (K / Gam).T), k=-1)
        Tm = np.linalg.inv(np.eye(L) + A)                    # UT transform
        W = Tm @ (b[:, None] * (K * Gam))
        U = Tm @ (b[:, None] * V)
        Ut = U - W @ S
        out[c0:c1] = (Q * Gam) @ S + np.tril((Q * Gam) @ (K / Gam).T) @ Ut
        S = gam[:, None] * S + (K * (gam[None, :] / Gam)).T @ Ut
    return out, S


def chunkwise(q, k, v, log_alpha, beta, init_state=None, cu_seqlens=None, chunk_size=64):
    """Chunkwise evaluation with the same argument conventions as ``oracle.recurrent``."""
    q, k, v, g, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, log_alpha, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is None:
        segs = [(b, 0, T) for b in range(B)]
    else:
        cu = [int(x) for x in cu_seqlens]
        segs = [(0, cu[n], cu[n + 1]) for n in range(len(cu) - 1)]
    N = len(segs)
    out = np.zeros((B, T, H, dv), dtype=np.float64)
    fs = np.zeros((N, H, dk, dv), dtype=np.float64)
    for n, (b, t0, t1) in enumerate(segs):
        for h in range(H):
            S = np.zeros((dk, dv)) if init_state is None else np.array(init_state[n, h], dtype=np.float64)
            o, S = _chunk_pass(q[b, t0:t1, h], k[b, t0:t1, h], v[b, t0:t1, h], g[b, t0:t1, h],
                               beta[b, t0:t1, h], S, chunk_size)
            out[b, t0:t1, h] = o
            fs[n, h] = S
    return out, fs
