"""Seeded synthetic inputs for the KDA operator.

This module only draws random numbers and lays them out.  It holds none of the
operator's arithmetic, so the test oracle and the CUDA path can both take their
inputs from it without sharing any of the method.

Distributions (the same for every workload unless stated):
  * q, k ~ N(0, 1), then L2-normalised over d_k for every (token, head), in
    fp32 before any rounding to the storage dtype;
  * v ~ N(0, 1);
  * beta = sigmoid(N(0, 1)), one per (token, head);
  * log_alpha = logsigmoid(N(mu, 1)) per (token, head, key channel), so
    alpha = exp(log_alpha) lies in (0, 1);
  * initial states, where a workload has them, ~ N(0, 0.1^2) (std 0.1), fp32.

The random streams come from ``torch.Generator`` on the device the tensors are
made on, seeded with ``base_seed + workload id``; the same device and seed give
the same numbers.  Parity tests either build inputs on the CPU and copy them to
the GPU, or build them on the GPU and copy the sampled part to the CPU: in both
cases the oracle and the kernels see the same rounded values.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

BASE_SEED = 0x4B4441


@dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, dtype and the gate mean ``mu``."""
    wid: int
    name: str
    B: int
    T: int
    H: int
    dk: int
    dv: int
    dtype: torch.dtype
    mu: float
    init_state: bool
    chunk: int = 64
    varlen: int = 0                      # number of packed sequences (0: fixed-length batch)
    varlen_range: tuple = (1024, 16384)  # inclusive length range for packed sequences
    decode_steps: int = 0                # >0: a decode workload of this many steps
    notes: str = field(default="", compare=False)


WORKLOADS = {
    "tiny_fp32": Workload(1, "tiny_fp32", B=1, T=256, H=2, dk=64, dv=64, dtype=torch.float32,
                          mu=2.0, init_state=False,
                          notes="Tiny fp32 check: B1 H2 T256 d64, zero initial state"),
    "prefill_bf16": Workload(2, "prefill_bf16", B=2, T=4096, H=16, dk=128, dv=128,
                             dtype=torch.bfloat16, mu=2.0, init_state=False,
                             notes="Prefill bf16: B2 H16 T4096 d128, zero initial state"),
    "long_bf16": Workload(3, "long_bf16", B=1, T=65536, H=32, dk=128, dv=128,
                          dtype=torch.bfloat16, mu=4.0, init_state=True,
                          notes="Long-context prefill bf16: B1 H32 T65536 d128, N(0,0.1) initial state"),
    "varlen_bf16": Workload(4, "varlen_bf16", B=1, T=0, H=32, dk=128, dv=128,
                            dtype=torch.bfloat16, mu=2.0, init_state=True, varlen=8,
                            notes="Packed varlen bf16: 8 sequences, lengths U{1024..16384}, H32 d128"),
    "decode_bf16": Workload(5, "decode_bf16", B=256, T=1, H=32, dk=128, dv=128,
                            dtype=torch.bfloat16, mu=3.0, init_state=True, decode_steps=1024,
                            notes="Decode: B256 H32 d128, fp32 state in place, 1024 steps"),
}


def generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(int(seed))
    return g


def _normal(shape, gen, device, mean=0.0, std=1.0):
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    if mean != 0.0:
        x.add_(mean)
    return x


def _unit(shape, gen, device):
    x = _normal(shape, gen, device)
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def varlen_lengths(n: int, lo: int, hi: int, seed: int) -> list:
    """Sequence lengths drawn uniformly from the inclusive range [lo, hi] (CPU stream)."""
    g = generator(seed, "cpu")
    return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g)]


def token_inputs(B, T, H, dk, dv, mu, dtype, gen, device, raw=False):
    """q, k, v, log_alpha, beta for [B, T, H, .] in the storage dtype.

    With ``raw`` the same draws are returned before their activations (the raw projections):
    q and k not normalised, the gate's and beta's pre-activations N(mu, 1) and N(0, 1).
    """
    q = _normal((B, T, H, dk), gen, device) if raw else _unit((B, T, H, dk), gen, device)
    k = _normal((B, T, H, dk), gen, device) if raw else _unit((B, T, H, dk), gen, device)
    v = _normal((B, T, H, dv), gen, device)
    beta = _normal((B, T, H), gen, device)
    log_alpha = _normal((B, T, H, dk), gen, device, mean=mu)
    if not raw:
        beta = torch.sigmoid(beta)
        log_alpha = torch.nn.functional.logsigmoid(log_alpha)
    return tuple(x.to(dtype) for x in (q, k, v, log_alpha, beta))


def make_prefill(w: Workload | str, device="cpu", seed: int | None = None, raw: bool = False, **override):
    """Inputs for a prefill workload as a dict of tensors on ``device``.

    Keys: q, k, v, log_alpha, beta, init_state (None or fp32 [N,H,dk,dv]),
    cu_seqlens (None or int32 [N+1]).  ``override`` replaces Workload fields
    (e.g. T=300 for a shortened parity case).  With ``raw`` the keys q, k,
    log_alpha and beta hold the raw projections (see :func:`token_inputs`).
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    if override:
        w = Workload(**{**w.__dict__, **override})
    seed = BASE_SEED + w.wid if seed is None else seed
    gen = generator(seed, device)
    cu = None
    if w.varlen:
        lens = varlen_lengths(w.varlen, w.varlen_range[0], w.varlen_range[1], seed)
        total = sum(lens)
        B, T, N = 1, total, w.varlen
        cu = torch.tensor([0] + list(torch.tensor(lens).cumsum(0).tolist()), dtype=torch.int32,
                          device=device)
    else:
        B, T, N = w.B, w.T, w.B
    q, k, v, la, beta = token_inputs(B, T, w.H, w.dk, w.dv, w.mu, w.dtype, gen, device, raw=raw)
    s0 = _normal((N, w.H, w.dk, w.dv), gen, device, std=0.1) if w.init_state else None
    return dict(q=q, k=k, v=v, log_alpha=la, beta=beta, init_state=s0, cu_seqlens=cu,
                workload=w)


def make_decode(w: Workload | str = "decode_bf16", device="cpu", seed: int | None = None,
                steps: int | None = None, raw: bool = False, **override):
    """Inputs for a decode workload: per-step tokens stacked on a leading axis.

    Returns q, k, log_alpha [steps, B, H, dk], v [steps, B, H, dv], beta
    [steps, B, H] in the storage dtype, and state fp32 [B, H, dk, dv] (raw
    projections with ``raw``, as in :func:`make_prefill`).
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    if override:
        w = Workload(**{**w.__dict__, **override})
    seed = BASE_SEED + w.wid if seed is None else seed
    steps = w.decode_steps if steps is None else steps
    gen = generator(seed, device)
    state = _normal((w.B, w.H, w.dk, w.dv), gen, device, std=0.1)
    q, k, v, la, beta = token_inputs(steps, w.B, w.H, w.dk, w.dv, w.mu, w.dtype, gen, device, raw=raw)
    return dict(q=q, k=k, v=v, log_alpha=la, beta=beta, state=state, workload=w)
