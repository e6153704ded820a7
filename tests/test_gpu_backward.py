"""Gradient of the prefill (kda_chunk_bwd) on the GPU against the fp64 backward oracle
(oracle.backward, pinned in test_oracle_backward_pins.py): every gradient tensor, every element,
max |gpu - oracle| / rms(oracle) within the fp32 bound (the kernel computes in fp32 from the same
input values the oracle widens to fp64)."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_86_b200 import device_error, inputs, kda_chunk_bwd
from parity import FP32_TOL, NAMES, np64, rel_err

pytestmark = pytest.mark.gpu
GRADS = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "d_init_state")


def check(x, d_out, d_final=None, chunk=64, tol=FP32_TOL):
    dev = torch.device("cuda")
    args = [x[n].to(dev) for n in NAMES]
    s0 = None if x["init_state"] is None else x["init_state"].to(dev)
    cu = None if x["cu_seqlens"] is None else x["cu_seqlens"].to(dev)
    got = kda_chunk_bwd(*args, d_out.to(dev), initial_state=s0,
                        d_final_state=None if d_final is None else d_final.to(dev), cu_seqlens=cu, chunk_size=chunk)
    torch.cuda.synchronize()
    assert device_error() == 0
    ref = oracle.backward(*(np64(x[n]) for n in NAMES), np64(d_out), init_state=np64(x["init_state"]),
                          d_final_state=np64(d_final),
                          cu_seqlens=None if x["cu_seqlens"] is None else x["cu_seqlens"].cpu().numpy())
    errs = {}
    for name, g, r in zip(GRADS, got, ref):
        errs[name] = rel_err(g, r)
    assert all(e <= tol for e in errs.values()), errs
    return errs


def upstream(x, seed):
    g = torch.Generator().manual_seed(seed)
    B, T, H, dv = x["v"].shape
    N = B if x["cu_seqlens"] is None else x["cu_seqlens"].numel() - 1
    dk = x["q"].shape[-1]
    return torch.randn((B, T, H, dv), generator=g), torch.randn((N, H, dk, dv), generator=g)


@pytest.mark.parametrize("T", [1, 17, 64, 65, 200])
def test_backward_ragged(cuda_lib, T):
    x = inputs.make_prefill("prefill_bf16", device="cpu", B=1, T=T, H=3, init_state=True)
    do, dfin = upstream(x, T)
    check(x, do, dfin)


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64)])
def test_backward_head_sizes(cuda_lib, dk, dv):
    x = inputs.make_prefill("prefill_bf16", device="cpu", B=2, T=150, H=2, dk=dk, dv=dv, init_state=True)
    do, dfin = upstream(x, dk + dv)
    check(x, do, dfin)


@pytest.mark.parametrize("chunk", [32, 128, 256])
def test_backward_checkpoint_interval(cuda_lib, chunk):
    """The checkpoint interval changes no result."""
    x = inputs.make_prefill("prefill_bf16", device="cpu", B=1, T=300, H=2, init_state=True)
    do, dfin = upstream(x, chunk)
    check(x, do, dfin, chunk=chunk)


def test_backward_fp32_inputs_no_initial_state(cuda_lib):
    x = inputs.make_prefill("tiny_fp32", device="cpu")
    do, _ = upstream(x, 5)
    check(x, do, None)


def test_backward_bf16_upstream_gradient(cuda_lib):
    x = inputs.make_prefill("prefill_bf16", device="cpu", B=1, T=130, H=2, init_state=True)
    do, dfin = upstream(x, 6)
    check(x, do.to(torch.bfloat16), dfin)


def test_backward_varlen(cuda_lib):
    lens = [1, 0, 64, 130, 7, 65, 0, 100]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    x = inputs.make_prefill("prefill_bf16", device="cpu", B=1, T=int(cu[-1]), H=2, init_state=False)
    x["cu_seqlens"] = cu
    x["init_state"] = torch.randn((len(lens), 2, 128, 128), generator=torch.Generator().manual_seed(4)) * 0.1
    do, dfin = upstream(x, 7)
    check(x, do, dfin)


def test_backward_strong_decay(cuda_lib):
    """Fast forgetting (log-decays near -3 per token): the tensor-core forward takes its exact path
    there; the gradient has no such branch and must match all the same."""
    x = inputs.make_prefill("prefill_bf16", device="cpu", B=1, T=200, H=2, mu=-3.0, init_state=True)
    do, dfin = upstream(x, 8)
    check(x, do, dfin)


def test_backward_matches_autograd_free_directional_derivative(cuda_lib):
    """A directional derivative of the GPU forward (kda_recurrent_fwd in fp32, by central
    differences along a random direction of every input) agrees with <gradient, direction> from
    kda_chunk_bwd: the backward is the derivative of the library's own forward."""
    from gated_delta_rule_86_b200 import kda_recurrent_fwd
    x = inputs.make_prefill("tiny_fp32", device="cuda", T=48, H=2, init_state=True)
    g = torch.Generator(device="cuda").manual_seed(9)
    do = torch.randn(x["v"].shape, generator=g, device="cuda")
    base = [x[n] for n in NAMES] + [x["init_state"]]
    dirs = [torch.randn(t.shape, generator=g, device="cuda") for t in base]
    dirs[3] = dirs[3] * 0.1     # keep log_alpha <= 0 along the probe
    dirs[4] = dirs[4] * 0.1

    def loss(eps):
        a = [t + eps * d for t, d in zip(base, dirs)]
        a[3] = a[3].clamp(max=0.0)
        o, _ = kda_recurrent_fwd(*a[:5], initial_state=a[5])
        return float((o.double() * do.double()).sum())

    h = 1e-3
    fd = (loss(h) - loss(-h)) / (2 * h)
    grads = kda_chunk_bwd(*base[:5], do, initial_state=base[5])
    an = sum(float((gr.double() * d.double()).sum()) for gr, d in zip(grads, dirs))
    assert abs(fd - an) <= 2e-3 * max(1.0, abs(an)), (fd, an)


@pytest.mark.parametrize("varlen", [False, True])
def test_autograd_wrapper(cuda_lib, varlen):
    """kda_chunk (torch.autograd.Function over kda_chunk_fwd / kda_chunk_bwd): loss.backward() gives the
    gradients of kda_chunk_bwd called directly (bitwise, cast to each input's dtype), and those are the
    oracle's; the forward outputs are kda_chunk_fwd's."""
    from gated_delta_rule_86_b200 import kda_chunk, kda_chunk_fwd
    if varlen:
        x = inputs.make_prefill("varlen_bf16", device="cpu", H=2, varlen=3, varlen_range=(40, 150))
    else:
        x = inputs.make_prefill("prefill_bf16", device="cpu", B=2, T=130, H=3, init_state=True)
    dev = torch.device("cuda")
    cu = None if x["cu_seqlens"] is None else x["cu_seqlens"].to(dev)
    leaves = [x[n].to(dev).requires_grad_(True) for n in NAMES]
    s0 = x["init_state"].to(dev).requires_grad_(True)
    do, dfin = upstream(x, 11)
    out, fs = kda_chunk(*leaves, initial_state=s0, cu_seqlens=cu)
    ((out * do.to(dev)).sum() + (fs * dfin.to(dev)).sum()).backward()
    ref_out, ref_fs = kda_chunk_fwd(*(t.detach() for t in leaves), initial_state=s0.detach(), cu_seqlens=cu)
    assert torch.equal(out.detach(), ref_out) and torch.equal(fs.detach(), ref_fs)
    direct = kda_chunk_bwd(*(t.detach() for t in leaves), do.to(dev), initial_state=s0.detach(),
                           d_final_state=dfin.to(dev), cu_seqlens=cu)
    torch.cuda.synchronize()
    assert device_error() == 0
    for name, leaf, want in zip(GRADS, leaves + [s0], direct):
        assert leaf.grad is not None and leaf.grad.dtype == leaf.dtype, name
        assert torch.equal(leaf.grad, want.to(leaf.dtype)), name
    check(x, do, dfin)


@pytest.mark.parametrize("varlen", [False, True])
def test_backward_every_state_bitwise(cuda_lib, varlen):
    """chunk_size = 0 keeps the state before every token (no recompute pass): bitwise the gradients
    of the checkpointed schedule, and within the bound of the oracle."""
    if varlen:
        lens = [1, 0, 64, 130, 7, 65, 0, 100]
        cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
        x = inputs.make_prefill("prefill_bf16", device="cpu", B=1, T=int(cu[-1]), H=2, init_state=False)
        x["cu_seqlens"] = cu
        x["init_state"] = torch.randn((len(lens), 2, 128, 128), generator=torch.Generator().manual_seed(9)) * 0.1
    else:
        x = inputs.make_prefill("prefill_bf16", device="cpu", B=2, T=333, H=3, init_state=True)
    do, dfin = upstream(x, 12)
    dev = torch.device("cuda")
    a = [x[n].to(dev) for n in NAMES]
    s0 = x["init_state"].to(dev)
    cu = None if x["cu_seqlens"] is None else x["cu_seqlens"].to(dev)
    runs = [kda_chunk_bwd(*a, do.to(dev), initial_state=s0, d_final_state=dfin.to(dev), cu_seqlens=cu, chunk_size=c)
            for c in (64, 0)]
    torch.cuda.synchronize()
    assert device_error() == 0
    for name, g64, g0 in zip(GRADS, *runs):
        assert torch.equal(g64, g0), name
    check(x, do, dfin, chunk=0)


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64)])
def test_backward_every_state_head_sizes(cuda_lib, dk, dv):
    """chunk_size = 0 at the other head sizes: bitwise the checkpointed schedule's gradients."""
    x = inputs.make_prefill("prefill_bf16", device="cpu", B=2, T=97, H=2, dk=dk, dv=dv, init_state=True)
    do, dfin = upstream(x, dk + 3 * dv)
    dev = torch.device("cuda")
    a = [x[n].to(dev) for n in NAMES]
    runs = [kda_chunk_bwd(*a, do.to(dev), initial_state=x["init_state"].to(dev), d_final_state=dfin.to(dev),
                          chunk_size=c) for c in (32, 0)]
    torch.cuda.synchronize()
    assert device_error() == 0
    for name, g1, g0 in zip(GRADS, *runs):
        assert torch.equal(g1, g0), name
