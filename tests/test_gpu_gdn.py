"""Gated DeltaNet (one decay per head and token) and DeltaNet (no decay) on the GPU: parity of
gdn_chunk_fwd, gdn_recurrent_fwd and gdn_decode_step against the fp64 oracle, and agreement with
the KDA entry points given the same decay on every key channel."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_86_b200 import (device_error, gdn_chunk_fwd, gdn_decode_step, gdn_recurrent_fwd, inputs,
                                      kda_chunk_fwd, kda_decode_step)
from parity import BF16_TOL, FP32_TOL, check_heads_in_groups, np64, rel_err

pytestmark = pytest.mark.gpu

TOKENS = ("q", "k", "v")


def gdn_inputs(workload, gate=True, device="cpu", **kw):
    """Seeded workload inputs with a per-head gate: the first key channel's log-decay of the
    workload's gate (logsigmoid of a normal draw), or None for DeltaNet."""
    x = inputs.make_prefill(workload, device=device, **kw)
    x["log_g"] = x["log_alpha"][..., 0].contiguous() if gate else None
    return x


def run_and_check(fn, x, tol, heads=None):
    dev = torch.device("cuda")
    g = None if x["log_g"] is None else x["log_g"].to(dev)
    s0 = None if x["init_state"] is None else x["init_state"].to(dev)
    cu = None if x["cu_seqlens"] is None else x["cu_seqlens"].to(dev)
    out, fs = fn(*(x[n].to(dev) for n in TOKENS), g, x["beta"].to(dev), initial_state=s0, cu_seqlens=cu)
    torch.cuda.synchronize()
    assert device_error() == 0
    def sel(t, axis):
        return t if heads is None else t.index_select(axis, torch.as_tensor(heads, device=t.device))

    ref_o, ref_s = oracle.gdn_recurrent(
        *(np64(sel(x[n], 2)) for n in TOKENS), None if x["log_g"] is None else np64(sel(x["log_g"], 2)),
        np64(sel(x["beta"], 2)), init_state=None if s0 is None else np64(sel(x["init_state"], 1)),
        cu_seqlens=None if cu is None else x["cu_seqlens"].numpy())
    out, fs = sel(out.cpu(), 2), sel(fs.cpu(), 1)
    eo, es = rel_err(out, ref_o), rel_err(fs, ref_s)
    assert eo <= tol and es <= tol, f"out {eo:.3e} state {es:.3e} (tol {tol})"


@pytest.mark.parametrize("gate", [True, False])
@pytest.mark.parametrize("T", [1, 65, 200, 333])
def test_gdn_chunk_bf16_ragged(cuda_lib, T, gate):
    x = gdn_inputs("prefill_bf16", gate, B=1, T=T, H=2, init_state=True)
    run_and_check(gdn_chunk_fwd, x, BF16_TOL)


@pytest.mark.parametrize("dv", [64, 128])
def test_gdn_chunk_many_pairs(cuda_lib, dv):
    """80 (sequence, head) pairs: chains run several pairs in turn."""
    x = gdn_inputs("prefill_bf16", True, B=2, T=150, H=40, dv=dv, init_state=True)
    run_and_check(gdn_chunk_fwd, x, BF16_TOL)


def test_gdn_chunk_strong_decay_fallback(cuda_lib):
    """Per-head log-decays near -3 per token exceed the rebasing range: exact branch per chunk."""
    x = gdn_inputs("prefill_bf16", True, B=1, T=300, H=2, mu=-3.0, init_state=True)
    run_and_check(gdn_chunk_fwd, x, BF16_TOL)


def test_gdn_chunk_varlen(cuda_lib):
    lens = [1, 0, 64, 130, 7, 65, 0, 200]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    for gate in (True, False):
        x = gdn_inputs("prefill_bf16", gate, B=1, T=int(cu[-1]), H=3, init_state=False)
        x["cu_seqlens"] = cu
        x["init_state"] = torch.randn((len(lens), 3, 128, 128), generator=torch.Generator().manual_seed(9)) * 0.1
        run_and_check(gdn_chunk_fwd, x, BF16_TOL)
        run_and_check(gdn_recurrent_fwd, x, BF16_TOL)


@pytest.mark.parametrize("gate", [True, False])
def test_gdn_tiny_fp32(cuda_lib, gate):
    x = gdn_inputs("tiny_fp32", gate)
    run_and_check(gdn_chunk_fwd, x, FP32_TOL)      # fp32 I/O: the CUDA-core path
    run_and_check(gdn_recurrent_fwd, x, FP32_TOL)


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128)])
def test_gdn_recurrent_bf16(cuda_lib, dk, dv):
    x = gdn_inputs("prefill_bf16", True, B=2, T=97, H=3, dk=dk, dv=dv, init_state=True)
    run_and_check(gdn_recurrent_fwd, x, BF16_TOL)


def test_gdn_long_full(cuda_lib):
    """The long workload's shape (T = 65536, 32 heads) with a per-head gate, every head."""
    x = gdn_inputs("long_bf16", True, device="cuda")
    out, fs = gdn_chunk_fwd(*(x[n] for n in TOKENS), x["log_g"], x["beta"], initial_state=x["init_state"])
    torch.cuda.synchronize()
    assert device_error() == 0

    def ref(xs):
        return oracle.gdn_recurrent(*(np64(xs[n]) for n in TOKENS), np64(xs["log_g"]), np64(xs["beta"]),
                                    init_state=np64(xs["init_state"]))

    check_heads_in_groups(out, fs, x, ref, BF16_TOL, names=TOKENS + ("log_g", "beta"))


def test_gdn_equals_kda_with_shared_channel_decay(cuda_lib):
    """The per-head path and the per-channel path given the same decay on every channel compute
    the same arithmetic on the same values."""
    x = gdn_inputs("prefill_bf16", True, B=1, T=333, H=3, init_state=True)
    dev = torch.device("cuda")
    t = [x[n].to(dev) for n in TOKENS]
    g, b, s0 = x["log_g"].to(dev), x["beta"].to(dev), x["init_state"].to(dev)
    la = g[..., None].expand(*g.shape, 128).contiguous()
    o1, f1 = gdn_chunk_fwd(*t, g, b, initial_state=s0)
    o2, f2 = kda_chunk_fwd(*t, la, b, initial_state=s0)
    torch.cuda.synchronize()
    assert rel_err(o1, np64(o2)) <= 1e-5 and rel_err(f1, np64(f2)) <= 1e-5


@pytest.mark.parametrize("gate", [True, False])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_gdn_decode_small(cuda_lib, dk, dv, dtype, gate):
    d = inputs.make_decode("decode_bf16", device="cpu", steps=4, B=3, H=5, dk=dk, dv=dv, dtype=dtype)
    state = d["state"].cuda()
    ref_s = d["state"].numpy().astype(np.float64)
    tol = BF16_TOL if dtype == torch.bfloat16 else FP32_TOL
    for t in range(4):
        lg = d["log_alpha"][t][..., 0].contiguous() if gate else None
        o = gdn_decode_step(*(d[n][t].cuda() for n in TOKENS), None if lg is None else lg.cuda(),
                            d["beta"][t].cuda(), state)
        ref_o, ref_s = oracle.gdn_decode_step(*(np64(d[n][t]) for n in TOKENS), np64(lg), np64(d["beta"][t]),
                                              ref_s)
        assert rel_err(o, ref_o) <= tol
        assert rel_err(state, ref_s) <= tol
    assert device_error() == 0


def test_gdn_decode_equals_kda_decode(cuda_lib):
    d = inputs.make_decode("decode_bf16", device="cuda", steps=1, B=4, H=8)
    s1, s2 = d["state"].clone(), d["state"].clone()
    tok = [d[n][0] for n in TOKENS]
    lg = d["log_alpha"][0][..., 0].contiguous()
    o1 = gdn_decode_step(*tok, lg, d["beta"][0], s1)
    o2 = kda_decode_step(*tok, lg[..., None].expand_as(d["log_alpha"][0]).contiguous(), d["beta"][0], s2)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_gdn_chunk_length_32_and_key_width_64(cuda_lib):
    x = gdn_inputs("prefill_bf16", True, B=1, T=333, H=3, init_state=True)
    run_and_check(lambda *a, **kw: gdn_chunk_fwd(*a, chunk_size=32, **kw), x, BF16_TOL)
    y = gdn_inputs("prefill_bf16", True, B=2, T=150, H=3, dk=64, dv=64, init_state=True)
    run_and_check(gdn_chunk_fwd, y, BF16_TOL)
