"""KDA from the raw projections (kda_chunk_fwd_fused, kda_decode_step_fused) on the GPU: parity
against the fp64 oracle applied to oracle.prologue of the same raw values, and agreement with the
unfused calls given the activated inputs."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_86_b200 import (KdaError, device_error, inputs, kda_chunk_fwd, kda_chunk_fwd_fused,
                                      kda_decode_step_fused)
from parity import BF16_TOL, FP32_TOL, NAMES, check_heads_in_groups, np64, rel_err

pytestmark = pytest.mark.gpu


def check_chunk(x, heads=None):
    """x: raw inputs (inputs.make_prefill(..., raw=True)); compares kda_chunk_fwd_fused with the
    oracle recurrence on the activated inputs, on all heads or the listed ones."""
    dev = torch.device("cuda")
    s0 = None if x["init_state"] is None else x["init_state"].to(dev)
    cu = None if x["cu_seqlens"] is None else x["cu_seqlens"].to(dev)
    out, fs = kda_chunk_fwd_fused(*(x[n].to(dev) for n in NAMES), initial_state=s0, cu_seqlens=cu)
    torch.cuda.synchronize()
    assert device_error() == 0

    def sel(t, axis):
        return t if heads is None else t.index_select(axis, torch.as_tensor(heads, device=t.device))

    q, k, la, beta = oracle.prologue(*(np64(sel(x[n], 2)) for n in ("q", "k", "log_alpha", "beta")))
    ref_o, ref_s = oracle.recurrent(q, k, np64(sel(x["v"], 2)), la, beta,
                                    init_state=None if s0 is None else np64(sel(x["init_state"], 1)),
                                    cu_seqlens=None if cu is None else x["cu_seqlens"].cpu().numpy())
    out, fs = sel(out.cpu(), 2), sel(fs.cpu(), 1)
    eo, es = rel_err(out, ref_o), rel_err(fs, ref_s)
    assert eo <= BF16_TOL and es <= BF16_TOL, f"out {eo:.3e} state {es:.3e}"


@pytest.mark.parametrize("T", [1, 65, 200, 333])
def test_fused_chunk_ragged(cuda_lib, T):
    check_chunk(inputs.make_prefill("prefill_bf16", device="cpu", raw=True, B=1, T=T, H=2, init_state=True))


@pytest.mark.parametrize("dv", [64, 128])
def test_fused_chunk_many_pairs(cuda_lib, dv):
    x = inputs.make_prefill("prefill_bf16", device="cpu", raw=True, B=2, T=150, H=40, dv=dv, init_state=True)
    check_chunk(x)


def test_fused_chunk_strong_decay(cuda_lib):
    """Gate pre-activations near -3 (log-decays near -3 per token): the exact branch."""
    check_chunk(inputs.make_prefill("prefill_bf16", device="cpu", raw=True, B=1, T=300, H=2, mu=-3.0,
                                    init_state=True))


def test_fused_chunk_varlen(cuda_lib):
    lens = [1, 0, 64, 130, 7, 65, 0, 200]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    x = inputs.make_prefill("prefill_bf16", device="cpu", raw=True, B=1, T=int(cu[-1]), H=3, init_state=False)
    x["cu_seqlens"] = cu
    x["init_state"] = torch.randn((len(lens), 3, 128, 128), generator=torch.Generator().manual_seed(11)) * 0.1
    check_chunk(x)


def test_fused_long_full(cuda_lib):
    """The long workload from its raw projections, every head against oracle.prologue + the
    recurrence."""
    x = inputs.make_prefill("long_bf16", device="cuda", raw=True)
    out, fs = kda_chunk_fwd_fused(*(x[n] for n in NAMES), initial_state=x["init_state"])
    torch.cuda.synchronize()
    assert device_error() == 0

    def ref(xs):
        q, k, la, beta = oracle.prologue(*(np64(xs[n]) for n in ("q", "k", "log_alpha", "beta")))
        return oracle.recurrent(q, k, np64(xs["v"]), la, beta, init_state=np64(xs["init_state"]))

    check_heads_in_groups(out, fs, x, ref, BF16_TOL)


def test_fused_equals_unfused_on_activated_inputs(cuda_lib):
    """The same result as kda_chunk_fwd given the activated inputs.  Both are bf16-operand results
    that each lie within BF16_TOL of the oracle (the unfused one also rounds the activated inputs
    to bf16), so their difference is bounded by twice that."""
    x = inputs.make_prefill("prefill_bf16", device="cuda", raw=True, B=1, T=333, H=3, init_state=True)
    of, ff = kda_chunk_fwd_fused(*(x[n] for n in NAMES), initial_state=x["init_state"])
    qf, kf, gf, bf = (x[n].float() for n in ("q", "k", "log_alpha", "beta"))
    q = (qf * torch.rsqrt((qf * qf).sum(-1, keepdim=True) + 1e-6)).to(torch.bfloat16)
    k = (kf * torch.rsqrt((kf * kf).sum(-1, keepdim=True) + 1e-6)).to(torch.bfloat16)
    la = torch.nn.functional.logsigmoid(gf).to(torch.bfloat16)
    beta = torch.sigmoid(bf).to(torch.bfloat16)
    ou, fu = kda_chunk_fwd(q, k, x["v"], la, beta, initial_state=x["init_state"])
    torch.cuda.synchronize()
    assert rel_err(of, np64(ou)) <= 2 * BF16_TOL and rel_err(ff, np64(fu)) <= 2 * BF16_TOL


def test_fused_fp32_is_unsupported(cuda_lib):
    x = inputs.make_prefill("tiny_fp32", device="cuda", raw=True)
    with pytest.raises(KdaError):
        kda_chunk_fwd_fused(*(x[n] for n in NAMES))


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (64, 128)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_fused_decode_small(cuda_lib, dk, dv, dtype):
    d = inputs.make_decode("decode_bf16", device="cpu", raw=True, steps=4, B=3, H=5, dk=dk, dv=dv, dtype=dtype)
    state = d["state"].cuda()
    ref_s = d["state"].numpy().astype(np.float64)
    tol = BF16_TOL if dtype == torch.bfloat16 else FP32_TOL
    for t in range(4):
        o = kda_decode_step_fused(*(d[n][t].cuda() for n in NAMES), state)
        q, k, la, beta = oracle.prologue(*(np64(d[n][t]) for n in ("q", "k", "log_alpha", "beta")))
        ref_o, ref_s = oracle.decode_step(q, k, np64(d["v"][t]), la, beta, ref_s)
        assert rel_err(o, ref_o) <= tol
        assert rel_err(state, ref_s) <= tol
    assert device_error() == 0


def test_fused_chunk_length_32_and_key_width_64(cuda_lib):
    check_chunk(inputs.make_prefill("prefill_bf16", device="cpu", raw=True, B=1, T=200, H=2, dk=64, init_state=True))
    x = inputs.make_prefill("prefill_bf16", device="cpu", raw=True, B=1, T=333, H=2, init_state=True)
    dev = torch.device("cuda")
    out, fs = kda_chunk_fwd_fused(*(x[n].to(dev) for n in NAMES), initial_state=x["init_state"].to(dev),
                                  chunk_size=32)
    torch.cuda.synchronize()
    q, k, la, beta = oracle.prologue(*(np64(x[n]) for n in ("q", "k", "log_alpha", "beta")))
    ref_o, ref_s = oracle.recurrent(q, k, np64(x["v"]), la, beta, init_state=np64(x["init_state"]))
    assert rel_err(out, ref_o) <= BF16_TOL and rel_err(fs, ref_s) <= BF16_TOL
