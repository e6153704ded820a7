"""Decode step parity against the fp64 oracle (GPU)."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_86_b200 import device_error, inputs, kda_decode_step
from parity import BF16_TOL, FP32_TOL, NAMES, np64, rel_err

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64), (64, 128)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_decode_small(cuda_lib, dk, dv, dtype):
    d = inputs.make_decode("decode_bf16", device="cpu", steps=5, B=3, H=5, dk=dk, dv=dv, dtype=dtype)
    state = d["state"].cuda()
    ref_s = d["state"].numpy().astype(np.float64)
    tol = BF16_TOL if dtype == torch.bfloat16 else FP32_TOL
    for t in range(5):
        o = kda_decode_step(*(d[n][t].cuda() for n in NAMES), state)
        ref_o, ref_s = oracle.decode_step(*(np64(d[n][t]) for n in NAMES), ref_s)
        assert rel_err(o, ref_o) <= tol
        assert rel_err(state, ref_s) <= tol
    assert device_error() == 0


def test_decode_full_size_sampled(cuda_lib):
    """Decode workload (B256 H32 d128, 1024 steps): every head for 4 steps, 64 sampled heads for all steps."""
    w = inputs.WORKLOADS["decode_bf16"]
    steps = w.decode_steps
    d = inputs.make_decode(w, device="cuda")
    state = d["state"].clone()
    rng = np.random.default_rng(5)
    flat = rng.choice(w.B * w.H, size=64, replace=False)
    bsel, hsel = flat // w.H, flat % w.H
    ref_sample = np64(d["state"][bsel, hsel])                # [64, dk, dv]
    ref_all = np64(d["state"])
    worst_o = worst_s = 0.0
    for t in range(steps):
        o = kda_decode_step(*(d[n][t] for n in NAMES), state)
        tok = {n: d[n][t][bsel, hsel].unsqueeze(1) for n in NAMES}   # [64, 1, .]
        ro, rs = oracle.decode_step(*(np64(tok[n]) for n in NAMES), ref_sample[:, None])
        ref_sample = rs[:, 0]
        worst_o = max(worst_o, rel_err(o[bsel, hsel], ro[:, 0]))
        if t < 4:
            ro_all, ref_all = oracle.decode_step(*(np64(d[n][t]) for n in NAMES), ref_all)
            assert rel_err(o, ro_all) <= BF16_TOL
            assert rel_err(state, ref_all) <= BF16_TOL
    worst_s = rel_err(state[bsel, hsel], ref_sample)
    assert worst_o <= BF16_TOL and worst_s <= BF16_TOL, (worst_o, worst_s)
    assert device_error() == 0


def test_decode_bf16_output_is_rounded_fp32_output(cuda_lib):
    d = inputs.make_decode("decode_bf16", device="cpu", steps=1, B=4, H=8)
    s1, s2 = d["state"].cuda(), d["state"].cuda()
    tok = [d[n][0].cuda() for n in NAMES]
    o32 = kda_decode_step(*tok, s1)
    o16 = kda_decode_step(*tok, s2, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.equal(o16, o32.to(torch.bfloat16)) and torch.equal(s1, s2)
