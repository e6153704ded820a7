"""kda_chunk_fwd_static_ws: the prefill for callers that cannot allocate device memory.

Some callers (an engine that reserves all device memory up front and forbids
later allocations, code inside an allocation callback) cannot supply the
workspace kda_chunk_fwd asks for.  kda_chunk_fwd_static_ws takes its handoff
buffer from a fixed array inside the library instead.  This file checks,
through the C ABI, that two calls in a row give the same results as
kda_chunk_fwd (within the parity tolerance of the other tests; the array
keeps the previous call's contents, which must not leak into the next call),
also for more (sequence, head) pairs than the GPU runs chains at once.

Collected last on purpose (file name), and self-contained: it passes both
alone in a fresh process and after every other test.
"""
import ctypes

import pytest
import torch

import oracle
from gated_delta_rule_86_b200 import _lib, device_error, inputs, kda_chunk_fwd
from parity import BF16_TOL, NAMES, np64, rel_err

pytestmark = pytest.mark.gpu


def _static_ws(lib):
    vp, i32 = ctypes.c_void_p, ctypes.c_int32
    fn = lib.kda_chunk_fwd_static_ws
    fn.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, ctypes.c_int, ctypes.c_int, vp,
                   vp, vp]
    fn.restype = ctypes.c_int
    return fn


def _call(fn, x, out_dtype=torch.float32):
    q = x["q"]
    B, T, H, dk = q.shape
    dv = x["v"].shape[-1]
    cu = x["cu_seqlens"]
    N = B if cu is None else cu.numel() - 1
    out = torch.empty((B, T, H, dv), dtype=out_dtype, device="cuda")
    fs = torch.empty((N, H, dk, dv), dtype=torch.float32, device="cuda")
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = fn(*(ptr(x[n]) for n in NAMES), ptr(x["init_state"]), ptr(cu), N if cu is not None else 0, B, T, H, dk, dv,
            64, _lib.KDA_BF16, _lib.KDA_F32 if out_dtype == torch.float32 else _lib.KDA_BF16, ptr(out), ptr(fs),
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, out, fs


def _case(T, H, dv, seed, varlen=None):
    x = inputs.make_prefill("prefill_bf16", device="cuda", B=1, T=T, H=H, dv=dv, init_state=True, seed=seed)
    if varlen is not None:
        x["cu_seqlens"] = torch.tensor(varlen, dtype=torch.int32, device="cuda")
        x["init_state"] = torch.randn((len(varlen) - 1, H, 128, dv), device="cuda") * 0.1
    return x


def _check_same(fn, x):
    ref_o, ref_s = kda_chunk_fwd(*(x[n] for n in NAMES), initial_state=x["init_state"], cu_seqlens=x["cu_seqlens"])
    assert device_error() == 0
    st, out, fs = _call(fn, x)
    torch.cuda.synchronize()
    assert st == _lib.KDA_OK, _lib.status_string(st)
    assert device_error() == 0
    assert torch.equal(out, ref_o) and torch.equal(fs, ref_s)
    return out, fs


def test_two_calls_match_kda_chunk_fwd(cuda_lib):
    fn = _static_ws(cuda_lib)
    cases = [_case(T=700, H=6, dv=128, seed=11), _case(T=300, H=3, dv=64, seed=12, varlen=[0, 1, 130, 300])]
    for x in cases:
        _check_same(fn, x)
    # the first case once more: the array now holds the second case's images
    out, fs = _check_same(fn, cases[0])
    x = cases[0]
    ref_o, ref_s = oracle.recurrent(*(np64(x[n]) for n in NAMES), init_state=np64(x["init_state"]))
    assert rel_err(out, ref_o) <= BF16_TOL and rel_err(fs, ref_s) <= BF16_TOL


def test_more_pairs_than_chains(cuda_lib):
    # 70 (sequence, head) pairs: more than one wave of chains (at most a quarter of the SMs), so
    # chains run several pairs and the fixed array holds shallower rings
    fn = _static_ws(cuda_lib)
    x = _case(T=130, H=70, dv=128, seed=13)
    for _ in range(2):
        _check_same(fn, x)
