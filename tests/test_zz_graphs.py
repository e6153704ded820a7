"""CUDA graphs: the prefill's static-workspace entry point and the decode step captured into a
torch.cuda.CUDAGraph and replayed on new inputs (copied into the captured buffers) give bitwise the
results of eager calls on those inputs.

The static-workspace prefill allocates nothing, so it can be captured; its first call (before the
capture) looks up the library array's address.  Self-contained; collected after the other GPU tests.
"""
import ctypes

import pytest
import torch

from gated_delta_rule_86_b200 import _lib, device_error, inputs, kda_decode_step
from parity import NAMES

pytestmark = pytest.mark.gpu


def _static_ws(lib):
    vp, i32 = ctypes.c_void_p, ctypes.c_int32
    fn = lib.kda_chunk_fwd_static_ws
    fn.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, ctypes.c_int, ctypes.c_int, vp,
                   vp, vp]
    fn.restype = ctypes.c_int
    return fn


def _prefill(fn, x, out, fs, stream):
    B, T, H, dk = x["q"].shape
    dv = x["v"].shape[-1]
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    return fn(*(ptr(x[n]) for n in NAMES), ptr(x["init_state"]), None, 0, B, T, H, dk, dv, 64, _lib.KDA_BF16,
              _lib.KDA_F32, ptr(out), ptr(fs), ctypes.c_void_p(stream.cuda_stream))


def _inputs(seed):
    return inputs.make_prefill("prefill_bf16", device="cuda", B=1, T=333, H=4, init_state=True, seed=seed)


def test_prefill_static_ws_graph_replay(cuda_lib):
    fn = _static_ws(cuda_lib)
    x = _inputs(31)
    out = torch.empty(x["v"].shape, dtype=torch.float32, device="cuda")
    fs = torch.empty(x["init_state"].shape, dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        assert _prefill(fn, x, out, fs, s) == _lib.KDA_OK   # outside capture: looks the array up
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        st = _prefill(fn, x, out, fs, s)
    assert st == _lib.KDA_OK, _lib.status_string(st)
    for seed in (32, 33):
        y = _inputs(seed)
        for n in NAMES + ("init_state",):
            x[n].copy_(y[n])
        g.replay()
        torch.cuda.synchronize()
        ref_o = torch.empty_like(out)
        ref_s = torch.empty_like(fs)
        assert _prefill(fn, y, ref_o, ref_s, torch.cuda.current_stream()) == _lib.KDA_OK
        torch.cuda.synchronize()
        assert device_error() == 0
        assert torch.equal(out, ref_o) and torch.equal(fs, ref_s)
    del g


def test_decode_loop_graph_replay(cuda_lib):
    steps = 8
    d = inputs.make_decode("decode_bf16", device="cuda", steps=steps, B=8, H=4)
    tok = [d[n].clone() for n in NAMES]        # [steps, B, H, ...] static token buffers
    state = d["state"].clone()
    outs = torch.empty((steps,) + d["v"].shape[1:], dtype=torch.float32, device="cuda")

    def run(t, st, o):
        for i in range(steps):
            kda_decode_step(*(x[i] for x in t), st, out=o[i])

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run(tok, state.clone(), outs)   # warm-up outside capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        run(tok, state, outs)
    e = inputs.make_decode("decode_bf16", device="cuda", steps=steps, B=8, H=4, seed=77)
    for x, y in zip(tok, (e[n] for n in NAMES)):
        x.copy_(y)
    state.copy_(e["state"])
    g.replay()
    torch.cuda.synchronize()
    ref_state = e["state"].clone()
    ref_out = torch.empty_like(outs)
    run([e[n] for n in NAMES], ref_state, ref_out)
    torch.cuda.synchronize()
    assert device_error() == 0
    assert torch.equal(outs, ref_out) and torch.equal(state, ref_state)
    del g
