"""Python binding of the KDA C ABI (include/kda.h).

Argument marshalling only: shapes are checked, outputs are allocated with
torch (device memory is the only thing torch provides), pointers and the
current CUDA stream are passed to libkda_b200.so, and a non-OK status becomes
a :class:`KdaError`.  Every step of the computation runs in the library's
kernels; there is no CPU path.

Inputs that live in host memory (pinned CPU tensors) are copied to the current
CUDA device, and results are copied back into host tensors, on the same
stream: this is the end-to-end form of each call.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import KdaError  # noqa: F401  (re-exported)

_DTYPES = {torch.float32: _lib.KDA_F32, torch.bfloat16: _lib.KDA_BF16}


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _io_dtype(*ts):
    dt = ts[0].dtype
    if dt not in _DTYPES:
        raise TypeError(f"unsupported dtype {dt}; use torch.float32 or torch.bfloat16")
    for t in ts:
        if t is not None and t.dtype != dt:
            raise TypeError("q, k, v, the gate and beta must share one dtype")
    return _DTYPES[dt]


def _to_device(t, dev):
    if t is None or t.is_cuda:
        return t
    return t.to(dev, non_blocking=True)


def _prefill_prepare(q, k, v, log_alpha, beta, initial_state, cu_seqlens, per_head_gate=False):
    on_host = not q.is_cuda
    dev = torch.device("cuda", torch.cuda.current_device()) if on_host else q.device
    q, k, v, log_alpha, beta, initial_state, cu_seqlens = (
        _to_device(x, dev) for x in (q, k, v, log_alpha, beta, initial_state, cu_seqlens))
    q, k, v, beta = (x.contiguous() for x in (q, k, v, beta))
    if log_alpha is not None:
        log_alpha = log_alpha.contiguous()
    if q.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k must be [B, T, H, d_k] and v [B, T, H, d_v]")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    gate_shape = (B, T, H) if per_head_gate else q.shape
    if k.shape != q.shape or v.shape != (B, T, H, dv) or beta.shape != (B, T, H):
        raise ValueError("inconsistent shapes among q, k, v, beta")
    if log_alpha is None and not per_head_gate:
        raise ValueError("log_alpha is required")
    if log_alpha is not None and log_alpha.shape != gate_shape:
        raise ValueError(f"the gate must be {list(gate_shape)}")
    if cu_seqlens is not None:
        cu_seqlens = cu_seqlens.to(torch.int32).contiguous()
        if B != 1:
            raise ValueError("cu_seqlens requires B == 1")
        N = cu_seqlens.numel() - 1
    else:
        N = B
    if initial_state is not None:
        initial_state = initial_state.to(torch.float32).contiguous()
        if initial_state.shape != (N, H, dk, dv):
            raise ValueError(f"initial_state must be [{N}, {H}, {dk}, {dv}]")
    return on_host, (q, k, v, log_alpha, beta, initial_state, cu_seqlens), (B, T, H, dk, dv, N)


def _out_dtype(out_dtype):
    if out_dtype not in _DTYPES:
        raise TypeError(f"unsupported out_dtype {out_dtype}; use torch.float32 or torch.bfloat16")
    return _DTYPES[out_dtype]


def segment_bounds(T, segments, chunk_size):
    """Token ranges [a, b) of the host-buffer pipeline: at most ``segments`` of them, each starting at
    a multiple of ``chunk_size`` (so that the chunks are those of one call), covering [0, T)."""
    if T <= 0:
        return []
    seg = -(-T // max(1, segments))
    seg = -(-seg // chunk_size) * chunk_size
    return [(a, min(a + seg, T)) for a in range(0, T, seg)]


def _host_pipelined(fn_name, q, k, v, gate, beta, initial_state, chunk_size, out_dtype, segments):
    """The prefill of one sequence (B == 1) held in pinned host memory, in token segments whose
    host-to-device copies, kernels and device-to-host copies overlap: segment i's inputs travel on
    one copy stream while segment i-1 runs and segment i-2's output travels back on another.  The
    state passes from segment to segment on the device.  Segments start at multiples of the chunk
    length, so the chunks, and therefore the results, are exactly those of one call."""
    dev = torch.device("cuda", torch.cuda.current_device())
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    bounds = segment_bounds(T, segments, chunk_size)
    hosts = [q, k, v, gate, beta]
    devs = [None if t is None else torch.empty(t.shape, dtype=t.dtype, device=dev) for t in hosts]
    out_d = torch.empty((B, T, H, dv), dtype=out_dtype, device=dev)
    out_h = torch.empty((B, T, H, dv), dtype=out_dtype, pin_memory=True)
    st = [None, None]
    state = None
    if initial_state is not None:
        state = initial_state.to(dev, non_blocking=True).to(torch.float32).contiguous()
    compute = torch.cuda.current_stream()
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    h2d.wait_stream(compute)   # the device buffers are free for writing
    lib = _lib.load()
    dt = _io_dtype(*hosts)
    odt = _out_dtype(out_dtype)
    ws_bytes = ctypes.c_size_t(0)
    _lib.check(lib.kda_chunk_fwd_workspace_size(1, H, dk, dv, dt, ctypes.byref(ws_bytes)), "kda_chunk_fwd_workspace_size")
    ws = torch.empty(max(ws_bytes.value, 16), dtype=torch.uint8, device=dev)
    for i, (a, b) in enumerate(bounds):
        ev_in = torch.cuda.Event()
        with torch.cuda.stream(h2d):
            for hd, dd in zip(hosts, devs):
                if hd is not None:
                    dd[:, a:b].copy_(hd[:, a:b], non_blocking=True)
            ev_in.record(h2d)
        compute.wait_event(ev_in)
        fs = torch.empty((1, H, dk, dv), dtype=torch.float32, device=dev)
        st[i & 1] = fs
        segs = [None if dd is None else dd[:, a:b] for dd in devs]
        status = getattr(lib, fn_name)(*(_ptr(x) for x in segs), _ptr(state), None, ctypes.c_int32(0), 1, b - a, H, dk,
                                       dv, ctypes.c_int32(chunk_size), dt, odt, _ptr(out_d[:, a:b]), _ptr(fs),
                                       _ptr(ws), ctypes.c_size_t(ws.numel()), _stream_handle())
        _lib.check(status, fn_name)
        state = fs
        ev_out = torch.cuda.Event()
        ev_out.record(compute)
        d2h.wait_event(ev_out)
        with torch.cuda.stream(d2h):
            out_h[:, a:b].copy_(out_d[:, a:b], non_blocking=True)
    fs_h = None
    if state is not None:
        fs_h = torch.empty(state.shape, dtype=torch.float32, pin_memory=True)
        with torch.cuda.stream(d2h):
            fs_h.copy_(state, non_blocking=True)
    d2h.synchronize()
    compute.wait_stream(d2h)
    for t in devs + [out_d, ws] + st:
        if t is not None:
            t.record_stream(d2h)
    return out_h, fs_h


def _prefill(fn_name, q, k, v, log_alpha, beta, initial_state, cu_seqlens, output_final_state, chunk_size,
             out_dtype, host_segments=8):
    lib = _lib.load()
    if (host_segments and host_segments > 1 and not q.is_cuda and cu_seqlens is None and "_chunk_fwd" in fn_name
            and q.dim() == 4 and q.shape[0] == 1 and q.shape[1] >= 2 * host_segments * chunk_size
            and all(t is None or (t.is_pinned() and t.is_contiguous()) for t in (q, k, v, log_alpha, beta))):
        if log_alpha is None and not fn_name.startswith("gdn_"):
            raise ValueError("log_alpha is required")
        out_h, fs_h = _host_pipelined(fn_name, q, k, v, log_alpha, beta, initial_state, chunk_size, out_dtype,
                                      host_segments)
        return out_h, (fs_h if output_final_state else None)
    on_host, (q, k, v, la, beta, s0, cu), (B, T, H, dk, dv, N) = _prefill_prepare(
        q, k, v, log_alpha, beta, initial_state, cu_seqlens, per_head_gate=fn_name.startswith("gdn_"))
    dt = _io_dtype(q, k, v, la, beta)
    odt = _out_dtype(out_dtype)
    out = torch.empty((B, T, H, dv), dtype=out_dtype, device=q.device)
    fs = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device) if output_final_state else None
    args = [_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(beta), _ptr(s0), _ptr(cu),
            ctypes.c_int32(N if cu is not None else 0), B, T, H, dk, dv]
    if "_chunk_fwd" in fn_name:
        ws_bytes = ctypes.c_size_t(0)
        _lib.check(lib.kda_chunk_fwd_workspace_size(N, H, dk, dv, dt, ctypes.byref(ws_bytes)),
                   "kda_chunk_fwd_workspace_size")
        ws = torch.empty(ws_bytes.value, dtype=torch.uint8, device=q.device) if ws_bytes.value else None
        status = getattr(lib, fn_name)(*args, ctypes.c_int32(chunk_size), dt, odt, _ptr(out), _ptr(fs), _ptr(ws),
                                       ctypes.c_size_t(ws_bytes.value), _stream_handle())
    else:
        status = getattr(lib, fn_name)(*args, dt, odt, _ptr(out), _ptr(fs), _stream_handle())
    _lib.check(status, fn_name)
    if on_host:
        out_h = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        out_h.copy_(out, non_blocking=True)
        fs_h = None
        if fs is not None:
            fs_h = torch.empty(fs.shape, dtype=fs.dtype, pin_memory=True)
            fs_h.copy_(fs, non_blocking=True)
        torch.cuda.current_stream().synchronize()
        return out_h, fs_h
    return out, fs


def kda_chunk_fwd(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None, output_final_state=True,
                  chunk_size=64, out_dtype=torch.float32, host_segments=8):
    """Chunkwise-parallel KDA prefill; returns ``(out, final_state)``.

    q, k, log_alpha: [B, T, H, d_k]; v: [B, T, H, d_v]; beta: [B, T, H] (one
    dtype: bf16 or fp32).  initial_state: fp32 [N, H, d_k, d_v] or None;
    cu_seqlens: int32 [N+1] for packed sequences (B == 1) or None.  out has
    dtype ``out_dtype`` (fp32 by default, the accumulator precision).
    Inputs in pinned host memory are copied in and the results copied back;
    for one sequence (B == 1) this runs in ``host_segments`` token segments
    whose copies overlap the kernels (0 or 1: one copy in, one call, one
    copy out).
    """
    return _prefill("kda_chunk_fwd", q, k, v, log_alpha, beta, initial_state, cu_seqlens, output_final_state,
                    chunk_size, out_dtype, host_segments)


def kda_recurrent_fwd(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None, output_final_state=True,
                      out_dtype=torch.float32):
    """Token-by-token KDA prefill on CUDA cores (same contract as :func:`kda_chunk_fwd`)."""
    return _prefill("kda_recurrent_fwd", q, k, v, log_alpha, beta, initial_state, cu_seqlens, output_final_state,
                    64, out_dtype)


def _decode(fn_name, q, k, v, gate, beta, state, out, out_dtype):
    lib = _lib.load()
    if not state.is_cuda or state.dtype != torch.float32 or not state.is_contiguous():
        raise ValueError("state must be a contiguous fp32 CUDA tensor (it is updated in place)")
    on_host = not q.is_cuda
    q, k, v, beta = (_to_device(x, state.device).contiguous() for x in (q, k, v, beta))
    la = None if gate is None else _to_device(gate, state.device).contiguous()
    B, H, dk = q.shape
    dv = v.shape[-1]
    per_head = fn_name.startswith("gdn_")
    if la is None and not per_head:
        raise ValueError("log_alpha is required")
    if k.shape != q.shape or v.shape != (B, H, dv) or beta.shape != (B, H) or state.shape != (B, H, dk, dv) \
            or (la is not None and la.shape != ((B, H) if per_head else q.shape)):
        raise ValueError(f"inconsistent shapes for {fn_name}")
    dt = _io_dtype(q, k, v, la, beta)
    if out is not None:
        out_dtype = out.dtype
    odt = _out_dtype(out_dtype)
    o = out if (out is not None and out.is_cuda) else torch.empty((B, H, dv), dtype=out_dtype, device=state.device)
    status = getattr(lib, fn_name)(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(beta), _ptr(state), _ptr(o),
                                   B, H, dk, dv, dt, odt, _stream_handle())
    _lib.check(status, fn_name)
    if on_host:
        oh = out if out is not None else torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        oh.copy_(o, non_blocking=True)
        return oh
    return o


def kda_decode_step(q, k, v, log_alpha, beta, state, out=None, out_dtype=torch.float32):
    """One decode step; ``state`` (fp32 [B, H, d_k, d_v], on the GPU) is updated in place.

    q, k, log_alpha: [B, H, d_k]; v: [B, H, d_v]; beta: [B, H].  Returns out
    [B, H, d_v] of ``out_dtype`` (a host tensor when the token inputs were host
    tensors; ``out``, if given, receives the result).
    """
    return _decode("kda_decode_step", q, k, v, log_alpha, beta, state, out, out_dtype)


def gdn_chunk_fwd(q, k, v, log_g, beta, initial_state=None, cu_seqlens=None, output_final_state=True,
                  chunk_size=64, out_dtype=torch.float32, host_segments=8):
    """Gated DeltaNet prefill (one log-decay per head and token): :func:`kda_chunk_fwd` with
    ``log_g`` [B, T, H] in place of log_alpha; ``log_g=None`` is DeltaNet (no decay)."""
    return _prefill("gdn_chunk_fwd", q, k, v, log_g, beta, initial_state, cu_seqlens, output_final_state,
                    chunk_size, out_dtype, host_segments)


def gdn_recurrent_fwd(q, k, v, log_g, beta, initial_state=None, cu_seqlens=None, output_final_state=True,
                      out_dtype=torch.float32):
    """Token-by-token Gated DeltaNet / DeltaNet prefill (same contract as :func:`gdn_chunk_fwd`)."""
    return _prefill("gdn_recurrent_fwd", q, k, v, log_g, beta, initial_state, cu_seqlens, output_final_state,
                    64, out_dtype)


def gdn_decode_step(q, k, v, log_g, beta, state, out=None, out_dtype=torch.float32):
    """One Gated DeltaNet / DeltaNet decode step: :func:`kda_decode_step` with ``log_g`` [B, H]
    (or None: no decay) in place of log_alpha."""
    return _decode("gdn_decode_step", q, k, v, log_g, beta, state, out, out_dtype)


def kda_chunk_fwd_fused(q_raw, k_raw, v, g_raw, b_raw, initial_state=None, cu_seqlens=None,
                        output_final_state=True, chunk_size=64, out_dtype=torch.float32, host_segments=8):
    """:func:`kda_chunk_fwd` from the raw projections, activated inside the kernel's loads:
    q, k = L2-normalised q_raw, k_raw (over d_k, eps 1e-6 under the root), log_alpha =
    logsigmoid(g_raw), beta = sigmoid(b_raw).  Same shapes as kda_chunk_fwd; bf16 only."""
    return _prefill("kda_chunk_fwd_fused", q_raw, k_raw, v, g_raw, b_raw, initial_state, cu_seqlens,
                    output_final_state, chunk_size, out_dtype, host_segments)


def kda_decode_step_fused(q_raw, k_raw, v, g_raw, b_raw, state, out=None, out_dtype=torch.float32):
    """:func:`kda_decode_step` from the raw projections (see :func:`kda_chunk_fwd_fused`)."""
    return _decode("kda_decode_step_fused", q_raw, k_raw, v, g_raw, b_raw, state, out, out_dtype)


def kda_chunk_bwd(q, k, v, log_alpha, beta, d_out, initial_state=None, d_final_state=None, cu_seqlens=None,
                  chunk_size=64):
    """Gradient of :func:`kda_chunk_fwd` (reverse mode through the recurrence, fp32).

    Takes the forward's inputs and ``d_out`` = dLoss/dout ([B, T, H, d_v], fp32 or bf16) and,
    optionally, ``d_final_state`` = dLoss/dfinal_state (fp32 [N, H, d_k, d_v]).  Returns
    ``(dq, dk, dv, dlog_alpha, dbeta, d_initial_state)`` in fp32 with the shapes of q, k, v,
    log_alpha, beta and the initial state.  ``chunk_size`` is the checkpoint interval (0: the state
    before every token is kept, no recompute; more workspace, same result).
    """
    lib = _lib.load()
    on_host = not q.is_cuda
    _, (q, k, v, la, beta, s0, cu), (B, T, H, dk, dv, N) = _prefill_prepare(
        q, k, v, log_alpha, beta, initial_state, cu_seqlens)
    dt = _io_dtype(q, k, v, la, beta)
    d_out = _to_device(d_out, q.device).contiguous()
    if d_out.shape != (B, T, H, dv):
        raise ValueError("d_out must have the shape of the output")
    dodt = _out_dtype(d_out.dtype)
    dfin = None
    if d_final_state is not None:
        dfin = _to_device(d_final_state, q.device).to(torch.float32).contiguous()
        if dfin.shape != (N, H, dk, dv):
            raise ValueError(f"d_final_state must be [{N}, {H}, {dk}, {dv}]")
    f32 = dict(dtype=torch.float32, device=q.device)
    g = [torch.empty((B, T, H, dk), **f32), torch.empty((B, T, H, dk), **f32), torch.empty((B, T, H, dv), **f32),
         torch.empty((B, T, H, dk), **f32), torch.empty((B, T, H), **f32), torch.empty((N, H, dk, dv), **f32)]
    total = T if cu is not None else B * T
    ws_bytes = ctypes.c_size_t(0)
    _lib.check(lib.kda_chunk_bwd_workspace_size(N, H, total, dk, dv, chunk_size, ctypes.byref(ws_bytes)),
               "kda_chunk_bwd_workspace_size")
    ws = torch.empty(max(ws_bytes.value, 16), dtype=torch.uint8, device=q.device)
    status = lib.kda_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(beta), _ptr(s0), _ptr(cu),
                               ctypes.c_int32(N if cu is not None else 0), B, T, H, dk, dv,
                               ctypes.c_int32(chunk_size), dt, _ptr(d_out), dodt, _ptr(dfin),
                               *(_ptr(x) for x in g), _ptr(ws), ctypes.c_size_t(ws.numel()), _stream_handle())
    _lib.check(status, "kda_chunk_bwd")
    if on_host:
        out = []
        for x in g:
            hx = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
            hx.copy_(x, non_blocking=True)
            out.append(hx)
        torch.cuda.current_stream().synchronize()
        return tuple(out)
    return tuple(g)


class _KdaChunk(torch.autograd.Function):
    """Autograd wrapper: forward = kda_chunk_fwd, backward = kda_chunk_bwd (both in the library)."""

    @staticmethod
    def forward(ctx, q, k, v, log_alpha, beta, initial_state, cu_seqlens, chunk_size, out_dtype):
        out, fs = kda_chunk_fwd(q, k, v, log_alpha, beta, initial_state=initial_state, cu_seqlens=cu_seqlens,
                                output_final_state=True, chunk_size=chunk_size, out_dtype=out_dtype)
        ctx.save_for_backward(q, k, v, log_alpha, beta, initial_state, cu_seqlens)
        ctx.chunk_size = chunk_size
        return out, fs

    @staticmethod
    def backward(ctx, d_out, d_final_state):
        q, k, v, log_alpha, beta, s0, cu = ctx.saved_tensors
        if d_out is None:
            d_out = torch.zeros(v.shape, dtype=torch.float32, device=v.device)
        # the backward's chunk_size is its checkpoint interval (it changes no result)
        grads = kda_chunk_bwd(q, k, v, log_alpha, beta, d_out, initial_state=s0, d_final_state=d_final_state,
                              cu_seqlens=cu, chunk_size=ctx.chunk_size)
        dq, dk, dv, dla, db, ds0 = grads
        cast = [g.to(x.dtype) if (x is not None and ctx.needs_input_grad[i]) else None
                for i, (g, x) in enumerate(zip((dq, dk, dv, dla, db, ds0), (q, k, v, log_alpha, beta, s0)))]
        return (*cast, None, None, None)


def kda_chunk(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None, chunk_size=64,
              out_dtype=torch.float32):
    """Differentiable KDA prefill on CUDA tensors: ``(out, final_state)`` of :func:`kda_chunk_fwd`, with
    gradients (through :func:`kda_chunk_bwd`) for q, k, v, log_alpha, beta and the initial state, cast to
    their dtypes.  The gradient is that of the exact recurrence, evaluated in fp32."""
    if not q.is_cuda:
        raise ValueError("kda_chunk takes CUDA tensors")
    return _KdaChunk.apply(q, k, v, log_alpha, beta, initial_state, cu_seqlens, chunk_size, out_dtype)


def device_error() -> int:
    """Sync the current stream and return-and-clear the device error word (KDA_OK or KDA_ERR_TIMEOUT)."""
    return _lib.load().kda_get_last_device_error(_stream_handle())
