"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects malformed calls on the host before launching."""
import ctypes
import os
import re
import subprocess
import sys

import pytest
import torch

from gated_delta_rule_86_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "kda.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b((?:kda|gdn)_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from gated_delta_rule_86_b200 import build
    build.build_library()
    return _lib.load()


def test_header_matches_binding_list():
    assert declared_symbols() == sorted(_lib.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    names = [lib.kda_status_string(i).decode() for i in range(5)]
    assert names == ["KDA_OK", "KDA_ERR_INVALID_ARG", "KDA_ERR_UNSUPPORTED", "KDA_ERR_CUDA", "KDA_ERR_TIMEOUT"]
    assert lib.kda_version().decode().startswith("kda_b200")


FAKE = ctypes.c_void_p(1 << 20)        # aligned, never dereferenced: every call below is rejected first
ODD = ctypes.c_void_p((1 << 20) + 8)   # 8-byte aligned only


def chunk(lib, q=FAKE, B=1, T=128, H=2, dk=128, dv=128, chunk_size=64, dtype=_lib.KDA_BF16, cu=None, ns=0,
          s0=None, fs=None, out=FAKE, odt=_lib.KDA_F32, ws=FAKE, ws_bytes=1 << 30):
    return lib.kda_chunk_fwd(q, FAKE, FAKE, FAKE, FAKE, s0, cu, ns, B, T, H, dk, dv, chunk_size, dtype, odt, out,
                             fs, ws, ws_bytes, None)


def test_rejects_bad_arguments(lib):
    E, U = _lib.KDA_ERR_INVALID_ARG, _lib.KDA_ERR_UNSUPPORTED
    assert chunk(lib, q=None) == E
    assert chunk(lib, out=None) == E
    assert chunk(lib, B=0) == E
    assert chunk(lib, T=-1) == E
    assert chunk(lib, H=0) == E
    assert chunk(lib, q=ODD) == E
    assert chunk(lib, dtype=7) == E
    assert chunk(lib, odt=5) == E
    assert chunk(lib, chunk_size=0) == E
    assert chunk(lib, B=2, cu=FAKE, ns=3) == E          # packed batch needs B == 1
    assert chunk(lib, cu=FAKE, ns=0) == E
    assert chunk(lib, s0=FAKE, fs=ctypes.c_void_p((1 << 20) + 4096)) == E   # partial overlap
    assert chunk(lib, dk=96) == U
    assert chunk(lib, dv=256) == U
    assert chunk(lib, chunk_size=128) == U
    assert chunk(lib, dk=64, dtype=_lib.KDA_BF16) != U   # the tensor-core path takes d_k = 64 (zero-padded keys)
    assert chunk(lib, chunk_size=32) != U                # chunks of up to 64 tokens
    assert chunk(lib, ws=None) == E                      # tensor-core path needs its workspace
    assert chunk(lib, ws_bytes=1024) == E
    rec = lib.kda_recurrent_fwd(FAKE, FAKE, FAKE, FAKE, None, None, None, 0, 1, 8, 1, 64, 64, _lib.KDA_F32,
                                _lib.KDA_F32, FAKE, None, None)
    assert rec == E
    dec = lib.kda_decode_step
    assert dec(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1, 1, 128, 128, _lib.KDA_BF16, _lib.KDA_F32, None) == E
    assert dec(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 1, 128, 128, _lib.KDA_BF16, _lib.KDA_F32, None) == E
    assert dec(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 32, 128, _lib.KDA_BF16, _lib.KDA_F32, None) == U
    assert dec(ODD, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 128, _lib.KDA_BF16, _lib.KDA_F32, None) == E


def test_gdn_rejects_bad_arguments(lib):
    E, U = _lib.KDA_ERR_INVALID_ARG, _lib.KDA_ERR_UNSUPPORTED

    def gchunk(q=FAKE, gate=FAKE, B=1, T=128, dk=128, chunk_size=64, ws=FAKE, ws_bytes=1 << 30):
        return lib.gdn_chunk_fwd(q, FAKE, FAKE, gate, FAKE, None, None, 0, B, T, 2, dk, 128, chunk_size,
                                 _lib.KDA_BF16, _lib.KDA_F32, FAKE, None, ws, ws_bytes, None)

    assert gchunk(q=None) == E
    assert gchunk(B=0) == E
    assert gchunk(gate=ODD) == E                 # a given gate must be 16-byte aligned like every tensor
    assert gchunk(gate=None, ws=None) == E       # a null gate (DeltaNet) is fine; the missing workspace is not
    assert gchunk(dk=96) == U
    assert gchunk(chunk_size=128) == U
    # the per-channel gate of KDA stays mandatory
    assert lib.kda_chunk_fwd(FAKE, FAKE, FAKE, None, FAKE, None, None, 0, 1, 128, 2, 128, 128, 64, _lib.KDA_BF16,
                             _lib.KDA_F32, FAKE, None, FAKE, 1 << 30, None) == E
    assert lib.gdn_recurrent_fwd(FAKE, FAKE, FAKE, None, None, None, None, 0, 1, 8, 1, 64, 64, _lib.KDA_F32,
                                 _lib.KDA_F32, FAKE, None, None) == E   # beta missing
    dec = lib.gdn_decode_step
    assert dec(FAKE, FAKE, FAKE, None, FAKE, None, FAKE, 1, 1, 128, 128, _lib.KDA_BF16, _lib.KDA_F32, None) == E
    assert dec(FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, 1, 1, 32, 128, _lib.KDA_BF16, _lib.KDA_F32, None) == U
    assert lib.kda_decode_step(FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, 1, 1, 128, 128, _lib.KDA_BF16,
                               _lib.KDA_F32, None) == E


def test_fused_rejects_bad_arguments(lib):
    E, U = _lib.KDA_ERR_INVALID_ARG, _lib.KDA_ERR_UNSUPPORTED

    def fchunk(q=FAKE, g=FAKE, dtype=_lib.KDA_BF16, dk=128, ws=FAKE):
        return lib.kda_chunk_fwd_fused(q, FAKE, FAKE, g, FAKE, None, None, 0, 1, 128, 2, dk, 128, 64, dtype,
                                       _lib.KDA_F32, FAKE, None, ws, 1 << 30, None)

    assert fchunk(q=None) == E
    assert fchunk(g=None) == E                    # the gate's pre-activation is required
    assert fchunk(dtype=_lib.KDA_F32, dk=64) == U  # tensor-core path only
    assert fchunk(dk=64) != U
    assert fchunk(ws=None) == E
    dec = lib.kda_decode_step_fused
    assert dec(FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, 1, 1, 128, 128, _lib.KDA_BF16, _lib.KDA_F32, None) == E
    assert dec(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 96, 128, _lib.KDA_BF16, _lib.KDA_F32, None) == U


def test_workspace_size(lib):
    n = ctypes.c_size_t(7)
    assert lib.kda_chunk_fwd_workspace_size(2, 16, 128, 128, _lib.KDA_BF16, ctypes.byref(n)) == _lib.KDA_OK
    # schedule tables plus, for each of the 32 chains (one per (seq, head) pair), a ring of 12 chunk
    # images (-W, U^T, Qg, Kd, P, gamma: 73 KB at d_v = 128)
    assert n.value >= 32 * 12 * 73 * 1024 and n.value < 32 * 12 * 74 * 1024 + 16 * 1024
    assert lib.kda_chunk_fwd_workspace_size(2, 16, 128, 64, _lib.KDA_BF16, ctypes.byref(n)) == _lib.KDA_OK
    assert 32 * 12 * 64 * 1024 <= n.value < 32 * 12 * 73 * 1024
    # at most 64 rings, however many pairs
    assert lib.kda_chunk_fwd_workspace_size(64, 16, 128, 128, _lib.KDA_BF16, ctypes.byref(n)) == _lib.KDA_OK
    assert n.value < 64 * 12 * 74 * 1024 + 16 * 1024
    assert lib.kda_chunk_fwd_workspace_size(2, 16, 64, 64, _lib.KDA_F32, ctypes.byref(n)) == _lib.KDA_OK
    assert n.value == 0
    assert lib.kda_chunk_fwd_workspace_size(0, 16, 128, 128, _lib.KDA_BF16, ctypes.byref(n)) == \
        _lib.KDA_ERR_INVALID_ARG


def test_workspace_size_rejects_what_the_prefill_rejects(lib):
    """The size query answers KDA_ERR_UNSUPPORTED (size 0) exactly for the head sizes that
    kda_chunk_fwd itself rejects as unsupported, so a query never succeeds for a shape the
    prefill cannot run."""
    n = ctypes.c_size_t(7)
    for dk, dv, dt in [(96, 128, _lib.KDA_BF16), (128, 96, _lib.KDA_BF16), (96, 64, _lib.KDA_F32)]:
        n.value = 7
        assert lib.kda_chunk_fwd_workspace_size(2, 16, dk, dv, dt, ctypes.byref(n)) == _lib.KDA_ERR_UNSUPPORTED
        assert n.value == 0
    # shapes the prefill accepts get a size (fp32: the CUDA-core path, no workspace)
    for dk, dv, dt in [(128, 64, _lib.KDA_BF16), (64, 128, _lib.KDA_BF16), (64, 64, _lib.KDA_F32),
                       (64, 128, _lib.KDA_F32)]:
        assert lib.kda_chunk_fwd_workspace_size(2, 16, dk, dv, dt, ctypes.byref(n)) == _lib.KDA_OK


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", os.path.join(ROOT, "no_such_dir", "libkda_b200.so"))
    with pytest.raises(ImportError):
        _lib.load()


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the behaviour without a GPU")
def test_no_cpu_fallback_without_gpu():
    """Without a GPU every public call raises; nothing is computed on the CPU."""
    import gated_delta_rule_86_b200 as kda
    q = torch.zeros(1, 4, 1, 64)
    g = torch.zeros(1, 4, 1)
    calls = [
        lambda: kda.kda_chunk_fwd(q, q, q, q, g),
        lambda: kda.kda_recurrent_fwd(q, q, q, q, g),
        lambda: kda.gdn_chunk_fwd(q, q, q, g, g),
        lambda: kda.kda_chunk_fwd_fused(q, q, q, q, g),
        lambda: kda.kda_decode_step(q[:, 0], q[:, 0], q[:, 0], q[:, 0], g[:, 0], torch.zeros(1, 1, 64, 64)),
    ]
    for call in calls:
        with pytest.raises((RuntimeError, ValueError, AssertionError)):
            call()
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--steps", "1", "--warmup", "3",
                        "--no-cpu-baseline"], capture_output=True, text=True, cwd=ROOT, timeout=300)
    assert r.returncode != 0 and not any(ln.startswith("{") for ln in r.stdout.splitlines())


def test_backward_argument_checks(lib):
    """kda_chunk_bwd validates on the host before launching anything."""
    n = ctypes.c_size_t(7)
    assert lib.kda_chunk_bwd_workspace_size(2, 4, 1000, 128, 128, 64, ctypes.byref(n)) == _lib.KDA_OK
    # checkpoints (total/C + N + 1 per head) and one chunk of per-token states per (sequence, head)
    kv = 128 * 128 * 4
    assert n.value == 4 * (1000 // 64 + 2 + 1) * kv + 2 * 4 * 64 * kv
    assert lib.kda_chunk_bwd_workspace_size(2, 4, 1000, 96, 128, 64, ctypes.byref(n)) == _lib.KDA_ERR_UNSUPPORTED
    # chunk 0: the state before every token is kept (one state per token and head), no recompute
    assert lib.kda_chunk_bwd_workspace_size(2, 4, 1000, 128, 128, 0, ctypes.byref(n)) == _lib.KDA_OK
    assert n.value == 4 * 1000 * kv
    assert lib.kda_chunk_bwd_workspace_size(2, 4, 1000, 128, 128, -1, ctypes.byref(n)) == _lib.KDA_ERR_INVALID_ARG
    assert lib.kda_chunk_bwd_workspace_size(2, 4, 1000, 128, 128, 512, ctypes.byref(n)) == _lib.KDA_ERR_UNSUPPORTED
    F = ctypes.c_void_p(4096)
    bwd = lib.kda_chunk_bwd

    def call(dk=128, dq=F, ws=F, ws_bytes=1 << 40, chunk=64, T=16):
        return bwd(F, F, F, F, F, None, None, 0, 1, T, 2, dk, 128, chunk, _lib.KDA_BF16, F, _lib.KDA_F32, None,
                   dq, F, F, F, F, None, ws, ctypes.c_size_t(ws_bytes), None)

    assert call(dk=96) == _lib.KDA_ERR_UNSUPPORTED
    assert call(dq=None) == _lib.KDA_ERR_INVALID_ARG
    assert call(ws=None) == _lib.KDA_ERR_INVALID_ARG
    assert call(ws_bytes=16) == _lib.KDA_ERR_INVALID_ARG
    assert call(chunk=-1) == _lib.KDA_ERR_INVALID_ARG
    assert call(chunk=300) == _lib.KDA_ERR_UNSUPPORTED
    assert call(dq=ctypes.c_void_p(4100)) == _lib.KDA_ERR_INVALID_ARG   # misaligned
