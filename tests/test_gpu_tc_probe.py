"""tcgen05 building blocks: swizzled operand layouts, descriptors, TMEM readback.

Runs the test-only probe kernel (tests/csrc/tc_probe.cu), which uses the same
helpers and layouts as the chunk kernel, on each MMA shape the chunk kernel
issues, and compares D = A * B with a plain fp32 matmul of the same bf16 data.
"""
import ctypes
import os

import pytest
import torch

HERE = os.path.dirname(os.path.abspath(__file__))

# case id -> (M, N, K, A is MN-major, B is MN-major)
CASES = {0: (64, 64, 128, False, False), 1: (64, 128, 64, False, True), 2: (128, 64, 64, True, True),
         3: (64, 64, 128, False, True), 4: (64, 32, 128, False, True), 5: (128, 32, 64, True, True),
         6: (128, 128, 64, True, True), 7: (64, 128, 128, False, True),
         # A operand in TMEM (written with tcgen05.st), B K-major in shared memory
         8: (128, 64, 64, False, False), 9: (128, 128, 128, False, False)}


@pytest.fixture(scope="module")
def probe():
    if not torch.cuda.is_available():
        pytest.fail("GPU test collected without a CUDA device")
    lib = ctypes.CDLL(os.path.join(HERE, "csrc", "libtc_probe.so"))
    lib.tc_probe_run.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    lib.tc_probe_run.restype = ctypes.c_int
    return lib


@pytest.mark.gpu
@pytest.mark.parametrize("case", sorted(CASES))
def test_tcgen05_mma_layouts(probe, case):
    M, N, K, amn, bmn = CASES[case]
    g = torch.Generator(device="cuda").manual_seed(100 + case)
    A = torch.randn((K, M) if amn else (M, K), generator=g, device="cuda").to(torch.bfloat16)
    B = torch.randn((K, N) if bmn else (N, K), generator=g, device="cuda").to(torch.bfloat16)
    D = torch.full((M, N), float("nan"), device="cuda")
    assert probe.tc_probe_run(case, A.data_ptr(), B.data_ptr(), D.data_ptr()) == 0
    torch.cuda.synchronize()
    Am = A.float().t() if amn else A.float()
    Bm = B.float() if bmn else B.float().t()
    ref = Am @ Bm
    err = (D - ref).abs().max().item() / ref.abs().max().item()
    assert err < 1e-5, f"case {case}: rel err {err}"
