"""The prefill's failure path on the GPU, made to happen without a GPU fault.

Every wait of the tensor-core prefill on another CTA is bounded.  The library's
testing hook (kda_testing_set_chunk_fault) makes one producer leave one chunk
image unpublished and shortens the flag-wait limit to 20 ms.  The chain that
needs that image must then give up on its own: it records KDA_ERR_TIMEOUT in
the device error word and raises the launch's abort word, every CTA leaves its
loops, frees its Tensor Memory and returns.  The host reads the status, and a
normal call on the same device afterwards must still give correct results.
"""
import time

import pytest
import torch

import oracle
from gated_delta_rule_86_b200 import _lib, device_error, inputs, kda_chunk_fwd
from parity import BF16_TOL, NAMES, np64, rel_err

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("skip_item", [0, 5, 37])
def test_missing_chunk_image_times_out_and_recovers(cuda_lib, skip_item):
    # 4 (sequence, head) pairs of 16 chunks: 4 chains, 64 producer items
    x = inputs.make_prefill("prefill_bf16", device="cuda", B=1, T=1024, H=4, init_state=True, seed=21)
    assert device_error() == 0
    assert cuda_lib.kda_testing_set_chunk_fault(skip_item, 20000) == _lib.KDA_OK
    try:
        t0 = time.perf_counter()
        kda_chunk_fwd(*(x[n] for n in NAMES), initial_state=x["init_state"])
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
    finally:
        assert cuda_lib.kda_testing_set_chunk_fault(-1, 0) == _lib.KDA_OK
    assert device_error() == _lib.KDA_ERR_TIMEOUT
    assert elapsed < 5.0, f"the launch took {elapsed:.2f} s to give up"
    # the context is still usable and the next launch is correct
    out, fs = kda_chunk_fwd(*(x[n] for n in NAMES), initial_state=x["init_state"])
    torch.cuda.synchronize()
    assert device_error() == 0
    ref_o, ref_s = oracle.recurrent(*(np64(x[n]) for n in NAMES), init_state=np64(x["init_state"]))
    assert rel_err(out, ref_o) <= BF16_TOL and rel_err(fs, ref_s) <= BF16_TOL


def test_fault_hook_rejects_bad_item(cuda_lib):
    assert cuda_lib.kda_testing_set_chunk_fault(-2, 0) == _lib.KDA_ERR_INVALID_ARG
    assert cuda_lib.kda_testing_set_chunk_fault(-1, 0) == _lib.KDA_OK
