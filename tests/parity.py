"""Shared helpers of the parity tests: the error metric and input plumbing."""
import numpy as np
import torch

# max |x - ref| / rms(ref), per tensor
BF16_TOL = 2e-2
FP32_TOL = 1e-4

NAMES = ("q", "k", "v", "log_alpha", "beta")


def rel_err(x, ref):
    x = np.asarray(x.detach().float().cpu().numpy() if torch.is_tensor(x) else x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    assert np.all(np.isfinite(x)), "non-finite values in GPU result"
    rms = np.sqrt(np.mean(ref ** 2))
    return float(np.max(np.abs(x - ref)) / max(rms, 1e-300))


def np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64) if t is not None else None


def heads_slice(x, heads):
    """Inputs restricted to a subset of heads (index along the H axis)."""
    idx = torch.as_tensor(heads, device=x["q"].device)
    y = {n: x[n].index_select(2, idx) for n in NAMES}
    y["init_state"] = None if x["init_state"] is None else x["init_state"].index_select(1, idx)
    y["cu_seqlens"] = x["cu_seqlens"]
    return y
