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


def heads_slice(x, heads, names=NAMES):
    """Inputs restricted to a subset of heads (index along the H axis)."""
    idx = torch.as_tensor(heads, device=x["q"].device)
    y = {n: (None if x[n] is None else x[n].index_select(2, idx)) for n in names}
    y["init_state"] = None if x["init_state"] is None else x["init_state"].index_select(1, idx)
    y["cu_seqlens"] = x["cu_seqlens"]
    return y


def head_groups(H, group):
    return [list(range(h, min(h + group, H))) for h in range(0, H, group)]


def check_heads_in_groups(out, fs, x, ref_fn, tol, group=16, names=NAMES):
    """Compares a GPU result over ALL heads with the oracle, which runs on groups of `group` heads
    at a time so that the fp64 host copies stay bounded.  `ref_fn(xs)` returns the oracle's
    (out, final_state) for the head subset xs.  The metric is the same as rel_err over the whole
    tensors: the largest |gpu - oracle| over all heads divided by the rms of the whole oracle
    tensor.  Returns the (out, state) errors."""
    H = x["q"].shape[2]
    acc = {"o": [0.0, 0.0, 0], "s": [0.0, 0.0, 0]}   # max |d|, sum ref^2, count

    def add(key, got, ref):
        got = np.asarray(got.detach().float().cpu().numpy(), dtype=np.float64)
        ref = np.asarray(ref, dtype=np.float64)
        assert got.shape == ref.shape, (got.shape, ref.shape)
        assert np.all(np.isfinite(got)), "non-finite values in GPU result"
        a = acc[key]
        a[0] = max(a[0], float(np.max(np.abs(got - ref))) if got.size else 0.0)
        a[1] += float(np.sum(ref * ref))
        a[2] += ref.size

    for hs in head_groups(H, group):
        xs = heads_slice(x, hs, names)
        ref_o, ref_s = ref_fn(xs)
        idx = torch.as_tensor(hs, device=out.device)
        add("o", out.index_select(2, idx), ref_o)
        add("s", fs.index_select(1, idx), ref_s)
    eo, es = (a[0] / max(np.sqrt(a[1] / max(a[2], 1)), 1e-300) for a in (acc["o"], acc["s"]))
    assert eo <= tol and es <= tol, f"all {H} heads: out {eo:.3e} state {es:.3e} (tol {tol})"
    return eo, es
