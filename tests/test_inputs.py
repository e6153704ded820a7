"""The seeded input generator (CPU): the raw-projection option draws the same numbers as the
default stream, before their activations, and leaves the default stream unchanged."""
import torch

from gated_delta_rule_86_b200 import inputs


def _same_draws(a, b, rtol):
    """a: the default input; b: the activation of the raw input.  The raw side was rounded to bf16
    before its activation, the default side after it, so they differ by a few bf16 roundings (a
    gate g near 4 moves logsigmoid(g) by about |g| 2^-8 relative); other draws would differ at O(1)."""
    return torch.allclose(a.float(), b.float(), rtol=rtol, atol=1e-5)


def test_raw_option_is_the_default_stream_before_activation():
    kw = dict(device="cpu", B=1, T=50, H=2, init_state=True)
    x = inputs.make_prefill("prefill_bf16", **kw)
    r = inputs.make_prefill("prefill_bf16", raw=True, **kw)
    assert torch.equal(x["v"], r["v"]) and torch.equal(x["init_state"], r["init_state"])
    qr, kr = r["q"].float(), r["k"].float()
    assert _same_draws(x["q"], qr / qr.norm(dim=-1, keepdim=True), 1e-2)
    assert _same_draws(x["k"], kr / kr.norm(dim=-1, keepdim=True), 1e-2)
    assert _same_draws(x["beta"], torch.sigmoid(r["beta"].float()), 1e-2)
    assert _same_draws(x["log_alpha"], torch.nn.functional.logsigmoid(r["log_alpha"].float()), 3e-2)
    # and a different seed is far away
    y = inputs.make_prefill("prefill_bf16", seed=7, raw=True, **kw)
    assert not _same_draws(x["beta"], torch.sigmoid(y["beta"].float()), 0.2)


def test_decode_raw_option_matches():
    d = inputs.make_decode("decode_bf16", device="cpu", steps=2, B=2, H=3)
    r = inputs.make_decode("decode_bf16", device="cpu", steps=2, B=2, H=3, raw=True)
    assert torch.equal(d["state"], r["state"]) and torch.equal(d["v"], r["v"])
    assert _same_draws(d["beta"], torch.sigmoid(r["beta"].float()), 1e-2)


def test_seeds_are_deterministic():
    a = inputs.make_prefill("prefill_bf16", device="cpu", B=1, T=20, H=2)
    b = inputs.make_prefill("prefill_bf16", device="cpu", B=1, T=20, H=2)
    for n in ("q", "k", "v", "log_alpha", "beta"):
        assert torch.equal(a[n], b[n])
