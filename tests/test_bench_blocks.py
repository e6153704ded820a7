"""Host logic of bench.py's auxiliary measurement blocks, on CPU with the kernel call faked."""
import json
import os
import sys
from types import SimpleNamespace

import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
import gated_delta_rule_86_b200 as pkg  # noqa: E402


def test_gdn_prefill_block(monkeypatch):
    calls = []

    def fake_gdn(q, k, v, log_g, beta, initial_state=None):
        assert log_g.shape == q.shape[:3] and log_g.is_contiguous()
        assert torch.equal(log_g, calls_src[3][..., 0])
        calls.append(1)
        return None, None

    monkeypatch.setattr(pkg, "gdn_chunk_fwd", fake_gdn)
    monkeypatch.setattr(bench, "barrier", lambda world, device="cuda": None)

    def fake_time(fn, n):
        for i in range(n):
            fn(i)
        return 2.0 * n

    monkeypatch.setattr(bench, "event_time_ms", fake_time)
    B, T, H, d = 1, 128, 4, 128
    g = torch.Generator().manual_seed(0)
    calls_src = [torch.randn(B, T, H, d, generator=g) for _ in range(4)] + [torch.rand(B, T, H, generator=g)]
    out = bench.gdn_prefill_block(SimpleNamespace(warmup=3, steps=5), 1, calls_src, None, B * T, B * T * H, 6000.0)
    assert len(calls) == 8 and out["ms_per_step"] == 2.0
    assert out["tokens_per_s"] == B * T / 2e-3
    alg = bench.prefill_alg_bytes(B * T * H, B * H) - B * T * H * (d - 1) * 2
    assert out["roofline"]["alg_bytes_per_launch"] == alg
    assert abs(out["roofline"]["frac"] - alg / 2e-3 / 1e9 / 6000.0) < 1e-12
    json.dumps(out)
