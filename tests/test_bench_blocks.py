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


def test_prefill_block_bytes_follow_out_dtype(monkeypatch):
    seen = []

    def fake_chunk(q, k, v, la, beta, initial_state=None, cu_seqlens=None, out_dtype=None, chunk_size=64):
        seen.append(out_dtype)
        return None, None

    monkeypatch.setattr(pkg, "kda_chunk_fwd", fake_chunk)
    monkeypatch.setattr(bench, "barrier", lambda world, device="cuda": None)
    monkeypatch.setattr(bench, "event_time_ms", lambda fn, n: [fn(i) for i in range(n)] and 3.0 * n)
    B, T, H, d = 1, 256, 2, 128
    z = torch.zeros(B, T, H, d)
    from gated_delta_rule_86_b200 import inputs
    x = dict(q=z, k=z, v=z, log_alpha=z, beta=torch.zeros(B, T, H), init_state=None, cu_seqlens=None,
             workload=inputs.WORKLOADS["prefill_bf16"])
    args = SimpleNamespace(warmup=3, steps=4)
    o32 = bench.prefill_block(args, 1, x, 6000.0)
    o16 = bench.prefill_block(args, 1, x, 6000.0, out_dtype=torch.bfloat16)
    assert seen == [torch.float32] * 7 + [torch.bfloat16] * 7
    assert o32["ms_per_step"] == 3.0 and o32["tokens_per_s"] == B * T / 3e-3
    # fp32 output: 1538 B per token-head; bf16 output: 1282 B (plus the state once per sequence-head)
    state = B * H * 2 * d * d * 4
    assert o32["roofline"]["alg_bytes_per_launch"] == B * T * H * 1538 + state
    assert o16["roofline"]["alg_bytes_per_launch"] == B * T * H * 1282 + state
    json.dumps(o32)


def test_traffic_record_needs_the_current_build(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    for d in bench.LIB_SOURCES:
        (tmp_path / d).mkdir(parents=True)
    (tmp_path / "include" / "kda.h").write_text("int x;\n")
    csrc = tmp_path / bench.LIB_SOURCES[0]
    for f in {f for fs in bench.KERNEL_SOURCES.values() for f in fs}:
        (csrc / f).write_text("// " + f + "\n")
    (csrc / "kda_api.cu").write_text("// api\n")
    h = bench.build_hash()
    assert h == bench.build_hash() and len(h) == 16
    hk = bench.build_hash("kda_chunk_tc_kernel")
    assert len(hk) == 16 and hk != h and hk != bench.build_hash("kda_decode_kernel")
    rec = {"build": hk, "kernel": "kda_chunk_tc_kernel", "workload": "long_bf16", "dram_bytes": 1000, "units": 10}
    (tmp_path / "profiles" / "k.md").write_text("# summary\ntraffic-record: " + json.dumps(rec) + "\n")
    got = bench.traffic_record("kda_chunk_tc_kernel", "long_bf16")
    assert got is not None and got["dram_bytes"] == 1000 and got["file"] == os.path.join("profiles", "k.md")
    assert bench.traffic_record("kda_chunk_tc_kernel", "prefill_bf16") is None
    assert bench.traffic_record("kda_decode_kernel", "long_bf16") is None
    # changes outside the kernel's own sources leave the record valid ...
    (tmp_path / "include" / "kda.h").write_text("int y;\n")
    (csrc / "kda_api.cu").write_text("// api 2\n")
    (csrc / "kda_backward.cuh").write_text("// changed\n")
    assert bench.build_hash() != h and bench.build_hash("kda_chunk_tc_kernel") == hk
    assert bench.traffic_record("kda_chunk_tc_kernel", "long_bf16") is not None
    # ... and any change to one of them makes it stale
    (csrc / "tc_utils.cuh").write_text("// changed\n")
    assert bench.build_hash("kda_chunk_tc_kernel") != hk
    assert bench.traffic_record("kda_chunk_tc_kernel", "long_bf16") is None


def test_cpu_model_is_text_or_none():
    m = bench.cpu_model()
    assert m is None or (isinstance(m, str) and m)


class _FakeNvml:
    """Stands in for pynvml: fixed clocks and power, reason bits that change after a few samples."""
    NVML_CLOCK_SM = 1

    def __init__(self):
        self.calls = 0
        self.shutdown = False

    def nvmlInit(self):
        pass

    def nvmlShutdown(self):
        self.shutdown = True

    def nvmlDeviceGetHandleByUUID(self, uuid):
        return "h"

    def nvmlDeviceGetHandleByIndex(self, i):
        return "h"

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        assert kind == self.NVML_CLOCK_SM
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        self.calls += 1
        return 1965 if self.calls % 2 else 1950

    def nvmlDeviceGetPowerUsage(self, h):
        return 250000 + 1000 * self.calls   # mW

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return 0x4 if self.calls > 3 else 0x1   # sw_power_cap after a while; 0x1 (idle) is not reported


def test_clock_sampler_nvml_summary():
    import time
    fake = _FakeNvml()
    with bench.ClockSampler(0, nvml=fake) as clk:
        time.sleep(0.1)
    s = clk.summary()
    assert fake.shutdown and s["source"].startswith("nvml")
    assert s["samples"] >= 5 and s["sm_max_mhz"] == 1965 and s["sm_mhz"] in (1950, 1957.5, 1965)
    assert s["reasons"] == ["sw_power_cap"]
    assert s["power_w_max"] >= 250.0
    json.dumps(s)
