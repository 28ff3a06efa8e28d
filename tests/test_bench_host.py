"""Host-side logic of bench.py, on CPU: the roofline arithmetic, the gate on the
committed ncu traffic, and the sizing of the oracle sample in the reference arm."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from moe_inputs import CONFIGS  # noqa: E402

PEAKS = {"hbm_gbs": 6000.0, "bf16_tflops_sustained": 1000.0, "bf16_tflops": 1500.0}


def test_roof_entry_rates_and_binding_resource():
    # 2 launches per step, 2 ms each: per launch 1 TFLOP and 1 GB
    e = bench.roof_entry({"flop": 2e12, "byte": 2e9}, 2.0, 2, PEAKS)
    assert e["tensor"]["per_launch"] == 1e12 and e["hbm"]["per_launch"] == 1e9
    assert e["tensor"]["achieved"] == pytest.approx(500.0)     # TFLOP/s
    assert e["tensor"]["frac"] == pytest.approx(0.5)
    assert e["hbm"]["achieved"] == pytest.approx(500.0)        # GB/s
    assert e["hbm"]["frac"] == pytest.approx(500.0 / 6000.0)
    # ideal times 1 ms (tensor) against 0.17 ms (HBM): the tensor pipe binds
    assert e["bound"] == "tensor"
    # a byte-heavy kernel: 1 ms of HBM against 1 us of tensor
    assert bench.roof_entry({"flop": 1e9, "byte": 6e9}, 2.0, 1, PEAKS)["bound"] == "hbm"
    assert "tensor" not in bench.roof_entry({"byte": 1e6}, 1.0, 1, PEAKS)


def test_gate_up_forward_bytes_at_the_qwen_shape():
    # W_gu, sorted X, bf16(c XA), B_gu, and GU and H written, each once, in bf16
    cfg = CONFIGS["qwen3_30b_a3b"]
    P = cfg.T * cfg.k
    want = (cfg.E * cfg.m * 2 * cfg.n + P * cfg.m + P * 16 + cfg.E * 16 * 2 * cfg.n
            + P * 2 * cfg.n + P * cfg.n) * 2
    assert bench.kernel_work(cfg)["gemm_gateup_fwd"]["byte"] == want == 1_097_859_072
    # only the experts that received tokens have their weights read
    fewer = bench.kernel_work(cfg, active_experts=64)["gemm_gateup_fwd"]["byte"]
    assert want - fewer == 64 * (cfg.m * 2 * cfg.n + 16 * 2 * cfg.n) * 2


def test_rank_padding_of_the_lora_operands():
    # the [P, rp] rank-r operands are padded to 16, 32, 64 or 128 columns
    base = CONFIGS["qwen3_30b_a3b"]
    P = base.T * base.k
    from moe_inputs import LayerConfig
    for r, rp in ((8, 16), (16, 16), (24, 32), (48, 64), (64, 64), (96, 128), (128, 128)):
        cfg = LayerConfig("x", T=base.T, m=base.m, n=base.n, E=base.E, k=base.k, r=r, alpha=r)
        w = bench.kernel_work(cfg)
        assert w["rank_ha"]["byte"] == (P * cfg.n * 2 + cfg.E * cfg.n * r * 2 + P * r * 2
                                        + P * rp * 2)


def test_ncu_traffic_only_while_the_sources_match(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps(
        {"src_hash": "abc", "kernels": {"shape": {"gemm": {"dram_bytes_per_launch": 123}}}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "src_hash", lambda: "abc")
    assert bench.ncu_traffic("gemm", "shape") == 123
    assert bench.ncu_traffic("other", "shape") is None
    assert bench.ncu_traffic("gemm", "other") is None
    monkeypatch.setattr(bench, "src_hash", lambda: "changed")
    assert bench.ncu_traffic("gemm", "shape") is None


def test_src_hash_covers_every_kernel_source(tmp_path, monkeypatch):
    csrc = tmp_path / "mixture_experts_lora_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "a.cu").write_text("x")
    (csrc / "b.cuh").write_text("y")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.src_hash()
    (csrc / "b.cuh").write_text("y ")
    assert bench.src_hash() != h0


def test_oracle_sample_doubles_while_a_step_stays_under_half_the_budget(monkeypatch):
    cfg = CONFIGS["qwen3_30b_a3b"]
    seen = []

    def step_time(cfg_, cpu, W64, tok0, n):
        seen.append(n)
        return 0.2 + 0.001 * n              # a fixed part plus a part per token

    monkeypatch.setattr(bench, "time_oracle_sample", step_time)
    # 256 tokens take 0.456 s (< 0.5), 512 take 0.712 s: stop at 512
    assert bench.pick_sample_tokens(cfg, None, None, 1.0, 0) == 512
    assert seen[0] == 64 and max(seen) == 512
    # an explicit request wins, and the sample never exceeds the workload
    assert bench.pick_sample_tokens(cfg, None, None, 1.0, 77) == 77
    monkeypatch.setattr(bench, "time_oracle_sample", lambda *a: 1e-4)
    assert bench.pick_sample_tokens(cfg, None, None, 1.0, 0) == cfg.T
