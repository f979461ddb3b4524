"""The benchmark's roofline arithmetic on the CPU: algorithmic bytes and flops
per decode phase against the definitions written out by hand (quantized
latent: codes at 4/3 bits plus one fp16 scale per 32-channel group; scoring
2 r_h d flops per (token, query head); value contraction 2 r_v per (token,
query head); output 2 H r_v D per sequence)."""
import dataclasses
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from synth import gen  # noqa: E402


def test_latent_bytes_by_hand():
    spec = gen.config_spec(2)
    # rank 32 at 25 %: 8 channels x 4 bits + 24 x 3 bits = 104 bits = 13 B, two groups -> 4 B of scales
    assert bench.latent_bytes(spec, 32) == 13 + 4
    # rank 1024: 256 x 4 + 768 x 3 bits = 416 B, 8 + 24 groups -> 64 B of scales
    assert bench.latent_bytes(spec, 1024) == 416 + 64
    # rank 56: 14 x 4 + 42 x 3 = 182 bits = 22.75 B; groups 14 | 32 + 10 -> 3 scales
    assert bench.latent_bytes(spec, 56) == 22.75 + 6
    # the 20 % split: 0.2 * 40 is exactly 8 channels
    s20 = dataclasses.replace(spec, top_fraction=0.2)
    assert bench.latent_bytes(s20, 40) == (8 * 4 + 32 * 3) / 8 + 2 * 2
    # unquantized bf16
    assert bench.latent_bytes(gen.config_spec(1), 32) == 64


def test_phase_bytes_and_flops_by_hand():
    spec = gen.config_spec(2)
    B, T = 16, 32768
    key = sum(bench.latent_bytes(spec, r) for r in spec.key_ranks)
    pb = bench.phase_bytes(spec, B, T)
    assert pb[0] == B * T * key + 2 * 128 * 1024 + B * 32 * 128 * 2
    assert pb[1] == B * T * 480
    assert pb[2] == 0
    assert pb[3] == 2 * 32 * 1024 * 4096 + B * 4096 * 2
    pf = bench.phase_flops(spec, B, T)
    assert pf[0] == B * T * 2 * 128 * 1024          # sum of ranks 1024, MHA
    assert pf[1] == B * T * 2 * 1024 * 32
    assert pf[3] == B * 2 * 32 * 1024 * 4096
    # GQA: every query head of a group scores against its KV head's latent
    s3 = gen.config_spec(3, quantized=True)
    assert bench.phase_flops(s3, 1, 1)[0] == 2 * 128 * sum(s3.key_ranks) * (s3.n_heads // s3.n_kv_heads)


def test_job_throughput():
    assert bench.job_tokens_per_s(16, 1, 0.5) == pytest.approx(32000.0)
    assert bench.job_tokens_per_s(16, 8, 0.5) == pytest.approx(256000.0)


def test_reference_arm_reports_the_decode_steps_config():
    # Both arms print one config: the workload of the decode step (the oracle's sample is described in
    # cpu_baseline.sample, not in config).
    import argparse
    args = argparse.Namespace(steps=1, warmup=0, ref_ctx=64, unfused=False)
    res = bench.run_reference(args, 0, 1)
    B, ctx = bench.WORKLOAD["batch"], bench.WORKLOAD["ctx"]
    assert res["config"] == bench.decode_config(bench.workload_spec(), B, ctx, 0, 1, 1, False)
    assert res["impl"] == "reference" and res["cpu_baseline"]["kind"] == "oracle"
    assert res["e2e"]["h2d_bytes_per_step"] == 0 and res["value"] > 0
    assert bench.run_reference(args, 1, 2) is None          # only rank 0 runs it
