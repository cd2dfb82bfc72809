"""The seeded input generator: pinned to a pure-Python SplitMix64 and to the
statistics the workloads ask for."""
import math

import torch

from block_diffusion_speculative_03_b200 import inputs as I


def test_stream_matches_pure_python_splitmix64():
    z = I.raw_u64(0xDF1A5, 42, 1000, 64)
    got = [int(v) & ((1 << 64) - 1) for v in z]
    assert got == [I.splitmix64_ref(0xDF1A5, 42, 1000 + i) for i in range(64)]


def test_normal_statistics_and_determinism():
    a = I.normal(5, 9, (1 << 20,), 0.02, dtype=torch.float32)
    b = I.normal(5, 9, (1 << 20,), 0.02, dtype=torch.float32)
    assert torch.equal(a, b)
    assert abs(a.mean().item()) < 1e-4 and abs(a.std().item() - 0.02) < 1e-4
    g = I.normal(5, 10, (1 << 16,), 0.02, 1.0, dtype=torch.bfloat16)
    assert abs(g.float().mean().item() - 1.0) < 1e-3


def test_planned_acceptance_means():
    q = I.preset("qwen3_8b")
    a = I.plan_accept(q, 20000).float()
    assert a.min() >= 0 and a.max() <= 15 and abs(a.mean().item() - 6.0) < 0.15
    lc = I.preset("long_ctx")
    a = I.plan_accept(lc, 20000).float()
    assert abs(a.mean().item() - 5.0) < 0.15
    t = I.preset("tiny")
    a = I.plan_accept(t, 20000)
    assert set(a.flatten().tolist()) == {0, 1, 2, 3}


def test_randint_range_and_context_lengths():
    v = I.randint(1, 2, (100000,), 3, 17)
    assert v.min() == 3 and v.max() == 16
    b32 = I.preset("qwen3_8b_b32")
    assert len(b32.context) == 32 and min(b32.context) >= 512 and max(b32.context) <= 4096
