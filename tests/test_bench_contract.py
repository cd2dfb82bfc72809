"""The benchmark's output contract, checked on CPU through its reference arm
(the CPU oracle) on the tiny workload: one JSON line with the fields a driver
reads, and the same config description the GPU arm prints for that workload."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "2", "--warmup", "1"], capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["metric"] == "draft_blocks_per_s" and d["unit"] == "blocks/s"
    assert d["value"] > 0 and d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["steps"] >= 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    sys.path.insert(0, ROOT)
    import bench
    from block_diffusion_speculative_03_b200 import inputs as I
    w = I.preset("tiny")
    assert d["config"] == bench.config_of(w, 1, w.batch, w.context[0], w.gamma,
                                          bench.step_algorithmic_bytes(w, w.batch, w.gamma, w.context[0]))


def test_trace_attribution_partitions_the_traced_span():
    """bench.attribute_launches charges each launch from the previous launch's end to
    its own end: overlapping launches (programmatic dependent launch) are charged
    once, unused blocks (zero stamps) are ignored, and the shares add up to the span."""
    import numpy as np
    sys.path.insert(0, ROOT)
    import bench
    recs, words, off = [], [], 0
    # (kind, blocks, words per block, wait idx, exit idx, [(wait, exit) per used block])
    plan = [("embed", 2, 2, 0, 1, [(100, 400), (120, 380)]),
            ("gemm_qkv", 4, 8, 1, 6, [(300, 2000), (350, 2100), (0, 0), (500, 1900)]),   # starts before embed ends
            ("attention", 2, 8, 1, 7, [(2050, 2600), (2100, 2700)]),
            ("gemm_o", 3, 8, 1, 6, [(2400, 3500), (2600, 3300), (2500, 3600)])]
    buf = []
    for kind, blocks, w, wi, ei, st in plan:
        recs.append({"kind": kind, "blocks": blocks, "words": w, "wait_idx": wi, "exit_idx": ei, "offset": off})
        for a, b in st:
            row = [0] * w
            row[wi], row[ei] = a, b
            buf.extend(row)
        off += blocks * w
    out = bench.attribute_launches(recs, np.array(buf, dtype=np.int64))
    assert [o[0] for o in out] == ["embed", "gemm_qkv", "attention", "gemm_o"]
    assert [(o[1], o[2]) for o in out] == [(100, 400), (300, 2100), (2050, 2700), (2400, 3600)]
    assert [o[3] for o in out] == [300, 1700, 600, 900]
    assert sum(o[3] for o in out) == 3600 - 100


def test_step_flops_and_kernelwise_roofline_are_consistent():
    """The per-kind FLOPs times the step's launch counts add up to the step's FLOPs
    (both conditionings' draft parts), and the kernel-wise bound (each launch at its
    slower of bytes and FLOPs) is at least the step's byte bound and its FLOP bound."""
    sys.path.insert(0, ROOT)
    import bench
    from block_diffusion_speculative_03_b200 import inputs as I
    for name in ("qwen3_8b", "llama31_8b", "long_ctx", "tiny"):
        w = I.preset(name)
        B, g, T = w.batch, w.gamma, w.context[0]
        af = bench.algorithmic_flops(w, B, g, T)
        n = bench.step_launch_counts(w)
        assert sum(af[k] * c for k, c in n.items()) == bench.step_flops(w, B, g, T)
        ab = bench.algorithmic_bytes(w, B, g, T)
        assert sum(ab[k] * c for k, c in n.items()) == bench.step_algorithmic_bytes(w, B, g, T)
        bw, tf = 6541.0, 1385.0
        kw = bench.kernelwise_roof_ms(w, B, g, T, "kv-injection", bw, tf)
        t_bytes = bench.step_algorithmic_bytes(w, B, g, T) / (bw * 1e9) * 1e3
        t_flops = bench.step_flops(w, B, g, T) / (tf * 1e12) * 1e3
        assert kw >= max(t_bytes, t_flops) * (1 - 1e-12)


def test_gemm_traffic_constant_matches_its_profile():
    """The DRAM-traffic ratio the bench line multiplies by is the one the committed ncu
    summary reports (the capture that `bench.py` cites), and it is a plausible ratio of
    measured to algorithmic bytes (every weight byte read once, partials in L2)."""
    import re
    sys.path.insert(0, ROOT)
    import bench
    with open(os.path.join(ROOT, "profiles", "k_gemm_tc_m16_n24576_k4096.md")) as f:
        text = f.read()
    m = re.search(r"reports `roofline\.traffic` as ([0-9.]+)", text)
    assert m, "the profile states the ratio the bench uses"
    assert float(m.group(1)) == bench.GEMM_TRAFFIC["ratio"]
    assert 1.0 <= bench.GEMM_TRAFFIC["ratio"] < 1.05
    assert re.fullmatch(r"[0-9a-f]{64}", bench.GEMM_TRAFFIC["sources_sha256"])
