#!/usr/bin/env python
"""Benchmark of the DFlash draft step (draft blocks/s and drafted tok/s at
gamma = 16) on B200.

One step = one steady-state speculative cycle of every request of the batch:
  draft_block (the block of gamma positions through every draft layer, shared
  LM head, argmax) -> verification stand-in (one tiny kernel building the
  target's tokens from the drafts and a planned acceptance length) ->
  fuse_context + inject_kv of the gamma verified rows -> accept (commit /
  roll back) -> reset of the context length to the workload's context.
The reset keeps every step at the workload's context length (2048 rows for
the Qwen3-8B-shaped batch-1 drafter), so the timed steps are identical work.

Inputs are seeded synthetic tensors (weights N(0, 0.02), gains N(1, 0.02),
target hiddens N(0, 1)) already resident in HBM.  Each step streams ~3.4 GB of
weights, more than the 126 MB L2, so no L2 flush is needed between steps.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl dflash|reference]
Under torchrun (N > 1) every rank runs its own replica (weak scaling, no
collective in the step); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

HBM_FALLBACK_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024
BF16_FALLBACK_TFLOPS = 1590.0

# NVML clock-event reason bits
_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
            0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
            0x80: "hw_power_brake_slowdown", 0x100: "display_clock"}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["dflash", "reference"], default="dflash")
    ap.add_argument("--workload", default="qwen3_8b")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-profile-pass", action="store_true")
    ap.add_argument("--eager", action="store_true", help="time eager launches instead of CUDA-graph replays")
    ap.add_argument("--no-pdl", action="store_true", help="plain stream-ordered launches")
    ap.add_argument("--conditioning", choices=["kv-injection", "input-fusion"], default="kv-injection",
                    help="how the verified rows condition the drafter: injected into every layer's K/V (DFlash), "
                         "or passed through the draft layers as input hidden states (the ablation)")
    ap.add_argument("--separate-pre-step", action="store_true",
                    help="fuse_context + inject_kv as two calls instead of one fuse_inject call")
    ap.add_argument("--no-fold", action="store_true", help="separate RMSNorm kernels in the draft step")
    ap.add_argument("--fold-head", action="store_true", help="fold the final RMSNorm into the LM head too")
    ap.add_argument("--inject-whole", type=int, default=None, help="1: injection GEMM over whole tiles, 0: split-K slabs")
    ap.add_argument("--trace-dump", default=None,
                    help="write the traced step's raw per-block stamps and launch records to this .npz file")
    ap.add_argument("--o-beside", type=int, default=None,
                    help="1: O-projection on the SMs the attention leaves free (default), 0: on all SMs")
    ap.add_argument("--pre-stages", type=int, default=None,
                    help="ring stages each GEMM CTA fills with weights before its dependency wait (0 = all; library default 6)")
    ap.add_argument("--gemm-cluster", type=int, default=None,
                    help="largest thread-block cluster for 16-token GEMMs (0 = whole-grid split-K only, the library default)")
    ap.add_argument("--o-late-deficit", type=int, default=None,
                    help="k-block units fewer for O-projection CTAs that start after the attention (library default 9)")
    ap.add_argument("--gemm-tail", type=int, nargs=2, default=None, metavar=("CTAS", "UNITS"),
                    help="the last CTAS CTAs of the other whole-grid GEMMs take UNITS fewer k-block units "
                         "(library default 24 3)")
    ap.add_argument("--last-arriver", action="store_true",
                    help="split GEMM tiles finished by the contributor that counts in last (default: by the first)")
    ap.add_argument("--l2-prefetch", type=int, default=None,
                    help="weight tiles each GEMM CTA prefetches into L2 before its dependency wait")
    return ap.parse_args()


def env_int(name, default):
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


# DRAM traffic of k_gemm_tc relative to its algorithmic bytes
# (dram__bytes_read.sum + dram__bytes_write.sum over (weights + activations in +
# outputs)), from one ncu capture of a single GEMM launch of the step's shape
# class (M = 16 tokens, weights larger than L2).  It describes the kernel sources
# it was taken on: once they change, the figure is void and the line reports null.
GEMM_TRAFFIC = {"ratio": 1.0028,
                "sources_sha256": "d709f5ee59cf7207c5a610c04b91e0856bdc0d6ac1418ae97d875c870f2f33c3"}


def gemm_sources_sha256():
    import hashlib
    h = hashlib.sha256()
    for f in ("gemm_tc.cu", "gemm.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "block_diffusion_speculative_03_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic(workload):
    """DRAM bytes per algorithmic byte of the GEMM kernel, or None when not measured for these sources."""
    try:
        if GEMM_TRAFFIC["ratio"] and gemm_sources_sha256() == GEMM_TRAFFIC["sources_sha256"]:
            return GEMM_TRAFFIC["ratio"]
    except OSError:
        pass
    return None


def traced_step(D, h, step, i0, K, st, ab, dump=None):
    """Replay one graph-captured step with the library's step trace on; return
    ({kind: [launches, ms summed over replays]}, info)."""
    import torch
    words = 1 << 22
    buf = torch.zeros(words, dtype=torch.int64, device=st.device)
    D.dflash_diag_step_trace(h, buf.data_ptr(), words)
    gr = torch.cuda.CUDAGraph()
    cs = torch.cuda.Stream()
    with torch.cuda.graph(gr, stream=cs):
        step(i0)
    recs = D.dflash_diag_step_trace_records(h)
    D.dflash_diag_step_trace(h, None)
    for _ in range(3):
        gr.replay()
    R = max(3, min(K, 50))
    hist = torch.empty(R, words, dtype=torch.int64, device=st.device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    tot = 0.0
    for r in range(R):
        e0.record(st)
        gr.replay()
        e1.record(st)
        hist[r].copy_(buf)
        torch.cuda.synchronize()
        tot += e0.elapsed_time(e1)
    H = hist.cpu().numpy()
    del hist, buf, gr
    if dump:
        import numpy as np
        np.savez_compressed(dump, stamps=H[-1], kinds=np.array([r["kind"] for r in recs]),
                            recs=np.array([[r["blocks"], r["words"], r["wait_idx"], r["exit_idx"], r["offset"]]
                                           for r in recs], dtype=np.int64))
    kern = {}
    for r in range(R):
        for kind, start, end, excl in attribute_launches(recs, H[r]):
            e = kern.setdefault(kind, [0, 0.0])
            e[0] += 1
            e[1] += excl / 1e6
    info = {"replays": R, "traced_ms_per_step": tot / R, "launches": len(recs)}
    return kern, info


def attribute_launches(recs, stamps):
    """Per traced launch (kind, start, end, exclusive ns) from one replay's stamps.

    start = the earliest block's stamp past its dependency wait, end = the latest
    block's exit stamp (blocks a launch did not use hold 0 and are ignored).  A
    launch's exclusive time runs from the previous launch's end to its own end
    (the first launch: from its own start), so kernels that overlap under
    programmatic dependent launch are charged once and the exclusive times add up
    to the traced span (first start to last end)."""
    out = []
    prev_end = None
    for rec in recs:
        blk = stamps[rec["offset"]:rec["offset"] + rec["blocks"] * rec["words"]].reshape(rec["blocks"], rec["words"])
        used = blk[:, rec["exit_idx"]] != 0
        if not used.any():
            continue
        start = int(blk[used, rec["wait_idx"]].min())
        end = int(blk[used, rec["exit_idx"]].max())
        excl = end - (prev_end if prev_end is not None else start)
        prev_end = max(end, prev_end) if prev_end is not None else end
        out.append((rec["kind"], start, end, max(excl, 0)))
    return out


def workload_description(w, B, T, g):
    family = ("LLaMA-3.1-8B-shaped" if w.name.startswith("llama")
              else "Qwen3-4B-shaped" if w.name.startswith("qwen3_4b")
              else "Qwen3-Coder-30B-A3B-target-shaped" if w.name.startswith("qwen3_coder")
              else "Qwen3-8B-shaped" if w.name.startswith(("qwen3_8b", "long_ctx"))
              else "%s (%s, parity-size)" % (w.name, w.dtype))
    return ("%s drafter (hidden %d, %d layers, %d/%d heads, d %d, intermediate %d, vocab %d, %s LM head), "
            "batch %d per GPU, context %d, gamma %d"
            % (family, w.hidden, w.n_layers, w.n_q_heads, w.n_kv_heads, w.head_dim, w.intermediate, w.vocab,
               "tied" if w.tied_lm_head else "separate", B, T, g))


def config_of(w, world, B, T, g, step_bytes):
    """The config object of a bench line (the GPU arm and the reference arm report the same)."""
    return {"workload": workload_description(w, B, T, g), "global_batch": world * B, "seq_len": T, "gamma": g,
            "parallelism": "replicas x%d" % world,
            "l2": ("inputs larger than L2 (%.2f GB of weights streamed per step)" % (step_bytes / 1e9)
                   if step_bytes > L2_BYTES else "inputs fit in L2 (%.1f MB per step; a parity-size workload, "
                   "not flushed)" % (step_bytes / 1e6))}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    return HBM_FALLBACK_GBS, BF16_FALLBACK_TFLOPS, "fallback"


# ---------------------------------------------------------------------------
# Replicas across ranks: every rank runs its own requests (no collective in the
# step); a timed region's length is the max over ranks and the rate counts the
# units of all ranks.
# ---------------------------------------------------------------------------
def max_over_ranks(ms: float, device) -> float:
    """Max of this rank's time over all ranks (the value itself without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(ms)
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, units_per_rank_step: int, steps: int, ms: float) -> float:
    """Units per second of the whole job: all ranks' units over the slowest rank's time."""
    return world * units_per_rank_step * steps / (ms / 1e3)


# ---------------------------------------------------------------------------
# Algorithmic bytes per launch group (each weight byte once, activations in and
# out once, each KV byte once per request and layer).
# ---------------------------------------------------------------------------
def algorithmic_bytes(w, B, gamma, ctx_len):
    H, d = w.hidden, w.head_dim
    Nq, Nkv, I, V = w.n_q_heads * d, w.n_kv_heads * d, w.intermediate, w.vocab
    es = 2
    M, Mlm, R = B * gamma, B * (gamma - 1), B * gamma
    Kc = w.n_sel * w.target_hidden
    return {
        "gemm_qkv": ((Nq + 2 * Nkv) * H + M * H + M * (Nq + 2 * Nkv)) * es,
        "gemm_o": (Nq * H + M * Nq + 2 * M * H) * es,
        "gemm_swiglu": (2 * I * H + M * H + M * I) * es,
        "gemm_down": (H * I + M * I + 2 * M * H) * es,
        "gemm_lmhead": (V * H + Mlm * H) * es + Mlm * ((V + 127) // 128) * 16,
        "gemm_fuse": (H * Kc + R * Kc + R * H) * es,
        "gemm_inject": (w.n_layers * 2 * Nkv * H + R * H + R * w.n_layers * 2 * Nkv) * es,
        "attention": (B * w.n_kv_heads * (ctx_len + gamma) * d * 2 + 2 * M * Nq) * es,
        "rmsnorm": (2 * M * H + H) * es,
    }


def step_algorithmic_bytes(w, B, gamma, ctx_len, conditioning="kv-injection"):
    ab = algorithmic_bytes(w, B, gamma, ctx_len)
    L = w.n_layers
    draft = (L * (ab["gemm_qkv"] + ab["gemm_o"] + ab["gemm_swiglu"] + ab["gemm_down"] + ab["attention"])
             + ab["gemm_lmhead"] + ab["gemm_fuse"])
    if conditioning == "input-fusion":
        # the gamma verified rows through every layer's QKV, and all but the last
        # layer's attention, O-projection and MLP (causal over the context)
        return draft + L * ab["gemm_qkv"] + (L - 1) * (ab["gemm_o"] + ab["gemm_swiglu"] + ab["gemm_down"]
                                                       + ab["attention"])
    return draft + ab["gemm_inject"]


def algorithmic_flops(w, B, gamma, ctx_len):
    """Multiply-add FLOPs of one launch of each kernel kind (the same kinds as
    algorithmic_bytes)."""
    H, d = w.hidden, w.head_dim
    Nq, Nkv, I, V = w.n_q_heads * d, w.n_kv_heads * d, w.intermediate, w.vocab
    M, Mlm = B * gamma, B * (gamma - 1)
    return {
        "gemm_qkv": 2 * M * H * (Nq + 2 * Nkv),
        "gemm_o": 2 * M * Nq * H,
        "gemm_swiglu": 2 * M * H * 2 * I,
        "gemm_down": 2 * M * I * H,
        "gemm_lmhead": 2 * Mlm * H * V,
        "gemm_fuse": 2 * M * w.n_sel * w.target_hidden * H,
        "gemm_inject": 2 * M * H * w.n_layers * 2 * Nkv,
        "attention": 4 * B * w.n_q_heads * gamma * (ctx_len + gamma) * d,
        "rmsnorm": 0,
    }


def step_launch_counts(w, conditioning="kv-injection"):
    """Launches of each kernel kind in one step (those algorithmic_bytes counts)."""
    L = w.n_layers
    n = {"gemm_qkv": L, "gemm_o": L, "gemm_swiglu": L, "gemm_down": L, "attention": L,
         "gemm_lmhead": 1, "gemm_fuse": 1, "gemm_inject": 1}
    if conditioning == "input-fusion":
        n["gemm_inject"] = 0
        n["gemm_qkv"] += L
        for k in ("gemm_o", "gemm_swiglu", "gemm_down", "attention"):
            n[k] += L - 1
    return n


def kernelwise_roof_ms(w, B, gamma, ctx_len, conditioning, hbm_gbs, tflops):
    """Sum over the step's launches of max(bytes at the HBM peak, FLOPs at the tensor
    peak): a launch cannot beat its own slower bound."""
    ab, af = algorithmic_bytes(w, B, gamma, ctx_len), algorithmic_flops(w, B, gamma, ctx_len)
    return sum(c * max(ab[k] / (hbm_gbs * 1e9), af[k] / (tflops * 1e12))
               for k, c in step_launch_counts(w, conditioning).items()) * 1e3


def step_flops(w, B, gamma, ctx_len):
    H, d = w.hidden, w.head_dim
    Nq, Nkv, I, V = w.n_q_heads * d, w.n_kv_heads * d, w.intermediate, w.vocab
    M, Mlm = B * gamma, B * (gamma - 1)
    per_layer = 2 * M * H * (Nq + 2 * Nkv) + 2 * M * Nq * H + 2 * M * H * 2 * I + 2 * M * I * H
    per_layer += 4 * B * w.n_q_heads * gamma * (ctx_len + gamma) * d
    return (w.n_layers * per_layer + 2 * Mlm * H * V + 2 * M * w.n_sel * w.target_hidden * H
            + 2 * M * H * w.n_layers * 2 * Nkv)


# ---------------------------------------------------------------------------
# CPU oracle cycle (the reference arm and the cpu_baseline leg)
# ---------------------------------------------------------------------------
def _np(t):
    """Host numpy copy: bf16 as uint16 bit patterns, fp32 as float32."""
    import numpy as np
    import torch
    t = t.detach().cpu()
    return t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.numpy()


class OracleCycle:
    """One request's steady-state cycle in the CPU oracle, on the workload's
    shapes: draft_block over a context of the workload's length + fuse/inject of
    gamma verified rows + accept, then the same length reset as the GPU step."""

    def __init__(self, w, weights_np, acc32=0):
        from oracle import oracle as O
        from block_diffusion_speculative_03_b200 import inputs as I
        shape = dict(hidden=w.hidden, n_layers=w.n_layers, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                     head_dim=w.head_dim, intermediate=w.intermediate, vocab=w.vocab, n_sel=w.n_sel,
                     target_hidden=w.target_hidden, mask_id=w.mask_token,
                     storage="f32" if w.dtype == "f32" else "bf16", rope_theta=w.rope_theta, rms_eps=w.rms_eps,
                     acc32=acc32)
        self.w = w
        self.od = O.OracleDrafter(shape, weights_np)
        T = w.context[0]
        self.T = T
        self.cache = self.od.new_cache(T + 2 * w.gamma)
        for l in range(w.n_layers):
            for kind, key in ((0, "k"), (1, "v")):
                self.cache[key][l, :, :T] = I.synthetic_cache_rows(w, l, kind, 0, T).double().numpy()
        self.cache["len"] = self.cache["committed"] = T
        self.hid = [_np(x) for x in I.make_hiddens(w, w.gamma, stream=4242)]
        self.anchor = int(I.make_anchors(w)[0])
        self.plan = I.plan_accept(w, 64).numpy()[:, 0]
        self.rnd = I.random_tokens(w, (64, w.gamma)).numpy()
        self.i = 0

    def _target(self, drafts, a, rnd):
        t = rnd.astype("int32").copy()
        t[:a] = drafts[:a]
        if a < self.w.gamma - 1 and t[a] == drafts[a]:
            t[a] = (t[a] + 1) % self.w.vocab
        return t

    def cycle(self):
        g = self.w.gamma
        drafts, margin, _ = self.od.draft_block(self.cache, self.anchor, g)
        target = self._target(drafts, int(self.plan[self.i % 64]), self.rnd[self.i % 64])
        ctx = self.od.fuse_context(self.hid)
        self.od.inject_kv(self.cache, ctx)
        st, a, nxt = self.od.accept(self.cache, drafts, target)
        self.anchor = nxt
        self.cache["len"] = self.cache["committed"] = self.T
        self.i += 1


def oracle_weights_from(weights):
    """Host copies of the seeded weights in the oracle's numpy form."""
    out = {k: _np(weights[k]) for k in ("w_fc", "g_fc", "embed", "lm_head", "g_final")}
    out["layers"] = [{k: _np(v) for k, v in lw.items()} for lw in weights["layers"]]
    return out


def run_reference(args):
    """--impl reference: the CPU oracle timed on the host cores, rank 0 only."""
    rank = env_int("RANK", 0)
    if rank != 0:
        return 0
    import torch
    from block_diffusion_speculative_03_b200 import inputs as I
    from oracle import oracle as O
    w_full = I.preset(args.workload)
    w = I.preset(args.workload)
    w.batch = 1
    w.context = w.context[:1]
    # Seeded inputs: generated with plain torch ops (on the GPU when there is
    # one, only to save time), then handed to the oracle as host arrays.
    gen_dev = "cuda" if torch.cuda.is_available() else "cpu"
    weights = I.make_weights(w, device=gen_dev)
    oc = OracleCycle(w, oracle_weights_from(weights))
    del weights
    for _ in range(min(args.warmup, 1)):
        oc.cycle()
    # Each step is one full cycle of the request; the run is capped at ~90 s of
    # cycles (at least 2) so that the arm ends within a few minutes.
    n, t0 = 0, time.perf_counter()
    while n < args.steps and (n < 2 or time.perf_counter() - t0 < 90.0):
        oc.cycle()
        n += 1
    dt = time.perf_counter() - t0
    bps = n / dt
    line = {
        "impl": "reference", "metric": "draft_blocks_per_s", "value": bps, "unit": "blocks/s",
        "n_gpus": args.gpus, "steps": n, "warmup": min(args.warmup, 1), "ms_per_step": 1e3 * dt / n,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "drafted_tok_per_s": bps * (w.gamma - 1),
        "config": config_of(w_full, args.gpus, w_full.batch, w_full.context[0], w_full.gamma,
                            step_algorithmic_bytes(w_full, w_full.batch, w_full.gamma, w_full.context[0])),
        "cpu_baseline": {"value": bps, "unit": "blocks/s", "cores": O.num_threads(), "kind": "oracle",
                         "sample": "%d full oracle cycles (draft block + fuse/inject of %d rows + accept) of one "
                                   "request (of %d requested steps; capped at ~90 s)" % (n, w.gamma, args.steps)},
        "e2e": {"value": bps, "unit": "blocks/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def start_sampler(gpu_index):
    try:
        p = subprocess.Popen([sys.executable, "-m", "block_diffusion_speculative_03_b200.clock_sampler",
                              str(gpu_index), "0.01"], stdin=subprocess.PIPE, stdout=subprocess.PIPE,
                             stderr=subprocess.DEVNULL, text=True, cwd=ROOT)
        line = p.stdout.readline()    # "max_sm,<MHz>" once NVML is up
        return p, int(line.strip().split(",")[1]) if line.startswith("max_sm") else None
    except Exception:
        return None, None


def stop_sampler(p, max_sm, t0, t1):
    if p is None:
        return None
    try:
        out, _ = p.communicate(input="", timeout=10)
    except Exception:
        p.kill()
        return None
    sms, reasons = [], 0
    allr = []
    for ln in out.splitlines():
        parts = ln.split(",")
        if len(parts) != 4:
            continue
        ts, sm, rs = float(parts[0]), int(parts[1]), int(parts[2])
        if t0 <= ts <= t1:
            sms.append(sm)
            reasons |= rs
        allr.append(sm)
    if not sms and allr:
        sms = allr[-3:]
    names = [n for bit, n in _REASONS.items() if reasons & bit]
    return {"sm_mhz": statistics.median(sms) if sms else None, "sm_max_mhz": max_sm, "reasons": names,
            "samples": len(sms)}


def run_gpu(args):
    import torch
    import torch.distributed as dist
    from block_diffusion_speculative_03_b200 import dflash as D
    from block_diffusion_speculative_03_b200 import inputs as I
    from block_diffusion_speculative_03_b200.drafter import Drafter, shape_from_workload

    rank, world, local = env_int("RANK", 0), env_int("WORLD_SIZE", 1), env_int("LOCAL_RANK", 0)
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    dev = torch.device("cuda", local)
    w = I.preset(args.workload)
    B, g = w.batch, w.gamma
    T = w.context[0]
    assert all(c == T for c in w.context), "bench workloads use one context length"
    K, W = args.steps, args.warmup
    cap = T + 2 * g + 8
    weights = I.make_weights(w, device=dev)
    if w.tied_lm_head:
        weights["lm_head"] = weights["embed"]
    drafter = Drafter(shape_from_workload(w), weights, max_batch=B, max_rows=max(B * T, B * g),
                      max_position=cap, max_gamma=g, device=dev)
    cache = drafter.new_cache(B, cap)
    st = torch.cuda.current_stream()
    # prefill through the library: fuse + inject of B*T seeded target-hidden rows,
    # once to fill the cache and twice more timed (prefill ingestion, reported apart)
    hid = I.make_hiddens(w, B * T, stream=0, device=dev)
    lens = torch.full((B,), T, dtype=torch.int32, device=dev)
    zeros = torch.zeros(B, dtype=torch.int32, device=dev)
    starts = torch.arange(0, B * T, T, dtype=torch.int32, device=dev)
    # library switches (process-wide) before any call, the prefill included
    D.dflash_diag_set_launch_mode(not args.no_pdl)
    D.dflash_diag_set_norm_fold(0 if args.no_fold else 2 if args.fold_head else 1)
    if args.inject_whole is not None:
        D.dflash_diag_set_inject_partition(bool(args.inject_whole))
    if args.l2_prefetch is not None:
        D.dflash_diag_set_gemm_prefetch(args.l2_prefetch)
    if args.pre_stages is not None:
        D.dflash_diag_set_gemm_pre_stages(args.pre_stages)
    if args.o_beside is not None:
        D.dflash_diag_set_o_beside_attention(bool(args.o_beside))
    D.dflash_diag_set_split_finisher(args.last_arriver)
    if args.o_late_deficit is not None:
        D.dflash_diag_set_o_late_deficit(args.o_late_deficit)
    if args.gemm_tail is not None:
        D.dflash_diag_set_gemm_tail(*args.gemm_tail)
    if args.gemm_cluster is not None:
        D.dflash_diag_set_gemm_max_cluster(args.gemm_cluster)
    pre_ms = []
    for rep in range(3):
        cache.set_len(zeros)
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        p0.record()
        ctx = drafter.fuse_context(hid)
        drafter.inject_kv(cache, ctx, starts, lens)
        p1.record()
        torch.cuda.synchronize()
        if rep:
            pre_ms.append(p0.elapsed_time(p1))
        del ctx
    cache.set_len(lens)
    del hid
    pre_t = statistics.median(pre_ms)
    pre_flops = 2.0 * B * T * w.hidden * (w.n_sel * w.target_hidden + w.n_layers * 2 * w.n_kv_heads * w.head_dim)
    prefill = {"rows": B * T, "ms": round(pre_t, 3), "rows_per_s": round(B * T / (pre_t / 1e3), 1),
               "tflops": round(pre_flops / (pre_t / 1e3) / 1e12, 1),
               "what": "fuse_context + inject_kv of the whole context (all requests), median of 2, "
                       "allocation of the context buffer included"}
    # per-step inputs resident in HBM (a pool of distinct verified-row sets)
    POOL = 32
    step_hid = [I.make_hiddens(w, B * g, stream=1000 + i, device=dev) for i in range(POOL)]
    a_plan = I.plan_accept(w, POOL).to(dev)
    rnd = I.random_tokens(w, (POOL, B, g), device=dev)
    anchor = I.make_anchors(w, device=dev)
    drafts = torch.empty(B, g - 1, dtype=torch.int32, device=dev)
    target = torch.empty(B, g, dtype=torch.int32, device=dev)
    acc = torch.empty(B, dtype=torch.int32, device=dev)
    ctx_step = torch.empty(B * g, w.hidden, dtype=torch.bfloat16, device=dev)
    rs = torch.arange(0, B * g, g, dtype=torch.int32, device=dev)
    rc = torch.full((B,), g, dtype=torch.int32, device=dev)
    h, c = drafter.handle, cache.handle

    def step(i, hid_list=None):
        sp = torch.cuda.current_stream().cuda_stream
        D.dflash_draft_block(h, c, anchor.data_ptr(), g, drafts.data_ptr(), None, None, sp)
        j = i % POOL
        D.dflash_diag_synth_target(drafts.data_ptr(), a_plan[j].data_ptr(), rnd[j].data_ptr(), B, g, w.vocab,
                                   target.data_ptr(), sp)
        hl = hid_list if hid_list is not None else step_hid[i % POOL]
        if args.conditioning == "input-fusion":
            D.dflash_fuse_context(h, [x.data_ptr() for x in hl], w.target_hidden, B * g, ctx_step.data_ptr(), sp)
            D.dflash_ingest_fused_input(h, c, ctx_step.data_ptr(), g, None, sp)
        elif args.separate_pre_step:
            D.dflash_fuse_context(h, [x.data_ptr() for x in hl], w.target_hidden, B * g, ctx_step.data_ptr(), sp)
            D.dflash_inject_kv(h, c, ctx_step.data_ptr(), rs.data_ptr(), rc.data_ptr(), B * g, sp)
        else:   # the verify-side pre-step: fuse + inject of the verified rows in one call
            D.dflash_fuse_inject(h, c, [x.data_ptr() for x in hl], w.target_hidden, rs.data_ptr(), rc.data_ptr(),
                                 B * g, None, sp)
        D.dflash_accept(h, c, drafts.data_ptr(), target.data_ptr(), g, acc.data_ptr(), anchor.data_ptr(), sp)
        D.dflash_cache_set_len(c, lens.data_ptr(), sp)

    i = 0
    for _ in range(W):
        step(i)
        i += 1
    torch.cuda.synchronize()
    assert cache.status() == 0, "device status after warm-up"
    if world > 1:
        dist.barrier()

    # launches of one step (library counter; + the verification stand-in kernel)
    n0 = drafter.launch_count()
    step(i)
    i += 1
    per_step_launches = drafter.launch_count() - n0 + 1
    graphs = None
    if not args.eager:
        # one CUDA graph per input-pool slot; each replays one whole step
        graphs = []
        cs = torch.cuda.Stream()
        for j in range(POOL):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=cs):
                step(j)
            graphs.append(gr)
        torch.cuda.synchronize()
        for j in range(min(W, POOL)):          # warm replays
            graphs[(i + j) % POOL].replay()
        i += min(W, POOL)
        torch.cuda.synchronize()
        assert cache.status() == 0, "device status after graph warm-up"

    # ---- timed pass
    sampler, max_sm = start_sampler(local) if rank == 0 else (None, None)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t_wall0 = time.time()
    e0.record(st)
    for _ in range(K):
        if graphs is not None:
            graphs[i % POOL].replay()
        else:
            step(i)
        i += 1
    e1.record(st)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    launches = per_step_launches * K
    ms = e0.elapsed_time(e1)
    clocks = stop_sampler(sampler, max_sm, t_wall0, t_wall1)
    if world > 1:
        dist.barrier()
    ms = max_over_ranks(ms, dev)
    status = cache.status()
    assert status == 0, "device status %d" % status
    ms_step = ms / K
    blocks_per_s = whole_job_rate(world, B, K, ms)

    hbm_peak, tc_peak, peak_src = measured_peaks()
    ab = algorithmic_bytes(w, B, g, T)
    step_bytes = step_algorithmic_bytes(w, B, g, T, args.conditioning)
    t_roof_ms = step_bytes / (hbm_peak * 1e9) * 1e3
    t_flops_ms = step_flops(w, B, g, T) / (tc_peak * 1e12) * 1e3
    t_kw_ms = kernelwise_roof_ms(w, B, g, T, args.conditioning, hbm_peak, tc_peak)

    # ---- traced pass: the same step captured in one CUDA graph with the library's
    # step trace on (every kernel stamps %globaltimer per block past its dependency
    # wait and at exit), replayed like the timed pass.  Launch k's time is charged
    # from the end of launch k-1 to its own end (the first launch from its start),
    # so the per-kernel times partition the traced part of the step and add up to
    # no more than the step.
    kern, traced = {}, None
    if not args.no_profile_pass and graphs is not None:
        kern, traced = traced_step(D, h, step, i, K, st, ab, args.trace_dump)
        i += max(3, min(K, 50)) + 3
    gemm_names = ["gemm_qkv", "gemm_o", "gemm_swiglu", "gemm_down", "gemm_lmhead", "gemm_fuse", "gemm_inject"]
    roofline = None
    if kern:
        gl = sum(kern[n][0] for n in gemm_names if n in kern)
        gms = sum(kern[n][1] for n in gemm_names if n in kern)
        gbytes = sum(kern[n][0] * ab[n] for n in gemm_names if n in kern)
        achieved = gbytes / (gms / 1e3) / 1e9
        traffic = measured_traffic(args.workload)
        roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                    "frac": round(achieved / hbm_peak, 4),
                    "traffic": (round(traffic * gbytes / max(gl, 1)) if traffic else None),
                    "kernel": "k_gemm_tc (all %d launches of one step, %d replays)" % (gl // max(traced["replays"], 1),
                                                                                  traced["replays"]),
                    "algorithmic_bytes_per_launch": round(gbytes / max(gl, 1)),
                    "time_source": "per-kernel share of the graph-replayed step from the kernels' own %globaltimer "
                                   "stamps (launch end minus previous launch end)",
                    "peak_source": peak_src + " (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured" else peak_src}
    reps = traced["replays"] if traced else 1
    per_kernel = {n: {"launches": v[0] // reps, "ms_per_step": round(v[1] / reps, 4),
                      "GB_per_s": (round(ab[n] * v[0] / (v[1] / 1e3) / 1e9, 1) if n in ab and v[1] > 0 else None)}
                  for n, v in sorted(kern.items(), key=lambda kv: -kv[1][1])}

    # ---- end-to-end pass: host inputs in, results out, through the C ABI
    e2e = None
    if not args.no_e2e:
        pin_hid = [[x.cpu().pin_memory() for x in step_hid[j]] for j in range(8)]
        dev_hid = [torch.empty_like(x) for x in step_hid[0]]
        out_dr = torch.empty(B, g - 1, dtype=torch.int32).pin_memory()
        out_acc = torch.empty(B, dtype=torch.int32).pin_memory()
        out_nxt = torch.empty(B, dtype=torch.int32).pin_memory()
        # The library calls of a step are graph-captured like a serving loop would
        # (one graph per input slot, reading the fixed device input buffers); the
        # host->device copy of the step's inputs and the read-back of its results
        # are issued every step, outside the graphs, inside the timed region.
        e2e_graphs = None
        if graphs is not None:
            e2e_graphs = []
            cs2 = torch.cuda.Stream()
            for j in range(POOL):
                gr = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gr, stream=cs2):
                    step(j, dev_hid)
                e2e_graphs.append(gr)
            for j in range(min(W, POOL)):
                e2e_graphs[(i + j) % POOL].replay()
            i += min(W, POOL)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0.record(st)
        for k in range(K):
            for dst, src in zip(dev_hid, pin_hid[k % 8]):
                dst.copy_(src, non_blocking=True)
            if e2e_graphs is not None:
                e2e_graphs[i % POOL].replay()
            else:
                step(i, dev_hid)
            out_dr.copy_(drafts, non_blocking=True)
            out_acc.copy_(acc, non_blocking=True)
            out_nxt.copy_(anchor, non_blocking=True)
            i += 1
        e1.record(st)
        torch.cuda.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1), dev)
        h2d = sum(x.numel() * x.element_size() for x in pin_hid[0])
        d2h = (out_dr.numel() + out_acc.numel() + out_nxt.numel()) * 4
        e2e = {"value": whole_job_rate(world, B, K, ems), "unit": "blocks/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": ems / K,
               "launch": "C-ABI calls replayed from CUDA graphs" if e2e_graphs is not None else "eager C-ABI calls"}
        del e2e_graphs
    assert cache.status() == 0

    # ---- CPU oracle baseline (rank 0, one GPU only)
    cpu = cpu32 = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # The oracle runs its requests one after another, so its blocks/s is its
        # cycle rate on one request, whatever the batch.
        from oracle import oracle as O
        wc = I.preset(args.workload)
        wc.batch, wc.context = 1, wc.context[:1]
        host_w = oracle_weights_from(weights)

        def time_cycles(acc32, max_n, max_s):
            oc = OracleCycle(wc, host_w, acc32=acc32)
            oc.cycle()                          # warm (first-touch of the host arrays)
            n, t0 = 0, time.perf_counter()
            while n < max_n and (n < 2 or time.perf_counter() - t0 < max_s):
                oc.cycle()
                n += 1
            return n, time.perf_counter() - t0

        n, dt = time_cycles(0, 8, 12.0)
        cpu = {"value": n / dt, "unit": "blocks/s", "cores": O.num_threads(), "kind": "oracle",
               "cpu_model": cpu_model(),
               "sample": "%d oracle cycles (fp64 accumulation, the parity mode) of one request: draft block + "
                         "fuse/inject of %d rows + accept" % (n, g)}
        n, dt = time_cycles(1, 8, 8.0)
        cpu32 = {"value": n / dt, "unit": "blocks/s", "cores": O.num_threads(), "kind": "oracle",
                 "sample": "%d oracle cycles with fp32 accumulation (the oracle's sensitivity mode), "
                           "one request" % n}

    if rank == 0:
        line = {
            "metric": "draft_blocks_per_s", "value": round(blocks_per_s, 2), "unit": "blocks/s",
            "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": round(ms_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,0.02) weights, N(0,1) target hiddens; benchmark datasets not used)",
            "config": dict(config_of(w, world, B, T, g, step_bytes),
                           **({"conditioning": "input fusion (the ablation KV injection is compared against)"}
                              if args.conditioning == "input-fusion" else {})),
            "drafted_tok_per_s": round(blocks_per_s * (g - 1), 1),
            "roofline": roofline,
            "step_roofline": {"algorithmic_bytes": step_bytes, "flops": step_flops(w, B, g, T),
                              "t_roof_ms": round(t_roof_ms, 4), "frac": round(t_roof_ms / ms_step, 4),
                              "peak_gbs": hbm_peak, "peak_source": peak_src,
                              # the mixed bound: the step cannot beat its bytes at the HBM peak
                              # nor its FLOPs at the (sustained) bf16 tensor peak
                              "t_flops_ms": round(t_flops_ms, 4), "peak_tflops": tc_peak,
                              "t_roof_mixed_ms": round(max(t_roof_ms, t_flops_ms), 4),
                              "frac_mixed": round(max(t_roof_ms, t_flops_ms) / ms_step, 4),
                              "t_roof_kernelwise_ms": round(t_kw_ms, 4), "frac_kernelwise": round(t_kw_ms / ms_step, 4)},
            "per_kernel": per_kernel,
            "traced_step": ({"ms_per_step": round(traced["traced_ms_per_step"], 4),
                             "traced_launches": traced["launches"],
                             "attributed_ms": round(sum(v["ms_per_step"] for v in per_kernel.values()), 4)}
                            if traced else None),
            "cpu_baseline": cpu,
            "cpu_baseline_fp32_accumulation": cpu32,
            "prefill": prefill,
            "e2e": e2e,
            "gpu_launches": launches,
            "step_options": {"conditioning": args.conditioning,
                             "pre_step": ("fuse_context + ingest_fused_input" if args.conditioning == "input-fusion"
                                          else "two calls" if args.separate_pre_step else "fuse_inject (one call)"),
                             "norm_fold": "off" if args.no_fold else "with the LM head" if args.fold_head else "on",
                             "gemm_l2_prefetch_tiles": D.dflash_diag_gemm_prefetch(),
                             "split_tile_finisher": "last arriver" if args.last_arriver else "first contributor",
                             "gemm_pre_stages": args.pre_stages if args.pre_stages is not None else "library default (6)",
                             "gemm_max_cluster": args.gemm_cluster if args.gemm_cluster is not None else "library default (0)",
                             "o_late_deficit": args.o_late_deficit if args.o_late_deficit is not None else "library default (9)",
                             "gemm_tail": args.gemm_tail if args.gemm_tail is not None else "library default (24, 3)",
                             "gemm_resident_clusters": {str(c): D.dflash_diag_gemm_max_active_clusters(c) for c in (2, 3, 4)}},
            "launch_mode": ("eager" if args.eager else "cuda-graph replay") + (", plain launches" if args.no_pdl
                                                                              else ", programmatic dependent launch"),
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
