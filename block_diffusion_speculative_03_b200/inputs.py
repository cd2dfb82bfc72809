"""Seeded synthetic inputs and workload presets.

This module holds no arithmetic of the draft step.  It only produces seeded
inputs (weights, target hidden states, tokens, planned acceptance lengths) and
names the workload shapes; both the CUDA path and the CPU oracle consume the
same tensors from here.

Generator: a counter-based SplitMix64 stream keyed by (seed, tensor id,
element index).  SplitMix64 is Steele, Lea and Flood, "Fast splittable
pseudorandom number generators" (OOPSLA 2014); the finaliser constants are the
published ones.  Two 53-bit uniforms per element feed a Box-Muller transform in
fp64; the result is scaled and rounded to the storage dtype.  The arithmetic is
done with torch int64 tensors (wrapping multiply, masked logical shifts) so the
same code runs on the CPU and on a GPU; a given run generates each tensor on
one device and copies it where else it is needed.

Shapes follow the DFlash summaries' experiments (Qwen3-8B and LLaMA-3.1-8B
targets, a 5-layer drafter, blocks of 16, serving concurrency up to 32, long
thinking-mode contexts).  The benchmarks the pages evaluate on are not in this
environment; these seeded inputs stand in for them, and no benchmark item is
reproduced.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import torch

_MASK64 = (1 << 64) - 1


def _s64(x: int) -> int:
    """Two's-complement int64 view of an unsigned 64-bit constant."""
    x &= _MASK64
    return x - (1 << 64) if x >= (1 << 63) else x


_GOLDEN = _s64(0x9E3779B97F4A7C15)
_M1 = _s64(0xBF58476D1CE4E5B9)
_M2 = _s64(0x94D049BB133111EB)


def _lsr(z: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 bit patterns."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def _mix(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _lsr(z, 30)) * _M1
    z = (z ^ _lsr(z, 27)) * _M2
    return z ^ _lsr(z, 31)


def splitmix64_ref(seed: int, tensor_id: int, index: int) -> int:
    """Pure-Python reference of one stream element (used to pin the tensor version)."""
    def mix(z):
        z &= _MASK64
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
        return z ^ (z >> 31)
    key = mix((seed ^ ((tensor_id * 0x9E3779B97F4A7C15) & _MASK64)) & _MASK64)
    return mix((key + (index + 1) * 0x9E3779B97F4A7C15) & _MASK64)


def _key(seed: int, tensor_id: int) -> int:
    t = torch.tensor([_s64(seed ^ ((tensor_id * 0x9E3779B97F4A7C15) & _MASK64))], dtype=torch.int64)
    return int(_mix(t)[0])


def raw_u64(seed: int, tensor_id: int, start: int, count: int, device="cpu") -> torch.Tensor:
    """Stream elements [start, start+count) as int64 bit patterns."""
    key = _key(seed, tensor_id)
    idx = torch.arange(start + 1, start + count + 1, dtype=torch.int64, device=device)
    return _mix(idx * _GOLDEN + key)


def _uniform53(z: torch.Tensor) -> torch.Tensor:
    return _lsr(z, 11).to(torch.float64) * (1.0 / (1 << 53))


_CHUNK = 1 << 24


def normal(seed: int, tensor_id: int, shape, std: float = 1.0, mean: float = 0.0,
           dtype=torch.bfloat16, device="cpu") -> torch.Tensor:
    """Seeded N(mean, std^2) tensor, Box-Muller in fp64, rounded to dtype."""
    n = 1
    for s in shape:
        n *= int(s)
    out = torch.empty(n, dtype=dtype, device=device)
    for c0 in range(0, n, _CHUNK):
        cnt = min(_CHUNK, n - c0)
        z = raw_u64(seed, tensor_id, 2 * c0, 2 * cnt, device=device).view(cnt, 2)
        u1 = _uniform53(z[:, 0])
        u2 = _uniform53(z[:, 1])
        g = torch.sqrt(-2.0 * torch.log1p(-u1)) * torch.cos((2.0 * math.pi) * u2)
        out[c0:c0 + cnt] = (g * std + mean).to(dtype)
    return out.view(*shape)


def randint(seed: int, tensor_id: int, shape, low: int, high: int, device="cpu") -> torch.Tensor:
    """Seeded integers uniform in [low, high) as int32."""
    n = 1
    for s in shape:
        n *= int(s)
    z = raw_u64(seed, tensor_id, 0, n, device=device)
    u = _uniform53(z)
    v = torch.clamp((u * (high - low)).floor().to(torch.int64), max=high - low - 1) + low
    return v.to(torch.int32).view(*shape)


def uniform(seed: int, tensor_id: int, shape, device="cpu") -> torch.Tensor:
    n = 1
    for s in shape:
        n *= int(s)
    return _uniform53(raw_u64(seed, tensor_id, 0, n, device=device)).view(*shape)


# ---------------------------------------------------------------------------
# Workload presets
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class Workload:
    name: str
    hidden: int
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    intermediate: int
    vocab: int
    n_sel: int
    target_hidden: int
    rope_theta: float
    rms_eps: float
    dtype: str                 # "f32" or "bf16"
    batch: int
    gamma: int
    context: List[int]         # per-request context length
    tied_lm_head: bool = True
    mask_id: int = -1          # -1: vocab - 1
    accept_kind: str = "geometric"   # "uniform" (0..gamma-1) or "geometric"
    accept_q: float = 0.87358
    cycles: int = 1
    seed: int = 0xDF1A5
    gammas: Optional[List[int]] = None   # block sizes swept on the same weights

    @property
    def mask_token(self) -> int:
        return self.vocab - 1 if self.mask_id < 0 else self.mask_id

    def capacity(self) -> int:
        return max(self.context) + self.cycles * self.gamma + self.gamma


def _ctx_lengths(seed: int, batch: int, lo: int, hi: int) -> List[int]:
    return [int(v) for v in randint(seed, 9001, (batch,), lo, hi + 1)]


def preset(name: str) -> Workload:
    """Named workloads: the five drafter configurations plus reduced parity cases."""
    if name == "tiny":
        return Workload("tiny", 256, 2, 4, 2, 64, 768, 1024, 3, 256, 1e4, 1e-6, "f32",
                        batch=1, gamma=4, context=[64], mask_id=1023, accept_kind="uniform",
                        seed=0xDF1A5 + 0)
    if name == "qwen3_8b":
        return Workload("qwen3_8b", 4096, 5, 32, 8, 128, 12288, 151936, 5, 4096, 1e6, 1e-6, "bf16",
                        batch=1, gamma=16, context=[2048], seed=0xDF1A5 + 1)
    if name == "qwen3_8b_b32":
        seed = 0xDF1A5 + 2
        return Workload("qwen3_8b_b32", 4096, 5, 32, 8, 128, 12288, 151936, 5, 4096, 1e6, 1e-6, "bf16",
                        batch=32, gamma=16, context=_ctx_lengths(seed, 32, 512, 4096), cycles=16,
                        seed=seed)
    if name == "long_ctx":
        return Workload("long_ctx", 4096, 5, 32, 8, 128, 12288, 151936, 5, 4096, 1e6, 1e-6, "bf16",
                        batch=4, gamma=16, context=[32768] * 4, accept_q=0.84448,
                        gammas=[16, 8, 4], seed=0xDF1A5 + 3)
    if name == "llama31_8b":
        return Workload("llama31_8b", 4096, 5, 32, 8, 128, 14336, 128256, 5, 4096, 5e5, 1e-5, "bf16",
                        batch=16, gamma=16, context=[8192] * 16, tied_lm_head=False,
                        seed=0xDF1A5 + 4)
    # The same draft step on a deeper drafter, and on a Qwen3-4B-shaped one
    # (hidden 2560 with 32 query heads of 128: the attention width exceeds the
    # hidden size).
    if name == "qwen3_8b_depth8":
        return Workload("qwen3_8b_depth8", 4096, 8, 32, 8, 128, 12288, 151936, 5, 4096, 1e6, 1e-6, "bf16",
                        batch=1, gamma=16, context=[2048], seed=0xDF1A5 + 5)
    if name == "qwen3_4b":
        return Workload("qwen3_4b", 2560, 5, 32, 8, 128, 9728, 151936, 5, 2560, 1e6, 1e-6, "bf16",
                        batch=1, gamma=16, context=[2048], seed=0xDF1A5 + 6)
    # A drafter for a Qwen3-Coder-30B-A3B-shaped target: the target's hidden size
    # (2048), 32 query heads of 128 over 4 key/value heads (8 query heads per kv
    # head: 128 query rows per kv head at gamma 16), a dense SwiGLU of 3 x hidden
    # (the target's experts are not part of the drafter), the Qwen3 vocabulary and
    # a long-context RoPE base.
    if name == "qwen3_coder_30b":
        return Workload("qwen3_coder_30b", 2048, 5, 32, 4, 128, 6144, 151936, 5, 2048, 1e7, 1e-6, "bf16",
                        batch=1, gamma=16, context=[2048], seed=0xDF1A5 + 7)
    # Reduced bf16 shapes that span several GEMM tiles and ragged tails but
    # that the oracle finishes in seconds.
    if name == "small_bf16":
        return Workload("small_bf16", 512, 2, 8, 2, 128, 1536, 4000, 3, 384, 1e6, 1e-6, "bf16",
                        batch=2, gamma=16, context=[300, 173], cycles=3, seed=0xDF1A5 + 10)
    if name == "small_bf16_untied":
        return Workload("small_bf16_untied", 384, 2, 6, 3, 64, 1024, 2500, 2, 256, 5e5, 1e-5, "bf16",
                        batch=3, gamma=8, context=[97, 260, 0], tied_lm_head=False, cycles=3,
                        seed=0xDF1A5 + 11)
    raise KeyError(name)


PRESETS = ["tiny", "qwen3_8b", "qwen3_8b_b32", "long_ctx", "llama31_8b", "qwen3_8b_depth8", "qwen3_4b",
           "qwen3_coder_30b", "small_bf16", "small_bf16_untied"]


# Tensor ids of the generator streams.
def _tid_layer(l: int, k: int) -> int:
    return 100 + 16 * l + k


def torch_dtype(w: Workload):
    return torch.float32 if w.dtype == "f32" else torch.bfloat16


def make_weights(w: Workload, device="cpu") -> Dict[str, object]:
    """Drafter weights: matrices N(0, 0.02), RMSNorm gains N(1, 0.02)."""
    dt = torch_dtype(w)
    s = w.seed
    H, d = w.hidden, w.head_dim
    out: Dict[str, object] = {}
    out["w_fc"] = normal(s, 1, (H, w.n_sel * w.target_hidden), 0.02, dtype=dt, device=device)
    out["g_fc"] = normal(s, 2, (H,), 0.02, 1.0, dtype=dt, device=device)
    out["embed"] = normal(s, 3, (w.vocab, H), 0.02, dtype=dt, device=device)
    out["lm_head"] = out["embed"] if w.tied_lm_head else normal(s, 4, (w.vocab, H), 0.02, dtype=dt, device=device)
    out["g_final"] = normal(s, 5, (H,), 0.02, 1.0, dtype=dt, device=device)
    layers = []
    for l in range(w.n_layers):
        layers.append({
            "g_in": normal(s, _tid_layer(l, 0), (H,), 0.02, 1.0, dtype=dt, device=device),
            "wq": normal(s, _tid_layer(l, 1), (w.n_q_heads * d, H), 0.02, dtype=dt, device=device),
            "wk": normal(s, _tid_layer(l, 2), (w.n_kv_heads * d, H), 0.02, dtype=dt, device=device),
            "wv": normal(s, _tid_layer(l, 3), (w.n_kv_heads * d, H), 0.02, dtype=dt, device=device),
            "wo": normal(s, _tid_layer(l, 4), (H, w.n_q_heads * d), 0.02, dtype=dt, device=device),
            "g_post": normal(s, _tid_layer(l, 5), (H,), 0.02, 1.0, dtype=dt, device=device),
            "w_gate": normal(s, _tid_layer(l, 6), (w.intermediate, H), 0.02, dtype=dt, device=device),
            "w_up": normal(s, _tid_layer(l, 7), (w.intermediate, H), 0.02, dtype=dt, device=device),
            "w_down": normal(s, _tid_layer(l, 8), (H, w.intermediate), 0.02, dtype=dt, device=device),
        })
    out["layers"] = layers
    return out


def make_hiddens(w: Workload, rows: int, stream: int = 0, device="cpu") -> List[torch.Tensor]:
    """n_sel target-layer hidden states, each [rows, target_hidden], N(0, 1)."""
    dt = torch_dtype(w)
    return [normal(w.seed, 5000 + 64 * stream + i, (rows, w.target_hidden), 1.0, dtype=dt, device=device)
            for i in range(w.n_sel)]


def make_anchors(w: Workload, stream: int = 0, device="cpu") -> torch.Tensor:
    return randint(w.seed, 7000 + stream, (w.batch,), 0, w.vocab, device=device)


def plan_accept(w: Workload, cycles: int, gamma: Optional[int] = None, stream: int = 0) -> torch.Tensor:
    """Planned acceptance lengths a* in [0, gamma-1], shape [cycles, batch].

    uniform: a* uniform in 0..gamma-1.  geometric: P(a) = (1-q) q^a truncated at
    gamma-1 (q = 0.87358 gives mean 6.0 at gamma = 16; q = 0.84448 gives mean 5).
    """
    g = w.gamma if gamma is None else gamma
    u = uniform(w.seed, 8000 + stream, (cycles, w.batch))
    if w.accept_kind == "uniform":
        a = torch.clamp((u * g).floor().to(torch.int64), max=g - 1)
    else:
        a = torch.floor(torch.log1p(-u) / math.log(w.accept_q)).to(torch.int64)
        a = torch.clamp(a, max=g - 1)
    return a.to(torch.int32)


def random_tokens(w: Workload, shape, stream: int = 0, device="cpu") -> torch.Tensor:
    return randint(w.seed, 9000 + stream, shape, 0, w.vocab, device=device)


def synthetic_cache_rows(w: Workload, layer: int, kind: int, request: int, rows: int, device="cpu") -> torch.Tensor:
    """Seeded K or V rows [n_kv_heads, rows, head_dim] with the spread of injected
    keys/values (N(0, 1.28^2): unit-RMS features through N(0, 0.02) weights of
    fan-in 4096).  Used where a test or benchmark fills a context cache directly
    instead of injecting thousands of rows."""
    dt = torch_dtype(w)
    return normal(w.seed, 20000 + 64 * (request * w.n_layers + layer) + kind,
                  (w.n_kv_heads, rows, w.head_dim), 0.02 * math.sqrt(w.hidden), dtype=dt, device=device)
