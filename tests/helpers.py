"""Test helpers: marshal seeded torch tensors into the oracle's numpy form."""
from __future__ import annotations

import numpy as np
import torch

from block_diffusion_speculative_03_b200 import inputs as I
from oracle import oracle as O


def to_np(t: torch.Tensor) -> np.ndarray:
    """bf16 -> uint16 bit patterns; fp32 -> float32 (host copy)."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16).copy()
    if t.dtype == torch.float32:
        return t.numpy().copy()
    raise TypeError(t.dtype)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().to(torch.float64).numpy()


def shape_of(w: I.Workload) -> dict:
    return dict(hidden=w.hidden, n_layers=w.n_layers, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                head_dim=w.head_dim, intermediate=w.intermediate, vocab=w.vocab, n_sel=w.n_sel,
                target_hidden=w.target_hidden, mask_id=w.mask_token,
                storage="f32" if w.dtype == "f32" else "bf16", rope_theta=w.rope_theta, rms_eps=w.rms_eps)


def oracle_weights(weights: dict) -> dict:
    out = {k: to_np(weights[k]) for k in ("w_fc", "g_fc", "embed", "lm_head", "g_final")}
    out["layers"] = [{k: to_np(v) for k, v in lw.items()} for lw in weights["layers"]]
    return out


def oracle_drafter(w: I.Workload, weights: dict) -> O.OracleDrafter:
    return O.OracleDrafter(shape_of(w), oracle_weights(weights))


def synth_target(drafts: np.ndarray, a_star: int, rand_tokens: np.ndarray, vocab: int) -> np.ndarray:
    """Target tokens for one verified block of gamma = len(rand_tokens): equal to
    the drafts before a_star, different from the draft at a_star, seeded random
    after it.  Stands in for the target model's greedy verification."""
    gamma = rand_tokens.size
    t = rand_tokens.astype(np.int32).copy()
    t[:a_star] = drafts[:a_star]
    if a_star < gamma - 1 and t[a_star] == drafts[a_star]:
        t[a_star] = (t[a_star] + 1) % vocab
    return t


def gamma_schedule(w: I.Workload, cycles: int, candidates, decay: float = 0.5, cost_fixed: float = 1.0,
                   cost_per_token: float = 0.05, prior=(1.0, 1.0)):
    """Block sizes the library's gamma policy picks over `cycles` cycles of
    workload w, with each cycle's planned acceptance lengths (the workload's plan
    for its largest block, clipped to the block picked: the same truncated
    geometric law).  Host values only, fed alike to the GPU path and the oracle."""
    from block_diffusion_speculative_03_b200 import dflash as D
    plan = I.plan_accept(w, cycles, gamma=max(candidates)).numpy()
    p = D.dflash_gamma_policy_init(list(candidates), decay, cost_fixed, cost_per_token, prior[0], prior[1])
    out = []
    for c in range(cycles):
        g = D.dflash_gamma_policy_choose(p)
        a = np.minimum(plan[c], g - 1).astype(np.int32)
        D.dflash_gamma_policy_observe(p, a.tolist(), g)
        out.append((g, a))
    return out
