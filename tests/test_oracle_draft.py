"""Pins of the oracle's composed draft step (fuse, inject, draft block).

The references here are independent of the oracle's code: torch fp64 library
routines (linear, rms_norm, scaled_dot_product_attention, silu), RoPE written
as a complex rotation, structural properties the DFlash summaries state (one
pass per block, conditioning at every layer, shared embedding/LM head), and
invariants of attention.
"""
import dataclasses

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from block_diffusion_speculative_03_b200 import inputs as I
from oracle import oracle as O
from tests.helpers import oracle_drafter, to_f64, to_np


def micro(dtype="f32", **kw):
    base = I.Workload("micro", 64, 2, 4, 2, 16, 96, 200, 3, 32, 1e4, 1e-6, dtype,
                      batch=1, gamma=5, context=[20], seed=77)
    return dataclasses.replace(base, **kw)


def _rope_t(x: torch.Tensor, pos: torch.Tensor, theta: float) -> torch.Tensor:
    """x [..., rows, heads, d] with positions [rows]; complex-rotation RoPE."""
    d = x.shape[-1]
    h = d // 2
    freqs = torch.tensor([theta ** (-2.0 * i / d) for i in range(h)], dtype=torch.float64)
    ang = pos.to(torch.float64)[:, None] * freqs[None, :]
    rot = torch.polar(torch.ones_like(ang), ang)[:, None, :]
    z = torch.complex(x[..., :h], x[..., h:]) * rot
    return torch.cat([z.real, z.imag], dim=-1)


def _R(t: torch.Tensor, bf16: bool) -> torch.Tensor:
    return t.to(torch.float32).to(torch.bfloat16).to(torch.float64) if bf16 else t


def torch_reference(w: I.Workload, W: dict, hiddens, gamma, anchor):
    """Whole draft step from torch fp64 library routines: fuse + inject the
    context, then draft one block.  Returns (ctx, K, V, logits)."""
    bf = w.dtype == "bf16"
    f = lambda t: t.to(torch.float64)
    H, d, nq, nkv = w.hidden, w.head_dim, w.n_q_heads, w.n_kv_heads
    cat = torch.cat([f(h) for h in hiddens], dim=1)
    y = _R(F.linear(cat, f(W["w_fc"])), bf)
    ctx = _R(F.rms_norm(y, (H,), f(W["g_fc"]), eps=w.rms_eps), bf)
    T = ctx.shape[0]
    pos_ctx = torch.arange(T)
    Ks, Vs = [], []
    for lw in W["layers"]:
        k = F.linear(ctx, f(lw["wk"])).view(T, nkv, d)
        Ks.append(_R(_rope_t(k, pos_ctx, w.rope_theta), bf))
        Vs.append(_R(F.linear(ctx, f(lw["wv"])).view(T, nkv, d), bf))
    toks = torch.tensor([anchor] + [w.mask_token] * (gamma - 1))
    x = f(W["embed"])[toks]
    pos_b = torch.arange(T, T + gamma)
    G = nq // nkv
    for l, lw in enumerate(W["layers"]):
        h = _R(F.rms_norm(x, (H,), f(lw["g_in"]), eps=w.rms_eps), bf)
        q = _R(_rope_t(F.linear(h, f(lw["wq"])).view(gamma, nq, d), pos_b, w.rope_theta), bf)
        kb = _R(_rope_t(F.linear(h, f(lw["wk"])).view(gamma, nkv, d), pos_b, w.rope_theta), bf)
        vb = _R(F.linear(h, f(lw["wv"])).view(gamma, nkv, d), bf)
        K = torch.cat([Ks[l], kb], 0).permute(1, 0, 2).repeat_interleave(G, 0)
        V = torch.cat([Vs[l], vb], 0).permute(1, 0, 2).repeat_interleave(G, 0)
        o = F.scaled_dot_product_attention(q.permute(1, 0, 2), K, V)      # no mask
        o = _R(o.permute(1, 0, 2).reshape(gamma, nq * d), bf)
        x = _R(x + F.linear(o, f(lw["wo"])), bf)
        h2 = _R(F.rms_norm(x, (H,), f(lw["g_post"]), eps=w.rms_eps), bf)
        m = _R(F.silu(F.linear(h2, f(lw["w_gate"]))) * F.linear(h2, f(lw["w_up"])), bf)
        x = _R(x + F.linear(m, f(lw["w_down"])), bf)
    hf = _R(F.rms_norm(x[1:], (H,), f(W["g_final"]), eps=w.rms_eps), bf)
    logits = F.linear(hf, f(W["lm_head"]))
    return ctx, Ks, Vs, logits


def _run_oracle(w, W, hiddens, gamma, anchor):
    od = oracle_drafter(w, W)
    ctx = od.fuse_context([to_np(h) for h in hiddens])
    cache = od.new_cache(hiddens[0].shape[0] + gamma)
    od.inject_kv(cache, ctx)
    cache["committed"] = cache["len"]
    drafts, margin, logits = od.draft_block(cache, anchor, gamma, want_logits=True)
    return od, ctx, cache, drafts, margin, logits


def test_draft_step_matches_torch_library_composition_fp32():
    w = micro("f32")
    W = I.make_weights(w)
    hid = I.make_hiddens(w, 20)
    od, ctx, cache, drafts, margin, logits = _run_oracle(w, W, hid, 5, 17)
    rctx, Ks, Vs, rlog = torch_reference(w, W, hid, 5, 17)
    assert np.allclose(ctx, rctx.numpy(), rtol=1e-10, atol=1e-12)
    for l in range(w.n_layers):
        assert np.allclose(cache["k"][l, :, :20], Ks[l].permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)
        assert np.allclose(cache["v"][l, :, :20], Vs[l].permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)
    assert np.allclose(logits, rlog.numpy(), rtol=1e-9, atol=1e-11)
    assert np.array_equal(drafts, rlog.argmax(1).numpy())
    top2 = torch.topk(rlog, 2, dim=1).values
    assert np.allclose(margin, (top2[:, 0] - top2[:, 1]).numpy(), atol=1e-10)


def test_draft_step_matches_torch_library_composition_bf16():
    w = micro("bf16")
    W = I.make_weights(w)
    hid = I.make_hiddens(w, 20)
    od, ctx, cache, drafts, margin, logits = _run_oracle(w, W, hid, 5, 3)
    rctx, Ks, Vs, rlog = torch_reference(w, W, hid, 5, 3)
    # torch rounds to bf16 through fp32 (double rounding is possible but rare)
    assert np.mean(ctx == rctx.numpy()) > 0.999
    assert np.max(np.abs(logits - rlog.numpy())) < 2e-2
    ok = margin > 0.05
    assert np.array_equal(drafts[ok], rlog.argmax(1).numpy()[ok])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_empty_context_is_a_bidirectional_encoder_over_the_block(dtype):
    # T = 0: nothing injected, so the block attends only to itself, at positions
    # 0..gamma-1, with no mask: a plain bidirectional encoder over the block.
    w = micro(dtype, context=[0])
    W = I.make_weights(w)
    od = oracle_drafter(w, W)
    cache = od.new_cache(8)
    cache["committed"] = cache["len"]
    assert cache["len"] == 0
    drafts, margin, logits = od.draft_block(cache, 23, 6, want_logits=True)
    empty = [h[:0] for h in I.make_hiddens(w, 1)]
    _, _, _, rlog = torch_reference(w, W, empty, 6, 23)
    if dtype == "f32":
        assert np.allclose(logits, rlog.numpy(), rtol=1e-9, atol=1e-11)
        assert np.array_equal(drafts, rlog.argmax(1).numpy())
    else:
        assert np.max(np.abs(logits - rlog.numpy())) < 2e-2
        ok = margin > 0.05
        assert np.array_equal(drafts[ok], rlog.argmax(1).numpy()[ok])


def test_fuse_concat_order_and_projection():
    # W_fc = [0 | I | 0] picks exactly the second selected layer: ctx = RMSNorm(h_1) * g
    w = micro("f32", hidden=32, target_hidden=32)
    W = I.make_weights(w)
    wfc = torch.zeros(32, 3 * 32)
    wfc[:, 32:64] = torch.eye(32)
    W["w_fc"] = wfc
    hid = I.make_hiddens(w, 6)
    od = oracle_drafter(w, W)
    ctx = od.fuse_context([to_np(h) for h in hid])
    g = to_f64(W["g_fc"])
    for r in range(6):
        x = to_f64(hid[1][r])
        exp = x / np.sqrt(np.mean(x * x) + w.rms_eps) * g
        assert np.allclose(ctx[r], exp, rtol=1e-12)
    # a non-symmetric W_fc: out[n] depends on row n of W_fc (not column n)
    wfc2 = torch.zeros(32, 96)
    wfc2[0, 95] = 1.0
    W["w_fc"] = wfc2
    ctx2 = oracle_drafter(w, W).fuse_context([to_np(h) for h in hid])
    assert np.all(ctx2[:, 1:] == 0) and np.all(ctx2[:, 0] != 0)
    assert np.allclose(np.sign(ctx2[:, 0]), np.sign(to_f64(hid[2][:, 31])) * np.sign(to_f64(W["g_fc"][0])))


def test_fuse_is_scale_invariant_per_row():
    w = micro("f32", rms_eps=0.0)
    W = I.make_weights(w)
    hid = I.make_hiddens(w, 4)
    od = oracle_drafter(w, W)
    a = od.fuse_context([to_np(h) for h in hid])
    b = od.fuse_context([to_np(h * 8.0) for h in hid])
    assert np.allclose(a, b, rtol=1e-9)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_inject_in_chunks_equals_all_at_once(dtype):
    w = micro(dtype)
    W = I.make_weights(w)
    hid = I.make_hiddens(w, 20)
    od = oracle_drafter(w, W)
    ctx = od.fuse_context([to_np(h) for h in hid])
    c1 = od.new_cache(32)
    od.inject_kv(c1, ctx)
    c2 = od.new_cache(32)
    od.inject_kv(c2, ctx[:7])
    od.inject_kv(c2, ctx[7:13])
    od.inject_kv(c2, ctx[13:])
    assert c1["len"] == c2["len"] == 20
    assert np.array_equal(c1["k"], c2["k"]) and np.array_equal(c1["v"], c2["v"])


def test_inject_writes_every_layer_with_its_own_weights():
    w = micro("f32")
    W = I.make_weights(w)
    od = oracle_drafter(w, W)
    ctx = np.random.default_rng(0).standard_normal((3, w.hidden))
    c = od.new_cache(8)
    od.inject_kv(c, ctx)
    for l in range(w.n_layers):
        v = ctx @ to_f64(W["layers"][l]["wv"]).T                 # V: no rotation
        assert np.allclose(c["v"][l, :, :3].transpose(1, 0, 2).reshape(3, -1), v, rtol=1e-12)
        k0 = ctx[0] @ to_f64(W["layers"][l]["wk"]).T             # position 0: RoPE is the identity
        assert np.allclose(c["k"][l, :, 0].reshape(-1), k0, rtol=1e-12)
    assert not np.allclose(c["k"][0], c["k"][1])


def test_draft_ignores_cache_row_order():
    # attention has no mask, so the committed context is a set: permuting the
    # cached rows (keys and values together, already rotated) changes nothing
    w = micro("f32")
    W = I.make_weights(w)
    hid = I.make_hiddens(w, 20)
    od, ctx, cache, drafts, margin, logits = _run_oracle(w, W, hid, 5, 9)
    perm = np.random.default_rng(1).permutation(20)
    c2 = dict(cache)
    c2["k"] = cache["k"].copy()
    c2["v"] = cache["v"].copy()
    c2["k"][:, :, :20] = cache["k"][:, :, perm]
    c2["v"][:, :, :20] = cache["v"][:, :, perm]
    d2, m2, l2 = od.draft_block(c2, 9, 5, want_logits=True)
    assert np.allclose(l2, logits, rtol=1e-10, atol=1e-12)


def test_block_is_one_bidirectional_pass():
    # In one block-diffusion pass every block position attends to every other.
    # So the first mask position's logits change with the block size, which a
    # causal (autoregressive) drafter would never do; and the anchor token
    # changes every mask position's logits.
    w = micro("f32")
    W = I.make_weights(w)
    hid = I.make_hiddens(w, 20)
    od = oracle_drafter(w, W)
    ctx = od.fuse_context([to_np(h) for h in hid])
    c = od.new_cache(40)
    od.inject_kv(c, ctx)
    c["committed"] = c["len"]
    _, _, l4 = od.draft_block(c, 9, 4, want_logits=True)
    _, _, l8 = od.draft_block(c, 9, 8, want_logits=True)
    assert not np.allclose(l4[0], l8[0])
    _, _, l8b = od.draft_block(c, 10, 8, want_logits=True)
    assert all(not np.allclose(l8[j], l8b[j]) for j in range(7))


def test_injected_context_conditions_every_layer():
    # Changing only the deepest layer's injected K/V changes the drafts' logits:
    # the context reaches the last layer directly, not only through layer 0.
    w = micro("f32")
    W = I.make_weights(w)
    hid = I.make_hiddens(w, 20)
    od, ctx, cache, drafts, margin, logits = _run_oracle(w, W, hid, 5, 9)
    c2 = dict(cache)
    c2["v"] = cache["v"].copy()
    c2["v"][w.n_layers - 1, :, :20] *= -1.0
    _, _, l2 = od.draft_block(c2, 9, 5, want_logits=True)
    assert not np.allclose(l2, logits)


def test_zero_layer_drafter_is_norm_then_shared_head():
    # With no draft layers the block's mask positions are the mask embedding,
    # so every draft row is argmax(E . RMSNorm(E[mask]) * g).
    w = micro("f32", n_layers=0)
    W = I.make_weights(w)
    od = oracle_drafter(w, W)
    c = od.new_cache(8)
    drafts, margin, logits = od.draft_block(c, 3, 4, want_logits=True)
    E = to_f64(W["embed"])
    e = E[w.mask_token]
    hf = e / np.sqrt(np.mean(e * e) + w.rms_eps) * to_f64(W["g_final"])
    exp = E @ hf
    for j in range(3):
        assert np.allclose(logits[j], exp, rtol=1e-12)
        assert drafts[j] == int(np.argmax(exp))


def test_argmax_ties_go_to_lowest_index():
    w = micro("f32", n_layers=0, vocab=16)
    W = I.make_weights(w)
    E = torch.zeros(16, w.hidden)
    E[5] = 1.0
    E[11] = 1.0
    E[15] = 1.0       # the mask row: rows 5, 11 and 15 give identical logits
    W["embed"] = E
    W["lm_head"] = E
    od = oracle_drafter(w, W)
    c = od.new_cache(8)
    drafts, margin, logits = od.draft_block(c, 0, 3, want_logits=True)
    assert logits[0][5] == logits[0][11] == logits[0][15] > 0
    assert list(drafts) == [5, 5]
    assert np.all(margin == 0.0)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_piecewise_draft_equals_one_call(dtype):
    # embed -> every layer -> final norm -> LM head, called one piece at a time
    # (the form the call-local GPU parity tests feed the GPU's own inputs to),
    # reproduces the one-call draft bit for bit
    w = micro(dtype)
    W = I.make_weights(w)
    hid = I.make_hiddens(w, 20)
    od, ctx, cache, drafts, margin, logits = _run_oracle(w, W, hid, 5, 11)
    x = od.embed_block(11, 5)
    for l in range(w.n_layers):
        x = od.draft_layer(cache, l, x)
    hf = od.final_norm(x)
    d2, m2, l2 = od.lm_head(hf)
    assert np.array_equal(d2, drafts) and np.array_equal(m2, margin) and np.array_equal(l2, logits)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_layer_stages_compose_to_the_layer(dtype):
    # norm -> qkv -> attention -> O-proj -> norm -> MLP (= SwiGLU, then down), one stage at a time (the form
    # the per-stage GPU parity tests feed the GPU's own inputs to), equals one layer call
    w = micro(dtype)
    W = I.make_weights(w)
    hid = I.make_hiddens(w, 20)
    od, ctx, cache, drafts, margin, logits = _run_oracle(w, W, hid, 5, 11)
    x = od.embed_block(11, 5)
    for l in range(w.n_layers):
        h = od.norm_rows("g_in", l, x)
        q, k, v = od.layer_qkv(l, h, cache["len"])
        o = od.layer_attention(cache, l, q, k, v)
        xm = od.layer_oproj(l, o, x)
        m, x2 = od.layer_mlp(l, od.norm_rows("g_post", l, xm), xm)
        assert np.array_equal(x2, od.layer_down(l, m, xm))
        assert np.array_equal(x2, od.draft_layer(cache, l, x))
        x = x2
