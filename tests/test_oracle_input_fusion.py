"""Pins of the oracle's input-fusion ablation (the conditioning KV injection is
compared against): the context rows pass through the draft layers as input
hidden states, causal over the context, and every layer caches the K/V of its
own normed state.  References independent of the oracle's code: a composition
of torch fp64 library routines with a causal mask, and structural properties
(appending in chunks = appending at once; one layer = injecting the normed
feature; different from KV injection)."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from block_diffusion_speculative_03_b200 import inputs as I
from tests.helpers import oracle_drafter, to_np
from tests.test_oracle_draft import _R, _rope_t, micro


def torch_input_fusion(w, W, ctx: torch.Tensor):
    """Per-layer cached K, V [T, nkv, d] of the input-fusion drafter over T context
    rows at positions 0..T-1, from torch fp64 library routines."""
    bf = w.dtype == "bf16"
    f = lambda t: t.to(torch.float64)
    H, d, nq, nkv = w.hidden, w.head_dim, w.n_q_heads, w.n_kv_heads
    T = ctx.shape[0]
    pos = torch.arange(T)
    G = nq // nkv
    x = ctx.clone()
    Ks, Vs = [], []
    for l, lw in enumerate(W["layers"]):
        h = _R(F.rms_norm(x, (H,), f(lw["g_in"]), eps=w.rms_eps), bf)
        k = _R(_rope_t(F.linear(h, f(lw["wk"])).view(T, nkv, d), pos, w.rope_theta), bf)
        v = _R(F.linear(h, f(lw["wv"])).view(T, nkv, d), bf)
        Ks.append(k)
        Vs.append(v)
        if l == w.n_layers - 1:
            break
        q = _R(_rope_t(F.linear(h, f(lw["wq"])).view(T, nq, d), pos, w.rope_theta), bf)
        K = k.permute(1, 0, 2).repeat_interleave(G, 0)
        V = v.permute(1, 0, 2).repeat_interleave(G, 0)
        o = F.scaled_dot_product_attention(q.permute(1, 0, 2), K, V, is_causal=True)
        o = _R(o.permute(1, 0, 2).reshape(T, nq * d), bf)
        x = _R(x + F.linear(o, f(lw["wo"])), bf)
        h2 = _R(F.rms_norm(x, (H,), f(lw["g_post"]), eps=w.rms_eps), bf)
        m = _R(F.silu(F.linear(h2, f(lw["w_gate"]))) * F.linear(h2, f(lw["w_up"])), bf)
        x = _R(x + F.linear(m, f(lw["w_down"])), bf)
    return Ks, Vs


def _ingest(w, W, T, chunks=None):
    od = oracle_drafter(w, W)
    hid = I.make_hiddens(w, T)
    ctx = od.fuse_context([to_np(h) for h in hid])
    cache = od.new_cache(T + 8)
    for a, b in (chunks or [(0, T)]):
        od.ingest_fused_input(cache, ctx[a:b])
    return od, ctx, cache


def test_input_fusion_matches_torch_composition_fp32():
    w = micro("f32", n_layers=3)
    W = I.make_weights(w)
    od, ctx, cache = _ingest(w, W, 20)
    Ks, Vs = torch_input_fusion(w, W, torch.from_numpy(ctx))
    for l in range(w.n_layers):
        assert np.allclose(cache["k"][l, :, :20], Ks[l].permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)
        assert np.allclose(cache["v"][l, :, :20], Vs[l].permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)


def test_input_fusion_matches_torch_composition_bf16():
    # torch weights the values with unrounded softmax probabilities, the oracle with
    # bf16-rounded ones (the path's reading), so deeper layers agree to a few ulps
    w = micro("bf16", n_layers=3)
    W = I.make_weights(w)
    od, ctx, cache = _ingest(w, W, 20)
    Ks, Vs = torch_input_fusion(w, W, torch.from_numpy(ctx))
    assert np.array_equal(cache["k"][0, :, :20], Ks[0].permute(1, 0, 2).numpy())   # no attention before layer 0
    for l in range(w.n_layers):
        ref_k = Ks[l].permute(1, 0, 2).numpy()
        assert np.max(np.abs(cache["k"][l, :, :20] - ref_k)) <= 2.0 ** -6 * np.max(np.abs(ref_k))
        assert np.mean(cache["k"][l, :, :20] == ref_k) > 0.75


def test_appending_in_chunks_equals_appending_at_once():
    w = micro("f32", n_layers=3)
    W = I.make_weights(w)
    _, _, once = _ingest(w, W, 20)
    _, _, parts = _ingest(w, W, 20, chunks=[(0, 7), (7, 8), (8, 20)])
    assert parts["len"] == once["len"] == 20
    assert np.array_equal(parts["k"], once["k"]) and np.array_equal(parts["v"], once["v"])


def test_one_layer_caches_the_normed_feature_projection():
    # With one layer nothing runs before its K/V: they are the KV injection of
    # R(RMSNorm(ctx) g_in) rather than of ctx itself.
    w = micro("f32", n_layers=1)
    W = I.make_weights(w)
    od, ctx, cache = _ingest(w, W, 12)
    g = W["layers"][0]["g_in"].double()
    normed = F.rms_norm(torch.from_numpy(ctx), (w.hidden,), g, eps=w.rms_eps).numpy()
    ref = od.new_cache(20)
    od.inject_kv(ref, normed)
    assert np.allclose(cache["k"][:, :, :12], ref["k"][:, :, :12], rtol=1e-12, atol=1e-14)
    assert np.allclose(cache["v"][:, :, :12], ref["v"][:, :, :12], rtol=1e-12, atol=1e-14)
    inj = od.new_cache(20)
    od.inject_kv(inj, ctx)
    assert not np.allclose(cache["k"][:, :, :12], inj["k"][:, :, :12])


def test_block_drafts_over_the_fused_input_cache():
    # The block pass is the same over either cache; the two conditionings differ.
    w = micro("f32", n_layers=2)
    W = I.make_weights(w)
    od, ctx, cache = _ingest(w, W, 20)
    cache["committed"] = cache["len"]
    d_f, m_f, l_f = od.draft_block(cache, 9, 5, want_logits=True)
    inj = od.new_cache(28)
    od.inject_kv(inj, ctx)
    inj["committed"] = inj["len"]
    d_i, m_i, l_i = od.draft_block(inj, 9, 5, want_logits=True)
    assert l_f.shape == l_i.shape == (4, w.vocab)
    assert not np.allclose(l_f, l_i)
