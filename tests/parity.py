"""Shared machinery of the GPU parity tests: one workload driven through the
CUDA library (C ABI via the Drafter binding) and through the CPU oracle on the
same seeded inputs, with comparisons under the agreement rules:

  * drafted tokens, acceptance lengths, next anchors and cache lengths: exact
    (draft tokens compared only where the oracle's top-1 minus top-2 logit
    margin exceeds 0.1);
  * fp32 storage: logits within max relative error 1e-4 (max |g - r| / max |r|);
  * bf16 storage: logits within max absolute error 3e-2.
"""
from __future__ import annotations

import numpy as np
import torch

from block_diffusion_speculative_03_b200 import inputs as I
from block_diffusion_speculative_03_b200.drafter import Drafter, shape_from_workload
from tests.helpers import oracle_drafter, synth_target, to_np

MARGIN = 0.1
F32_LOGIT_REL = 1e-4
BF16_LOGIT_ABS = 3e-2


def rel_err(g: np.ndarray, r: np.ndarray) -> float:
    return float(np.max(np.abs(g - r)) / max(np.max(np.abs(r)), 1e-30))


def check_float(w: I.Workload, got: np.ndarray, ref: np.ndarray, what: str, bf16_rel: float = 2.0 ** -6,
                min_same: float = 0.9):
    """fp32: relative 1e-4; bf16 storage values: within 2^-6 of the tensor's scale, with at
    least 90 % of elements identical (the rest single rounding flips)."""
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    if got.size == 0:
        return
    if w.dtype == "f32":
        e = rel_err(got, ref)
        assert e <= F32_LOGIT_REL, (what, e)
    else:
        scale = max(float(np.max(np.abs(ref))), 1e-30)
        e = float(np.max(np.abs(got - ref)))
        assert e <= bf16_rel * scale, (what, e, scale)
        same = float(np.mean(got == ref))
        assert same >= min_same, (what, same)   # differences are single rounding flips, not systematic


MAX_SEEN = {"logits": 0.0}


def check_logits(w: I.Workload, got: np.ndarray, ref: np.ndarray, bf16_tol: float = BF16_LOGIT_ABS):
    if w.dtype == "f32":
        e = rel_err(got, ref)
        assert e <= F32_LOGIT_REL, ("logits rel", e)
    else:
        e = float(np.max(np.abs(got - ref)))
        assert e <= bf16_tol, ("logits abs", e, bf16_tol)
    MAX_SEEN["logits"] = max(MAX_SEEN["logits"], e)
    print("%s logits %s error %.3g" % (w.name, "max rel" if w.dtype == "f32" else "max abs", e))
    return e


def check_drafts(got: np.ndarray, ref: np.ndarray, margin: np.ndarray):
    ok = margin > MARGIN
    assert np.array_equal(got[ok], ref[ok]), (got[ok], ref[ok])
    return int(ok.sum())


class Pair:
    """The same workload on the GPU and in the oracle."""

    def __init__(self, w: I.Workload, max_rows: int = None, capacity: int = None, weights=None):
        self.w = w
        self.W = weights if weights is not None else I.make_weights(w)
        self.gW = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in self.W.items() if k != "layers"}
        self.gW["layers"] = [{k: v.cuda() for k, v in lw.items()} for lw in self.W["layers"]]
        if w.tied_lm_head:
            self.gW["lm_head"] = self.gW["embed"]
        self.cap = capacity or w.capacity()
        total = sum(w.context)
        self.max_rows = max_rows or max(total, w.batch * w.gamma, 1)
        self.gpu = Drafter(shape_from_workload(w), self.gW, max_batch=w.batch, max_rows=self.max_rows,
                           max_position=self.cap, max_gamma=max(w.gammas or [w.gamma]))
        self.cache = self.gpu.new_cache(w.batch, self.cap)
        self.ora = oracle_drafter(w, self.W)
        self.ocache = [self.ora.new_cache(self.cap) for _ in range(w.batch)]
        self.dt = I.torch_dtype(w)

    # -- prefill -----------------------------------------------------------
    def prefill(self, check: bool = True, stream: int = 0):
        w = self.w
        total = sum(w.context)
        starts = np.cumsum([0] + w.context[:-1]).astype(np.int32)
        if total == 0:
            return
        hid = I.make_hiddens(w, total, stream=stream)
        ctx_g = self.gpu.fuse_context([h.cuda() for h in hid])
        rs = torch.tensor(starts, dtype=torch.int32, device="cuda")
        rc = torch.tensor(w.context, dtype=torch.int32, device="cuda")
        self.gpu.inject_kv(self.cache, ctx_g, rs, rc)
        torch.cuda.synchronize()
        assert self.cache.status() == 0
        ctx_g_np = ctx_g.double().cpu().numpy()
        for b in range(w.batch):
            T = w.context[b]
            if T == 0:
                continue
            s0 = int(starts[b])
            ctx_o = self.ora.fuse_context([to_np(h[s0:s0 + T]) for h in hid])
            if check:
                check_float(w, ctx_g_np[s0:s0 + T], ctx_o, "ctx[%d]" % b)
            # the oracle injects the GPU's ctx (compared just above), so that the
            # cache comparison tests the injection and not an inherited ctx flip
            self.ora.inject_kv(self.ocache[b], ctx_g_np[s0:s0 + T])
            self.ocache[b]["committed"] = self.ocache[b]["len"]
        self.cache.set_len(torch.tensor(w.context, dtype=torch.int32))
        if check:
            self.check_cache()

    def check_cache(self, rows=None):
        slab = self.cache.slab()
        lens = self.cache.len.cpu().numpy()
        for b in range(self.w.batch):
            oc = self.ocache[b]
            assert lens[b] == oc["len"], (b, lens[b], oc["len"])
            n = oc["len"]
            if n == 0:
                continue
            sel = slice(None) if rows is None else rows
            g = slab[b, :, :, :, :n].double().cpu().numpy()      # [L, 2, nkv, n, d]
            check_float(self.w, g[:, 0][..., sel, :], oc["k"][:, :, :n][..., sel, :], "K[%d]" % b)
            check_float(self.w, g[:, 1][..., sel, :], oc["v"][:, :, :n][..., sel, :], "V[%d]" % b)

    # -- one draft / verify / accept cycle ----------------------------------
    def draft(self, anchors: np.ndarray, gamma: int):
        w = self.w
        B = w.batch
        nd = gamma - 1
        logits = torch.zeros(B, max(nd, 1), w.vocab, dtype=torch.float32, device="cuda")
        margin = torch.zeros(B, max(nd, 1), dtype=torch.float32, device="cuda")
        anc = torch.tensor(anchors, dtype=torch.int32, device="cuda")
        drafts = self.gpu.draft_block(self.cache, anc, gamma, logits=logits, margin=margin)
        torch.cuda.synchronize()
        st = self.cache.status()
        assert st == 0, st
        g_dr = drafts.cpu().numpy()[:, :nd]
        g_lg = logits.cpu().numpy()[:, :nd].astype(np.float64)
        g_mg = margin.cpu().numpy()[:, :nd]
        o_dr, o_mg = [], []
        compared = 0
        for b in range(B):
            d_o, m_o, l_o = self.ora.draft_block(self.ocache[b], int(anchors[b]), gamma, want_logits=True)
            check_logits(w, g_lg[b], l_o)
            compared += check_drafts(g_dr[b], d_o, m_o)
            ok = m_o > MARGIN
            assert np.allclose(g_mg[b][ok], m_o[ok], atol=(BF16_LOGIT_ABS * 2 if w.dtype == "bf16" else 1e-3))
            o_dr.append(d_o)
            o_mg.append(m_o)
        return np.array(o_dr, dtype=np.int32).reshape(B, nd), g_dr, compared

    def verify_and_accept(self, o_drafts: np.ndarray, gamma: int, a_star: np.ndarray, cycle: int,
                          order: str = "speculative"):
        """Target tokens from the oracle's drafts (teacher forcing); inject the
        gamma verified rows; accept.  Returns next anchors."""
        w = self.w
        B = w.batch
        rnd = I.random_tokens(w, (B, gamma), stream=100 + cycle).numpy()
        target = np.stack([synth_target(o_drafts[b], int(a_star[b]), rnd[b], w.vocab) for b in range(B)])
        hid = I.make_hiddens(w, B * gamma, stream=200 + cycle)
        ctx_g = self.gpu.fuse_context([h.cuda() for h in hid])
        rs = torch.arange(0, B * gamma, gamma, dtype=torch.int32, device="cuda")
        dr_g = torch.tensor(o_drafts if gamma > 1 else np.zeros((B, 1), np.int32), dtype=torch.int32, device="cuda")
        tg_g = torch.tensor(target, dtype=torch.int32, device="cuda")
        acc = torch.empty(B, dtype=torch.int32, device="cuda")
        nxt = torch.empty(B, dtype=torch.int32, device="cuda")
        if order == "speculative":
            rc = torch.full((B,), gamma, dtype=torch.int32, device="cuda")
            self.gpu.inject_kv(self.cache, ctx_g, rs, rc)
            self.gpu.accept(self.cache, dr_g, tg_g, acc, nxt)
        else:
            self.gpu.accept(self.cache, dr_g, tg_g, acc, nxt)
            rc = acc + 1
            self.gpu.inject_kv(self.cache, ctx_g, rs, rc)
        torch.cuda.synchronize()
        assert self.cache.status() == 0
        acc_g, nxt_g = acc.cpu().numpy(), nxt.cpu().numpy()
        ctx_g_np = ctx_g.double().cpu().numpy()
        out = []
        for b in range(B):
            ctx_o = self.ora.fuse_context([to_np(h[b * gamma:(b + 1) * gamma]) for h in hid])
            check_float(w, ctx_g_np[b * gamma:(b + 1) * gamma], ctx_o, "ctx rows [%d]" % b)
            ctx_o = ctx_g_np[b * gamma:(b + 1) * gamma]   # the oracle injects the GPU's ctx
            oc = self.ocache[b]
            if order == "speculative":
                self.ora.inject_kv(oc, ctx_o)
                st, a, nx = self.ora.accept(oc, o_drafts[b], target[b])
            else:
                st, a, nx = self.ora.accept(oc, o_drafts[b], target[b])
                self.ora.inject_kv(oc, ctx_o[:a + 1])
            assert st == 0
            assert a == int(a_star[b]) and acc_g[b] == a and nxt_g[b] == nx, (b, a, acc_g[b], nx, nxt_g[b])
            out.append(nx)
        lens = self.cache.len.cpu().numpy()
        comm = self.cache.committed.cpu().numpy()
        for b in range(B):
            assert lens[b] == self.ocache[b]["len"] and comm[b] == self.ocache[b]["committed"]
        return np.array(out, dtype=np.int32)
