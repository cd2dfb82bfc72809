"""Python wrapper of the CPU oracle (test infrastructure only).

Loads liboracle.so (built from dflash_oracle.cpp) and marshals numpy arrays.
Only the tests, the package smoke check and the benchmark's CPU-baseline leg
use this module; the GPU library never imports it.  It imports nothing from
the GPU package either: callers pass numpy arrays (bf16 tensors as uint16 bit
patterns, fp32 as float32) and a plain dict of shapes.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Dict, List, Optional, Sequence

import numpy as np

from . import build as _build

_lib = None


class _Cfg(C.Structure):
    _fields_ = [("hidden", C.c_int), ("n_layers", C.c_int), ("n_q_heads", C.c_int),
                ("n_kv_heads", C.c_int), ("head_dim", C.c_int), ("intermediate", C.c_int),
                ("vocab", C.c_int), ("n_sel", C.c_int), ("target_hidden", C.c_int),
                ("mask_id", C.c_int), ("storage", C.c_int),
                ("rope_theta", C.c_double), ("rms_eps", C.c_double), ("acc32", C.c_int)]


class _W(C.Structure):
    _fields_ = [("w_fc", C.c_void_p), ("g_fc", C.c_void_p), ("embed", C.c_void_p),
                ("lm_head", C.c_void_p), ("g_final", C.c_void_p)] + \
               [(n, C.c_void_p * 16) for n in ("g_in", "wq", "wk", "wv", "wo", "g_post",
                                                "w_gate", "w_up", "w_down")]


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        dp = C.POINTER(C.c_double)
        ip = C.POINTER(C.c_int)
        L.oracle_round_bf16.restype = C.c_double
        L.oracle_round_bf16.argtypes = [C.c_double]
        L.oracle_round_bf16_array.argtypes = [dp, dp, C.c_long]
        L.oracle_rmsnorm.argtypes = [dp, dp, C.c_int, C.c_double, dp]
        L.oracle_rope.argtypes = [dp, C.c_int, C.c_long, C.c_double]
        L.oracle_attention.argtypes = [dp, C.c_int, C.c_int, dp, dp, C.c_int, C.c_int, C.c_int, C.c_int, dp]
        L.oracle_attention_block.argtypes = [dp, C.c_int, C.c_int, dp, dp, C.c_int, C.c_int, C.c_int, C.c_int,
                                             dp, dp, dp]
        L.oracle_layer_ids.argtypes = [C.c_int, C.c_int, ip]
        L.oracle_loss_weights.argtypes = [C.c_int, dp]
        L.oracle_fuse_context.argtypes = [C.POINTER(_Cfg), C.POINTER(_W), C.POINTER(C.c_void_p),
                                          C.c_long, C.c_int, dp]
        L.oracle_inject_kv.argtypes = [C.POINTER(_Cfg), C.POINTER(_W), dp, C.c_int, C.c_int, dp, dp, C.c_int]
        L.oracle_ingest_fused_input.argtypes = [C.POINTER(_Cfg), C.POINTER(_W), dp, C.c_int, C.c_int, dp, dp,
                                                C.c_int]
        L.oracle_draft_block.argtypes = [C.POINTER(_Cfg), C.POINTER(_W), dp, dp, C.c_int, C.c_int,
                                         C.c_int, C.c_int, ip, dp, dp]
        L.oracle_draft_layer.argtypes = [C.POINTER(_Cfg), C.POINTER(_W), C.c_int, dp, dp, C.c_int, C.c_int,
                                         C.c_int, dp]
        L.oracle_norm_rows.argtypes = [C.POINTER(_Cfg), C.c_void_p, dp, C.c_int, dp]
        L.oracle_layer_qkv.argtypes = [C.POINTER(_Cfg), C.POINTER(_W), C.c_int, dp, C.c_int, C.c_int, dp, dp, dp]
        L.oracle_layer_attention.argtypes = [C.POINTER(_Cfg), C.c_int, dp, dp, dp, dp, dp, C.c_int, C.c_int,
                                             C.c_int, dp]
        L.oracle_layer_oproj.argtypes = [C.POINTER(_Cfg), C.POINTER(_W), C.c_int, dp, dp, C.c_int, dp]
        L.oracle_layer_mlp.argtypes = [C.POINTER(_Cfg), C.POINTER(_W), C.c_int, dp, dp, C.c_int, dp, dp]
        L.oracle_layer_down.argtypes = [C.POINTER(_Cfg), C.POINTER(_W), C.c_int, dp, dp, C.c_int, dp]
        L.oracle_embed_block.argtypes = [C.POINTER(_Cfg), C.POINTER(_W), C.c_int, C.c_int, dp]
        L.oracle_final_norm.argtypes = [C.POINTER(_Cfg), C.POINTER(_W), dp, C.c_int, dp]
        L.oracle_lm_head.argtypes = [C.POINTER(_Cfg), C.POINTER(_W), dp, C.c_int, ip, dp, dp]
        L.oracle_accept.restype = C.c_int
        L.oracle_accept.argtypes = [C.c_int, C.c_int, ip, ip, ip, ip, ip, ip]
        L.oracle_num_threads.restype = C.c_int
        _lib = L
    return _lib


def _dp(a: np.ndarray):
    assert a.dtype == np.float64 and a.flags.c_contiguous
    return a.ctypes.data_as(C.POINTER(C.c_double))


def _ip(a: np.ndarray):
    assert a.dtype == np.int32 and a.flags.c_contiguous
    return a.ctypes.data_as(C.POINTER(C.c_int))


def num_threads() -> int:
    return lib().oracle_num_threads()


# ---------------------------------------------------------------------------
# Building blocks
# ---------------------------------------------------------------------------

def round_bf16(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty_like(x)
    lib().oracle_round_bf16_array(_dp(x), _dp(y), x.size)
    return y


def rmsnorm(x, g, eps: float) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    g = np.ascontiguousarray(g, dtype=np.float64)
    y = np.empty_like(x)
    lib().oracle_rmsnorm(_dp(x), _dp(g), x.size, eps, _dp(y))
    return y


def rope(v, pos: int, theta: float) -> np.ndarray:
    v = np.array(v, dtype=np.float64, copy=True)
    lib().oracle_rope(_dp(v), v.size, pos, theta)
    return v


def attention(q, k, v, round_p: bool = False) -> np.ndarray:
    """q: [nrow, nq, d]; k, v: [nkv, n, d] -> o [nrow, nq, d]."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    nrow, nq, d = q.shape
    nkv, n, _ = k.shape
    o = np.empty_like(q)
    lib().oracle_attention(_dp(q), nrow, nq, _dp(k), _dp(v), n, nkv, d, int(round_p), _dp(o))
    return o


def attention_block(q, k, v, round_p: bool = False):
    """Unnormalised attention over one block of keys: q [nrow, nq, d]; k, v
    [nkv, n, d] -> (num [nrow, nq, d], z [nrow, nq], base [nrow, nq]) with
    o = num / z and base the block's integer base-2 shift."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    nrow, nq, d = q.shape
    nkv, n, _ = k.shape
    num = np.empty_like(q)
    z = np.empty((nrow, nq), dtype=np.float64)
    base = np.empty((nrow, nq), dtype=np.float64)
    lib().oracle_attention_block(_dp(q), nrow, nq, _dp(k), _dp(v), n, nkv, d, int(round_p), _dp(num), _dp(z),
                                 _dp(base))
    return num, z, base


def layer_ids(n_target_layers: int, n_sel: int) -> List[int]:
    out = np.zeros(n_sel, dtype=np.int32)
    lib().oracle_layer_ids(n_target_layers, n_sel, _ip(out))
    return [int(v) for v in out]


def loss_weights(gamma: int) -> np.ndarray:
    w = np.zeros(gamma, dtype=np.float64)
    lib().oracle_loss_weights(gamma, _dp(w))
    return w


# ---------------------------------------------------------------------------
# The draft step
# ---------------------------------------------------------------------------

class OracleDrafter:
    """The oracle's drafter.  ``shape`` keys: hidden, n_layers, n_q_heads,
    n_kv_heads, head_dim, intermediate, vocab, n_sel, target_hidden, mask_id,
    storage ("bf16" | "f32"), rope_theta, rms_eps.  ``weights``: numpy arrays
    (uint16 bf16 bits or float32) named like the GPU library's weight table:
    w_fc, g_fc, embed, lm_head, g_final, and per layer (list ``layers``) g_in,
    wq, wk, wv, wo, g_post, w_gate, w_up, w_down."""

    def __init__(self, shape: Dict, weights: Dict):
        self.shape = dict(shape)
        st = 1 if shape["storage"] == "bf16" else 0
        self._np_dtype = np.uint16 if st == 1 else np.float32
        self.cfg = _Cfg(shape["hidden"], shape["n_layers"], shape["n_q_heads"], shape["n_kv_heads"],
                        shape["head_dim"], shape["intermediate"], shape["vocab"], shape["n_sel"],
                        shape["target_hidden"], shape["mask_id"], st,
                        float(shape["rope_theta"]), float(shape["rms_eps"]), int(shape.get("acc32", 0)))
        self._keep = []
        w = _W()

        def ptr(a):
            a = np.ascontiguousarray(a)
            assert a.dtype == self._np_dtype, (a.dtype, self._np_dtype)
            self._keep.append(a)
            return a.ctypes.data

        w.w_fc = ptr(weights["w_fc"])
        w.g_fc = ptr(weights["g_fc"])
        w.embed = ptr(weights["embed"])
        w.lm_head = ptr(weights["lm_head"])
        w.g_final = ptr(weights["g_final"])
        for l, lw in enumerate(weights["layers"]):
            for name in ("g_in", "wq", "wk", "wv", "wo", "g_post", "w_gate", "w_up", "w_down"):
                getattr(w, name)[l] = ptr(lw[name])
        self.w = w

    # -- cache of one request: k, v [L, nkv, cap, d] fp64 -------------------
    def new_cache(self, cap: int):
        s = self.shape
        k = np.zeros((s["n_layers"], s["n_kv_heads"], cap, s["head_dim"]), dtype=np.float64)
        return {"k": k, "v": np.zeros_like(k), "cap": cap, "len": 0, "committed": 0}

    def fuse_context(self, hiddens: Sequence[np.ndarray]) -> np.ndarray:
        """hiddens: n_sel arrays [rows, target_hidden] -> ctx [rows, hidden] fp64."""
        hs = [np.ascontiguousarray(h) for h in hiddens]
        for h in hs:
            assert h.dtype == self._np_dtype
        rows = hs[0].shape[0]
        arr = (C.c_void_p * len(hs))(*[h.ctypes.data for h in hs])
        out = np.empty((rows, self.shape["hidden"]), dtype=np.float64)
        lib().oracle_fuse_context(C.byref(self.cfg), C.byref(self.w), arr, hs[0].shape[1], rows, _dp(out))
        return out

    def inject_kv(self, cache: Dict, ctx: np.ndarray) -> None:
        ctx = np.ascontiguousarray(ctx, dtype=np.float64)
        rows = ctx.shape[0]
        if cache["len"] + rows > cache["cap"]:
            raise ValueError("capacity")
        lib().oracle_inject_kv(C.byref(self.cfg), C.byref(self.w), _dp(ctx), rows, cache["len"],
                               _dp(cache["k"]), _dp(cache["v"]), cache["cap"])
        cache["len"] += rows

    def ingest_fused_input(self, cache: Dict, ctx: np.ndarray) -> None:
        """Input-fusion ablation: the context rows pass through the draft layers as
        input hidden states (causal over the context) and every layer caches the
        K/V of its own normed state, in place of inject_kv."""
        ctx = np.ascontiguousarray(ctx, dtype=np.float64)
        rows = ctx.shape[0]
        if cache["len"] + rows > cache["cap"]:
            raise ValueError("capacity")
        lib().oracle_ingest_fused_input(C.byref(self.cfg), C.byref(self.w), _dp(ctx), rows, cache["len"],
                                        _dp(cache["k"]), _dp(cache["v"]), cache["cap"])
        cache["len"] += rows

    def draft_block(self, cache: Dict, anchor: int, gamma: int, want_logits: bool = False):
        """Returns (drafts [gamma-1] int32, margin [gamma-1], logits or None)."""
        if cache["len"] + gamma > cache["cap"]:
            raise ValueError("capacity")
        nd = max(gamma - 1, 0)
        drafts = np.zeros(max(nd, 1), dtype=np.int32)
        margin = np.zeros(max(nd, 1), dtype=np.float64)
        logits = np.zeros((max(nd, 1), self.shape["vocab"]), dtype=np.float64) if want_logits else None
        lib().oracle_draft_block(C.byref(self.cfg), C.byref(self.w), _dp(cache["k"]), _dp(cache["v"]),
                                 cache["cap"], cache["len"], int(anchor), int(gamma), _ip(drafts),
                                 _dp(logits) if logits is not None else None, _dp(margin))
        return drafts[:nd], margin[:nd], (logits[:nd] if logits is not None else None)

    # -- the draft step one piece at a time (call-local parity: each piece can
    #    be fed the GPU's own inputs) ----------------------------------------
    def embed_block(self, anchor: int, gamma: int) -> np.ndarray:
        x = np.empty((gamma, self.shape["hidden"]), dtype=np.float64)
        lib().oracle_embed_block(C.byref(self.cfg), C.byref(self.w), int(anchor), int(gamma), _dp(x))
        return x

    def draft_layer(self, cache: Dict, layer: int, x: np.ndarray) -> np.ndarray:
        """Layer `layer` on the block's hidden states x [gamma, hidden] over the
        cache's committed context; returns the layer's output (x is not changed)."""
        y = np.array(x, dtype=np.float64, copy=True, order="C")
        gamma = y.shape[0]
        if cache["len"] + gamma > cache["cap"]:
            raise ValueError("capacity")
        lib().oracle_draft_layer(C.byref(self.cfg), C.byref(self.w), int(layer), _dp(cache["k"]), _dp(cache["v"]),
                                 cache["cap"], cache["len"], gamma, _dp(y))
        return y

    # -- one layer one stage at a time --------------------------------------
    def norm_rows(self, gain: str, layer: int, x: np.ndarray) -> np.ndarray:
        """R(RMSNorm(x) * g) of rows x [rows, hidden]; gain one of g_in, g_post (per
        layer), g_final, g_fc."""
        x = np.ascontiguousarray(x, dtype=np.float64)
        gp = getattr(self.w, gain)[layer] if gain in ("g_in", "g_post") else getattr(self.w, gain)
        out = np.empty_like(x)
        lib().oracle_norm_rows(C.byref(self.cfg), gp, _dp(x), x.shape[0], _dp(out))
        return out

    def layer_qkv(self, layer: int, h: np.ndarray, pos0: int):
        """q [rows, nq*d], k, v [rows, nkv*d] of normalised rows h at positions pos0 + j."""
        s = self.shape
        h = np.ascontiguousarray(h, dtype=np.float64)
        g = h.shape[0]
        q = np.empty((g, s["n_q_heads"] * s["head_dim"]))
        k = np.empty((g, s["n_kv_heads"] * s["head_dim"]))
        v = np.empty_like(k)
        lib().oracle_layer_qkv(C.byref(self.cfg), C.byref(self.w), int(layer), _dp(h), int(pos0), g, _dp(q),
                               _dp(k), _dp(v))
        return q, k, v

    def layer_attention(self, cache: Dict, layer: int, q: np.ndarray, kb: np.ndarray, vb: np.ndarray) -> np.ndarray:
        """o [rows, nq*d]: the block queries over the cache's committed rows then the block's kb, vb."""
        q = np.ascontiguousarray(q, dtype=np.float64)
        kb = np.ascontiguousarray(kb, dtype=np.float64)
        vb = np.ascontiguousarray(vb, dtype=np.float64)
        o = np.empty_like(q)
        lib().oracle_layer_attention(C.byref(self.cfg), int(layer), _dp(q), _dp(kb), _dp(vb), _dp(cache["k"]),
                                     _dp(cache["v"]), cache["cap"], cache["len"], q.shape[0], _dp(o))
        return o

    def layer_oproj(self, layer: int, o: np.ndarray, x: np.ndarray) -> np.ndarray:
        o = np.ascontiguousarray(o, dtype=np.float64)
        x = np.ascontiguousarray(x, dtype=np.float64)
        out = np.empty_like(x)
        lib().oracle_layer_oproj(C.byref(self.cfg), C.byref(self.w), int(layer), _dp(o), _dp(x), x.shape[0], _dp(out))
        return out

    def layer_mlp(self, layer: int, h2: np.ndarray, x: np.ndarray):
        """(m [rows, intermediate], x_out [rows, hidden])."""
        h2 = np.ascontiguousarray(h2, dtype=np.float64)
        x = np.ascontiguousarray(x, dtype=np.float64)
        m = np.empty((x.shape[0], self.shape["intermediate"]))
        out = np.empty_like(x)
        lib().oracle_layer_mlp(C.byref(self.cfg), C.byref(self.w), int(layer), _dp(h2), _dp(x), x.shape[0], _dp(m),
                               _dp(out))
        return m, out

    def layer_down(self, layer: int, m: np.ndarray, x: np.ndarray) -> np.ndarray:
        """x_out [rows, hidden] = R(x + m . Wd^T) from the SwiGLU output m [rows, intermediate]."""
        m = np.ascontiguousarray(m, dtype=np.float64)
        x = np.ascontiguousarray(x, dtype=np.float64)
        out = np.empty_like(x)
        lib().oracle_layer_down(C.byref(self.cfg), C.byref(self.w), int(layer), _dp(m), _dp(x), x.shape[0], _dp(out))
        return out

    def final_norm(self, x: np.ndarray) -> np.ndarray:
        """hf rows of the mask positions 1..gamma-1 of x [gamma, hidden]."""
        x = np.ascontiguousarray(x, dtype=np.float64)
        gamma = x.shape[0]
        hf = np.empty((max(gamma - 1, 1), self.shape["hidden"]), dtype=np.float64)
        lib().oracle_final_norm(C.byref(self.cfg), C.byref(self.w), _dp(x), gamma, _dp(hf))
        return hf[:gamma - 1]

    def lm_head(self, hf: np.ndarray):
        """Shared LM head + argmax on normalised rows hf [rows, hidden] ->
        (drafts [rows] int32, margin [rows], logits [rows, vocab])."""
        hf = np.ascontiguousarray(hf, dtype=np.float64)
        rows = hf.shape[0]
        drafts = np.zeros(max(rows, 1), dtype=np.int32)
        margin = np.zeros(max(rows, 1), dtype=np.float64)
        logits = np.zeros((max(rows, 1), self.shape["vocab"]), dtype=np.float64)
        lib().oracle_lm_head(C.byref(self.cfg), C.byref(self.w), _dp(hf), rows, _ip(drafts), _dp(logits),
                             _dp(margin))
        return drafts[:rows], margin[:rows], logits[:rows]

    def accept(self, cache: Dict, drafts, target) -> tuple:
        """Returns (status, accept_len, next_anchor) and updates cache lengths."""
        target = np.ascontiguousarray(target, dtype=np.int32)
        gamma = target.size
        d = np.ascontiguousarray(drafts, dtype=np.int32)
        if d.size == 0:
            d = np.zeros(1, dtype=np.int32)
        a = np.zeros(1, dtype=np.int32)
        nxt = np.zeros(1, dtype=np.int32)
        ln = np.array([cache["len"]], dtype=np.int32)
        cm = np.array([cache["committed"]], dtype=np.int32)
        st = lib().oracle_accept(gamma, self.shape["vocab"], _ip(d), _ip(target), _ip(a), _ip(nxt), _ip(ln), _ip(cm))
        cache["len"], cache["committed"] = int(ln[0]), int(cm[0])
        return st, int(a[0]), int(nxt[0])
