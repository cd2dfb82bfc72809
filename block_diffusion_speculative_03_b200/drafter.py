"""Torch-memory convenience layer over the C ABI.

:class:`Drafter` owns the device workspace and borrows the weight tensors;
:class:`Cache` owns the cache memory of a batch of requests; :class:`GammaPolicy`
holds the host-side block-size policy between cycles.  All arithmetic
happens in libdflash; this module allocates device memory with torch, passes
pointers and the current CUDA stream, and checks statuses.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence

import torch

from . import dflash as D

_DT = {"bf16": (D.DFLASH_BF16, torch.bfloat16), "f32": (D.DFLASH_F32, torch.float32)}


def _aligned_empty(nbytes: int, device, align: int = 1024):
    """uint8 device buffer and a pointer into it aligned to `align` bytes."""
    buf = torch.empty(nbytes + align, dtype=torch.uint8, device=device)
    p = buf.data_ptr()
    return buf, (p + align - 1) // align * align


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


class Cache:
    """Draft KV cache of `batch` requests with `capacity` positions each."""

    def __init__(self, drafter: "Drafter", batch: int, capacity: int):
        self.drafter = drafter
        self.batch, self.capacity = batch, capacity
        self.nbytes = D.dflash_cache_bytes(drafter.handle, batch, capacity)
        self._buf, self.ptr = _aligned_empty(self.nbytes, drafter.device)
        self.handle = D.dflash_cache_init(drafter.handle, self.ptr, self.nbytes, batch, capacity, _stream())
        self.info = D.dflash_cache_get_info(self.handle)

    def _i32(self, addr: int, n: int) -> torch.Tensor:
        base = self._buf.data_ptr()
        off = addr - base
        return self._buf[off:off + 4 * n].view(torch.int32)

    @property
    def len(self) -> torch.Tensor:
        return self._i32(self.info.len, self.batch)

    @property
    def committed(self) -> torch.Tensor:
        return self._i32(self.info.committed, self.batch)

    def slab(self) -> torch.Tensor:
        """The K/V slab as a tensor view [batch, L, 2, n_kv_heads, capacity, head_dim]."""
        d = self.drafter
        off = self.info.slab - self._buf.data_ptr()
        n = self.batch * d.n_layers * 2 * d.n_kv_heads * self.capacity * d.head_dim
        es = 2 if d.torch_dtype == torch.bfloat16 else 4
        return self._buf[off:off + n * es].view(d.torch_dtype).view(
            self.batch, d.n_layers, 2, d.n_kv_heads, self.capacity, d.head_dim)

    def set_len(self, lens: torch.Tensor) -> None:
        lens = lens.to(device=self.drafter.device, dtype=torch.int32).contiguous()
        D.dflash_cache_set_len(self.handle, lens.data_ptr(), _stream())

    def status(self) -> int:
        return D.dflash_cache_status(self.drafter.handle, self.handle, _stream())

    def __del__(self):
        try:
            if getattr(self, "handle", None):
                D.dflash_cache_release(self.handle)
                self.handle = None
        except Exception:
            pass


class Drafter:
    """A DFlash drafter bound to weights already resident on the GPU.

    weights: dict with w_fc, g_fc, embed, lm_head, g_final and a list `layers`
    of dicts (g_in, wq, wk, wv, wo, g_post, w_gate, w_up, w_down), every tensor
    contiguous, on `device`, in the storage dtype.
    """

    def __init__(self, shape: Dict, weights: Dict, max_batch: int, max_rows: int, max_position: int,
                 max_gamma: int = 16, device="cuda"):
        self.device = torch.device(device)
        if self.device.type == "cuda" and self.device.index is None:
            self.device = torch.device("cuda", torch.cuda.current_device())
        dt, self.torch_dtype = _DT[shape["dtype"]]
        self.n_layers = shape["n_layers"]
        self.n_kv_heads = shape["n_kv_heads"]
        self.head_dim = shape["head_dim"]
        self.hidden = shape["hidden"]
        self.vocab = shape["vocab"]
        self.n_sel = shape["n_sel"]
        self.target_hidden = shape["target_hidden"]
        self.max_gamma = max_gamma
        c = D.dflash_config()
        c.hidden, c.n_layers = shape["hidden"], shape["n_layers"]
        c.n_q_heads, c.n_kv_heads, c.head_dim = shape["n_q_heads"], shape["n_kv_heads"], shape["head_dim"]
        c.intermediate, c.vocab = shape["intermediate"], shape["vocab"]
        c.n_sel, c.target_hidden, c.mask_id = shape["n_sel"], shape["target_hidden"], shape["mask_id"]
        c.max_gamma, c.dtype = max_gamma, dt
        c.max_batch, c.max_rows, c.max_position = max_batch, max_rows, max_position
        c.rope_theta, c.rms_eps = float(shape["rope_theta"]), float(shape["rms_eps"])
        self.cfg = c
        self._weights = weights          # keep the borrowed tensors alive
        w = D.dflash_weights()
        w.w_fc, w.g_fc = weights["w_fc"].data_ptr(), weights["g_fc"].data_ptr()
        w.embed, w.lm_head = weights["embed"].data_ptr(), weights["lm_head"].data_ptr()
        w.g_final = weights["g_final"].data_ptr()
        for l, lw in enumerate(weights["layers"]):
            for name in ("g_in", "wq", "wk", "wv", "wo", "g_post", "w_gate", "w_up", "w_down"):
                t = lw[name]
                assert t.is_contiguous() and t.dtype == self.torch_dtype and t.device == self.device
                getattr(w, name)[l] = t.data_ptr()
        self.ws_bytes = D.dflash_workspace_bytes(c)
        self._ws, self.ws_ptr = _aligned_empty(self.ws_bytes, self.device)
        torch.cuda.synchronize(self.device)
        self.handle = D.dflash_create(c, w, self.ws_ptr, self.ws_bytes)

    def new_cache(self, batch: int, capacity: int) -> Cache:
        return Cache(self, batch, capacity)

    def launch_count(self) -> int:
        return D.dflash_launch_count(self.handle)

    # -- the four calls ----------------------------------------------------
    def fuse_context(self, hiddens: Sequence[torch.Tensor], out: Optional[torch.Tensor] = None) -> torch.Tensor:
        rows = hiddens[0].shape[0]
        stride = hiddens[0].stride(0)
        for h in hiddens:
            assert h.dtype == self.torch_dtype and h.stride(1) == 1 and h.stride(0) == stride and h.shape[0] == rows
        if out is None:
            out = torch.empty(rows, self.hidden, dtype=self.torch_dtype, device=self.device)
        D.dflash_fuse_context(self.handle, [h.data_ptr() for h in hiddens], stride, rows, out.data_ptr(), _stream())
        return out

    def inject_kv(self, cache: Cache, ctx: torch.Tensor, row_start: torch.Tensor, row_count: torch.Tensor) -> None:
        assert ctx.is_contiguous() and ctx.dtype == self.torch_dtype
        D.dflash_inject_kv(self.handle, cache.handle, ctx.data_ptr(), row_start.data_ptr(), row_count.data_ptr(),
                           ctx.shape[0], _stream())

    def fuse_inject(self, cache: Cache, hiddens: Sequence[torch.Tensor], row_start: torch.Tensor,
                    row_count: torch.Tensor, ctx_out: Optional[torch.Tensor] = None) -> Optional[torch.Tensor]:
        """fuse_context + inject_kv of the same rows in one library call."""
        rows = hiddens[0].shape[0]
        stride = hiddens[0].stride(0)
        for h in hiddens:
            assert h.dtype == self.torch_dtype and h.stride(1) == 1 and h.stride(0) == stride and h.shape[0] == rows
        D.dflash_fuse_inject(self.handle, cache.handle, [h.data_ptr() for h in hiddens], stride, row_start.data_ptr(),
                             row_count.data_ptr(), rows, ctx_out.data_ptr() if ctx_out is not None else None,
                             _stream())
        return ctx_out

    def ingest_fused_input(self, cache: Cache, ctx: torch.Tensor, rows: int,
                           row_count: Optional[torch.Tensor] = None) -> None:
        """Input-fusion ablation: append `rows` context rows per request (ctx [batch*rows, H])
        through the draft layers instead of injecting them."""
        assert ctx.is_contiguous() and ctx.dtype == self.torch_dtype and ctx.shape[0] == cache.batch * rows
        D.dflash_ingest_fused_input(self.handle, cache.handle, ctx.data_ptr(), rows,
                                    row_count.data_ptr() if row_count is not None else None, _stream())

    def draft_block(self, cache: Cache, anchor: torch.Tensor, gamma: int, drafts: Optional[torch.Tensor] = None,
                    logits: Optional[torch.Tensor] = None, margin: Optional[torch.Tensor] = None) -> torch.Tensor:
        if drafts is None:
            drafts = torch.empty(cache.batch, max(gamma - 1, 1), dtype=torch.int32, device=self.device)
        D.dflash_draft_block(self.handle, cache.handle, anchor.data_ptr(), gamma, drafts.data_ptr(),
                             logits.data_ptr() if logits is not None else None,
                             margin.data_ptr() if margin is not None else None, _stream())
        return drafts

    def accept(self, cache: Cache, drafts: torch.Tensor, target: torch.Tensor, accept_len: torch.Tensor,
               next_anchor: torch.Tensor) -> None:
        gamma = target.shape[1]
        D.dflash_accept(self.handle, cache.handle, drafts.data_ptr(), target.data_ptr(), gamma,
                        accept_len.data_ptr(), next_anchor.data_ptr(), _stream())

    def __del__(self):
        try:
            if getattr(self, "handle", None):
                D.dflash_destroy(self.handle)
                self.handle = None
        except Exception:
            pass


class GammaPolicy:
    """Block size for the next cycle from the acceptance lengths seen so far
    (include/dflash_policy.h): a geometric acceptance estimate with forgetting
    factor `decay`, and the candidate with the most expected committed tokens per
    unit of cycle cost (cost_fixed + cost_per_token * gamma).  Host only."""

    def __init__(self, candidates: Sequence[int] = (4, 8, 16), decay: float = 0.5, cost_fixed: float = 1.0,
                 cost_per_token: float = 0.02, prior_accepts: float = 1.0, prior_rejects: float = 1.0):
        self.state = D.dflash_gamma_policy_init(list(candidates), decay, cost_fixed, cost_per_token,
                                                prior_accepts, prior_rejects)

    def choose(self) -> int:
        return D.dflash_gamma_policy_choose(self.state)

    def observe(self, accept_len, gamma: int) -> None:
        """accept_len: the cycle's acceptance lengths (host sequence or tensor)."""
        if torch.is_tensor(accept_len):
            accept_len = accept_len.cpu().tolist()
        D.dflash_gamma_policy_observe(self.state, list(accept_len), gamma)

    @property
    def alpha(self) -> float:
        return D.dflash_gamma_policy_alpha(self.state)


def shape_from_workload(w) -> Dict:
    """Shape dict of a workload preset (inputs.Workload)."""
    return dict(hidden=w.hidden, n_layers=w.n_layers, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                head_dim=w.head_dim, intermediate=w.intermediate, vocab=w.vocab, n_sel=w.n_sel,
                target_hidden=w.target_hidden, mask_id=w.mask_token, dtype=w.dtype, rope_theta=w.rope_theta,
                rms_eps=w.rms_eps)
