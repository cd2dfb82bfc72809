"""ctypes binding of libdflash (include/dflash.h, include/dflash_ablation.h,
include/dflash_diag.h, include/dflash_policy.h).

Functions carry the C names and only marshal arguments: every step of the
draft step runs in the library's CUDA kernels.  Pointers are passed as ints
(device addresses, e.g. ``tensor.data_ptr()``); streams as ``cudaStream_t``
ints (``torch.cuda.current_stream().cuda_stream``).  Non-zero statuses raise
:class:`DflashError` unless ``check=False``.

Loading fails loudly when libdflash.so has not been built: there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdflash.so")

DFLASH_F32, DFLASH_BF16 = 0, 1
DFLASH_MAX_LAYERS = 16
STATUS = {0: "OK", -1: "INVALID_ARG", -2: "UNSUPPORTED", -3: "CUDA", -4: "WORKSPACE", -5: "CAPACITY",
          -6: "STATE", -7: "TOKEN_RANGE", -8: "TIMEOUT"}


class DflashError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = status
        super().__init__("%s: %s (%d)" % (where, STATUS.get(status, "?"), status))


class dflash_config(C.Structure):
    _fields_ = [("hidden", C.c_int), ("n_layers", C.c_int), ("n_q_heads", C.c_int), ("n_kv_heads", C.c_int),
                ("head_dim", C.c_int), ("intermediate", C.c_int), ("vocab", C.c_int), ("n_sel", C.c_int),
                ("target_hidden", C.c_int), ("mask_id", C.c_int), ("max_gamma", C.c_int), ("dtype", C.c_int),
                ("max_batch", C.c_int), ("max_rows", C.c_int), ("max_position", C.c_int), ("reserved", C.c_int),
                ("rope_theta", C.c_double), ("rms_eps", C.c_double)]


_PL = C.c_void_p * DFLASH_MAX_LAYERS


class dflash_weights(C.Structure):
    _fields_ = [("w_fc", C.c_void_p), ("g_fc", C.c_void_p), ("embed", C.c_void_p), ("lm_head", C.c_void_p),
                ("g_final", C.c_void_p), ("g_in", _PL), ("wq", _PL), ("wk", _PL), ("wv", _PL), ("wo", _PL),
                ("g_post", _PL), ("w_gate", _PL), ("w_up", _PL), ("w_down", _PL)]


class dflash_cache_info(C.Structure):
    _fields_ = [("batch", C.c_int), ("capacity", C.c_int), ("status", C.c_void_p), ("len", C.c_void_p),
                ("committed", C.c_void_p), ("slab", C.c_void_p), ("stride_kv", C.c_int64),
                ("stride_kind", C.c_int64), ("stride_layer", C.c_int64), ("stride_request", C.c_int64)]


DFLASH_POLICY_MAX_CANDIDATES = 8


class dflash_gamma_policy(C.Structure):
    _fields_ = [("n_candidates", C.c_int), ("candidates", C.c_int * DFLASH_POLICY_MAX_CANDIDATES),
                ("decay", C.c_double), ("cost_fixed", C.c_double), ("cost_per_token", C.c_double),
                ("prior_accepts", C.c_double), ("prior_rejects", C.c_double), ("accepts", C.c_double),
                ("rejects", C.c_double)]


_lib = None


def lib():
    """Load libdflash.so (raises if it is missing; build it with build.py)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError("libdflash.so is not built (run block_diffusion_speculative_03_b200/build.py); "
                          "there is no fallback implementation")
    L = C.CDLL(LIB_PATH)
    vp, i32, i64, sz = C.c_void_p, C.c_int, C.c_int64, C.c_size_t
    sig = {
        "dflash_workspace_bytes": (i32, [C.POINTER(dflash_config), C.POINTER(sz)]),
        "dflash_create": (i32, [C.POINTER(dflash_config), C.POINTER(dflash_weights), vp, sz, C.POINTER(vp)]),
        "dflash_destroy": (None, [vp]),
        "dflash_cache_bytes": (i32, [vp, i32, i32, C.POINTER(sz)]),
        "dflash_cache_init": (i32, [vp, vp, sz, i32, i32, C.POINTER(vp), vp]),
        "dflash_cache_release": (None, [vp]),
        "dflash_cache_get_info": (i32, [vp, C.POINTER(dflash_cache_info)]),
        "dflash_cache_set_len": (i32, [vp, vp, vp]),
        "dflash_cache_status": (i32, [vp, vp, vp]),
        "dflash_fuse_context": (i32, [vp, C.POINTER(vp), i64, i32, vp, vp]),
        "dflash_inject_kv": (i32, [vp, vp, vp, vp, vp, i32, vp]),
        "dflash_fuse_inject": (i32, [vp, vp, C.POINTER(vp), i64, vp, vp, i32, vp, vp]),
        "dflash_ingest_fused_input": (i32, [vp, vp, vp, i32, vp, vp]),
        "dflash_draft_block": (i32, [vp, vp, vp, i32, vp, vp, vp, vp]),
        "dflash_accept": (i32, [vp, vp, vp, vp, i32, vp, vp, vp]),
        "dflash_status_string": (C.c_char_p, [i32]),
        "dflash_launch_count": (i64, [vp]),
        "dflash_diag_gemm_scratch_bytes": (i32, [i32, i32, i32, C.POINTER(sz)]),
        "dflash_diag_gemm_bf16": (i32, [vp, vp, vp, i32, i32, i32, vp, sz, i32, vp]),
        "dflash_diag_partition": (i32, [i64, i32, i32, i64, C.POINTER(i32), C.POINTER(i32)]),
        "dflash_diag_synth_target": (i32, [vp, vp, vp, i32, i32, i32, vp, vp]),
        "dflash_diag_arch": (C.c_char_p, []),
        "dflash_diag_timing_enable": (i32, [vp, i32]),
        "dflash_diag_timing_read": (i32, [vp, vp, C.POINTER(i32), C.POINTER(C.c_float), i32, C.POINTER(i32)]),
        "dflash_diag_timing_disable": (i32, [vp]),
        "dflash_diag_timed_name": (C.c_char_p, [i32]),
        "dflash_diag_set_launch_mode": (i32, [i32]),
        "dflash_diag_set_gemm_prefetch": (i32, [i32]),
        "dflash_diag_gemm_prefetch": (i32, []),
        "dflash_diag_set_gemm_pre_stages": (i32, [i32]),
        "dflash_diag_set_split_finisher": (i32, [i32]),
        "dflash_diag_set_gemm_max_cluster": (i32, [i32]),
        "dflash_diag_set_o_late_deficit": (i32, [i32]),
        "dflash_diag_set_gemm_tail": (i32, [i32, i32]),
        "dflash_diag_gemm_max_active_clusters": (i32, [i32]),
        "dflash_diag_set_norm_fold": (i32, [i32]),
        "dflash_diag_set_inject_partition": (i32, [i32]),
        "dflash_diag_set_o_beside_attention": (i32, [i32]),
        "dflash_diag_wait_selftest": (i32, [vp, vp, vp]),
        "dflash_diag_attention": (i32, [vp, vp, vp, vp, i32, i32, vp]),
        "dflash_diag_gemm_bf16_traced": (i32, [vp, vp, vp, i32, i32, i32, vp, sz, i32, vp, vp]),
        "dflash_diag_attention_traced": (i32, [vp, vp, vp, vp, i32, i32, vp, C.POINTER(i32), vp]),
        "dflash_diag_gemm_bf16_noalloc": (i32, [vp, vp, vp, i32, i32, i32, i32, vp]),
        "dflash_diag_draft_capture": (i32, [vp, vp, vp]),
        "dflash_diag_draft_capture_stages": (i32, [vp, vp, vp, vp, vp, vp, vp]),
        "dflash_diag_step_trace": (i32, [vp, vp, i64]),
        "dflash_diag_step_trace_records": (i32, [vp, C.POINTER(C.c_int32), C.POINTER(i64), i32, C.POINTER(i32)]),
        "dflash_diag_gemm_bf16_noalloc_status": (i32, [C.POINTER(C.c_int32), vp]),
        "dflash_gamma_policy_init": (i32, [C.POINTER(dflash_gamma_policy), C.POINTER(i32), i32, C.c_double,
                                           C.c_double, C.c_double, C.c_double, C.c_double]),
        "dflash_gamma_policy_observe": (i32, [C.POINTER(dflash_gamma_policy), C.POINTER(C.c_int32), i32, i32]),
        "dflash_gamma_policy_alpha": (i32, [C.POINTER(dflash_gamma_policy), C.POINTER(C.c_double)]),
        "dflash_gamma_policy_expected_tokens": (i32, [C.c_double, i32, C.POINTER(C.c_double)]),
        "dflash_gamma_policy_choose": (i32, [C.POINTER(dflash_gamma_policy), C.POINTER(i32)]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def exported_symbols() -> list:
    return ["dflash_workspace_bytes", "dflash_create", "dflash_destroy", "dflash_cache_bytes", "dflash_cache_init",
            "dflash_cache_release", "dflash_cache_get_info", "dflash_cache_set_len", "dflash_cache_status",
            "dflash_fuse_context", "dflash_inject_kv", "dflash_fuse_inject", "dflash_draft_block", "dflash_accept",
            "dflash_ingest_fused_input",
            "dflash_status_string", "dflash_launch_count", "dflash_diag_gemm_scratch_bytes",
            "dflash_diag_gemm_bf16", "dflash_diag_partition", "dflash_diag_synth_target", "dflash_diag_arch",
            "dflash_diag_timing_enable", "dflash_diag_timing_read", "dflash_diag_timing_disable",
            "dflash_diag_timed_name", "dflash_diag_set_launch_mode", "dflash_diag_set_gemm_prefetch", "dflash_diag_gemm_prefetch",
            "dflash_diag_set_gemm_pre_stages", "dflash_diag_set_split_finisher", "dflash_diag_set_gemm_max_cluster",
            "dflash_diag_set_o_late_deficit", "dflash_diag_set_gemm_tail",
            "dflash_diag_gemm_max_active_clusters",
            "dflash_diag_set_norm_fold", "dflash_diag_set_inject_partition",
            "dflash_diag_set_o_beside_attention",
            "dflash_diag_wait_selftest",
            "dflash_diag_attention", "dflash_diag_gemm_bf16_traced",
            "dflash_diag_attention_traced", "dflash_diag_gemm_bf16_noalloc", "dflash_diag_draft_capture",
            "dflash_diag_draft_capture_stages",
            "dflash_diag_gemm_bf16_noalloc_status", "dflash_diag_step_trace", "dflash_diag_step_trace_records",
            "dflash_gamma_policy_init", "dflash_gamma_policy_observe", "dflash_gamma_policy_alpha",
            "dflash_gamma_policy_expected_tokens", "dflash_gamma_policy_choose"]


def _chk(st: int, where: str, check: bool = True) -> int:
    if check and st != 0:
        raise DflashError(st, where)
    return st


# ---------------------------------------------------------------------------
# C entry points
# ---------------------------------------------------------------------------

def dflash_workspace_bytes(cfg: dflash_config, check: bool = True):
    n = C.c_size_t(0)
    st = _chk(lib().dflash_workspace_bytes(C.byref(cfg), C.byref(n)), "dflash_workspace_bytes", check)
    return n.value if st == 0 else st


def dflash_create(cfg: dflash_config, w: dflash_weights, workspace: int, ws_bytes: int, check: bool = True):
    h = C.c_void_p()
    st = _chk(lib().dflash_create(C.byref(cfg), C.byref(w), workspace, ws_bytes, C.byref(h)), "dflash_create", check)
    return h.value if st == 0 else st


def dflash_destroy(h: int) -> None:
    lib().dflash_destroy(h)


def dflash_cache_bytes(h: int, batch: int, capacity: int, check: bool = True):
    n = C.c_size_t(0)
    st = _chk(lib().dflash_cache_bytes(h, batch, capacity, C.byref(n)), "dflash_cache_bytes", check)
    return n.value if st == 0 else st


def dflash_cache_init(h: int, mem: int, nbytes: int, batch: int, capacity: int, stream: int = 0, check: bool = True):
    c = C.c_void_p()
    st = _chk(lib().dflash_cache_init(h, mem, nbytes, batch, capacity, C.byref(c), stream), "dflash_cache_init", check)
    return c.value if st == 0 else st


def dflash_cache_release(c: int) -> None:
    lib().dflash_cache_release(c)


def dflash_cache_get_info(c: int) -> dflash_cache_info:
    info = dflash_cache_info()
    _chk(lib().dflash_cache_get_info(c, C.byref(info)), "dflash_cache_get_info")
    return info


def dflash_cache_set_len(c: int, lens: int, stream: int = 0, check: bool = True) -> int:
    return _chk(lib().dflash_cache_set_len(c, lens, stream), "dflash_cache_set_len", check)


def dflash_cache_status(h: int, c: int, stream: int = 0) -> int:
    return lib().dflash_cache_status(h, c, stream)


def dflash_fuse_context(h: int, hiddens: Sequence[int], row_stride: int, total_rows: int, ctx_out: int,
                        stream: int = 0, check: bool = True) -> int:
    arr = (C.c_void_p * max(1, len(hiddens)))(*hiddens)
    return _chk(lib().dflash_fuse_context(h, arr, row_stride, total_rows, ctx_out, stream), "dflash_fuse_context", check)


def dflash_inject_kv(h: int, c: int, ctx: int, row_start: int, row_count: int, total_rows: int, stream: int = 0,
                     check: bool = True) -> int:
    return _chk(lib().dflash_inject_kv(h, c, ctx, row_start, row_count, total_rows, stream), "dflash_inject_kv", check)


def dflash_fuse_inject(h: int, c: int, hiddens: Sequence[int], row_stride: int, row_start: int, row_count: int,
                       total_rows: int, ctx_out: Optional[int] = None, stream: int = 0, check: bool = True) -> int:
    arr = (C.c_void_p * max(1, len(hiddens)))(*hiddens)
    return _chk(lib().dflash_fuse_inject(h, c, arr, row_stride, row_start, row_count, total_rows, ctx_out, stream),
                "dflash_fuse_inject", check)


def dflash_ingest_fused_input(h: int, c: int, ctx: int, rows: int, row_count: Optional[int] = None, stream: int = 0,
                              check: bool = True) -> int:
    return _chk(lib().dflash_ingest_fused_input(h, c, ctx, rows, row_count, stream), "dflash_ingest_fused_input",
                check)


def dflash_draft_block(h: int, c: int, anchor: int, gamma: int, drafts: int, logits: Optional[int] = None,
                       margin: Optional[int] = None, stream: int = 0, check: bool = True) -> int:
    return _chk(lib().dflash_draft_block(h, c, anchor, gamma, drafts, logits, margin, stream),
                "dflash_draft_block", check)


def dflash_accept(h: int, c: int, drafts: int, target: int, gamma: int, accept_len: int, next_anchor: int,
                  stream: int = 0, check: bool = True) -> int:
    return _chk(lib().dflash_accept(h, c, drafts, target, gamma, accept_len, next_anchor, stream),
                "dflash_accept", check)


def dflash_status_string(status: int) -> str:
    return lib().dflash_status_string(status).decode()


def dflash_launch_count(h: int) -> int:
    return lib().dflash_launch_count(h)


def dflash_diag_gemm_scratch_bytes(M: int, N: int, K: int) -> int:
    n = C.c_size_t(0)
    _chk(lib().dflash_diag_gemm_scratch_bytes(M, N, K, C.byref(n)), "dflash_diag_gemm_scratch_bytes")
    return n.value


def dflash_diag_gemm_bf16(X: int, W: int, Y: int, M: int, N: int, K: int, scratch: int, scratch_bytes: int,
                          grid: int = 0, stream: int = 0, check: bool = True) -> int:
    return _chk(lib().dflash_diag_gemm_bf16(X, W, Y, M, N, K, scratch, scratch_bytes, grid, stream),
                "dflash_diag_gemm_bf16", check)


DFLASH_NOALLOC_SCRATCH_BYTES = 6 << 20


def dflash_diag_gemm_bf16_noalloc(X: int, W: int, Y: int, M: int, N: int, K: int, grid: int = 0, stream: int = 0,
                                  check: bool = True) -> int:
    """The same GEMM with its scratch in the library's static device array (no allocation)."""
    return _chk(lib().dflash_diag_gemm_bf16_noalloc(X, W, Y, M, N, K, grid, stream),
                "dflash_diag_gemm_bf16_noalloc", check)


def dflash_diag_gemm_bf16_noalloc_status(stream: int = 0) -> int:
    """Status word of the last no-allocation GEMM on this device (syncs `stream`)."""
    v = C.c_int32(0)
    _chk(lib().dflash_diag_gemm_bf16_noalloc_status(C.byref(v), stream), "dflash_diag_gemm_bf16_noalloc_status")
    return v.value


def dflash_diag_partition(units: int, kb: int, ctas: int, tile: int):
    f, n = C.c_int(0), C.c_int(0)
    st = lib().dflash_diag_partition(units, kb, ctas, tile, C.byref(f), C.byref(n))
    if st != 0:
        raise DflashError(st, "dflash_diag_partition")
    return f.value, n.value


def dflash_diag_synth_target(drafts: int, a_plan: int, rand_tokens: int, batch: int, gamma: int, vocab: int,
                             target: int, stream: int = 0) -> int:
    return _chk(lib().dflash_diag_synth_target(drafts, a_plan, rand_tokens, batch, gamma, vocab, target, stream),
                "dflash_diag_synth_target")


def dflash_diag_arch() -> str:
    return lib().dflash_diag_arch().decode()


def dflash_diag_timing_enable(h: int, max_launches: int) -> int:
    return _chk(lib().dflash_diag_timing_enable(h, max_launches), "dflash_diag_timing_enable")


def dflash_diag_timing_read(h: int, stream: int = 0, max_entries: int = 1 << 16):
    """List of (kind name, milliseconds) in launch order."""
    kinds = (C.c_int * max_entries)()
    ms = (C.c_float * max_entries)()
    n = C.c_int(0)
    _chk(lib().dflash_diag_timing_read(h, stream, kinds, ms, max_entries, C.byref(n)), "dflash_diag_timing_read")
    return [(dflash_diag_timed_name(kinds[i]), float(ms[i])) for i in range(n.value)]


def dflash_diag_timing_disable(h: int) -> int:
    return _chk(lib().dflash_diag_timing_disable(h), "dflash_diag_timing_disable")


def dflash_diag_timed_name(kind: int) -> str:
    return lib().dflash_diag_timed_name(kind).decode()


def dflash_diag_set_launch_mode(programmatic: bool) -> int:
    return _chk(lib().dflash_diag_set_launch_mode(1 if programmatic else 0), "dflash_diag_set_launch_mode")


def dflash_diag_step_trace(h: int, buf: Optional[int], words: int = 0) -> int:
    return _chk(lib().dflash_diag_step_trace(h, buf, words if buf else 0), "dflash_diag_step_trace")


def dflash_diag_step_trace_records(h: int, max_records: int = 4096):
    """List of dicts (kind name, blocks, words, wait_idx, exit_idx, offset) in launch order."""
    recs = (C.c_int32 * (5 * max_records))()
    offs = (C.c_int64 * max_records)()
    n = C.c_int(0)
    _chk(lib().dflash_diag_step_trace_records(h, recs, offs, max_records, C.byref(n)),
         "dflash_diag_step_trace_records")
    out = []
    for i in range(min(n.value, max_records)):
        out.append({"kind": dflash_diag_timed_name(recs[5 * i]), "blocks": recs[5 * i + 1], "words": recs[5 * i + 2],
                    "wait_idx": recs[5 * i + 3], "exit_idx": recs[5 * i + 4], "offset": offs[i]})
    return out


def dflash_diag_draft_capture(h: int, x_layers: Optional[int], hf: Optional[int]) -> int:
    return _chk(lib().dflash_diag_draft_capture(h, x_layers, hf), "dflash_diag_draft_capture")


def dflash_diag_set_gemm_prefetch(tiles: int) -> int:
    return _chk(lib().dflash_diag_set_gemm_prefetch(int(tiles)), "dflash_diag_set_gemm_prefetch")


def dflash_diag_set_gemm_pre_stages(stages: int) -> int:
    return _chk(lib().dflash_diag_set_gemm_pre_stages(int(stages)), "dflash_diag_set_gemm_pre_stages")


def dflash_diag_set_split_finisher(last_arriver: bool) -> int:
    return _chk(lib().dflash_diag_set_split_finisher(int(bool(last_arriver))), "dflash_diag_set_split_finisher")


def dflash_diag_set_gemm_max_cluster(max_cluster: int) -> int:
    return _chk(lib().dflash_diag_set_gemm_max_cluster(int(max_cluster)), "dflash_diag_set_gemm_max_cluster")


def dflash_diag_gemm_max_active_clusters(cluster_size: int) -> int:
    return int(lib().dflash_diag_gemm_max_active_clusters(int(cluster_size)))


def dflash_diag_set_o_late_deficit(units: int) -> int:
    return _chk(lib().dflash_diag_set_o_late_deficit(int(units)), "dflash_diag_set_o_late_deficit")


def dflash_diag_set_gemm_tail(ctas: int, units: int) -> int:
    return _chk(lib().dflash_diag_set_gemm_tail(int(ctas), int(units)), "dflash_diag_set_gemm_tail")


def dflash_diag_gemm_prefetch() -> int:
    return lib().dflash_diag_gemm_prefetch()


def dflash_diag_set_o_beside_attention(on: bool) -> int:
    return _chk(lib().dflash_diag_set_o_beside_attention(1 if on else 0), "dflash_diag_set_o_beside_attention")


def dflash_diag_set_inject_partition(whole_tiles: bool) -> int:
    return _chk(lib().dflash_diag_set_inject_partition(1 if whole_tiles else 0), "dflash_diag_set_inject_partition")


def dflash_diag_set_norm_fold(on) -> int:
    """0: no fold; 1 / True: fold the layer norms; 2: also fold the final norm into the LM head."""
    return _chk(lib().dflash_diag_set_norm_fold(int(on)), "dflash_diag_set_norm_fold")


def dflash_diag_draft_capture_stages(h: int, h_in=None, q=None, o=None, x_mid=None, h2=None, act=None) -> int:
    return _chk(lib().dflash_diag_draft_capture_stages(h, h_in, q, o, x_mid, h2, act),
                "dflash_diag_draft_capture_stages")


def dflash_diag_wait_selftest(h: int, out: int, stream: int = 0) -> int:
    return _chk(lib().dflash_diag_wait_selftest(h, out, stream), "dflash_diag_wait_selftest")


def dflash_diag_attention(h: int, c: int, q: int, out: int, layer: int, gamma: int, stream: int = 0) -> int:
    return _chk(lib().dflash_diag_attention(h, c, q, out, layer, gamma, stream), "dflash_diag_attention")


def dflash_diag_gemm_bf16_traced(X: int, W: int, Y: int, M: int, N: int, K: int, scratch: int, scratch_bytes: int,
                                 grid: int, trace: int, stream: int = 0) -> int:
    return _chk(lib().dflash_diag_gemm_bf16_traced(X, W, Y, M, N, K, scratch, scratch_bytes, grid, trace, stream),
                "dflash_diag_gemm_bf16_traced")


def dflash_diag_attention_traced(h: int, c: int, q: int, out: int, layer: int, gamma: int, trace: int,
                                 stream: int = 0) -> int:
    """Returns the split count the kernel used."""
    sp = C.c_int(0)
    _chk(lib().dflash_diag_attention_traced(h, c, q, out, layer, gamma, trace, C.byref(sp), stream),
         "dflash_diag_attention_traced")
    return sp.value


# -- block-size policy (include/dflash_policy.h; host arithmetic, no device) -------
def dflash_gamma_policy_init(candidates: Sequence[int], decay: float, cost_fixed: float, cost_per_token: float,
                             prior_accepts: float, prior_rejects: float, check: bool = True):
    """Returns a new dflash_gamma_policy (or the status when check=False and it fails)."""
    p = dflash_gamma_policy()
    arr = (C.c_int * max(len(candidates), 1))(*candidates)
    st = lib().dflash_gamma_policy_init(C.byref(p), arr, len(candidates), decay, cost_fixed, cost_per_token,
                                        prior_accepts, prior_rejects)
    _chk(st, "dflash_gamma_policy_init", check)
    return p if st == 0 else st


def dflash_gamma_policy_observe(p: dflash_gamma_policy, accept_len: Sequence[int], gamma: int,
                                check: bool = True) -> int:
    arr = (C.c_int32 * max(len(accept_len), 1))(*[int(a) for a in accept_len])
    return _chk(lib().dflash_gamma_policy_observe(C.byref(p), arr, len(accept_len), gamma),
                "dflash_gamma_policy_observe", check)


def dflash_gamma_policy_alpha(p: dflash_gamma_policy) -> float:
    out = C.c_double()
    _chk(lib().dflash_gamma_policy_alpha(C.byref(p), C.byref(out)), "dflash_gamma_policy_alpha")
    return out.value


def dflash_gamma_policy_expected_tokens(alpha: float, gamma: int, check: bool = True):
    out = C.c_double()
    st = lib().dflash_gamma_policy_expected_tokens(alpha, gamma, C.byref(out))
    _chk(st, "dflash_gamma_policy_expected_tokens", check)
    return out.value if st == 0 else st


def dflash_gamma_policy_choose(p: dflash_gamma_policy) -> int:
    out = C.c_int()
    _chk(lib().dflash_gamma_policy_choose(C.byref(p), C.byref(out)), "dflash_gamma_policy_choose")
    return out.value
