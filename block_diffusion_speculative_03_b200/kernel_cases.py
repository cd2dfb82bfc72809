"""Single-kernel cases of libdflash for profiling (e.g. under Nsight Compute).

  python -m block_diffusion_speculative_03_b200.kernel_cases gemm --M 16 --N 24576 --K 4096 --iters 3
  python -m block_diffusion_speculative_03_b200.kernel_cases attention --batch 4 --context 32768 --gamma 16

`gemm` runs the tensor-core split-K GEMM (fp32 output) through the diagnostic
entry point on seeded bf16 operands; `attention` runs one layer's block
attention over a cache filled with seeded rows.  Each prints the CUDA-event
time of its last iteration.  Operands are sized by the caller: pick weights
larger than the 126 MB L2 so that DRAM counters mean something.
"""
from __future__ import annotations

import argparse

import torch

from . import dflash as D
from . import inputs as I
from .drafter import Drafter, shape_from_workload


def _time(fn, iters):
    ms = 0.0
    for _ in range(iters):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
    return ms


def gemm(M, N, K, grid, iters):
    X = I.normal(5, 1, (M, K), 1.0, dtype=torch.bfloat16, device="cuda")
    W = I.normal(5, 2, (N, K), 0.02, dtype=torch.bfloat16, device="cuda")
    Y = torch.empty(M, N, dtype=torch.float32, device="cuda")
    nbytes = D.dflash_diag_gemm_scratch_bytes(M, N, K)
    scratch = torch.zeros(nbytes + 256, dtype=torch.uint8, device="cuda")
    sp = (scratch.data_ptr() + 255) // 256 * 256
    st = torch.cuda.current_stream().cuda_stream
    ms = _time(lambda: D.dflash_diag_gemm_bf16(X.data_ptr(), W.data_ptr(), Y.data_ptr(), M, N, K, sp, nbytes,
                                               grid, st), iters)
    byts = (N * K + M * K) * 2 + M * N * 4
    print("gemm M=%d N=%d K=%d: %.1f us, %.0f GB/s (operands once)" % (M, N, K, ms * 1e3, byts / ms / 1e6))


def attention(B, T, gamma, nq, nkv, d, iters):
    w = I.Workload("attn", 512, 1, nq, nkv, d, 1024, 1024, 1, 512, 1e6, 1e-6, "bf16", batch=B, gamma=gamma,
                   context=[T] * B, seed=9)
    W = I.make_weights(w, device="cuda")
    cap = T + 2 * gamma + 8
    dr = Drafter(shape_from_workload(w), W, max_batch=B, max_rows=1, max_position=cap, max_gamma=gamma)
    cache = dr.new_cache(B, cap)
    slab = cache.slab()
    for b in range(B):
        for kind in (0, 1):
            slab[b, 0, kind, :, :T + gamma] = I.synthetic_cache_rows(w, 0, kind, b, T + gamma, device="cuda")
    cache.set_len(torch.tensor([T] * B, dtype=torch.int32))
    q = I.normal(9, 777, (B * gamma, nq * d), 1.3, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    st = torch.cuda.current_stream().cuda_stream
    ms = _time(lambda: D.dflash_diag_attention(dr.handle, cache.handle, q.data_ptr(), out.data_ptr(), 0, gamma, st),
               iters)
    kv = B * nkv * (T + gamma) * d * 2 * 2
    print("attention B=%d T=%d gamma=%d: %.1f us, KV %.1f MB, %.0f GB/s" % (B, T, gamma, ms * 1e3, kv / 1e6,
                                                                            kv / ms / 1e6))
    assert cache.status() == 0


def main():
    ap = argparse.ArgumentParser()
    sub = ap.add_subparsers(dest="case", required=True)
    g = sub.add_parser("gemm")
    g.add_argument("--M", type=int, default=16)
    g.add_argument("--N", type=int, default=24576)
    g.add_argument("--K", type=int, default=4096)
    g.add_argument("--grid", type=int, default=0)
    g.add_argument("--iters", type=int, default=3)
    a = sub.add_parser("attention")
    a.add_argument("--batch", type=int, default=4)
    a.add_argument("--context", type=int, default=32768)
    a.add_argument("--gamma", type=int, default=16)
    a.add_argument("--nq", type=int, default=32)
    a.add_argument("--nkv", type=int, default=8)
    a.add_argument("--d", type=int, default=128)
    a.add_argument("--iters", type=int, default=3)
    args = ap.parse_args()
    torch.cuda.set_device(0)
    if args.case == "gemm":
        gemm(args.M, args.N, args.K, args.grid, args.iters)
    else:
        attention(args.batch, args.context, args.gamma, args.nq, args.nkv, args.d, args.iters)


if __name__ == "__main__":
    main()
