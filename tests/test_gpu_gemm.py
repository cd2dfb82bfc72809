"""Kernel-level checks of the sm_100a tcgen05 split-K GEMM (through the C ABI's
diagnostic entry point) against an fp64 CPU product of the same bf16 inputs."""
import pytest
import torch

from block_diffusion_speculative_03_b200 import dflash as D
from block_diffusion_speculative_03_b200 import inputs as I

pytestmark = pytest.mark.gpu


def _run(M, N, K, grid=0, seed=3, calls=1):
    X = I.normal(seed, 1, (M, K), 1.0, dtype=torch.bfloat16)
    W = I.normal(seed, 2, (N, K), 0.02, dtype=torch.bfloat16)
    ref = X.double() @ W.double().T
    Xd, Wd = X.cuda(), W.cuda()
    nbytes = D.dflash_diag_gemm_scratch_bytes(M, N, K)
    scratch = torch.zeros(nbytes + 256, dtype=torch.uint8, device="cuda")
    sp = (scratch.data_ptr() + 255) // 256 * 256
    outs = []
    for _ in range(calls):
        Y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        D.dflash_diag_gemm_bf16(Xd.data_ptr(), Wd.data_ptr(), Y.data_ptr(), M, N, K, sp, nbytes, grid,
                                torch.cuda.current_stream().cuda_stream)
        torch.cuda.synchronize()
        outs.append(Y.cpu().double())
    return ref, outs


def _close(ref, got, K):
    # fp32 accumulation of K bf16 products: error << 1e-3 of the row scale
    scale = ref.abs().max().item() + 1e-30
    err = (got - ref).abs().max().item()
    assert err <= 2e-4 * scale * max(1.0, (K / 1024) ** 0.5), (err, scale)


@pytest.mark.parametrize("M,N,K", [(16, 128, 64), (1, 128, 64), (15, 6144, 4096), (7, 300, 200), (16, 4096, 12288),
                                   (40, 640, 512), (100, 1000, 520), (300, 256, 1024), (513, 384, 256)])
def test_gemm_matches_fp64(M, N, K):
    ref, (got,) = _run(M, N, K)
    assert not torch.isnan(got).any()
    _close(ref, got, K)


@pytest.mark.parametrize("grid", [1, 3, 7, 64])
def test_gemm_split_tiles_and_repeat_calls(grid):
    # few CTAs over many k-blocks: every tile is split across CTAs and finished
    # by one of them; repeated calls check the counters are left at zero
    M, N, K = 16, 512, 2048
    ref, outs = _run(M, N, K, grid=grid, calls=3)
    for got in outs:
        _close(ref, got, K)
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])


def test_gemm_result_does_not_depend_on_partition_much():
    M, N, K = 16, 1024, 4096
    ref, (a,) = _run(M, N, K, grid=0)
    _, (b,) = _run(M, N, K, grid=5)
    _close(ref, a, K)
    _close(ref, b, K)


@pytest.mark.parametrize("M,N,K,grid", [(16, 512, 2048, 7), (16, 128, 12288, 0), (33, 1000, 4096, 0),
                                        (200, 640, 1024, 64), (16, 4096, 4096, 0), (5, 384, 704, 100),
                                        (256, 6144, 4096, 0), (256, 4096, 4096, 0), (256, 2048, 4096, 0),
                                        (256, 1024, 4096, 0), (128, 1024, 4096, 0), (64, 2048, 4096, 0),
                                        (250, 4096, 14336, 0)])
def test_split_tile_finishers_agree_bitwise(M, N, K, grid):
    """A split tile finished by its first contributor (waiting for the others'
    partials) and by its last arriver adds the same partials in the same order:
    identical bits, every call.  (16, 128, 12288) on the full grid splits one tile
    over all CTAs, so the first contributor waits for every other one.  The 64- to
    256-token tiles cover the chunked landing of wide partials at every depth (about
    3, 5, 10 and 18 contributors per tile: three, two and one chunk ahead, and the
    register path past the ring's capacity)."""
    try:
        D.dflash_diag_set_split_finisher(True)
        _, last = _run(M, N, K, grid=grid, calls=2)
        D.dflash_diag_set_split_finisher(False)
        ref, first = _run(M, N, K, grid=grid, calls=2)
    finally:
        D.dflash_diag_set_split_finisher(False)
        D.dflash_diag_set_gemm_max_cluster(0)
    _close(ref, first[0], K)
    for got in last + first[1:]:
        assert torch.equal(got, first[0])


@pytest.mark.parametrize("M,N,K", [(16, 6144, 4096), (16, 4096, 4096), (16, 24576, 4096), (5, 1024, 12288),
                                   (16, 128, 256), (1, 384, 704), (9, 640, 1024)])
def test_cluster_partition_matches_fp64_and_repeats(M, N, K):
    """16-token tiles in thread-block clusters (tiles owned by clusters, split
    tiles reduced through distributed shared memory; on a single tile the whole
    cluster contributes to it) against the fp64 product and against the
    whole-grid partition, with identical bits on repeated calls."""
    try:
        D.dflash_diag_set_gemm_max_cluster(4)
        ref, clu = _run(M, N, K, calls=3)
        D.dflash_diag_set_gemm_max_cluster(0)
        _, (grid,) = _run(M, N, K)
    finally:
        D.dflash_diag_set_gemm_max_cluster(0)
    for got in clu + [grid]:
        assert not torch.isnan(got).any()
        _close(ref, got, K)
    assert torch.equal(clu[0], clu[1]) and torch.equal(clu[1], clu[2])
