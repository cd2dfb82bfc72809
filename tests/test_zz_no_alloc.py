"""The GEMM entry point that keeps its scratch in the library's static device
array (dflash_diag_gemm_bf16_noalloc), called through the C ABI: two calls in
a row must agree with the caller-scratch entry point (dflash_diag_gemm_bf16)
and with an fp64 product of the same bf16 inputs, must report a clear status
word, must not change the device's free memory, and sizes whose scratch
exceeds the array must be refused.

The file name sorts last so that the test also runs after every other GPU test
has used the library in the same process."""
import pytest
import torch

from block_diffusion_speculative_03_b200 import dflash as D
from block_diffusion_speculative_03_b200 import inputs as I

pytestmark = pytest.mark.gpu


def _close(ref, got, K):
    # fp32 accumulation of K bf16 products (same bound as the caller-scratch GEMM tests)
    scale = ref.abs().max().item() + 1e-30
    err = (got - ref).abs().max().item()
    assert err <= 2e-4 * scale * max(1.0, (K / 1024) ** 0.5), (err, scale)


@pytest.mark.parametrize("M,N,K,grid", [(16, 4096, 4096, 0), (32, 1000, 520, 0), (7, 300, 200, 0),
                                        (16, 512, 2048, 3), (64, 640, 512, 32), (1, 128, 64, 0)])
def test_noalloc_matches_caller_scratch_gemm(M, N, K, grid):
    X = I.normal(11, 1, (M, K), 1.0, dtype=torch.bfloat16)
    W = I.normal(11, 2, (N, K), 0.02, dtype=torch.bfloat16)
    ref64 = X.double() @ W.double().T
    Xd, Wd = X.cuda(), W.cuda()
    st = torch.cuda.current_stream().cuda_stream

    nbytes = D.dflash_diag_gemm_scratch_bytes(M, N, K)
    scratch = torch.zeros(nbytes + 256, dtype=torch.uint8, device="cuda")
    sp = (scratch.data_ptr() + 255) // 256 * 256
    Y0 = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    D.dflash_diag_gemm_bf16(Xd.data_ptr(), Wd.data_ptr(), Y0.data_ptr(), M, N, K, sp, nbytes, grid, st)

    Ys = [torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda") for _ in range(2)]
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    for Y in Ys:
        D.dflash_diag_gemm_bf16_noalloc(Xd.data_ptr(), Wd.data_ptr(), Y.data_ptr(), M, N, K, grid, st)
        # the status word in the static array: no bounded wait ran out
        assert D.dflash_diag_gemm_bf16_noalloc_status(st) == 0
    torch.cuda.synchronize()
    free_after = torch.cuda.mem_get_info()[0]
    # the first call on this device may have loaded the module (and with it the
    # array) only if no earlier noalloc call did; later calls allocate nothing
    D.dflash_diag_gemm_bf16_noalloc(Xd.data_ptr(), Wd.data_ptr(), Ys[1].data_ptr(), M, N, K, grid, st)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_after
    assert free_after <= free_before

    ref = Y0.cpu().double()
    _close(ref64, ref, K)
    for Y in Ys:
        got = Y.cpu().double()
        assert not torch.isnan(got).any()
        _close(ref64, got, K)
        _close(ref, got, K)


def test_noalloc_refuses_scratch_beyond_the_array():
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    M, N, K = 256, 1024, 4096        # nt = 256: 256 KiB of partials per CTA
    need = 2 * min(sms, 160) * 256 * 128 * 4
    assert need > D.DFLASH_NOALLOC_SCRATCH_BYTES
    X = torch.zeros(M, K, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(N, K, dtype=torch.bfloat16, device="cuda")
    Y = torch.full((M, N), 7.0, dtype=torch.float32, device="cuda")
    st = D.dflash_diag_gemm_bf16_noalloc(X.data_ptr(), W.data_ptr(), Y.data_ptr(), M, N, K, 0,
                                         torch.cuda.current_stream().cuda_stream, check=False)
    torch.cuda.synchronize()
    assert st == -4                  # DFLASH_WORKSPACE
    assert torch.all(Y == 7.0)       # nothing was launched
    # a grid small enough for the array runs
    D.dflash_diag_gemm_bf16_noalloc(X.data_ptr(), W.data_ptr(), Y.data_ptr(), M, N, K, 8,
                                    torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert torch.all(Y == 0.0)
