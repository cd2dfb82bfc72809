"""Injection is bit-exact under chunking on the GPU (the oracle's own invariant,
DFlash-ja section 2.2, KV-injection bullet: the context feature of every
verified row is appended to every layer's cache): a 2048-row context of the
Qwen3-8B-shaped drafter injected in one call, in 16-row chunks, and in ragged
chunks writes identical K/V bits.  Under either work partition of the injection
GEMM (split-K per slab of tile rows, or whole output tiles) the summation order
of every element depends only on the weight shape and the grid, never on the
number of rows."""
import pytest
import torch

from block_diffusion_speculative_03_b200 import inputs as I
from block_diffusion_speculative_03_b200.drafter import Drafter, shape_from_workload

pytestmark = pytest.mark.gpu


def _inject(dr, cache, ctx, pieces):
    r0 = 0
    for n in pieces:
        dr.inject_kv(cache, ctx, torch.tensor([r0], dtype=torch.int32, device="cuda"),
                     torch.tensor([n], dtype=torch.int32, device="cuda"))
        r0 += n
    torch.cuda.synchronize()
    assert cache.status() == 0


@pytest.mark.parametrize("whole_tiles", [False, True])
def test_inject_2048_rows_in_chunks_is_bit_exact(whole_tiles):
    from block_diffusion_speculative_03_b200 import dflash as D
    D.dflash_diag_set_inject_partition(whole_tiles)
    try:
        _chunked(whole_tiles)
    finally:
        D.dflash_diag_set_inject_partition(True)


def _chunked(whole_tiles):
    w = I.preset("qwen3_8b")
    T = w.context[0]
    W = I.make_weights(w, device="cuda")
    W["lm_head"] = W["embed"]
    dr = Drafter(shape_from_workload(w), W, max_batch=1, max_rows=T, max_position=T + 64, max_gamma=w.gamma)
    hid = I.make_hiddens(w, T, stream=77, device="cuda")
    ctx = dr.fuse_context(hid)
    splits = {"one call": [T], "16-row chunks": [16] * (T // 16),
              "ragged": [1, 15, 100, 257, 640, 1035]}
    assert all(sum(v) == T for v in splits.values())
    slabs = {}
    for name, pieces in splits.items():
        cache = dr.new_cache(1, T + 64)
        _inject(dr, cache, ctx, pieces)
        assert int(cache.len.cpu()[0]) == T
        slabs[name] = cache.slab()[0, :, :, :, :T].clone()
        del cache
    ref = slabs["one call"]
    assert ref.abs().sum().item() > 0
    for name, s in slabs.items():
        assert torch.equal(s, ref), name
