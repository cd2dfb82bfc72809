"""The verify-side pre-step (dflash_fuse_inject: fuse + inject of the same rows in
one call, RMSNorm folded into the injection GEMM for small batches of rows)
against the oracle's fuse followed by its inject (DFlash-ja section 2.2,
context-feature and KV-injection bullets), call-locally: the context feature
the call reports is compared with the oracle's fuse of the same hidden rows,
and the cache rows with the oracle's inject of that feature."""
import numpy as np
import pytest
import torch

from block_diffusion_speculative_03_b200 import inputs as I
from block_diffusion_speculative_03_b200.drafter import Drafter, shape_from_workload
from tests.helpers import oracle_drafter, to_np
from tests.parity import Pair, check_float

pytestmark = pytest.mark.gpu


def _check(w, od, cache, ctx_g, hid, starts, counts, lens0):
    ctx_np = ctx_g.double().cpu().numpy()
    slab = cache.slab()
    cap = slab.shape[4]
    for b in range(w.batch):
        s0, n = int(starts[b]), int(counts[b])
        if n == 0:
            continue
        ctx_o = od.fuse_context([to_np(h[s0:s0 + n].cpu()) for h in hid])
        check_float(w, ctx_np[s0:s0 + n], ctx_o, "ctx[%d]" % b)
        oc = od.new_cache(cap)
        oc["len"] = int(lens0[b])
        od.inject_kv(oc, ctx_np[s0:s0 + n])
        new = slice(int(lens0[b]), int(lens0[b]) + n)
        check_float(w, slab[b, :, 0, :, new].double().cpu().numpy(), oc["k"][:, :, new], "K[%d]" % b)
        check_float(w, slab[b, :, 1, :, new].double().cpu().numpy(), oc["v"][:, :, new], "V[%d]" % b)


@pytest.mark.parametrize("name", ["small_bf16", "small_bf16_untied"])
def test_fuse_inject_small_prefill_then_cycle_rows(name):
    w = I.preset(name)
    pr = Pair(w)
    od = pr.ora
    # prefill of every request's context (wide token tiles: the two calls in sequence)
    total = sum(w.context)
    starts = np.cumsum([0] + w.context[:-1]).astype(np.int32)
    hid = [h.cuda() for h in I.make_hiddens(w, total, stream=31)]
    ctx = torch.empty(total, w.hidden, dtype=torch.bfloat16, device="cuda")
    lens0 = pr.cache.len.cpu().numpy().copy()
    pr.gpu.fuse_inject(pr.cache, hid, torch.tensor(starts, device="cuda"),
                       torch.tensor(w.context, dtype=torch.int32, device="cuda"), ctx_out=ctx)
    torch.cuda.synchronize()
    assert pr.cache.status() == 0
    assert np.array_equal(pr.cache.len.cpu().numpy(), lens0 + np.array(w.context))
    _check(w, od, pr.cache, ctx, hid, starts, w.context, lens0)
    pr.cache.set_len(torch.tensor(pr.cache.len.cpu().numpy(), dtype=torch.int32))
    # gamma verified rows per request (small token tiles: the folded path), twice
    for cyc in range(2):
        g = w.gamma
        hid = [h.cuda() for h in I.make_hiddens(w, w.batch * g, stream=40 + cyc)]
        starts = np.arange(0, w.batch * g, g, dtype=np.int32)
        counts = np.full(w.batch, g, dtype=np.int32)
        ctx = torch.empty(w.batch * g, w.hidden, dtype=torch.bfloat16, device="cuda")
        lens0 = pr.cache.len.cpu().numpy().copy()
        pr.gpu.fuse_inject(pr.cache, hid, torch.tensor(starts, device="cuda"), torch.tensor(counts, device="cuda"),
                           ctx_out=ctx)
        torch.cuda.synchronize()
        assert pr.cache.status() == 0
        assert np.array_equal(pr.cache.len.cpu().numpy(), lens0 + g)
        _check(w, od, pr.cache, ctx, hid, starts, counts, lens0)
    # without ctx_out: the same V rows as the call with it, injected again after them
    # (K rows differ only by their positions' rotation)
    lens0 = pr.cache.len.cpu().numpy().copy()
    pr.gpu.fuse_inject(pr.cache, hid, torch.tensor(starts, device="cuda"), torch.tensor(counts, device="cuda"))
    torch.cuda.synchronize()
    assert pr.cache.status() == 0
    slab = pr.cache.slab()
    for b in range(w.batch):
        a = slice(int(lens0[b]) - w.gamma, int(lens0[b]))
        bb = slice(int(lens0[b]), int(lens0[b]) + w.gamma)
        assert torch.equal(slab[b, :, 1, :, a], slab[b, :, 1, :, bb])


def test_fuse_inject_full_size_verified_block():
    # Qwen3-8B-shaped drafter: 16 verified rows of one request after a 2048-row context
    w = I.preset("qwen3_8b")
    W = I.make_weights(w, device="cuda")
    W["lm_head"] = W["embed"]
    T, g = w.context[0], w.gamma
    dr = Drafter(shape_from_workload(w), W, max_batch=1, max_rows=T, max_position=T + 64, max_gamma=g)
    cache = dr.new_cache(1, T + 64)
    cache.set_len(torch.tensor([T], dtype=torch.int32))
    hid = I.make_hiddens(w, g, stream=9, device="cuda")
    ctx = torch.empty(g, w.hidden, dtype=torch.bfloat16, device="cuda")
    dr.fuse_inject(cache, hid, torch.zeros(1, dtype=torch.int32, device="cuda"),
                   torch.full((1,), g, dtype=torch.int32, device="cuda"), ctx_out=ctx)
    torch.cuda.synchronize()
    assert cache.status() == 0 and int(cache.len.cpu()[0]) == T + g
    Wh = {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in W.items() if k != "layers"}
    Wh["layers"] = [{k: v.cpu() for k, v in lw.items()} for lw in W["layers"]]
    od = oracle_drafter(w, Wh)
    _check(w, od, cache, ctx, hid, np.array([0]), np.array([g]), np.array([T]))
