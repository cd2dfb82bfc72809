"""The input-fusion drafter (the conditioning KV injection is compared against:
DFlash-ja section 3, contribution 2, and section 4, KV-injection ablation
bullet) on the GPU against the oracle's oracle_ingest_fused_input: the context
rows pass through the draft layers, causal over the context, and every layer
caches the K/V of its own normed state; then a block is drafted over that
cache.  The oracle ingests the GPU's own context feature (compared first with
the oracle's fuse of the same hidden rows)."""
import dataclasses

import numpy as np
import pytest
import torch

from block_diffusion_speculative_03_b200 import inputs as I
from tests.helpers import to_np
from tests.parity import Pair, check_float

pytestmark = pytest.mark.gpu


def _ingest_all(pr, ctx_g, starts, chunk):
    """Ingest every request's context rows in calls of `chunk` rows per request."""
    w = pr.w
    B, H = w.batch, w.hidden
    done = [0] * B
    while any(done[b] < w.context[b] for b in range(B)):
        counts = [min(chunk, w.context[b] - done[b]) for b in range(B)]
        rows = torch.zeros(B * chunk, H, dtype=ctx_g.dtype, device="cuda")
        for b in range(B):
            if counts[b]:
                s0 = int(starts[b]) + done[b]
                rows[b * chunk:b * chunk + counts[b]] = ctx_g[s0:s0 + counts[b]]
        pr.gpu.ingest_fused_input(pr.cache, rows, chunk, torch.tensor(counts, dtype=torch.int32, device="cuda"))
        for b in range(B):
            done[b] += counts[b]
    torch.cuda.synchronize()
    assert pr.cache.status() == 0


@pytest.mark.parametrize("name,chunk", [("small_bf16", 16), ("small_bf16_untied", 8)])
def test_input_fusion_ingest_and_draft(name, chunk):
    w = dataclasses.replace(I.preset(name), context=[c for c in I.preset(name).context], cycles=1)
    if name == "small_bf16":
        w.context = [150, 90]            # the oracle ingests row by row; keep it quick
    pr = Pair(w)
    total = sum(w.context)
    starts = np.cumsum([0] + w.context[:-1]).astype(np.int32)
    hid = I.make_hiddens(w, total, stream=3)
    ctx_g = pr.gpu.fuse_context([h.cuda() for h in hid])
    torch.cuda.synchronize()
    ctx_np = ctx_g.double().cpu().numpy()
    _ingest_all(pr, ctx_g, starts, chunk)
    lens = pr.cache.len.cpu().numpy()
    assert np.array_equal(lens, np.array(w.context))
    slab = pr.cache.slab()
    for b in range(w.batch):
        T = w.context[b]
        s0 = int(starts[b])
        check_float(w, ctx_np[s0:s0 + T], pr.ora.fuse_context([to_np(h[s0:s0 + T]) for h in hid]), "ctx[%d]" % b)
        oc = pr.ocache[b]
        if T:
            pr.ora.ingest_fused_input(oc, ctx_np[s0:s0 + T])
        oc["committed"] = oc["len"]
        for l in range(w.n_layers):
            g = slab[b, l, :, :, :T].double().cpu().numpy()
            check_float(w, g[0], oc["k"][l, :, :T], "K[layer %d, b %d]" % (l, b))
            check_float(w, g[1], oc["v"][l, :, :T], "V[layer %d, b %d]" % (l, b))
    pr.cache.set_len(torch.tensor(w.context, dtype=torch.int32))
    anchors = I.make_anchors(w).numpy()
    _, _, compared = pr.draft(anchors, w.gamma)
    assert compared > 0


def test_input_fusion_rejects_rows_past_capacity():
    w = dataclasses.replace(I.preset("small_bf16"), context=[10, 20])
    pr = Pair(w, capacity=40)
    rows = 16
    ctx = torch.zeros(w.batch * rows, w.hidden, dtype=torch.bfloat16, device="cuda")
    pr.cache.set_len(torch.tensor([10, 30], dtype=torch.int32))   # request 1: 30 + 16 > 40
    pr.gpu.ingest_fused_input(pr.cache, ctx, rows)
    torch.cuda.synchronize()
    assert pr.cache.status() == -5                                  # DFLASH_CAPACITY
    assert np.array_equal(pr.cache.len.cpu().numpy(), [26, 30])     # request 0 appended, request 1 skipped
