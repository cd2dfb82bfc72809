"""GPU path vs the CPU oracle, element by element, on reduced shapes that span
several GEMM tiles and ragged tails: prefill (fuse + inject), then chained
draft -> verify -> accept cycles with planned acceptance lengths.  The accept
step consumes the oracle's drafts (teacher forcing) so both sides follow the
same length trajectory; the GPU's own drafts are compared every cycle."""
import numpy as np
import pytest
import torch

from block_diffusion_speculative_03_b200 import inputs as I
from tests.helpers import gamma_schedule
from tests.parity import Pair

pytestmark = pytest.mark.gpu


def _chain(name, cycles=None, order="speculative", gamma=None):
    w = I.preset(name)
    if cycles is not None:
        w.cycles = cycles
    g = gamma or w.gamma
    pr = Pair(w)
    pr.prefill()
    anchors = I.make_anchors(w).numpy()
    plan = I.plan_accept(w, w.cycles, gamma=g).numpy()
    compared = 0
    for cyc in range(w.cycles):
        o_dr, g_dr, n = pr.draft(anchors, g)
        compared += n
        anchors = pr.verify_and_accept(o_dr, g, plan[cyc], cyc, order=order)
        pr.check_cache()
    return compared


def test_tiny_fp32_chain():
    # hidden 256, 2 layers, 4/2 heads, d 64, vocab 1024, 64 context rows, gamma 4
    n = _chain("tiny", cycles=6)
    assert n > 0


@pytest.mark.parametrize("fold", [1, 2, 0])
def test_small_bf16_chain_speculative_order(fold):
    # fold 1: each layer RMSNorm applied inside the GEMM that consumes it (the
    # default for token tiles up to 64 wide); 2: the final norm folded into the LM
    # head as well; 0: one normalisation kernel before each consumer
    from block_diffusion_speculative_03_b200 import dflash as D
    D.dflash_diag_set_norm_fold(fold)
    try:
        n = _chain("small_bf16")
    finally:
        D.dflash_diag_set_norm_fold(1)
    assert n > 0


def test_small_bf16_chain_commit_order():
    _chain("small_bf16", cycles=2, order="commit")


def test_small_bf16_untied_ragged_heads_and_empty_context():
    # d 64, 3 kv heads (K/V sections not multiples of 128), vocab 2500, one
    # request with an empty context, separate LM head
    n = _chain("small_bf16_untied")
    assert n > 0


def test_small_bf16_chain_dynamic_block_size():
    # The block size follows the host-side gamma policy from cycle to cycle
    # (4 -> 8 -> 16 -> 8 ...), through the same cache: every cycle's drafts,
    # acceptance, next anchor and cache rows against the oracle.
    w = I.preset("small_bf16")
    w.cycles = 6
    sched = gamma_schedule(w, w.cycles, (4, 8, 16), decay=0.5, cost_per_token=0.02)
    assert len({g for g, _ in sched}) == 3
    pr = Pair(w)
    pr.prefill()
    anchors = I.make_anchors(w).numpy()
    compared = 0
    for cyc, (g, a_star) in enumerate(sched):
        o_dr, g_dr, n = pr.draft(anchors, g)
        compared += n
        anchors = pr.verify_and_accept(o_dr, g, a_star, cyc)
        pr.check_cache()
    assert compared > 0


@pytest.mark.parametrize("gamma", [1, 2, 5, 8])
def test_small_bf16_other_block_sizes(gamma):
    w = I.preset("small_bf16")
    pr = Pair(w)
    pr.prefill(check=False)
    anchors = I.make_anchors(w).numpy()
    if gamma == 1:
        drafts = torch.empty(w.batch, 1, dtype=torch.int32, device="cuda")
        pr.gpu.draft_block(pr.cache, torch.tensor(anchors, dtype=torch.int32, device="cuda"), 1, drafts=drafts)
        torch.cuda.synchronize()
        assert pr.cache.status() == 0
        return
    pr.draft(anchors, gamma)


def test_inject_in_chunks_equals_all_at_once_on_gpu():
    w = I.preset("small_bf16")
    a = Pair(w)
    a.prefill(check=False)
    b = Pair(w, weights=a.W)
    total = sum(w.context)
    hid = I.make_hiddens(w, total)
    ctx = b.gpu.fuse_context([h.cuda() for h in hid])
    starts = np.cumsum([0] + w.context[:-1])
    # inject each request's rows in two pieces of different sizes
    for piece in range(2):
        rs, rc = [], []
        for r in range(w.batch):
            T = w.context[r]
            cut = T // 3
            rs.append(int(starts[r]) + (0 if piece == 0 else cut))
            rc.append(cut if piece == 0 else T - cut)
        b.gpu.inject_kv(b.cache, ctx, torch.tensor(rs, dtype=torch.int32, device="cuda"),
                        torch.tensor(rc, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(a.cache.len.cpu(), b.cache.len.cpu())
    sa, sb = a.cache.slab(), b.cache.slab()
    for r in range(w.batch):
        T = w.context[r]
        assert torch.equal(sa[r, :, :, :, :T], sb[r, :, :, :, :T])


def test_small_bf16_long_context_multi_tile_splits():
    # 2000 / 1500 context rows: every attention split holds several K/V tiles
    import dataclasses
    w = dataclasses.replace(I.preset("small_bf16"), context=[2000, 1500], cycles=2)
    pr = Pair(w)
    pr.prefill()
    anchors = I.make_anchors(w).numpy()
    plan = I.plan_accept(w, w.cycles).numpy()
    for cyc in range(w.cycles):
        o_dr, g_dr, n = pr.draft(anchors, w.gamma)
        anchors = pr.verify_and_accept(o_dr, w.gamma, plan[cyc], cyc)


def test_small_bf16_wide_gqa_128_query_rows():
    # 8 query heads on one kv head at gamma 16: 128 query rows per kv head (one copy
    # of each row in the attention tile), through draft / verify / accept cycles
    import dataclasses
    w = dataclasses.replace(I.preset("small_bf16"), n_kv_heads=1, cycles=2)
    pr = Pair(w)
    pr.prefill()
    anchors = I.make_anchors(w).numpy()
    plan = I.plan_accept(w, w.cycles).numpy()
    compared = 0
    for cyc in range(w.cycles):
        o_dr, g_dr, n = pr.draft(anchors, w.gamma)
        compared += n
        anchors = pr.verify_and_accept(o_dr, w.gamma, plan[cyc], cyc)
        pr.check_cache()
    assert compared > 0


@pytest.mark.parametrize("batch,gamma", [(3, 16), (5, 16), (13, 16), (7, 13)])
def test_small_bf16_wide_token_tiles_ragged(batch, gamma):
    # B x gamma = 48, 80, 208 and 91 rows: 64-, 128- and 256-token tiles whose last
    # 32-token chunk is ragged, with split tiles finished from landed chunks of the
    # peers' partials, of the residual rows and of the RoPE rows (runs of positions
    # that break at request boundaries inside a chunk when gamma is 13)
    import dataclasses
    ctx = [300 - 17 * r for r in range(batch)]
    w = dataclasses.replace(I.preset("small_bf16"), batch=batch, gamma=gamma, context=ctx, cycles=2)
    pr = Pair(w)
    pr.prefill()
    anchors = I.make_anchors(w).numpy()
    plan = I.plan_accept(w, w.cycles, gamma=gamma).numpy()
    compared = 0
    for cyc in range(w.cycles):
        o_dr, g_dr, n = pr.draft(anchors, gamma)
        compared += n
        anchors = pr.verify_and_accept(o_dr, gamma, plan[cyc], cyc)
        pr.check_cache()
    assert compared > 0
