"""Error behaviour of the C ABI on the GPU, with no GPU fault: host-detected
argument errors enqueue nothing; device-detected errors (state, capacity, token
range) land in the cache's sticky status word, skip only the affected request,
and are cleared by reading them; a bounded device wait that runs out reports
DFLASH_TIMEOUT and leaves the context usable."""
import numpy as np
import pytest
import torch

from block_diffusion_speculative_03_b200 import dflash as D
from block_diffusion_speculative_03_b200 import inputs as I
from tests.parity import Pair

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pair():
    w = I.preset("small_bf16")
    pr = Pair(w)
    pr.prefill(check=False)
    return pr


def _stream():
    return torch.cuda.current_stream().cuda_stream


def test_host_errors_enqueue_nothing(pair):
    h, c = pair.gpu.handle, pair.cache.handle
    B = pair.w.batch
    anc = torch.zeros(B, dtype=torch.int32, device="cuda")
    dr = torch.zeros(B, 32, dtype=torch.int32, device="cuda")
    n0 = pair.gpu.launch_count()
    assert D.dflash_draft_block(h, c, anc.data_ptr(), 0, dr.data_ptr(), stream=_stream(), check=False) == -1
    assert D.dflash_draft_block(h, c, anc.data_ptr(), 17, dr.data_ptr(), stream=_stream(), check=False) == -1
    assert D.dflash_draft_block(h, c, 0, 4, dr.data_ptr(), stream=_stream(), check=False) == -1
    assert D.dflash_accept(h, c, dr.data_ptr(), 0, 4, dr.data_ptr(), dr.data_ptr(), stream=_stream(), check=False) == -1
    assert D.dflash_inject_kv(h, c, dr.data_ptr(), anc.data_ptr(), anc.data_ptr(), 10 ** 7, _stream(), check=False) == -1
    assert D.dflash_fuse_context(h, [0] * pair.w.n_sel, pair.w.target_hidden, 4, dr.data_ptr(), _stream(),
                                 check=False) == -1
    assert pair.gpu.launch_count() == n0
    assert pair.cache.status() == 0


def test_state_error_skips_only_that_request(pair):
    w = pair.w
    B, g = w.batch, w.gamma
    lens0 = pair.cache.len.clone()
    # request 1 gets uncommitted rows (len != committed)
    rows = 3
    hid = I.make_hiddens(w, rows, stream=77)
    ctx = pair.gpu.fuse_context([x.cuda() for x in hid])
    pair.gpu.inject_kv(pair.cache, ctx, torch.tensor([0, 0], dtype=torch.int32, device="cuda"),
                       torch.tensor([0, rows], dtype=torch.int32, device="cuda"))
    anc = I.make_anchors(w).cuda()
    drafts = pair.gpu.draft_block(pair.cache, anc, g)
    torch.cuda.synchronize()
    assert pair.cache.status() == -6          # DFLASH_STATE
    assert pair.cache.status() == 0           # read clears it
    d = drafts.cpu().numpy()
    assert np.all(d[1] == -1)
    assert np.all((d[0] >= 0) & (d[0] < w.vocab))
    # restore
    pair.cache.set_len(lens0)
    torch.cuda.synchronize()
    assert pair.cache.status() == 0


def test_capacity_error_leaves_lengths(pair):
    w = pair.w
    lens0 = pair.cache.len.clone()
    big = pair.cap - int(lens0[0]) + 1        # one row more than request 0 can take
    hid = I.make_hiddens(w, big + 1, stream=78)
    ctx = pair.gpu.fuse_context([x.cuda() for x in hid])
    pair.gpu.inject_kv(pair.cache, ctx, torch.tensor([0, big], dtype=torch.int32, device="cuda"),
                       torch.tensor([big, 1], dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert pair.cache.status() == -5          # DFLASH_CAPACITY
    lens = pair.cache.len.cpu()
    assert int(lens[0]) == int(lens0[0]) and int(lens[1]) == int(lens0[1]) + 1
    pair.cache.set_len(lens0)
    torch.cuda.synchronize()
    assert pair.cache.status() == 0


def test_token_range_errors(pair):
    w = pair.w
    B, g = w.batch, w.gamma
    anc = torch.tensor([w.vocab, 5], dtype=torch.int32, device="cuda")
    drafts = pair.gpu.draft_block(pair.cache, anc, g)
    torch.cuda.synchronize()
    assert pair.cache.status() == -7
    assert np.all(drafts.cpu().numpy()[0] == -1)
    target = torch.zeros(B, g, dtype=torch.int32, device="cuda")
    target[1, 3] = -4
    acc = torch.empty(B, dtype=torch.int32, device="cuda")
    nxt = torch.empty(B, dtype=torch.int32, device="cuda")
    comm0 = pair.cache.committed.clone()
    pair.gpu.accept(pair.cache, drafts, target, acc, nxt)
    torch.cuda.synchronize()
    assert pair.cache.status() == -7
    assert int(acc[1]) == -1 and int(nxt[1]) == -1
    assert int(pair.cache.committed[1]) == int(comm0[1])
    assert int(acc[0]) >= 0
    pair.cache.set_len(pair.cache.len.clone())


def test_bounded_wait_times_out_and_context_survives(pair):
    out = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    D.dflash_diag_wait_selftest(pair.gpu.handle, out.data_ptr(), _stream())
    torch.cuda.synchronize()
    assert int(out.item()) == 0
    assert pair.cache.status() == -8          # DFLASH_TIMEOUT, reported once
    assert pair.cache.status() == 0
    x = torch.ones(4, device="cuda") * 2      # the context still works
    assert float(x.sum()) == 8.0
