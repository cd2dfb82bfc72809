"""The block-attention kernel alone against the oracle's attention, on seeded
q / K / V, for context lengths that give one to many K/V tiles per split,
every split count the planner picks (cluster merge through distributed
shared memory), and query-row counts G * gamma on both sides of 32 (four or
two copies of the rows in the tile, each row's keys split over as many
threads), padded windows included."""
import numpy as np
import pytest
import torch

from block_diffusion_speculative_03_b200 import dflash as D
from block_diffusion_speculative_03_b200 import inputs as I
from block_diffusion_speculative_03_b200.drafter import Drafter, shape_from_workload
from oracle import oracle as O

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("lens,gamma,nq,nkv,d", [([2048], 16, 32, 8, 128), ([100, 3000], 16, 8, 2, 128),
                                                 ([5000, 17, 700], 8, 6, 3, 64), ([64], 4, 8, 2, 128),
                                                 ([32768], 16, 32, 8, 128), ([4000], 8, 32, 8, 128),
                                                 ([1500, 250], 11, 12, 4, 128),
                                                 # 8 and 12 query heads per kv head: 128 and 120 query rows
                                                 ([2048, 300], 16, 32, 4, 128), ([700], 10, 24, 2, 64)])
def test_attention_kernel_matches_oracle(lens, gamma, nq, nkv, d):
    B = len(lens)
    w = I.Workload("attn", 512, 1, nq, nkv, d, 1024, 1024, 1, 512, 1e6, 1e-6, "bf16", batch=B, gamma=gamma,
                   context=lens, seed=99)
    W = I.make_weights(w, device="cuda")
    cap = max(lens) + gamma + 8
    dr = Drafter(shape_from_workload(w), W, max_batch=B, max_rows=1, max_position=cap, max_gamma=gamma)
    cache = dr.new_cache(B, cap)
    slab = cache.slab()
    for b in range(B):
        n = lens[b] + gamma
        for kind in (0, 1):
            slab[b, 0, kind, :, :n] = I.synthetic_cache_rows(w, 0, kind, b, n, device="cuda")
    cache.set_len(torch.tensor(lens, dtype=torch.int32))
    q = I.normal(99, 777, (B * gamma, nq * d), 1.3, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    D.dflash_diag_attention(dr.handle, cache.handle, q.data_ptr(), out.data_ptr(), 0, gamma,
                            torch.cuda.current_stream().cuda_stream)
    got = out.double().cpu().numpy().reshape(B, gamma, nq, d)
    qn = q.double().cpu().numpy().reshape(B, gamma, nq, d)
    for b in range(B):
        n = lens[b] + gamma
        k = slab[b, 0, 0, :, :n].double().cpu().numpy()
        v = slab[b, 0, 1, :, :n].double().cpu().numpy()
        ref = O.attention(qn[b], k, v, round_p=True)
        ref_r = O.round_bf16(ref)
        err = np.max(np.abs(got[b] - ref_r))
        scale = np.max(np.abs(ref))
        # The kernel rounds the same softmax weights as the oracle (integer base-2
        # shift), so outputs differ only where fp32 accumulation order moves a
        # value across a bf16 rounding boundary: one ulp, rarely.
        same = float(np.mean(got[b] == ref_r))
        print("attention lens=%s b=%d: max|err| %.3g (scale %.3g), identical %.4f" % (lens, b, err, scale, same))
        assert err <= 2.0 ** -7 * scale, (b, err, scale)
        assert same > 0.95, same
