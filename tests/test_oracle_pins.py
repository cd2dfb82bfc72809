"""Pins of the CPU oracle against things other than itself.

Each test checks an oracle function against a closed form, an invariant, a
brute-force search, an independent library routine (torch fp64) or a value
table from the DFlash summaries, chosen so that a dropped term, a wrong sign
or index, or a transposed operand in the oracle fails at least one of them.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


# ---------------------------------------------------------------------------
# R(): round to nearest even bf16
# ---------------------------------------------------------------------------

def _bf16_neighbours(x: float):
    """The two bf16 values around x found by brute force over fp32 bit patterns."""
    f = np.float32(x)
    bits = int(np.array([f], dtype=np.float32).view(np.uint32)[0])
    lo_bits = bits & 0xFFFF0000
    cands = []
    for b in (lo_bits - 0x10000, lo_bits, lo_bits + 0x10000):
        b &= 0xFFFFFFFF
        v = float(np.array([b], dtype=np.uint32).view(np.float32)[0])
        if np.isfinite(v):
            cands.append((v, b))
    return cands


def test_round_bf16_matches_torch_on_fp32_values():
    # 10^6 fp32 values: random bit patterns (normals and subnormals), and exact ties.
    bits = rng.integers(0, 2**32, size=600_000, dtype=np.uint64).astype(np.uint32)
    ties = (rng.integers(0, 2**16, size=200_000, dtype=np.uint64).astype(np.uint32) << 16) | 0x8000
    sub = rng.integers(0, 0x007FFFFF, size=200_000, dtype=np.uint64).astype(np.uint32)
    allb = np.concatenate([bits, ties, sub])
    x = allb.view(np.float32).astype(np.float64)
    keep = np.isfinite(x) & (np.abs(x) < 3.3e38)
    x = x[keep]
    ours = O.round_bf16(x)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(ours, ref)


def test_round_bf16_is_nearest_even_by_brute_force():
    xs = np.concatenate([rng.standard_normal(2000) * 10.0 ** rng.integers(-40, 38, 2000),
                         rng.standard_normal(200) * 1e-39])
    for x in xs:
        r = O.round_bf16([x])[0]
        cands = _bf16_neighbours(x)
        best = min(abs(v - x) for v, _ in cands)
        assert abs(r - x) == best
        ties = [(v, b) for v, b in cands if abs(v - x) == best]
        if len(ties) == 2:  # exact tie: even mantissa (bit 16 of the fp32 pattern clear)
            even = [v for v, b in ties if ((b >> 16) & 1) == 0][0]
            assert r == even


def test_round_bf16_exact_values_and_specials():
    assert O.round_bf16([1.0])[0] == 1.0
    assert O.round_bf16([1.0 + 2**-8])[0] == 1.0            # tie -> even
    assert O.round_bf16([1.0 + 3 * 2**-8])[0] == 1.0 + 2**-6  # tie -> even (up)
    assert O.round_bf16([1.0 + 2**-8 + 2**-30])[0] == 1.0 + 2**-7
    assert O.round_bf16([2.0**-133])[0] == 2.0**-133         # smallest subnormal
    assert O.round_bf16([2.0**-135])[0] == 0.0
    assert np.isinf(O.round_bf16([3.5e38])[0])


# ---------------------------------------------------------------------------
# RMSNorm
# ---------------------------------------------------------------------------

def test_rmsnorm_matches_torch_and_unit_rms():
    for n in (7, 256, 4096):
        x = rng.standard_normal(n) * 3.0
        g = 1.0 + 0.02 * rng.standard_normal(n)
        eps = 1e-6
        ours = O.rmsnorm(x, g, eps)
        ref = F.rms_norm(torch.from_numpy(x), (n,), torch.from_numpy(g), eps=eps).numpy()
        assert np.allclose(ours, ref, rtol=1e-13, atol=1e-13)
        ones = O.rmsnorm(x, np.ones(n), 0.0)
        assert math.isclose(float(np.sqrt(np.mean(ones ** 2))), 1.0, rel_tol=1e-12)
    # scale invariance (eps = 0) and the role of the gain
    x = rng.standard_normal(64)
    g = rng.standard_normal(64)
    assert np.allclose(O.rmsnorm(5.0 * x, g, 0.0), O.rmsnorm(x, g, 0.0), rtol=1e-13)
    assert np.allclose(O.rmsnorm(x, 2.0 * g, 1e-5), 2.0 * O.rmsnorm(x, g, 1e-5), rtol=1e-13)


# ---------------------------------------------------------------------------
# RoPE
# ---------------------------------------------------------------------------

def _rope_complex(v: np.ndarray, pos: int, theta: float) -> np.ndarray:
    """Rotary embedding written as a complex rotation of (v_i + j v_{i+d/2})."""
    d = v.size
    h = d // 2
    z = torch.complex(torch.from_numpy(v[:h]), torch.from_numpy(v[h:]))
    freqs = torch.tensor([theta ** (-2.0 * i / d) for i in range(h)], dtype=torch.float64)
    rot = torch.polar(torch.ones(h, dtype=torch.float64), pos * freqs)
    out = z * rot
    return np.concatenate([out.real.numpy(), out.imag.numpy()])


def test_rope_identity_at_zero_and_complex_rotation():
    for d in (8, 64, 128):
        v = rng.standard_normal(d)
        assert np.array_equal(O.rope(v, 0, 1e4), v)
        for pos in (1, 17, 2047, 32790):
            assert np.allclose(O.rope(v, pos, 1e6), _rope_complex(v, pos, 1e6), rtol=0, atol=1e-12)


def test_rope_preserves_pair_norms_and_is_relative():
    d = 128
    q = rng.standard_normal(d)
    k = rng.standard_normal(d)
    for m, n, s in ((5, 3, 100), (0, 2000, 7), (4096, 1, 31000)):
        a = np.dot(O.rope(q, m, 1e6), O.rope(k, n, 1e6))
        b = np.dot(O.rope(q, m + s, 1e6), O.rope(k, n + s, 1e6))
        assert math.isclose(a, b, rel_tol=1e-9, abs_tol=1e-9)
        r = O.rope(q, m, 1e6)
        assert np.allclose(r[:64] ** 2 + r[64:] ** 2, q[:64] ** 2 + q[64:] ** 2, rtol=1e-12)


def test_rope_pairs_first_frequency_closed_form():
    # pair 0 rotates by exactly pos radians (theta^0 = 1)
    d = 16
    v = np.zeros(d)
    v[0] = 1.0
    r = O.rope(v, 3, 1e4)
    assert math.isclose(r[0], math.cos(3.0), abs_tol=1e-15)
    assert math.isclose(r[d // 2], math.sin(3.0), abs_tol=1e-15)
    assert np.count_nonzero(r) == 2


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------

def _sdpa_ref(q, k, v):
    """torch fp64 scaled_dot_product_attention, no mask, GQA by head repeat."""
    nrow, nq, d = q.shape
    nkv = k.shape[0]
    G = nq // nkv
    qt = torch.from_numpy(q).permute(1, 0, 2)                  # [nq, nrow, d]
    kt = torch.from_numpy(k).repeat_interleave(G, dim=0)       # [nq, n, d]
    vt = torch.from_numpy(v).repeat_interleave(G, dim=0)
    o = F.scaled_dot_product_attention(qt, kt, vt)
    return o.permute(1, 0, 2).numpy()


@pytest.mark.parametrize("nrow,nq,nkv,n,d", [(1, 1, 1, 1, 8), (4, 4, 2, 37, 64), (16, 8, 2, 300, 128), (3, 6, 3, 5, 16)])
def test_attention_matches_torch_sdpa(nrow, nq, nkv, n, d):
    q = rng.standard_normal((nrow, nq, d))
    k = rng.standard_normal((nkv, n, d))
    v = rng.standard_normal((nkv, n, d))
    assert np.allclose(O.attention(q, k, v), _sdpa_ref(q, k, v), rtol=1e-11, atol=1e-12)


def test_attention_closed_forms():
    d, n = 32, 50
    k = rng.standard_normal((2, n, d))
    v = rng.standard_normal((2, n, d))
    # q = 0: uniform weights -> mean of the value rows of the head's kv group
    o = O.attention(np.zeros((3, 4, d)), k, v)
    assert np.allclose(o[:, 0], v[0].mean(0)) and np.allclose(o[:, 1], v[0].mean(0))
    assert np.allclose(o[:, 2], v[1].mean(0)) and np.allclose(o[:, 3], v[1].mean(0))
    # a single key: output is that value row whatever q is
    q = rng.standard_normal((2, 2, d)) * 10
    o1 = O.attention(q, k[:, :1], v[:, :1])
    assert np.allclose(o1[:, 0], v[0, 0]) and np.allclose(o1[:, 1], v[1, 0])
    # softmax rows sum to 1: with V = 1 every output is 1
    o2 = O.attention(q, k, np.ones_like(v))
    assert np.allclose(o2, 1.0, rtol=0, atol=1e-12)
    # a strongly aligned key takes (almost) all the weight
    kk = k.copy()
    kk[0, 7] = q[0, 0] * 100
    o3 = O.attention(q[:1, :1], kk[:1], v[:1])
    assert np.allclose(o3[0, 0], v[0, 7], atol=1e-9)


def test_attention_gqa_equals_mha_with_duplicated_heads():
    d, n = 16, 20
    q = rng.standard_normal((5, 4, d))
    k = rng.standard_normal((2, n, d))
    v = rng.standard_normal((2, n, d))
    gqa = O.attention(q, k, v)
    mha = O.attention(q, np.repeat(k, 2, axis=0), np.repeat(v, 2, axis=0))
    assert np.array_equal(gqa, mha)


def test_attention_key_permutation_invariance_and_round_p():
    d, n = 64, 90
    q = rng.standard_normal((4, 2, d))
    k = rng.standard_normal((1, n, d))
    v = rng.standard_normal((1, n, d))
    perm = rng.permutation(n)
    a = O.attention(q, k, v)
    b = O.attention(q, k[:, perm], v[:, perm])
    assert np.allclose(a, b, rtol=1e-12, atol=1e-13)
    # rounding P to bf16 perturbs the output by at most ~2^-8 relative per weight
    c = O.attention(q, k, v, round_p=True)
    assert not np.array_equal(a, c)
    assert np.max(np.abs(a - c)) <= 2.0 ** -8 * np.max(np.abs(v)) + 1e-12


# ---------------------------------------------------------------------------
# Loss weights and layer ids
# ---------------------------------------------------------------------------

def _read_golden_wk():
    table = {}
    with open(os.path.join(GOLDEN, "loss_weights.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            g, rest = line.split(":")
            vals = [float(v) for v in rest.split()]
            table[int(g)] = vals
    return table


def test_loss_weights_golden_table():
    table = _read_golden_wk()
    assert set(table) == {16, 8, 4}
    for g, vals in table.items():
        w = O.loss_weights(g)
        assert w[0] == 1.0
        assert np.allclose(w, vals[:-1], rtol=0, atol=5e-5)
        assert math.isclose(float(w.sum()), vals[-1], abs_tol=5e-4)
        assert np.all(np.diff(w) < 0)


def test_layer_ids_uniform_shallow_to_deep():
    assert O.layer_ids(36, 5) == [0, 9, 18, 26, 35]
    assert O.layer_ids(32, 5) == [0, 8, 16, 23, 31]
    ids = O.layer_ids(28, 4)
    assert ids[0] == 0 and ids[-1] == 27 and ids == sorted(ids)


# ---------------------------------------------------------------------------
# Acceptance
# ---------------------------------------------------------------------------

def _brute_accept(drafts, target):
    gamma = len(target)
    for k in range(gamma - 1, -1, -1):
        if all(drafts[i] == target[i] for i in range(k)):
            return k
    return 0


class _Shape:
    pass


def _acceptor(vocab=50):
    shape = dict(hidden=8, n_layers=0, n_q_heads=1, n_kv_heads=1, head_dim=8, intermediate=8,
                 vocab=vocab, n_sel=1, target_hidden=8, mask_id=vocab - 1, storage="f32",
                 rope_theta=1e4, rms_eps=1e-6)
    z = np.zeros
    weights = dict(w_fc=z((8, 8), np.float32), g_fc=z(8, np.float32), embed=z((vocab, 8), np.float32),
                   lm_head=z((vocab, 8), np.float32), g_final=z(8, np.float32), layers=[])
    return O.OracleDrafter(shape, weights)


def test_accept_exhaustive_against_brute_force():
    o = _acceptor()
    for gamma in range(1, 9):
        target = rng.integers(0, 50, gamma).astype(np.int32)
        for pattern in itertools.product([0, 1], repeat=gamma - 1):
            drafts = np.array([target[i] if pattern[i] else (target[i] + 1) % 50
                               for i in range(gamma - 1)], dtype=np.int32)
            cache = {"len": 100 + gamma, "committed": 100}
            st, a, nxt = o.accept(cache, drafts, target)
            assert st == 0
            assert a == _brute_accept(drafts, target)
            assert nxt == target[a]
            assert cache["committed"] == 100 + a + 1
            assert cache["len"] == cache["committed"]          # speculative rows rolled back


def test_accept_commit_order_keeps_len():
    o = _acceptor()
    cache = {"len": 40, "committed": 40}
    st, a, nxt = o.accept(cache, np.array([1, 2, 3], np.int32), np.array([1, 2, 9, 4], np.int32))
    assert (st, a, nxt) == (0, 2, 9)
    assert cache == {"len": 40, "committed": 43}


def test_accept_rejects_out_of_range_target():
    o = _acceptor(vocab=10)
    cache = {"len": 5, "committed": 5}
    st, a, nxt = o.accept(cache, np.array([1], np.int32), np.array([1, 10], np.int32))
    assert st == -7 and a == -1 and nxt == -1 and cache == {"len": 5, "committed": 5}


def test_accept_is_lossless_against_greedy_sequence():
    # The committed stream must equal the target's greedy stream whatever the
    # drafts are (drafts here are random corruptions of the true continuation).
    o = _acceptor(vocab=7)
    greedy = rng.integers(0, 7, 400).astype(np.int32)
    pos = 0
    out = []
    cache = {"len": 0, "committed": 0}
    gamma = 6
    while pos + gamma < greedy.size:
        true = greedy[pos + 1: pos + gamma]          # tokens after the anchor
        drafts = np.where(rng.random(gamma - 1) < 0.7, true, (true + 1) % 7).astype(np.int32)
        target = greedy[pos + 1: pos + gamma + 1]    # target's argmax after each block position
        st, a, nxt = o.accept(cache, drafts, target)
        out.extend(list(drafts[:a]) + [nxt])
        pos += a + 1
    assert out == list(greedy[1:pos + 1])
    assert cache["committed"] == pos


def test_loss_weights_geometric_closed_forms():
    for g in (1, 2, 3, 4, 8, 16, 32):
        w = O.loss_weights(g)
        r = math.exp(-1.0 / g)
        assert np.allclose(w[1:] / w[:-1], r, rtol=1e-14)          # constant decay ratio
        assert math.isclose(float(w.sum()), (1 - math.exp(-1.0)) / (1 - r), rel_tol=1e-13)
        assert math.isclose(float(w[-1] * r), math.exp(-1.0), rel_tol=1e-13)   # w_{gamma+1} = 1/e
