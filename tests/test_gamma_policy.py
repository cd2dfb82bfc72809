"""The block-size (gamma) policy of include/dflash_policy.h, on the host: its
acceptance estimate against a brute-force maximum of the censored geometric
likelihood, its expected tokens against enumeration of the truncated geometric
law, its choice against a brute-force argmax, forgetting, argument checks,
convergence on the workloads' acceptance plans, and a chain of oracle cycles
whose block size changes from cycle to cycle."""
import math

import numpy as np
import pytest

from block_diffusion_speculative_03_b200 import build, dflash as D
from block_diffusion_speculative_03_b200 import inputs as I
from tests.helpers import gamma_schedule, oracle_drafter, synth_target, to_np


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    D.lib()


def _policy(cands=(4, 8, 16), decay=1.0, cf=1.0, ct=0.0, pa=1e-12, pr=1e-12):
    return D.dflash_gamma_policy_init(list(cands), decay, cf, ct, pa, pr)


def test_alpha_maximises_the_censored_geometric_likelihood():
    rng = np.random.default_rng(7)
    for _ in range(5):
        p = _policy()
        cycles = []
        for _ in range(int(rng.integers(3, 12))):
            g = int(rng.choice([4, 8, 16]))
            a = rng.integers(0, g, size=int(rng.integers(1, 4)))
            D.dflash_gamma_policy_observe(p, a.tolist(), g)
            cycles.append((g, a))
        # log L(alpha) = sum_i a_i log alpha + [a_i < g - 1] log(1 - alpha), on a fine grid
        grid = np.linspace(1e-6, 1 - 1e-6, 200001)
        ll = np.zeros_like(grid)
        for g, a in cycles:
            for ai in a:
                ll += ai * np.log(grid) + (np.log1p(-grid) if ai < g - 1 else 0.0)
        best = grid[int(np.argmax(ll))]
        assert abs(D.dflash_gamma_policy_alpha(p) - best) < 2e-5


def _tau_by_enumeration(alpha, gamma):
    # a = k with probability alpha^k (1 - alpha) for k < gamma - 1, and alpha^(gamma-1) at k = gamma - 1
    probs = [alpha ** k * (1 - alpha) for k in range(gamma - 1)] + [alpha ** (gamma - 1)]
    assert abs(sum(probs) - 1.0) < 1e-12
    return sum((k + 1) * pk for k, pk in enumerate(probs))


@pytest.mark.parametrize("alpha", [0.0, 0.25, 0.5, 0.84448, 0.87358, 0.99, 1.0])
def test_expected_tokens_is_the_mean_committed_per_cycle(alpha):
    for g in range(1, 33):
        tau = D.dflash_gamma_policy_expected_tokens(alpha, g)
        assert tau == pytest.approx(_tau_by_enumeration(alpha, g), rel=1e-12, abs=1e-12)
        if alpha < 1.0:
            assert tau == pytest.approx((1 - alpha ** g) / (1 - alpha), rel=1e-12)
        else:
            assert tau == g


def test_expected_tokens_at_the_workload_acceptance_law():
    # the synthetic plans use q = 0.87358 so that the mean acceptance length at gamma 16
    # is 6.0 tokens (so 7.0 committed with the target's own token), and q = 0.84448 for a
    # mean of 5 at gamma 16
    assert D.dflash_gamma_policy_expected_tokens(0.87358, 16) - 1 == pytest.approx(6.0, abs=2e-3)
    assert D.dflash_gamma_policy_expected_tokens(0.84448, 16) - 1 == pytest.approx(5.0, abs=2e-3)


def test_choose_is_the_argmax_of_tokens_per_cost():
    rng = np.random.default_rng(11)
    for _ in range(300):
        cands = sorted(set(int(v) for v in rng.integers(1, 33, size=int(rng.integers(1, 9)))))
        cf, ct = float(rng.uniform(0, 2)), float(rng.uniform(0, 0.3))
        if cf + ct * cands[0] <= 0:
            cf = 1.0
        pa, pr = float(rng.uniform(0.01, 50)), float(rng.uniform(0.01, 50))
        p = D.dflash_gamma_policy_init(cands, 1.0, cf, ct, pa, pr)
        alpha = pa / (pa + pr)
        assert D.dflash_gamma_policy_alpha(p) == pytest.approx(alpha, rel=1e-12)
        rates = [sum(alpha ** k for k in range(g)) / (cf + ct * g) for g in cands]
        best = max(rates)
        near = [g for g, r in zip(cands, rates) if r >= best * (1 - 1e-12)]
        got = D.dflash_gamma_policy_choose(p)
        assert got in near, (cands, rates, got)
        if len(near) == 1:
            assert got == near[0]


def test_ties_go_to_the_smaller_block():
    # alpha -> 0: every block commits one token; with a flat cost all rates tie
    p = _policy(cands=(2, 4, 8), cf=1.0, ct=0.0, pa=1e-300, pr=1.0)
    assert D.dflash_gamma_policy_choose(p) == 2


def test_limits_of_the_acceptance():
    hi = _policy(cf=1.0, ct=0.01)
    D.dflash_gamma_policy_observe(hi, [15] * 64, 16)    # every block fully accepted
    assert D.dflash_gamma_policy_alpha(hi) > 0.999999
    assert D.dflash_gamma_policy_choose(hi) == 16
    lo = _policy(cf=1.0, ct=0.01)
    D.dflash_gamma_policy_observe(lo, [0] * 64, 16)     # nothing accepted
    assert D.dflash_gamma_policy_alpha(lo) < 1e-6
    assert D.dflash_gamma_policy_choose(lo) == 4


def test_decay_forgets_old_cycles():
    p = _policy(decay=0.0)
    D.dflash_gamma_policy_observe(p, [15, 15], 16)
    D.dflash_gamma_policy_observe(p, [0, 3], 8)
    assert (p.accepts, p.rejects) == (3.0, 2.0)
    q = _policy(decay=0.5)
    D.dflash_gamma_policy_observe(q, [7], 8)             # 7 accepts, censored
    D.dflash_gamma_policy_observe(q, [2], 8)             # 2 accepts, 1 reject
    assert (q.accepts, q.rejects) == (0.5 * 7 + 2, 1.0)


def test_invalid_arguments_change_nothing():
    bad_init = [dict(cands=()), dict(cands=tuple(range(1, 10))), dict(cands=(8, 4)), dict(cands=(4, 4)),
                dict(cands=(0, 4)), dict(decay=-0.1), dict(decay=1.5), dict(decay=math.nan),
                dict(cf=0.0, ct=0.0), dict(cf=-1.0), dict(pa=0.0), dict(pr=-1.0), dict(ct=math.inf)]
    for kw in bad_init:
        args = dict(cands=(4, 8, 16), decay=1.0, cf=1.0, ct=0.0, pa=1.0, pr=1.0)
        args.update(kw)
        st = D.dflash_gamma_policy_init(list(args["cands"]), args["decay"], args["cf"], args["ct"], args["pa"],
                                        args["pr"], check=False)
        assert st == -1, kw
    p = _policy()
    before = (p.accepts, p.rejects)
    for acc, g in [([4], 4), ([-1], 8), ([0, 16], 16), ([0], 0)]:
        assert D.dflash_gamma_policy_observe(p, acc, g, check=False) == -1, (acc, g)
    assert (p.accepts, p.rejects) == before
    assert D.dflash_gamma_policy_expected_tokens(1.5, 4, check=False) == -1
    assert D.dflash_gamma_policy_expected_tokens(0.5, 0, check=False) == -1


@pytest.mark.parametrize("name", ["qwen3_8b", "long_ctx"])
def test_estimate_converges_on_the_workload_plan(name):
    w = I.preset(name)
    plan = I.plan_accept(w, 4000, gamma=16).numpy()
    p = _policy()
    for row in plan:
        D.dflash_gamma_policy_observe(p, row.tolist(), 16)
    assert D.dflash_gamma_policy_alpha(p) == pytest.approx(w.accept_q, abs=0.01)


def test_schedule_moves_between_block_sizes():
    w = I.preset("small_bf16")
    sched = gamma_schedule(w, 6, (4, 8, 16), decay=0.5, cost_per_token=0.02)
    used = [g for g, _ in sched]
    assert set(used) == {4, 8, 16}
    assert any(b < a for a, b in zip(used, used[1:]))     # it also moves down
    for g, a in sched:
        assert a.min() >= 0 and a.max() <= g - 1


def test_oracle_chain_with_a_changing_block_size():
    # tiny fp32 drafter, speculative order: inject the gamma verified rows, then accept
    # (roll back to a + 1); the block size follows the policy every cycle
    w = I.preset("tiny")
    sched = gamma_schedule(w, 8, (2, 4))
    assert len({g for g, _ in sched}) == 2
    W = I.make_weights(w)
    ora = oracle_drafter(w, W)
    cap = w.context[0] + 8 * 4 + 4
    oc = ora.new_cache(cap)
    hid = I.make_hiddens(w, w.context[0])
    ora.inject_kv(oc, ora.fuse_context([to_np(h) for h in hid]))
    oc["committed"] = oc["len"]
    anchor = int(I.make_anchors(w).numpy()[0])
    length = w.context[0]
    for cyc, (g, a_star) in enumerate(sched):
        drafts, margin, _ = ora.draft_block(oc, anchor, g, want_logits=True)
        assert drafts.shape == (g - 1,) and margin.shape == (g - 1,)
        rnd = I.random_tokens(w, (1, g), stream=100 + cyc).numpy()[0]
        target = synth_target(drafts, int(a_star[0]), rnd, w.vocab)
        hv = I.make_hiddens(w, g, stream=200 + cyc)
        ora.inject_kv(oc, ora.fuse_context([to_np(h) for h in hv]))
        assert oc["len"] == length + g
        st, a, nxt = ora.accept(oc, drafts, target)
        assert st == 0 and a == int(a_star[0]) and nxt == int(target[a])
        length += a + 1
        assert oc["len"] == length and oc["committed"] == length
        anchor = nxt


def test_convenience_class_matches_the_c_calls():
    import torch
    from block_diffusion_speculative_03_b200.drafter import GammaPolicy
    gp = GammaPolicy(candidates=(4, 8, 16), decay=0.5, cost_fixed=1.0, cost_per_token=0.02)
    p = D.dflash_gamma_policy_init([4, 8, 16], 0.5, 1.0, 0.02, 1.0, 1.0)
    w = I.preset("small_bf16")
    plan = I.plan_accept(w, 10, gamma=16).numpy()
    for row in plan:
        g = gp.choose()
        assert g == D.dflash_gamma_policy_choose(p)
        a = np.minimum(row, g - 1)
        gp.observe(torch.tensor(a, dtype=torch.int32), g)
        D.dflash_gamma_policy_observe(p, a.tolist(), g)
        assert gp.alpha == D.dflash_gamma_policy_alpha(p)
