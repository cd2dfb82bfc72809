"""Host-side checks of libdflash that need no GPU: the library loads, exports
every symbol the headers declare, validates configurations, and its split-K
work partition covers every k-block exactly once."""
import os
import re

import pytest

from block_diffusion_speculative_03_b200 import build, dflash as D

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return D.lib()


def _declared(header):
    src = open(os.path.join(ROOT, "include", header)).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dflash_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = (_declared("dflash.h") + _declared("dflash_ablation.h") + _declared("dflash_diag.h")
             + _declared("dflash_policy.h"))
    assert len(names) >= 20
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(D.exported_symbols())


def test_arch_and_status_strings(lib):
    assert D.dflash_diag_arch() == "sm_100a"
    for s in range(-8, 1):
        assert D.dflash_status_string(s) not in ("", "unknown status")
    assert D.dflash_status_string(-99) == "unknown status"


def _cfg(**kw):
    c = D.dflash_config(hidden=4096, n_layers=5, n_q_heads=32, n_kv_heads=8, head_dim=128, intermediate=12288,
                        vocab=151936, n_sel=5, target_hidden=4096, mask_id=151935, max_gamma=16, dtype=D.DFLASH_BF16,
                        max_batch=1, max_rows=2048, max_position=4096, rope_theta=1e6, rms_eps=1e-6)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def test_workspace_and_config_validation(lib):
    n = D.dflash_workspace_bytes(_cfg())
    assert 10e6 < n < 1e9
    assert D.dflash_workspace_bytes(_cfg(max_batch=32), check=False) > n
    bad = [dict(hidden=0), dict(mask_id=151936), dict(n_kv_heads=7), dict(dtype=5), dict(n_layers=17),
           dict(max_gamma=0), dict(rope_theta=0.0)]
    for kw in bad:
        assert D.dflash_workspace_bytes(_cfg(**kw), check=False) == -1, kw
    unsup = [dict(head_dim=96), dict(max_gamma=33), dict(hidden=4000), dict(max_gamma=32, n_kv_heads=4),
             dict(dtype=D.DFLASH_F32, max_position=20000)]
    for kw in unsup:
        assert D.dflash_workspace_bytes(_cfg(**kw), check=False) == -2, kw


def test_create_rejects_bad_arguments_without_touching_the_device(lib):
    w = D.dflash_weights()
    # null workspace / null weights / misaligned workspace: rejected before any CUDA call
    assert D.dflash_create(_cfg(), w, None, 1 << 30, check=False) == -1
    assert D.dflash_create(_cfg(), w, 1 << 20, 1 << 30, check=False) == -1
    assert D.dflash_create(_cfg(hidden=0), w, 1 << 20, 1 << 30, check=False) == -1


def _simulate(U, KB, P):
    """Brute force: the k-block ranges of each CTA and the contributors per tile."""
    begins = [p * U // P for p in range(P + 1)]
    contrib = {}
    for p in range(P):
        for u in range(begins[p], begins[p + 1]):
            contrib.setdefault(u // KB, []).append(p)
    return begins, {t: sorted(set(v)) for t, v in contrib.items()}


@pytest.mark.parametrize("U,KB,P", [(3072, 64, 148), (75968, 64, 148), (64, 64, 64), (1001, 7, 33),
                                    (130, 13, 10), (48, 16, 48), (6144, 192, 148), (10240, 320, 148)])
def test_partition_matches_brute_force(lib, U, KB, P):
    begins, contrib = _simulate(U, KB, P)
    for t, ps in contrib.items():
        f, n = D.dflash_diag_partition(U, KB, P, t)
        assert f == ps[0] and n == len(ps) and ps == list(range(f, f + n))
    # every CTA has at most two split segments: its first and its last
    for p in range(P):
        b0, b1 = begins[p], begins[p + 1]
        assert b1 > b0
        tiles = range(b0 // KB, (b1 - 1) // KB + 1)
        split = [t for t in tiles if not (b0 <= t * KB and (t + 1) * KB <= b1)]
        assert len(split) <= 2
        assert all(t in (b0 // KB, (b1 - 1) // KB) for t in split)


def test_partition_rejects_bad_sizes(lib):
    with pytest.raises(D.DflashError):
        D.dflash_diag_partition(12, 3, 13, 0)      # more CTAs than units
    with pytest.raises(D.DflashError):
        D.dflash_diag_partition(10, 3, 2, 0)       # not a whole number of tiles
    with pytest.raises(D.DflashError):
        D.dflash_diag_partition(12, 3, 2, 4)       # tile out of range
