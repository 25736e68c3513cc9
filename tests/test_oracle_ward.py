"""Pins for the oracle's capped Ward clustering and bucket cache (essay
"《卡片柜》", ch. 2; Ward 1963): hand-derived merges, naive O(n^3) recompute vs
the nearest-neighbour variant, scipy's Ward linkage for the uncapped case, and
structural invariants of the bucket cache."""
import json
import os

import numpy as np
import pytest

import oracle
import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden", "ward_hand_example.json")


def _embed(x, dl=64):
    U = np.zeros((len(x), dl))
    U[:, 0] = x
    return U


def test_ward_hand_example():
    g = json.load(open(GOLD))
    U = _embed(g["x"])
    for case in g["cases"]:
        for naive in (False, True):
            if case["bucket_of"] is None:
                with pytest.raises(ValueError):
                    oracle.ward_block(U, case["m"], case["cap"], naive=naive)
            else:
                got, _ = oracle.ward_block(U, case["m"], case["cap"], naive=naive)
                assert got.tolist() == case["bucket_of"], (case, naive)
    for dd in g["deltas"]:
        sA = U[dd["A"]].sum(axis=0)
        sB = U[dd["B"]].sum(axis=0)
        assert oracle.ward_delta(sA, len(dd["A"]), sB, len(dd["B"])) == pytest.approx(dd["delta"], rel=1e-15)


def _partition(labels):
    groups = {}
    for i, l in enumerate(labels):
        groups.setdefault(int(l), []).append(i)
    return sorted(tuple(v) for v in groups.values())


@pytest.mark.parametrize("seed", range(6))
def test_ward_naive_equals_nearest_neighbour(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(5, 48))
    U = rng.standard_normal((n, 64)) * 0.2
    for cap in (2, 3, 4):
        m = (n + 1) // 2 if cap >= 2 else n
        a, _ = oracle.ward_block(U, m, cap, naive=False)
        b, mg = oracle.ward_block(U, m, cap, naive=True)
        assert np.array_equal(a, b)
        assert mg > 0


def test_ward_ties_lower_index_wins():
    """Duplicated and lattice points make exact Delta ties; both variants must
    break them the same way (lowest pair), and the result must be a valid
    capped partition."""
    base = np.array([0.0, 0.0, 1.0, 1.0, 2.0, 2.0, 0.0, 1.0, 3.0, 3.0])
    U = _embed(base)
    # zero-Delta pairs, lowest first: (0,1), (0,6), (2,3), (2,7), (4,5), (8,9)
    for naive in (False, True):
        lab, _ = oracle.ward_block(U, 4, 4, naive=naive)
        assert lab.tolist() == [0, 0, 1, 1, 2, 2, 0, 1, 3, 3]
        lab, _ = oracle.ward_block(U, 5, 4, naive=naive)
        assert lab.tolist() == [0, 0, 1, 1, 2, 2, 0, 1, 3, 4]
    # all-identical points: merges go (0,1), (0,2)... until the cap, lowest first
    U = _embed(np.zeros(8))
    lab, _ = oracle.ward_block(U, 2, 4, naive=False)
    assert lab.tolist() == [0, 0, 0, 0, 1, 1, 1, 1]


@pytest.mark.parametrize("seed", range(4))
def test_ward_uncapped_matches_scipy_linkage(seed):
    """With the cap lifted the rule is textbook Ward agglomeration; scipy's
    Ward linkage cut at m clusters must give the same partition."""
    from scipy.cluster.hierarchy import fcluster, linkage
    rng = np.random.default_rng(100 + seed)
    n = 40
    U = rng.standard_normal((n, 64))
    for m in (30, 20, 10, 4, 2):
        lab, _ = oracle.ward_block(U, m, 64, naive=False)
        Z = linkage(U, method="ward")
        ref = fcluster(Z, t=m, criterion="maxclust")
        assert _partition(lab) == _partition(ref), m


def test_ward_block_invariants_on_full_block():
    rng = np.random.default_rng(9)
    U = rng.standard_normal((128, 64))
    U /= np.linalg.norm(U, axis=1, keepdims=True)
    lab, _ = oracle.ward_block(U, 64, 4)
    assert sorted(set(lab.tolist())) == list(range(64))
    sizes = np.bincount(lab, minlength=64)
    assert sizes.min() >= 1 and sizes.max() <= 4 and sizes.sum() == 128
    # local bucket order = ascending lowest member
    first = [np.where(lab == b)[0][0] for b in range(64)]
    assert first == sorted(first)


def _brute_bucket_meta(c, h, b, pool, T, S):
    mem = c["members"][h, c["offsets"][h, b]:c["offsets"][h, b + 1]]
    keys = [p for j in mem for p in range(pool * j, min(pool * j + pool, T))]
    lr = [p for p in keys if p >= S]
    return mem, keys, lr


@pytest.mark.parametrize("T", [4096, 1000, 777, 524, 513, 4])
def test_bucket_cache_invariants(T):
    inp = synth.layer_inputs("prefill-4k", seed=3, T=T, parts=("K",))
    cfg = oracle.Cfg(k=512, sinks=4, window=256)
    U = oracle.key_latent_pool(inp["K"], inp["Wk"], 4)
    c = oracle.build_cache(U, T, cfg)
    NU = (T + 3) // 4
    nblk = (NU + 127) // 128
    assert c["NB"] == 64 * nblk
    h = 0
    # members are a permutation of the units, consistent with bucket_of_unit
    assert sorted(c["members"][h].tolist()) == list(range(NU))
    for blk in range(nblk):
        n = min(128, NU - 128 * blk)
        # a block's bucket count is the least that keeps its mean bucket at
        # most 8 keys (2 pooled units): 64 for a full block, and for a ragged
        # last block of n units the least m with n <= 2 m
        want_m = min(m for m in range(1, 65) if n <= 2 * m)
        sizes = np.diff(c["offsets"][h, 64 * blk:64 * blk + 65])
        assert (sizes[:want_m] >= 1).all() and (sizes[:want_m] <= 4).all()
        assert (sizes[want_m:] == 0).all()
        assert sizes.sum() == n
    for b in range(c["NB"]):
        mem, keys, lr = _brute_bucket_meta(c, h, b, 4, T, 4)
        assert list(mem) == sorted(mem)
        assert all(c["bucket_of_unit"][h, j] == b for j in mem)
        assert c["cnt_lr"][h, b] == len(lr)
        assert c["minlr"][h, b] == (min(lr) if lr else oracle.IMAX)
        assert c["maxpos"][h, b] == (max(keys) if keys else -1)
        s = U[h, mem].sum(axis=0) if len(mem) else np.zeros(64)
        assert np.allclose(c["sum"][h, b], s, atol=1e-13, rtol=0)
        cent = oracle.bf16_to_f64(c["cent"][h, b])
        if len(mem):
            # centroid = normalised mean, rounded to bf16 (relative error <= 2^-9)
            want = s / np.linalg.norm(s)
            assert np.all(np.abs(cent - want) <= np.abs(want) * 2.0 ** -8 + 1e-30)
        else:
            assert np.all(cent == 0)


def test_naive_and_fast_build_identical():
    inp = synth.layer_inputs("prefill-4k", seed=1, T=2048, parts=("K",))
    cfg = oracle.Cfg(k=512, sinks=4, window=256)
    U = oracle.key_latent_pool(inp["K"], inp["Wk"], 4)
    a = oracle.build_cache(U, 2048, cfg, naive=False)
    b = oracle.build_cache(U, 2048, cfg, naive=True)
    for key in ("bucket_of_unit", "members", "offsets", "cnt_lr", "minlr", "maxpos", "sum", "cent"):
        assert np.array_equal(a[key], b[key]), key
    assert np.all(b["ward_margin"] > 0)
