"""Pins for the oracle's selection (flat and tree), index assembly and
attention (essay "《卡片柜》", ch. 3-5; tutorial "隐空间稀疏注意力", section 二).

Independent checks: the all-buckets case reduces to full causal attention
(torch's scaled_dot_product_attention in fp64), with one and with 8 kv-heads
of 4 query heads; single-key lists (a closed form); the flat fill is a top set
under independently computed exact scores; structural invariants of each index
row; rows written out by hand on a hand-built cache (a bucket holding sink
keys, exact score ties); tree with a beam wider than every level equals flat;
beam 1 equals a greedy single-path descent and beams 2 and 3 a plain beam
search, both written here; comparison counts O(T/8) vs O(log T).
"""
import numpy as np
import pytest
import torch

import oracle
import synth


def _inputs(T, hkv=1, hq=4, seed=0, name="prefill-4k"):
    inp = synth.layer_inputs(name, seed=seed, T=T)
    if hkv != inp["K"].shape[1]:
        raise ValueError
    return inp


def _score_exact(y_bits, c_bits):
    """Exact dot products of bf16 vectors via integer-scaled arithmetic
    (python ints), independent of the oracle's fp64 loop."""
    from fractions import Fraction
    def fr(bits):
        u = (int(bits) << 16)
        s = -1 if u >> 31 else 1
        e = (u >> 23) & 0xFF
        m = u & 0x7FFFFF
        if e == 0:
            return s * Fraction(m, 1 << 149)
        return s * Fraction((1 << 23) | m, 1) * Fraction(2) ** (e - 150)
    return float(sum(fr(a) * fr(b) for a, b in zip(y_bits, c_bits)))


def _check_row(row, t, cfg, n_lr_expected=None):
    S, k, W = cfg.sinks, cfg.k, cfg.window
    sinks, lr, win = row[:S], row[S:S + k], row[S + k:]
    assert sinks[:min(S, t + 1)].tolist() == list(range(min(S, t + 1)))
    assert (sinks[min(S, t + 1):] == -1).all()
    w0 = max(S, t - W + 1)
    nw = t - w0 + 1 if t >= S else 0
    assert win[:nw].tolist() == list(range(w0, t + 1))
    assert (win[nw:] == -1).all()
    v = lr[lr >= 0]
    assert (lr[len(v):] == -1).all()
    assert len(set(v.tolist())) == len(v)
    assert ((v >= S) & (v <= t - W)).all()
    if n_lr_expected is not None:
        assert len(v) == n_lr_expected
    return v


def test_all_buckets_selected_equals_full_causal_attention():
    """k >= T: every eligible key is taken, so LSA is exact causal attention."""
    T = 600
    inp = _inputs(T)
    cfg = oracle.Cfg(k=T, sinks=4, window=64)
    r = oracle.layer(inp["Q"], inp["K"], inp["V"], inp["Wk"], inp["Wq"], cfg)
    for t in (0, 2, 3, 4, 67, 68, 69, 599):
        v = _check_row(r["idx"][t, 0], t, cfg, n_lr_expected=max(0, t - 64 - 4 + 1))
        full = set(r["idx"][t, 0][r["idx"][t, 0] >= 0].tolist())
        assert full == set(range(t + 1))
    q = torch.tensor(oracle.bf16_to_f64(inp["Q"])).permute(1, 0, 2)      # [hq, T, d]
    k = torch.tensor(oracle.bf16_to_f64(inp["K"])).permute(1, 0, 2).expand(4, T, 128)
    v = torch.tensor(oracle.bf16_to_f64(inp["V"])).permute(1, 0, 2).expand(4, T, 128)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)
    assert np.allclose(r["O"], ref.permute(1, 0, 2).numpy(), atol=1e-12, rtol=0)


def test_single_key_attention_and_padding():
    inp = _inputs(64)
    idx = np.full((1, 1, 8), -1, np.int32)
    idx[0, 0, 3] = 17
    O = oracle.attention(inp["Q"][:1], inp["K"], inp["V"], idx)
    assert np.array_equal(O[0], np.repeat(oracle.bf16_to_f64(inp["V"][17]), 4, axis=0))
    # permuting a list does not change the result beyond rounding
    idx = np.array([[[5, 9, -1, 30, 2, -1]]], np.int32)
    a = oracle.attention(inp["Q"][:1], inp["K"], inp["V"], idx)
    b = oracle.attention(inp["Q"][:1], inp["K"], inp["V"], idx[:, :, ::-1].copy())
    assert np.allclose(a, b, atol=1e-14)
    empty = oracle.attention(inp["Q"][:1], inp["K"], inp["V"], np.full((1, 1, 4), -1, np.int32))
    assert np.all(empty == 0)


@pytest.fixture(scope="module")
def built():
    T = 4096
    inp = _inputs(T)
    cfg = oracle.Cfg(k=512, sinks=4, window=256)
    U = oracle.key_latent_pool(inp["K"], inp["Wk"], 4)
    cache = oracle.build_cache(U, T, cfg)
    return inp, cfg, cache


def _weights(cache, h, b, t, cfg):
    lo, hi = cache["offsets"][h, b], cache["offsets"][h, b + 1]
    keys = [p for j in cache["members"][h, lo:hi] for p in range(4 * j, 4 * j + 4)]
    return [p for p in keys if cfg.sinks <= p <= t - cfg.window]


@pytest.mark.parametrize("agg", [0, 1])
def test_flat_fill_is_a_top_set_under_exact_scores(built, agg):
    inp, cfg, cache = built
    cfg = oracle.Cfg(k=cfg.k, sinks=cfg.sinks, window=cfg.window, agg=agg)
    tpos = np.array([259, 300, 777, 2048, 4095])
    Q = inp["Q"][tpos]
    Y = oracle.query_latent(Q, inp["Wq"], 1, agg)
    idx, mg, nc = oracle.select(cache, Y, tpos, cfg, G=4)
    for qi, t in enumerate(tpos):
        lr = _check_row(idx[qi, 0], t, cfg)
        elig = [b for b in range(cache["NB"]) if cache["minlr"][0, b] <= t - cfg.window]
        assert nc[qi, 0] == len(elig) * (4 if agg else 1)
        ys = Y[qi] if agg else Y[qi, :1]
        sc = {b: max(_score_exact(y, cache["cent"][0, b]) for y in ys) for b in elig}
        lrset = set(lr.tolist())
        total = sum(len(_weights(cache, 0, b, t, cfg)) for b in elig)
        assert len(lr) == min(cfg.k, total)
        full, part, none = [], [], []
        for b in elig:
            w = _weights(cache, 0, b, t, cfg)
            got = [p for p in w if p in lrset]
            if len(got) == len(w):
                full.append(b)
            elif got:
                part.append(b)
                assert got == w[:len(got)]  # truncation keeps the lowest keys
            else:
                none.append(b)
        assert len(part) <= 1
        taken = full + part
        if none and taken:
            # every taken bucket ranks above every untaken one (score desc, id asc)
            worst_taken = min(taken, key=lambda b: (sc[b], -b))
            best_none = max(none, key=lambda b: (sc[b], -b))
            assert (sc[worst_taken], -worst_taken) > (sc[best_none], -best_none)
        if part:
            assert all((sc[b], -b) > (sc[part[0]], -part[0]) for b in full)
        # every key of the row belongs to an eligible bucket and lies in R_t
        assert all(cache["bucket_of_unit"][0, p // 4] in sc for p in lr)


def test_native_with_one_head_equals_mean(built):
    inp, cfg, cache = built
    tpos = np.array([400, 1500, 4000])
    Q = inp["Q"][tpos][:, :1].copy()  # a single query head per group
    Ym = oracle.query_latent(Q, inp["Wq"], 1, 0)
    Yn = oracle.query_latent(Q, inp["Wq"], 1, 1)
    assert np.array_equal(Ym, Yn)
    a = oracle.select(cache, Ym, tpos, oracle.Cfg(k=512, sinks=4, window=256, agg=0), G=1)
    b = oracle.select(cache, Yn, tpos, oracle.Cfg(k=512, sinks=4, window=256, agg=1), G=1)
    assert np.array_equal(a[0], b[0])


def test_flat_comparisons_grow_like_T_over_8(built):
    inp, cfg, cache = built
    tpos = np.array([1279, 2303, 4095])
    Y = oracle.query_latent(inp["Q"][tpos], inp["Wq"], 1, 0)
    _, _, nc = oracle.select(cache, Y, tpos, cfg, G=4)
    # eligible buckets ~ (t - W) / 8
    for t, n in zip(tpos, nc[:, 0]):
        assert abs(n - (t - cfg.window) / 8) <= 64


def test_tree_wide_beam_equals_flat(built):
    inp, cfg, cache = built
    tpos = np.array([300, 1000, 2500, 4095])
    Y = oracle.query_latent(inp["Q"][tpos], inp["Wq"], 1, 0)
    flat = oracle.select(cache, Y, tpos, cfg, G=4)[0]
    wide = oracle.Cfg(k=512, sinks=4, window=256, beam=1024, mode=1)
    tree = oracle.select(cache, Y, tpos, wide, G=4)[0]
    assert np.array_equal(flat, tree)


def _greedy_path(tree, cache, y, t, cfg, lstar):
    """Beam-1 descent written as a plain greedy walk: from the root, step to
    the higher-scoring eligible child until level L*; return its leaves."""
    ln, lo = tree["level_n"], tree["level_off"]
    lvl, node = len(ln) - 1, 0
    if tree["minlr"][0, lo[lvl]] > t - cfg.window:
        return []
    while lvl > lstar:
        best = None
        for ch in (2 * node, 2 * node + 1):
            if ch >= ln[lvl - 1]:
                continue
            g = lo[lvl - 1] + ch
            if tree["minlr"][0, g] > t - cfg.window:
                continue
            s = _score_exact(y, tree["cent"][0, g])
            if best is None or s > best[0]:
                best = (s, ch)
        if best is None:
            return []
        node, lvl = best[1], lvl - 1
    return list(range(node << lstar, min((node + 1) << lstar, cache["NB"])))


def test_tree_beam1_is_greedy_descent(built):
    inp, cfg, cache = built
    tr = oracle.build_tree(cache)
    c1 = oracle.Cfg(k=64, sinks=4, window=256, beam=1, mode=1)  # L* = 3
    tpos = np.array([600, 1900, 3333, 4095])
    Y = oracle.query_latent(inp["Q"][tpos], inp["Wq"], 1, 0)
    idx, _, nc = oracle.select(cache, Y, tpos, c1, tree=tr, G=4)
    for qi, t in enumerate(tpos):
        leaves = _greedy_path(tr, cache, Y[qi, 0], t, c1, 3)
        lr = _check_row(idx[qi, 0], t, c1)
        allowed = set(p for b in leaves for p in _weights(cache, 0, b, t, c1))
        assert set(lr.tolist()) <= allowed
        assert len(lr) == min(c1.k, len(allowed))


def _beam_leaves(tree, cache, y, t, cfg, beam, lstar):
    """Beam descent written as a plain search: from the root to level L*,
    score the eligible children of the kept nodes exactly and keep the best
    `beam` (score desc, node index asc); return the buckets below them."""
    ln, lo = tree["level_n"], tree["level_off"]
    top = len(ln) - 1
    if tree["minlr"][0, lo[top]] > t - cfg.window:
        return []
    kept = [0]
    for lvl in range(top, lstar, -1):
        cands = []
        for node in kept:
            for ch in (2 * node, 2 * node + 1):
                if ch < ln[lvl - 1] and tree["minlr"][0, lo[lvl - 1] + ch] <= t - cfg.window:
                    cands.append((-_score_exact(y, tree["cent"][0, lo[lvl - 1] + ch]), ch))
        kept = [ch for _, ch in sorted(cands)[:beam]]
    return sorted(b for n in kept for b in range(n << lstar, min((n + 1) << lstar, cache["NB"])))


@pytest.mark.parametrize("beam", [2, 3])
def test_tree_beam_b_is_a_plain_beam_search(built, beam):
    inp, cfg, cache = built
    tr = oracle.build_tree(cache)
    k = 16 * beam * 2                    # L* = 2: beam * 8 * 2^2 = k
    cb = oracle.Cfg(k=k, sinks=4, window=256, beam=beam, mode=1)
    tpos = np.array([700, 1500, 2600, 3333, 4095])
    Y = oracle.query_latent(inp["Q"][tpos], inp["Wq"], 1, 0)
    idx, _, _ = oracle.select(cache, Y, tpos, cb, tree=tr, G=4)
    for qi, t in enumerate(tpos):
        leaves = _beam_leaves(tr, cache, Y[qi, 0], t, cb, beam, 2)
        assert len(leaves) == 4 * beam
        lr = _check_row(idx[qi, 0], t, cb)
        allowed = set(p for b in leaves for p in _weights(cache, 0, b, t, cb))
        assert set(lr.tolist()) <= allowed
        assert len(lr) == min(cb.k, len(allowed))


def test_tree_structure_and_log_comparisons(built):
    inp, cfg, cache = built
    tr = oracle.build_tree(cache)
    ln = tr["level_n"]
    assert ln[0] == cache["NB"] and ln[-1] == 1
    assert all(ln[i + 1] == (ln[i] + 1) // 2 for i in range(len(ln) - 1))
    # node sums are the sums of their leaves; minlr is the min over leaves
    for lvl in range(len(ln)):
        for i in range(ln[lvl]):
            b0, b1 = i << lvl, min((i + 1) << lvl, cache["NB"])
            node = tr["level_off"][lvl] + i
            assert np.allclose(tr["sum"][0, node], cache["sum"][0, b0:b1].sum(axis=0), atol=1e-12)
            assert tr["minlr"][0, node] == cache["minlr"][0, b0:b1].min()
    c2 = oracle.Cfg(k=512, sinks=4, window=256, beam=2, mode=1)  # L* = 5
    tpos = np.array([4095])
    Y = oracle.query_latent(inp["Q"][tpos], inp["Wq"], 1, 0)
    _, _, nc = oracle.select(cache, Y, tpos, c2, tree=tr, G=4)
    H = len(ln) - 1  # 9 levels above the leaves for 512 buckets
    assert nc[0, 0] <= 2 * 2 * (H - 5) + 2 * 2 ** 5


@pytest.fixture(scope="module")
def gqa_inputs():
    """160 tokens of the 8 kv-head / 32 query-head layer."""
    return _inputs(160, hkv=8, hq=32, name="prefill-128k")


def test_full_causal_attention_with_gqa_groups(gqa_inputs):
    """k >= T with 8 kv-heads of 4 query heads each: query head h attends
    with kv-head h // 4 (the GQA grouping), checked against SDPA in fp64."""
    T = 160
    inp = gqa_inputs
    cfg = oracle.Cfg(k=T, sinks=4, window=16)
    r = oracle.layer(inp["Q"], inp["K"], inp["V"], inp["Wk"], inp["Wq"], cfg)
    q = torch.tensor(oracle.bf16_to_f64(inp["Q"])).permute(1, 0, 2)      # [32, T, d]
    k = torch.tensor(oracle.bf16_to_f64(inp["K"])).permute(1, 0, 2).repeat_interleave(4, dim=0)
    v = torch.tensor(oracle.bf16_to_f64(inp["V"])).permute(1, 0, 2).repeat_interleave(4, dim=0)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)
    assert np.allclose(r["O"], ref.permute(1, 0, 2).numpy(), atol=1e-12, rtol=0)


def test_each_query_head_reads_its_groups_list(gqa_inputs):
    """One distinct key per kv-head list: a softmax over one key is 1, so
    query head h returns the V row of its group's key, V[key(h // 4), h // 4]."""
    inp = gqa_inputs
    idx = np.full((1, 8, 5), -1, np.int32)
    keys = [3 * g + 1 for g in range(8)]
    for g in range(8):
        idx[0, g, 2] = keys[g]
    O = oracle.attention(inp["Q"][:1], inp["K"], inp["V"], idx)
    Vf = oracle.bf16_to_f64(inp["V"])
    for h in range(32):
        assert np.array_equal(O[0, h], Vf[keys[h // 4], h // 4]), h


def _hand_cache(groups, T, S, vecs, dl=64, pool=4):
    """A one-head bucket cache made from explicit member lists; the bucket
    metadata follows its definition (unit j holds keys pool*j .. pool*j+3),
    and both the sum and the centroid of bucket b are the bf16-exact vector
    vecs[b] (the flat fill reads only the centroid; the tree reads sums)."""
    NU = (T + pool - 1) // pool
    NB = len(groups)
    members, offsets, cnt, mlr, mxp = [], [0], [], [], []
    bou = np.full((1, NU), -1, np.int32)
    for b, g in enumerate(groups):
        g = sorted(g)
        members += g
        offsets.append(len(members))
        keys = [p for j in g for p in range(pool * j, min(pool * j + pool, T))]
        lr = [p for p in keys if p >= S]
        cnt.append(len(lr))
        mlr.append(min(lr) if lr else oracle.IMAX)
        mxp.append(max(keys) if keys else -1)
        bou[0, g] = b
    assert sorted(members) == list(range(NU))
    V = np.zeros((1, NB, dl))
    V[0, :, :len(vecs[0])] = np.asarray(vecs, np.float64)
    cent = synth.f32_to_bf16_bits(V.astype(np.float32))
    assert np.array_equal(oracle.bf16_to_f64(cent), V)
    i32 = lambda a: np.asarray(a, np.int32)[None, :]
    return dict(T=T, H=1, NU=NU, NB=NB, nblk=1, bucket_of_unit=bou,
                members=i32(members), offsets=i32(offsets), cnt_lr=i32(cnt),
                minlr=i32(mlr), maxpos=i32(mxp), sum=V, cent=cent,
                ward_margin=np.zeros((1, 1)))


def _e0(dl=64):
    y = np.zeros((1, 1, dl), np.float32)
    y[0, 0, 0] = 1.0
    return synth.f32_to_bf16_bits(y)


def test_flat_fill_on_a_hand_built_cache():
    """Rows written out by hand from the definition of the flat fill.

    Bucket 0 holds the sink keys 0-3, keys 20-23 and keys 56-59, so at t = 40
    (R_t = [4, 32]) only its 4 keys 20-23 count. Buckets 1 and 2 score
    exactly the same; the lower bucket id wins the tie."""
    groups = [[0, 5, 14], [1, 2], [3, 4], [6, 7, 8, 9, 10, 11, 12, 13, 15]]
    c = _hand_cache(groups, 64, 4, [[1.0], [0.5], [0.5], [0.25]])
    y = _e0()
    cfg = oracle.Cfg(k=8, sinks=4, window=8)
    idx, _, _ = oracle.select(c, y, np.array([40]), cfg, G=1)
    assert idx[0, 0].tolist() == [0, 1, 2, 3,
                                  20, 21, 22, 23, 4, 5, 6, 7,
                                  33, 34, 35, 36, 37, 38, 39, 40]
    cfg = oracle.Cfg(k=24, sinks=4, window=8)
    rows = {}
    for t in (63, 5, 2):
        idx, _, _ = oracle.select(c, y, np.array([t]), cfg, G=1)
        rows[t] = idx[0, 0].tolist()
    # t = 63: R_t = [4, 55]; bucket 0 gives 20-23, bucket 1 (tie won) 4-11,
    # bucket 2 12-19, bucket 3 the lowest 4 of its keys in R_t
    assert rows[63] == [0, 1, 2, 3,
                        20, 21, 22, 23, *range(4, 12), *range(12, 20), 24, 25, 26, 27,
                        *range(56, 64)]
    # t = 5: no long-range key yet; window 4-5.  t = 2: sinks 0-2 only.
    assert rows[5] == [0, 1, 2, 3] + [-1] * 24 + [4, 5] + [-1] * 6
    assert rows[2] == [0, 1, 2, -1] + [-1] * 24 + [-1] * 8


def test_ties_take_the_lower_id_in_flat_and_tree():
    """Buckets 0 and 3 have one centroid, buckets 1 and 2 another, so both
    level-1 tree nodes have the same centroid: the beam of 1 keeps node 0 and
    the flat fill breaks both ties by the lower bucket id."""
    groups = [[0, 1], [2, 3], [4, 5], [6, 7]]
    c = _hand_cache(groups, 32, 4, [[2.0, 1.0], [1.0, 2.0], [1.0, 2.0], [2.0, 1.0]])
    # the flat fill reads centroids: make them the normalised sums, in bf16
    s = c["sum"][0]
    c["cent"] = oracle.bf16_rne(s / np.linalg.norm(s, axis=1, keepdims=True)).reshape(1, 4, 64)
    y = _e0()
    tr = oracle.build_tree(c)
    lo = tr["level_off"]
    assert np.array_equal(tr["cent"][0, lo[1]], tr["cent"][0, lo[1] + 1])
    t = np.array([31])                                  # R_t = [4, 27]
    flat = oracle.select(c, y, t, oracle.Cfg(k=16, sinks=4, window=4), G=1)[0][0, 0]
    # b0 and b3 tie first (b0 4-7, b3 24-27), then b1 beats b2 for the last 8
    assert flat.tolist() == [0, 1, 2, 3, *range(4, 16), 24, 25, 26, 27, 28, 29, 30, 31]
    cfg = oracle.Cfg(k=16, sinks=4, window=4, beam=1, mode=1)   # L* = 1
    tree = oracle.select(c, y, t, cfg, tree=tr, G=1)[0][0, 0]
    # node 0 (buckets 0, 1) wins the tie at level 1; both buckets fit
    assert tree.tolist() == [0, 1, 2, 3, *range(4, 16), -1, -1, -1, -1, 28, 29, 30, 31]
