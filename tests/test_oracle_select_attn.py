"""Pins for the oracle's selection (flat and tree), index assembly and
attention (essay "《卡片柜》", ch. 3-5; tutorial "隐空间稀疏注意力", section 二).

Independent checks: the all-buckets case reduces to full causal attention
(torch's scaled_dot_product_attention in fp64); the flat fill is a top set
under independently computed exact scores; structural invariants of each index
row; tree with a beam wider than every level equals flat; beam 1 equals a
greedy single-path descent written here; comparison counts O(T/8) vs O(log T).
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
