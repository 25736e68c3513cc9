"""Pins of the oracle's FP8 (e4m3) centroid cache (essay "《卡片柜》" ch. 8:
the bucket cache stacks with FP8 quantisation).

* e4m3 rounding: every finite code round-trips; on log-uniform random
  doubles the code is the nearest finite value, ties to the even mantissa,
  brute-forced over the 254 finite codes; saturation at +-448; torch's own
  float8_e4m3fn conversion agrees on fp32 inputs in range (a library
  routine, not this file's arithmetic);
* FP8 centroids: within half an e4m3 ulp of 2^8 times the fp64 normalised
  sum; signs and zeros kept; carried exactly by bf16;
* selection on the FP8 cache equals a brute-force fill whose scores are
  exact rational dot products of the bf16 query latent and the decoded e4m3
  values (fractions), and products of a bf16 and an e4m3 value are exact in
  fp64.
"""
from fractions import Fraction

import numpy as np
import torch

import oracle
import synth

FINITE = [c for c in range(256) if c not in (0x7F, 0xFF)]


def _table():
    return {c: float(oracle.e4m3_to_f64([c])[0]) for c in FINITE}


def test_e4m3_code_values():
    tab = _table()
    assert tab[0x00] == 0.0 and tab[0x38] == 1.0 and tab[0x7E] == 448.0 and tab[0x01] == 2.0 ** -9
    assert tab[0x08] == 2.0 ** -6 and tab[0x07] == 7 * 2.0 ** -9 and tab[0xB8] == -1.0
    vals = sorted(v for c, v in tab.items() if c < 0x80)
    assert len(set(vals)) == 127 and vals[0] == 0.0      # 0 and 126 positive values, all distinct
    assert np.isnan(oracle.e4m3_to_f64([0x7F])[0])


def test_e4m3_round_trip():
    codes = np.array(FINITE, np.uint8)
    back = oracle.e4m3_rne(oracle.e4m3_to_f64(codes))
    assert np.array_equal(back[codes != 0x80], codes[codes != 0x80])
    assert back[list(codes).index(0x80)] == 0x80        # -0 keeps its sign


def test_e4m3_nearest_even_brute_force():
    tab = _table()
    pos = sorted((v, c) for c, v in tab.items() if c < 0x80)
    rng = np.random.default_rng(5)
    xs = np.concatenate([np.exp(rng.uniform(np.log(2.0 ** -12), np.log(2000.0), 3000)),
                         [v for v, _ in pos[1:]],                             # exact values
                         [(a + b) / 2 for (a, _), (b, _) in zip(pos[:-1], pos[1:])]])  # exact ties
    xs = np.concatenate([xs, -xs])
    got = oracle.e4m3_rne(xs)
    for x, c in zip(xs, got):
        a = abs(x)
        if a >= 448.0:
            want = 0x7E
        else:
            best = min(abs(a - v) for v, _ in pos)
            near = [(v, cc) for v, cc in pos if abs(a - v) == best]
            want = near[0][1] if len(near) == 1 else [cc for v, cc in near if cc % 2 == 0][0]
        want |= 0x80 if x < 0 else 0
        assert c == want, (x, c, want)


def test_e4m3_agrees_with_torch_in_range():
    rng = np.random.default_rng(6)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-8, 5.5, 20000))).astype(np.float32)
    x = x[np.abs(x) <= 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_rne(x.astype(np.float64)), ref)


def _cache(T=4096, seed=0):
    inp = synth.layer_inputs("prefill-4k", seed=seed, T=T)
    cfg = oracle.Cfg(k=512, sinks=4, window=256)
    U = oracle.key_latent_pool(inp["K"], inp["Wk"], 4)
    return inp, cfg, oracle.build_cache(U, T, cfg)


def test_fp8_centroids_half_ulp_of_scaled_normalised_sum():
    _, _, c = _cache()
    s = c["sum"]
    nrm = np.sqrt((s * s).sum(axis=-1, keepdims=True))
    z = np.where(nrm > 0, s / np.where(nrm > 0, nrm, 1.0), 0.0) * 256.0
    v = oracle.e4m3_to_f64(oracle.cent_fp8(c)).reshape(s.shape)
    # half an ulp: 2^(e-4) for |z| in [2^(e-1), 2^e) (normals), 2^-10 below 2^-6
    e = np.floor(np.log2(np.maximum(np.abs(z), 2.0 ** -30))) + 1
    half = np.where(np.abs(z) >= 2.0 ** -6, np.ldexp(1.0, (e - 4).astype(int)), 2.0 ** -10)
    assert np.all(np.abs(v - z) <= half)
    assert np.all(np.sign(v) * np.sign(z) >= 0)
    assert np.all(v[nrm[..., 0] == 0] == 0)


def test_fp8_values_carried_exactly_by_bf16():
    codes = np.array(FINITE, np.uint8)
    b = oracle.fp8_as_bf16(codes)
    assert np.array_equal(oracle.bf16_to_f64(b), np.ldexp(oracle.e4m3_to_f64(codes), -8))


def test_bf16_times_e4m3_exact_in_fp64():
    rng = np.random.default_rng(7)
    y = oracle.bf16_to_f64(rng.integers(0, 0x7F7F, 5000).astype(np.uint16))
    v = np.ldexp(oracle.e4m3_to_f64(rng.choice(FINITE, 5000).astype(np.uint8)), -8)
    for a, b in zip(y[:500], v[:500]):
        assert Fraction(a) * Fraction(b) == Fraction(float(a * b))


def test_select_on_fp8_cache_is_the_exact_top_fill():
    inp, cfg, c = _cache()
    c8 = oracle.with_fp8_centroids(c)
    vals = np.ldexp(oracle.e4m3_to_f64(oracle.cent_fp8(c)), -8)[0]   # [NB, dl]
    tpos = np.array([300, 1333, 2900, 4095])
    Q = np.ascontiguousarray(inp["Q"][tpos])
    Y = oracle.query_latent(Q, inp["Wq"], 1, 0)
    idx, _, _ = oracle.select(c8, Y, tpos, cfg, G=4)
    off, mem = c["offsets"][0], c["members"][0]
    for qi, t in enumerate(tpos):
        lim = t - cfg.window
        y = [Fraction(float(v)) for v in oracle.bf16_to_f64(Y[qi, 0])]
        scored = []
        for b in range(c["NB"]):
            if c["minlr"][0, b] > lim:
                continue
            s = sum(yy * Fraction(float(cv)) for yy, cv in zip(y, vals[b]))
            keys = [p for m in mem[off[b]:off[b + 1]] for p in range(4 * m, 4 * m + 4)
                    if cfg.sinks <= p <= lim]
            scored.append((-s, b, keys))
        scored.sort()
        need, taken = cfg.k, {}
        for _, b, keys in scored:
            if need <= 0:
                break
            if keys:
                taken[b] = keys[:need]
                need -= len(taken[b])
        want = [p for b in sorted(taken) for p in taken[b]]
        got = [p for p in idx[qi, 0, cfg.sinks:cfg.sinks + cfg.k] if p >= 0]
        assert got == want, t
