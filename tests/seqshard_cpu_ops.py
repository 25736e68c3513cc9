"""A CPU restatement of the sequence-sharded calls, for the multi-rank
tests of the driver (clustered_key_indexing_b200.seqshard) on gloo ranks.
Each call redoes its step with the oracle's fp64 arithmetic:

* build       the oracle's cache of the rank's keys (sinks in the first
              shard only), positions local to the shard;
* candidates  the oracle's flat fill of k keys over that cache (essay
              "《卡片柜》" ch. 3); its long-range keys grouped by bucket give
              the records, each with its exact score (the oracle's sequence
              of fp64 adds over exact products);
* merge       the global fill over every rank's records (score desc, id
              asc, exactly k keys) and this rank's keys, window part, sinks;
* partial     exact softmax attention over the rank's entries in fp64, with
              the base-2 log-sum-exp of the scaled scores;
* combine     sum_r 2^(L_r - M) O_r / sum_r 2^(L_r - M).
Tensors are CPU torch tensors in the library's layouts (records as int32
[nq, hkv, cap, 4]: id, taken, fp64 score)."""
import math

import numpy as np
import torch

import oracle

LOG2E = 1.0 / math.log(2.0)


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _bf(b):
    return oracle.bf16_to_f64(np.asarray(b, np.uint16))


class OracleOps:
    def __init__(self, Wk_np, Wq_np, G):
        self.Wk, self.Wq, self.G = Wk_np, Wq_np, G

    @staticmethod
    def _ocfg(cfg, sinks):
        return oracle.Cfg(k=cfg.k, sinks=sinks, window=cfg.window, beam=cfg.beam, mode=0, agg=cfg.agg)

    def build(self, K_local, W_k, cfg, p0):
        n = K_local.shape[0]
        S_loc = cfg.sinks if p0 == 0 else 0
        oc = oracle.build_cache(oracle.key_latent_pool(_bits(K_local), self.Wk, 4), n, self._ocfg(cfg, S_loc))
        return dict(oc=oc, n=n, S_loc=S_loc)

    def cand_cap(self, cfg):
        return cfg.k // 4 + 4

    def candidates(self, Q, t0, W_q, cache, p0, cfg):
        oc, S_loc = cache["oc"], cache["S_loc"]
        H = oc["H"]
        nq = Q.shape[0]
        cap = self.cand_cap(cfg)
        rec = np.zeros((nq, H, cap, 4), np.int32)
        rec_n = np.zeros((nq, H), np.int32)
        Y = oracle.query_latent(_bits(Q), self.Wq, H, cfg.agg)
        ng = self.G if cfg.agg else 1
        base = p0 // 512 * 64
        for q in range(nq):
            t = t0 + q - p0
            if t - cfg.window < S_loc:
                continue
            idx, _, _ = oracle.select(oc, Y[q:q + 1], np.array([t]), self._ocfg(cfg, S_loc), G=self.G)
            for h in range(H):
                keys = idx[0, h, S_loc:S_loc + cfg.k]
                keys = keys[keys >= 0]
                bs = oc["bucket_of_unit"][h][keys // 4]
                order = sorted(set(int(b) for b in bs))
                assert len(order) <= cap
                yh = [Y[q, h * ng + g] if cfg.agg else Y[q, h] for g in range(ng)]
                for i, b in enumerate(order):
                    c = _bf(oc["cent"][h, b])
                    best = -math.inf
                    for y in yh:
                        s = 0.0
                        for a, cc in zip(_bf(y), c):
                            s = s + float(a) * float(cc)
                        best = max(best, s)
                    rec[q, h, i, 0] = base + b
                    rec[q, h, i, 1] = int((bs == b).sum())
                    rec[q, h, i, 2:4] = np.array([best], np.float64).view(np.int32)
                rec_n[q, h] = len(order)
        return torch.from_numpy(rec), torch.from_numpy(rec_n)

    def merge(self, rec_all, n_all, rank, t0, cache, p0, cfg):
        oc, S_loc, n_loc = cache["oc"], cache["S_loc"], cache["n"]
        rec_all, n_all = rec_all.numpy(), n_all.numpy()
        world, nq, H = n_all.shape
        S, k, W = cfg.sinks, cfg.k, cfg.window
        base = p0 // 512 * 64
        out = np.full((nq, H, S + k + W), -1, np.int32)
        off, mem = oc["offsets"], oc["members"]
        for q in range(nq):
            t = t0 + q
            lim = t - W
            for h in range(H):
                if p0 == 0:
                    for i in range(min(S, t + 1)):
                        out[q, h, i] = i
                w0, w1 = max(S, t - W + 1, p0), min(t + 1, p0 + n_loc)
                for i, p in enumerate(range(w0, w1)):
                    out[q, h, S + k + i] = p
                recs = []
                for r in range(world):
                    for i in range(n_all[r, q, h]):
                        x = rec_all[r, q, h, i]
                        recs.append((-float(x[2:4].copy().view(np.float64)[0]), int(x[0]), int(x[1]), r))
                recs.sort()
                need, mine = k, []
                for _, gid, w, r in recs:
                    if need <= 0:
                        break
                    take = min(w, need)
                    need -= take
                    if r == rank:
                        mine.append((gid, take))
                o = S
                for gid, take in sorted(mine):
                    b = gid - base
                    for m in mem[h][off[h][b]:off[h][b + 1]]:
                        for p in range(4 * m, min(4 * m + 4, n_loc)):
                            if take and S_loc <= p <= lim - p0:
                                out[q, h, o] = p + p0
                                o += 1
                                take -= 1
        return torch.from_numpy(out)

    def partial(self, Q, K_local, V_local, idx, p0):
        Qf, Kf, Vf = _bf(_bits(Q)), _bf(_bits(K_local)), _bf(_bits(V_local))
        idx = idx.numpy()
        nq, hq, d = Qf.shape
        H = Kf.shape[1]
        G = hq // H
        O = np.zeros((nq, hq, d))
        L = np.full((nq, hq), -np.inf)
        for q in range(nq):
            for hh in range(hq):
                e = idx[q, hh // G]
                e = e[e >= 0] - p0
                if e.size == 0:
                    continue
                s = (Kf[e, hh // G] @ Qf[q, hh]) / math.sqrt(d) * LOG2E
                m = s.max()
                p = np.exp2(s - m)
                O[q, hh] = (p @ Vf[e, hh // G]) / p.sum()
                L[q, hh] = m + math.log2(p.sum())
        return torch.from_numpy(O), torch.from_numpy(L)

    def combine(self, O_all, L_all):
        O_all, L_all = O_all.numpy(), L_all.numpy()
        M = L_all.max(axis=0)
        w = np.where(np.isfinite(L_all), np.exp2(L_all - np.where(np.isfinite(M), M, 0.0)[None]), 0.0)
        den = w.sum(axis=0)
        num = (w[..., None] * O_all).sum(axis=0)
        return torch.from_numpy(np.where(den[..., None] > 0, num / np.where(den > 0, den, 1.0)[..., None], 0.0))
