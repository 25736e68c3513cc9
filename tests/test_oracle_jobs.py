"""The GPU tests' oracle helpers (tests/oracle_jobs.py), checked on the CPU:
a cache cut to its first blocks equals the oracle's cache of those keys
alone, and the worker's decode rows equal the oracle's own calls."""
import numpy as np

import oracle
import oracle_jobs
import synth


def test_first_blocks_equals_build_of_prefix():
    inp = synth.layer_inputs("prefill-4k", seed=0, parts=("K",))
    K = inp["K"][:, :1]
    cfg = oracle.Cfg(k=512, sinks=4, window=256)
    full = oracle.build_cache(oracle.key_latent_pool(K, inp["Wk"], 4), 4096, cfg)
    for tb in (512, 1536, 3584):
        cut = oracle_jobs.first_blocks(full, tb)
        ref = oracle.build_cache(oracle.key_latent_pool(np.ascontiguousarray(K[:tb]), inp["Wk"], 4), tb, cfg)
        assert set(cut) == set(ref)
        for key, v in ref.items():
            if isinstance(v, np.ndarray):
                assert np.array_equal(cut[key], v), (tb, key)
            else:
                assert cut[key] == v, (tb, key)


def test_decode_context_rows_match_direct_calls(tmp_path):
    inp = synth.layer_inputs("decode-small", seed=0, parts=("Q", "K", "V"))
    h, G = 1, 4
    K = np.ascontiguousarray(inp["K"][:, h:h + 1])
    V = np.ascontiguousarray(inp["V"][:, h:h + 1])
    np.save(tmp_path / "K.npy", K)
    np.save(tmp_path / "V.npy", V)
    kw = dict(k=256, sinks=4, window=600, beam=2, agg=0)
    steps = [(0, 2046, None), (1, 2047, None), (2, 4000, None)]
    queries = [(s, t, np.ascontiguousarray(inp["Q"][t:t + 1, G * h:G * (h + 1)])) for s, t, _ in steps]
    out = oracle_jobs.decode_context_rows(dict(K=str(tmp_path / "K.npy"), V=str(tmp_path / "V.npy"),
                                               Wk=inp["Wk"], Wq=inp["Wq"], G=G, modes=(0, 1), cfg=kw,
                                               queries=queries))
    for s, t, Qt in queries:
        tb = 512 * ((t + 1) // 512)
        oc = oracle.build_cache(oracle.key_latent_pool(np.ascontiguousarray(K[:tb]), inp["Wk"], 4), tb,
                                oracle.Cfg(**kw))
        Y = oracle.query_latent(Qt, inp["Wq"], 1, 0)
        for mode in (0, 1):
            cfg = oracle.Cfg(**dict(kw, mode=mode))
            oidx, _, _ = oracle.select(oc, Y, np.array([t]), cfg, tree=oracle.build_tree(oc) if mode else None, G=G)
            got_idx, got_O = out[(mode, s)]
            assert np.array_equal(got_idx, oidx[0, 0]), (s, mode)
            assert np.array_equal(got_O, oracle.attention(Qt, K[:t + 1], V[:t + 1], oidx)[0]), (s, mode)
