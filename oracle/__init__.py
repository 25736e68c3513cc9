"""CPU oracle for the Latent Sparse Attention (LSA) indexer + attention path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  It
shares no code with the CUDA library (``clustered_key_indexing_b200``) and
never imports it; both sides meet only at the seeded input generators in
``synth``.

The arithmetic lives in ``lsa_oracle.c`` (plain single-threaded C, fp64,
ascending-index sums, no fused multiply-add); this module marshals numpy
arrays in and out of it.  Each function names the passage it restates:

* essay "《卡片柜》——当注意力学会先查目录再翻书" (zhichai.net), ch. 2
  (key latent, pool, Ward buckets, centroids), ch. 3 (flat search, sinks,
  window), ch. 4 (binary tree, beam descent), ch. 5 (one W_k/W_q pair per
  layer; native max over heads), ch. 6 (the natively trained variant's
  backward over saved key indices);
* tutorial "隐空间稀疏注意力 (LSA)" (diosapp.com.cn), section 二 (query in the
  same latent space; exact softmax attention over the selected keys);
* Ward (1963), cited by the essay: least increase of within-cluster SSE.

Every function is pinned by the ``-m "not gpu"`` tests in ``tests/`` against
closed forms, brute force, a library routine (scipy's Ward linkage, torch's
scaled-dot-product attention) or hand-derived values under ``tests/golden``.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lsa_oracle.c")
_SO = os.path.join(_HERE, "liblsa_oracle.so")
_lib = None

IMAX = 2147483647


def build(force: bool = False) -> str:
    """Compile ``lsa_oracle.c`` with gcc into ``liblsa_oracle.so``."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=gnu11", "-fPIC", "-shared", "-ffp-contract=off",
             "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _L():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        P = ctypes.c_void_p
        i32, i64 = ctypes.c_int32, ctypes.c_int64
        lib.lsao_bf16_rne.restype = ctypes.c_uint16
        lib.lsao_bf16_rne.argtypes = [ctypes.c_double]
        lib.lsao_bf16_rne_array.argtypes = [P, i64, P]
        lib.lsao_e4m3_rne.restype = ctypes.c_uint8
        lib.lsao_e4m3_rne.argtypes = [ctypes.c_double]
        lib.lsao_e4m3_to_double.restype = ctypes.c_double
        lib.lsao_e4m3_to_double.argtypes = [ctypes.c_uint8]
        lib.lsao_cent_fp8.argtypes = [P, i64, i32, P]
        lib.lsao_key_latent_pool.argtypes = [P, i64, i32, i32, P, i32, i32, P]
        lib.lsao_query_latent.argtypes = [P, i64, i32, i32, i32, P, i32, i32, P]
        lib.lsao_ward_delta.restype = ctypes.c_double
        lib.lsao_ward_delta.argtypes = [P, i32, P, i32, i32]
        lib.lsao_ward_block.argtypes = [P, i32, i32, i32, i32, i32, P, P]
        lib.lsao_build.argtypes = [P, i64, i32, i32, i32, i32, i32, i32, i32, i32,
                                   P, P, P, P, P, P, P, P, P]
        lib.lsao_tree_levels.restype = i32
        lib.lsao_tree_levels.argtypes = [i64, P, P]
        lib.lsao_build_tree.argtypes = [i64, i32, i32, P, P, P, P, P]
        lib.lsao_select.argtypes = [i64, i32, i32, i32, i64, P, P, P, P, P, P, P, P,
                                    P, i32, P, i64, i32, i32, i32, i32, i32, i32, i32,
                                    P, P, P]
        lib.lsao_attention.argtypes = [P, P, P, P, i64, i32, i32, i32, i32, P]
        lib.lsao_attention_backward.argtypes = [P, P, P, P, P, i64, i32, i32, i32, i32, i64,
                                                P, P, P]
        for f in ("lsao_key_latent_pool", "lsao_query_latent", "lsao_ward_block",
                  "lsao_build", "lsao_build_tree", "lsao_select", "lsao_attention",
                  "lsao_attention_backward"):
            getattr(lib, f).restype = i32
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


@dataclass
class Cfg:
    """Method parameters (names follow the pages' notation)."""
    d_head: int = 128
    d_latent: int = 64
    pool: int = 4            # keys pooled per unit (ch. 2)
    block: int = 512         # keys per cluster block (ch. 2)
    bucket_mean: int = 8     # mean keys per bucket (ch. 2)
    bucket_max: int = 16     # max keys per bucket (ch. 2)
    k: int = 2048            # long-range keys per query (ch. 3)
    sinks: int = 4           # S (ch. 3)
    window: int = 1024       # W (ch. 3)
    beam: int = 2            # tree beam width (ch. 4)
    mode: int = 0            # 0 flat, 1 tree
    agg: int = 0             # 0 mean over the GQA group, 1 max (native)

    @property
    def units_per_block(self) -> int:
        return self.block // self.pool

    @property
    def buckets_per_block(self) -> int:
        return self.block // self.bucket_mean

    @property
    def max_units(self) -> int:
        return self.bucket_max // self.pool

    @property
    def row(self) -> int:
        return self.sinks + self.k + self.window


# ------------------------------------------------------------------ bf16

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_rne(x) -> np.ndarray:
    """Round fp64 values straight to bf16 bits (ties to even)."""
    x = _c(np.atleast_1d(x), np.float64)
    out = np.empty(x.shape, np.uint16)
    _L().lsao_bf16_rne_array(_p(x), x.size, _p(out))
    return out


# -------------------------------------------------- fp8 centroids (ch. 8)

FP8_SCALE_EXP = 8   # a component c is stored as the e4m3 code of 2^8 * c


def e4m3_rne(x) -> np.ndarray:
    """fp64 values straight to OCP e4m3 codes (uint8), ties to even,
    saturating at +-448."""
    x = _c(np.atleast_1d(x), np.float64)
    L = _L()
    return np.array([L.lsao_e4m3_rne(float(v)) for v in x.ravel()], np.uint8).reshape(x.shape)


def e4m3_to_f64(codes) -> np.ndarray:
    c = np.atleast_1d(np.asarray(codes, np.uint8))
    L = _L()
    return np.array([L.lsao_e4m3_to_double(int(v)) for v in c.ravel()], np.float64).reshape(c.shape)


def cent_fp8(cache: dict) -> np.ndarray:
    """FP8 centroid cache (essay ch. 8: the bucket cache stacks with FP8
    quantisation): per bucket, the e4m3 code of 2^8 * s / |s| for its fp64
    unit sum s, rounded straight from fp64.  Returns uint8 [H, NB, dl]."""
    s = _c(cache["sum"], np.float64)
    H, NB, dl = s.shape
    out = np.empty((H, NB, dl), np.uint8)
    _L().lsao_cent_fp8(_p(s), H * NB, dl, _p(out))
    return out


def fp8_as_bf16(codes: np.ndarray) -> np.ndarray:
    """The values 2^-8 * e4m3(code) as bf16 bits (exact: 4 significant bits
    and exponents in bf16's range), so that the bf16 selection scores the FP8
    centroids exactly."""
    return bf16_rne(np.ldexp(e4m3_to_f64(codes), -FP8_SCALE_EXP)).reshape(np.shape(codes))


def with_fp8_centroids(cache: dict) -> dict:
    """The cache with its centroids replaced by the FP8 ones (as exact bf16
    values): selecting on it scores every bucket against its FP8 centroid."""
    return dict(cache, cent=fp8_as_bf16(cent_fp8(cache)))


# ----------------------------------------------------------- latents (ch. 2)

def key_latent_pool(K: np.ndarray, Wk: np.ndarray, pool: int = 4) -> np.ndarray:
    """Pooled unit latents U [H, ceil(T/pool), dl] (essay ch. 2): each key is
    projected by W_k, L2-normalised, and every `pool` consecutive keys are
    averaged (no re-normalisation)."""
    K = _c(K, np.uint16)
    Wk = _c(Wk, np.float32)
    T, H, d = K.shape
    dl = Wk.shape[1]
    NU = (T + pool - 1) // pool
    U = np.empty((H, NU, dl), np.float64)
    rc = _L().lsao_key_latent_pool(_p(K), T, H, d, _p(Wk), dl, pool, _p(U))
    assert rc == 0
    return U


def query_latent(Q: np.ndarray, Wq: np.ndarray, hkv: int, agg: int = 0) -> np.ndarray:
    """Query latents as bf16 bits (tutorial section 二; essay ch. 5):
    agg 0 -> [nq, hkv, dl] group means, agg 1 -> [nq, hq, dl] per head."""
    Q = _c(Q, np.uint16)
    Wq = _c(Wq, np.float32)
    nq, hq, d = Q.shape
    dl = Wq.shape[1]
    Y = np.empty((nq, hkv if agg == 0 else hq, dl), np.uint16)
    rc = _L().lsao_query_latent(_p(Q), nq, hq, hkv, d, _p(Wq), dl, agg, _p(Y))
    assert rc == 0
    return Y


# --------------------------------------------------------------- Ward (ch. 2)

def ward_delta(sA, nA, sB, nB) -> float:
    sA = _c(sA, np.float64)
    sB = _c(sB, np.float64)
    return _L().lsao_ward_delta(_p(sA), nA, _p(sB), nB, sA.size)


def ward_block(U: np.ndarray, m_target: int, max_units: int = 4, naive: bool = False):
    """Capped Ward clustering of one block's pooled units (essay ch. 2;
    Ward 1963).  Returns (bucket_of [n], margin)."""
    U = _c(U, np.float64)
    n, dl = U.shape
    out = np.empty(n, np.int32)
    mg = np.zeros(1, np.float64)
    rc = _L().lsao_ward_block(_p(U), n, dl, m_target, max_units, int(naive), _p(out), _p(mg))
    if rc != 0:
        raise ValueError("no eligible merge left")
    return out, float(mg[0])


def build_cache(U: np.ndarray, T: int, cfg: Cfg, naive: bool = False) -> dict:
    """Bucket cache of every kv-head (essay ch. 2-3)."""
    U = _c(U, np.float64)
    H, NU, dl = U.shape
    bu, bpb = cfg.units_per_block, cfg.buckets_per_block
    nblk = (NU + bu - 1) // bu
    NB = nblk * bpb
    c = dict(
        T=T, H=H, NU=NU, NB=NB, nblk=nblk,
        bucket_of_unit=np.full((H, NU), -1, np.int32),
        members=np.full((H, NU), -1, np.int32),
        offsets=np.zeros((H, NB + 1), np.int32),
        cnt_lr=np.zeros((H, NB), np.int32),
        minlr=np.zeros((H, NB), np.int32),
        maxpos=np.zeros((H, NB), np.int32),
        sum=np.zeros((H, NB, dl), np.float64),
        cent=np.zeros((H, NB, dl), np.uint16),
        ward_margin=np.zeros((H, nblk), np.float64),
    )
    rc = _L().lsao_build(_p(U), T, H, dl, cfg.pool, bu, bpb, cfg.max_units, cfg.sinks,
                         int(naive), _p(c["bucket_of_unit"]), _p(c["members"]),
                         _p(c["offsets"]), _p(c["cnt_lr"]), _p(c["minlr"]),
                         _p(c["maxpos"]), _p(c["sum"]), _p(c["cent"]),
                         _p(c["ward_margin"]))
    if rc != 0:
        raise ValueError("Ward clustering failed")
    return c


def tree_levels(NB: int):
    ln = np.zeros(64, np.int64)
    lo = np.zeros(64, np.int64)
    L = _L().lsao_tree_levels(NB, _p(ln), _p(lo))
    return [int(x) for x in ln[:L]], [int(x) for x in lo[:L]]


def build_tree(cache: dict) -> dict:
    """Complete binary tree of merged centroids (essay ch. 4)."""
    H, NB = cache["H"], cache["NB"]
    dl = cache["sum"].shape[2]
    ln, lo = tree_levels(NB)
    ntot = lo[-1] + ln[-1]
    t = dict(levels=len(ln), level_n=ln, level_off=lo, ntot=ntot,
             sum=np.zeros((H, ntot, dl), np.float64),
             minlr=np.zeros((H, ntot), np.int32),
             cent=np.zeros((H, ntot, dl), np.uint16))
    rc = _L().lsao_build_tree(NB, H, dl, _p(cache["sum"]), _p(cache["minlr"]),
                              _p(t["sum"]), _p(t["minlr"]), _p(t["cent"]))
    assert rc == 0
    return t


# --------------------------------------------------------- selection (ch. 3-4)

def select(cache: dict, Y: np.ndarray, tpos, cfg: Cfg, tree: dict | None = None, G: int = 1):
    """Index lists [nq, H, S+k+W] for query positions `tpos` (essay ch. 3-4).
    Returns (idx, margin [nq, H], ncmp [nq, H])."""
    Y = _c(Y, np.uint16)
    tpos = _c(tpos, np.int64)
    nq = tpos.size
    H, NB, dl = cache["H"], cache["NB"], cache["cent"].shape[2]
    if cfg.mode == 1 and tree is None:
        tree = build_tree(cache)
    if tree is None:
        tminlr = np.zeros(1, np.int32)
        tcent = np.zeros(1, np.uint16)
    else:
        tminlr, tcent = tree["minlr"], tree["cent"]
    idx = np.empty((nq, H, cfg.row), np.int32)
    mg = np.empty((nq, H), np.float64)
    nc = np.empty((nq, H), np.int64)
    rc = _L().lsao_select(NB, H, dl, cfg.pool, cache["T"], _p(cache["offsets"]),
                          _p(cache["members"]), _p(cache["cnt_lr"]), _p(cache["minlr"]),
                          _p(cache["maxpos"]), _p(cache["cent"]), _p(tminlr), _p(tcent),
                          _p(Y), G, _p(tpos), nq, cfg.k, cfg.sinks, cfg.window, cfg.beam,
                          cfg.bucket_mean, cfg.mode, cfg.agg, _p(idx), _p(mg), _p(nc))
    assert rc == 0
    return idx, mg, nc


# -------------------------------------------------------- attention (sec. 二)

def attention(Q: np.ndarray, K: np.ndarray, V: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """Exact softmax attention over index lists; Q [nq, hq, d] rows aligned
    with idx [nq, hkv, n]; returns fp64 O [nq, hq, d] (tutorial section 二)."""
    Q = _c(Q, np.uint16)
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    idx = _c(idx, np.int32)
    nq, hq, d = Q.shape
    hkv = K.shape[1]
    O = np.empty((nq, hq, d), np.float64)
    rc = _L().lsao_attention(_p(Q), _p(K), _p(V), _p(idx), nq, hq, hkv, d, idx.shape[2], _p(O))
    assert rc == 0
    return O


def _f64(x) -> np.ndarray:
    """bf16 bits (uint16) to fp64; any other array is taken as real values."""
    x = np.asarray(x)
    return bf16_to_f64(x) if x.dtype == np.uint16 else _c(x, np.float64)


def attention_backward(Q, K, V, idx: np.ndarray, dO):
    """Gradients (dQ, dK, dV) of the exact sparse attention over saved index
    lists, in fp64 (tutorial section 二 for the attention; essay ch. 6: the
    natively trained variant keeps each query's selected key indices for its
    backward pass).  The discrete selection carries no gradient.

    Q, dO [nq, hq, d]; K, V [T, hkv, d]; each as bf16 bits or real values.
    idx [nq, hkv, n] as for ``attention``.  Returns dQ [nq, hq, d] and
    dK, dV [T, hkv, d], fp64."""
    Qf, Kf, Vf, gf = _f64(Q), _f64(K), _f64(V), _f64(dO)
    idx = _c(idx, np.int32)
    nq, hq, d = Qf.shape
    T, hkv, _ = Kf.shape
    assert gf.shape == Qf.shape and Vf.shape == Kf.shape and idx.shape[:2] == (nq, hkv)
    dQ = np.empty_like(Qf)
    dK = np.empty_like(Kf)
    dV = np.empty_like(Vf)
    rc = _L().lsao_attention_backward(_p(Qf), _p(Kf), _p(Vf), _p(gf), _p(idx), nq, hq, hkv, d,
                                      idx.shape[2], T, _p(dQ), _p(dK), _p(dV))
    assert rc == 0
    return dQ, dK, dV


# ------------------------------------------------------------ whole layer

def layer(Q, K, V, Wk, Wq, cfg: Cfg, tpos=None, cache=None, tree=None):
    """The whole path for the query positions `tpos` (default: all T):
    build -> (tree) -> query latent -> select -> attention.
    Returns dict with U, cache, tree, Y, idx, margin, ncmp, O."""
    T, hkv, _ = K.shape
    hq = Q.shape[1]
    G = hq // hkv
    if tpos is None:
        tpos = np.arange(T, dtype=np.int64)
    tpos = np.asarray(tpos, np.int64)
    U = None
    if cache is None:
        U = key_latent_pool(K, Wk, cfg.pool)
        cache = build_cache(U, T, cfg)
    if cfg.mode == 1 and tree is None:
        tree = build_tree(cache)
    Qs = np.ascontiguousarray(np.asarray(Q)[tpos])
    Y = query_latent(Qs, Wq, hkv, cfg.agg)
    idx, mg, nc = select(cache, Y, tpos, cfg, tree=tree, G=G)
    O = attention(Qs, K, V, idx)
    return dict(U=U, cache=cache, tree=tree, Y=Y, idx=idx, margin=mg, ncmp=nc, O=O)


# ------------------------------------------- training-free PCA projection

def fit_pca(K: np.ndarray, d_latent: int = 64):
    """Training-free projection of the distilled variant: the first d_latent
    principal directions of the layer's keys (tutorial "隐空间稀疏注意力
    (LSA)" and the essay's closing remarks: PCA of the keys, the leading 64
    directions taken as the projection, no training).

    Readings: the covariance is the centred one, (1/N) sum (k - mean)(k -
    mean)^T over the keys of every kv-head (one projection per layer);
    directions are ordered by eigenvalue, largest first, equal eigenvalues by
    eigh's order; each direction's sign makes its largest-magnitude component
    (the first such) positive.

    K: bf16 bits [T, hkv, d].  Returns (W fp32 [d, d_latent] with the
    directions as columns, eigenvalues fp64 [d] descending, V fp64 [d, d])."""
    X = bf16_to_f64(np.asarray(K, np.uint16)).reshape(-1, K.shape[-1])
    N = X.shape[0]
    mean = X.sum(axis=0) / N
    Xc = X - mean
    C = (Xc.T @ Xc) / N
    lam, V = np.linalg.eigh(C)                    # ascending
    order = np.argsort(-lam, kind="stable")
    lam, V = lam[order], V[:, order]
    for j in range(V.shape[1]):
        i = int(np.argmax(np.abs(V[:, j])))
        if V[i, j] < 0:
            V[:, j] = -V[:, j]
    return np.ascontiguousarray(V[:, :d_latent], dtype=np.float32), lam, V
