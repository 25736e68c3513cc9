"""PyTorch-facing calls of the LSA library (marshalling only).

Tensors are CUDA tensors: Q/K/V/O torch.bfloat16, W_k/W_q torch.float32
[128, 64], index lists torch.int32.  Streams default to torch's current
stream.  Each call maps one-to-one onto an entry point of include/lsa.h.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass, fields

import torch

from . import _lib
from ._lib import check, lib


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


BF16, F32, I32 = torch.bfloat16, torch.float32, torch.int32
W_SHAPE = (128, 64)  # W_k, W_q: d_head x d_latent


def _spec(t, name, dtype, shape=None):
    """One tensor argument's dtype and, where given, its shape (None entries
    match any size); the library reads every argument as this dense layout,
    so a mismatch is refused before any call."""
    if t is None:
        return
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if shape is not None and (t.dim() != len(shape) or
                              any(n is not None and t.shape[i] != n for i, n in enumerate(shape))):
        want = tuple("*" if n is None else n for n in shape)
        raise ValueError(f"{name}: expected shape {want}, got {tuple(t.shape)}")


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("LSA calls take CUDA tensors (there is no CPU implementation)")
        if t is not None and not t.is_contiguous():
            raise ValueError("LSA calls take contiguous tensors")


@dataclass
class Config:
    """Method parameters (see lsa_cfg in include/lsa.h)."""
    d_head: int = 128
    d_latent: int = 64
    pool: int = 4
    block: int = 512
    bucket_mean: int = 8
    bucket_max: int = 16
    k: int = 2048
    sinks: int = 4
    window: int = 1024
    beam: int = 2
    mode: int = 0   # 0 flat, 1 tree
    agg: int = 0    # 0 group mean, 1 max over heads (native)

    def c(self) -> _lib.lsa_cfg:
        return _lib.lsa_cfg(*[getattr(self, f.name) for f in fields(self)])

    @property
    def row(self) -> int:
        return self.sinks + self.k + self.window


class Cache:
    """Device arrays of one layer's bucket cache (lsa_cache), sized for
    `cap_tokens` tokens per head."""

    def __init__(self, hkv: int, cap_tokens: int, cfg: Config | None = None, device="cuda",
                 with_units: bool = True, fp8: bool = False):
        """fp8: also keep FP8 (e4m3) centroids, which the flat decode step
        then scores (lsa_cache.cent8)."""
        cfg = cfg or Config()
        cc = cfg.c()
        L = lib()
        self.hkv = hkv
        self.cap_units = int(L.lsa_cache_units(ctypes.byref(cc), cap_tokens))
        self.cap_buckets = int(L.lsa_cache_buckets(ctypes.byref(cc), cap_tokens))
        dl = cfg.d_latent
        z = dict(device=device)
        # pooled unit latents (the decode state keeps only a block ring instead)
        self.U = torch.zeros((hkv, self.cap_units if with_units else 1, dl), dtype=torch.float64, **z)
        self.bucket_of_unit = torch.full((hkv, self.cap_units), -1, dtype=torch.int32, **z)
        self.members = torch.full((hkv, self.cap_units), -1, dtype=torch.int32, **z)
        self.offsets = torch.zeros((hkv, self.cap_buckets + 1), dtype=torch.int32, **z)
        self.cnt_lr = torch.zeros((hkv, self.cap_buckets), dtype=torch.int32, **z)
        self.minlr = torch.zeros((hkv, self.cap_buckets), dtype=torch.int32, **z)
        self.maxpos = torch.zeros((hkv, self.cap_buckets), dtype=torch.int32, **z)
        self.sum = torch.zeros((hkv, self.cap_buckets, dl), dtype=torch.float64, **z)
        self.cent = torch.zeros((hkv, self.cap_buckets, dl), dtype=torch.bfloat16, **z)
        self.units = torch.zeros((hkv, self.cap_buckets), dtype=torch.int32, **z)
        self.cent8 = torch.zeros((hkv, self.cap_buckets, dl), dtype=torch.uint8, **z) if fp8 else None
        self.c = _lib.lsa_cache(hkv, 0, self.cap_units, self.cap_buckets, *[
            t.data_ptr() for t in (self.U, self.bucket_of_unit, self.members, self.offsets,
                                   self.cnt_lr, self.minlr, self.maxpos, self.sum, self.cent,
                                   self.units)], self.cent8.data_ptr() if fp8 else None)

    @property
    def n_tokens(self) -> int:
        return int(self.c.n_tokens)

    @property
    def n_buckets(self) -> int:
        nu = -(-self.n_tokens // 4)
        return -(-nu // 128) * 64


class Tree:
    """Device arrays of the binary centroid tree (lsa_tree) over a cache."""

    def __init__(self, cache: "Cache", device="cuda"):
        self.t = _lib.lsa_tree()
        check(lib().lsa_tree_layout(cache.cap_buckets, ctypes.byref(self.t)), "lsa_tree_layout")
        n, hkv = int(self.t.n_nodes), cache.hkv
        self.sum = torch.zeros((hkv, n, 64), dtype=torch.float64, device=device)
        self.minlr = torch.zeros((hkv, n), dtype=torch.int32, device=device)
        self.cent = torch.zeros((hkv, n, 64), dtype=torch.bfloat16, device=device)
        self.t.sum, self.t.minlr, self.t.cent = self.sum.data_ptr(), self.minlr.data_ptr(), self.cent.data_ptr()

    @property
    def levels(self):
        return int(self.t.levels)

    @property
    def level_n(self):
        return [int(self.t.level_n[i]) for i in range(self.levels)]

    @property
    def level_off(self):
        return [int(self.t.level_off[i]) for i in range(self.levels)]


def check_device_error():
    """Raise if a kernel set the device-side error word (synchronous)."""
    check(lib().lsa_check_device_error(), "device")


def build_buckets(K: torch.Tensor, W_k: torch.Tensor, cfg: Config, cache: Cache, stream=None):
    """lsa_build_buckets: key latents, pooling, Ward buckets, centroids."""
    _spec(K, "K", BF16, (None, None, 128))
    _spec(W_k, "W_k", F32, W_SHAPE)
    _need_cuda(K, W_k)
    T, hkv, _ = K.shape
    check(lib().lsa_build_buckets(_ptr(K), T, hkv, _ptr(W_k), ctypes.byref(cfg.c()),
                                  ctypes.byref(cache.c), _stream(stream)), "lsa_build_buckets")
    return cache


def build_tree(cache: Cache, cfg: Config, tree: Tree | None = None, stream=None) -> Tree:
    """lsa_build_tree: binary tree of merged centroids."""
    tree = tree or Tree(cache)
    check(lib().lsa_build_tree(ctypes.byref(cache.c), ctypes.byref(cfg.c()), ctypes.byref(tree.t),
                               _stream(stream)), "lsa_build_tree")
    return tree


def query_latent(Q: torch.Tensor, W_q: torch.Tensor, hkv: int, cfg: Config, stream=None):
    """lsa_query_latent: bf16 latents [nq, hkv, 64] (mean) or [nq, hq, 64] (native)."""
    _spec(Q, "Q", BF16, (None, None, 128))
    _spec(W_q, "W_q", F32, W_SHAPE)
    _need_cuda(Q, W_q)
    nq, hq, _ = Q.shape
    Y = torch.empty((nq, hkv if cfg.agg == 0 else hq, cfg.d_latent), dtype=torch.bfloat16, device=Q.device)
    check(lib().lsa_query_latent(_ptr(Q), nq, hq, hkv, _ptr(W_q), ctypes.byref(cfg.c()), _ptr(Y),
                                 _stream(stream)), "lsa_query_latent")
    return Y


def select_workspace_bytes(cfg: Config, nq: int, hq: int, cache: Cache) -> int:
    return int(lib().lsa_select_workspace_bytes(ctypes.byref(cfg.c()), nq, hq, ctypes.byref(cache.c)))


def select(Q: torch.Tensor, t0: int, W_q: torch.Tensor, cache: Cache, cfg: Config,
           tree: Tree | None = None, idx: torch.Tensor | None = None, Y_out: torch.Tensor | None = None,
           ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """lsa_select: index lists [nq, hkv, S + k + W] for positions t0 .. t0+nq-1."""
    _spec(Q, "Q", BF16, (None, None, 128))
    _spec(W_q, "W_q", F32, W_SHAPE)
    nq, hq, _ = Q.shape
    _spec(idx, "idx", I32, (nq, cache.hkv, cfg.row))
    _spec(Y_out, "Y_out", BF16, (nq, cache.hkv if cfg.agg == 0 else hq, 64))
    _spec(ws, "ws", torch.uint8, (None,))
    _need_cuda(Q, W_q, idx, Y_out, ws)
    if idx is None:
        idx = torch.empty((nq, cache.hkv, cfg.row), dtype=torch.int32, device=Q.device)
    need = select_workspace_bytes(cfg, nq, hq, cache)
    if ws is None or ws.numel() < need:
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=Q.device)
    check(lib().lsa_select(_ptr(Q), t0, nq, hq, _ptr(W_q), ctypes.byref(cache.c),
                           ctypes.byref(tree.t) if tree is not None else None, ctypes.byref(cfg.c()),
                           _ptr(idx), _ptr(Y_out), _ptr(ws), ws.numel(), _stream(stream)), "lsa_select")
    return idx


def sparse_attn(Q, K, V, idx, T: int | None = None, O=None, stream=None) -> torch.Tensor:
    """lsa_sparse_attn: exact softmax attention over index lists."""
    _spec(Q, "Q", BF16, (None, None, 128))
    _spec(K, "K", BF16, (None, None, 128))
    _spec(V, "V", BF16, tuple(K.shape))
    nq, hq, d = Q.shape
    hkv = K.shape[1]
    _spec(idx, "idx", I32, (nq, hkv, None))
    _spec(O, "O", BF16, (nq, hq, 128))
    _need_cuda(Q, K, V, idx, O)
    if O is None:
        O = torch.empty((nq, hq, d), dtype=torch.bfloat16, device=Q.device)
    T = K.shape[0] if T is None else T
    check(lib().lsa_sparse_attn(_ptr(Q), _ptr(K), _ptr(V), _ptr(idx), nq, hq, hkv, idx.shape[2], T,
                                _ptr(O), _stream(stream)), "lsa_sparse_attn")
    return O


def attn_backward(Q, K, V, O, dO, idx, T: int | None = None, dK=None, dV=None, stream=None):
    """lsa_attn_backward: gradients of the sparse attention over saved index
    lists.  Returns (dQ [nq, hq, 128], dK, dV [T, hkv, 128]), fp32; dK and dV
    are added to when given (so query chunks accumulate), else zero-started."""
    _spec(Q, "Q", BF16, (None, None, 128))
    nq, hq, d = Q.shape
    _spec(O, "O", BF16, tuple(Q.shape))
    _spec(dO, "dO", BF16, tuple(Q.shape))
    _spec(K, "K", BF16, (None, None, 128))
    _spec(V, "V", BF16, tuple(K.shape))
    hkv = K.shape[1]
    _spec(idx, "idx", I32, (nq, hkv, None))
    _spec(dK, "dK", F32, tuple(K.shape))
    _spec(dV, "dV", F32, tuple(K.shape))
    _need_cuda(Q, K, V, O, dO, idx, dK, dV)
    T = K.shape[0] if T is None else T
    dQ = torch.empty((nq, hq, d), dtype=torch.float32, device=Q.device)
    if dK is None:
        dK = torch.zeros((K.shape[0], hkv, d), dtype=torch.float32, device=Q.device)
    if dV is None:
        dV = torch.zeros((V.shape[0], hkv, d), dtype=torch.float32, device=Q.device)
    check(lib().lsa_attn_backward(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(dO), _ptr(idx), nq, hq, hkv,
                                  idx.shape[2], T, _ptr(dQ), _ptr(dK), _ptr(dV), _stream(stream)),
          "lsa_attn_backward")
    return dQ, dK, dV


def select_attn_workspace_bytes(nq: int, hq: int) -> int:
    return int(lib().lsa_select_attn_workspace_bytes(nq, hq))


def select_attn(Q, K, V, idx, t0: int, cfg: Config, T: int | None = None, O=None, ws=None,
                stream=None) -> torch.Tensor:
    """lsa_select_attn: attention over lsa_select's index rows (window as a band)."""
    _spec(Q, "Q", BF16, (None, None, 128))
    _spec(K, "K", BF16, (None, None, 128))
    _spec(V, "V", BF16, tuple(K.shape))
    nq, hq, d = Q.shape
    hkv = K.shape[1]
    _spec(idx, "idx", I32, (nq, hkv, cfg.row))
    _spec(O, "O", BF16, (nq, hq, 128))
    _spec(ws, "ws", torch.uint8, (None,))
    _need_cuda(Q, K, V, idx, O, ws)
    if O is None:
        O = torch.empty((nq, hq, d), dtype=torch.bfloat16, device=Q.device)
    T = K.shape[0] if T is None else T
    need = select_attn_workspace_bytes(nq, hq)
    if ws is None:
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=Q.device)
    check(lib().lsa_select_attn(_ptr(Q), _ptr(K), _ptr(V), _ptr(idx), t0, nq, hq, hkv, T,
                                ctypes.byref(cfg.c()), _ptr(O), _ptr(ws), ws.numel(), _stream(stream)),
          "lsa_select_attn")
    return O


def fit_pca(K: torch.Tensor, d_latent: int = 64, stream=None):
    """lsa_fit_pca: the training-free projection, the leading d_latent
    principal directions of the keys K [T, hkv, 128] (all heads).  Returns
    (W fp32 [128, d_latent], eigenvalues fp64 [128], descending)."""
    _spec(K, "K", BF16, (None, None, 128))
    _need_cuda(K)
    T, hkv = int(K.shape[0]), int(K.shape[1])
    W = torch.empty((128, d_latent), dtype=torch.float32, device=K.device)
    eig = torch.empty(128, dtype=torch.float64, device=K.device)
    ws = torch.empty(int(lib().lsa_fit_pca_workspace_bytes(T, hkv)) or 1, dtype=torch.uint8, device=K.device)
    check(lib().lsa_fit_pca(_ptr(K), T, hkv, d_latent, _ptr(W), _ptr(eig), _ptr(ws), ws.numel(), _stream(stream)),
          "lsa_fit_pca")
    return W, eig


def prefill_chunk(cfg: Config, T: int, hq: int, hkv: int, chunk: int = 0) -> int:
    """The query chunk lsa_prefill uses for a requested chunk (0: its own choice)."""
    return int(lib().lsa_prefill_chunk(ctypes.byref(cfg.c()), T, hq, hkv, chunk))


def prefill_workspace_bytes(cfg: Config, T: int, hq: int, hkv: int, chunk: int) -> int:
    return int(lib().lsa_prefill_workspace_bytes(ctypes.byref(cfg.c()), T, hq, hkv, chunk))


def prefill(Q, K, V, W_k, W_q, cfg: Config, cache: Cache | None = None, tree: Tree | None = None,
            O=None, chunk: int = 16384, ws=None, stream=None) -> torch.Tensor:
    """lsa_prefill: a whole LSA attention layer over a T-token prompt."""
    _spec(Q, "Q", BF16, (None, None, 128))
    T, hq, d = Q.shape
    _spec(K, "K", BF16, (T, None, 128))
    _spec(V, "V", BF16, tuple(K.shape))
    _spec(W_k, "W_k", F32, W_SHAPE)
    _spec(W_q, "W_q", F32, W_SHAPE)
    _spec(O, "O", BF16, (T, hq, 128))
    _need_cuda(Q, K, V, W_k, W_q, O)
    hkv = K.shape[1]
    cache = cache or Cache(hkv, T, cfg, device=Q.device)
    if cfg.mode == 1 and tree is None:
        tree = Tree(cache, device=Q.device)
    if O is None:
        O = torch.empty_like(Q)
    need = prefill_workspace_bytes(cfg, T, hq, hkv, chunk)
    if ws is None or ws.numel() < need:
        ws = torch.empty(need, dtype=torch.uint8, device=Q.device)
    check(lib().lsa_prefill(_ptr(Q), _ptr(K), _ptr(V), T, hq, hkv, _ptr(W_k), _ptr(W_q),
                            ctypes.byref(cfg.c()), ctypes.byref(cache.c),
                            ctypes.byref(tree.t) if tree is not None else None, _ptr(O), chunk,
                            _ptr(ws), ws.numel(), _stream(stream)), "lsa_prefill")
    return O


def prefill_host(hQ, hK, hV, W_k, W_q, cfg: Config, hO=None, dev_bufs=None, cache: Cache | None = None,
                 tree: Tree | None = None, chunk: int = 16384, ws=None, stream=None, h2d_stream=None,
                 d2h_stream=None) -> torch.Tensor:
    """lsa_prefill_host: the whole layer from pinned host Q/K/V into pinned
    host O, uploads and downloads overlapped with the compute.  dev_bufs:
    optional (Q, K, V, O) device buffers; streams: the compute stream (default
    current) and two copy streams (default: new ones)."""
    _spec(hQ, "hQ", BF16, (None, None, 128))
    T, hq, d = hQ.shape
    _spec(hK, "hK", BF16, (T, None, 128))
    _spec(hV, "hV", BF16, tuple(hK.shape))
    _spec(hO, "hO", BF16, tuple(hQ.shape))
    _spec(W_k, "W_k", F32, W_SHAPE)
    _spec(W_q, "W_q", F32, W_SHAPE)
    if dev_bufs is not None:
        for name, t, like in zip(("Q", "K", "V", "O"), dev_bufs, (hQ, hK, hV, hQ)):
            _spec(t, name, BF16, tuple(like.shape))
        _need_cuda(*dev_bufs)
    _need_cuda(W_k, W_q)
    for t in (hQ, hK, hV) + ((hO,) if hO is not None else ()):
        if t.is_cuda or not t.is_pinned() or not t.is_contiguous():
            raise ValueError("lsa_prefill_host takes contiguous pinned host tensors")
    hkv = hK.shape[1]
    dev = W_k.device
    if hO is None:
        hO = torch.empty_like(hQ).pin_memory()
    if dev_bufs is None:
        dev_bufs = (torch.empty(hQ.shape, dtype=hQ.dtype, device=dev), torch.empty(hK.shape, dtype=hK.dtype, device=dev),
                    torch.empty(hV.shape, dtype=hV.dtype, device=dev), torch.empty(hQ.shape, dtype=hQ.dtype, device=dev))
    Q, K, V, O = dev_bufs
    cache = cache or Cache(hkv, T, cfg, device=dev)
    if cfg.mode == 1 and tree is None:
        tree = Tree(cache, device=dev)
    need = prefill_workspace_bytes(cfg, T, hq, hkv, chunk)
    if ws is None or ws.numel() < need:
        ws = torch.empty(need, dtype=torch.uint8, device=dev)
    up = h2d_stream or torch.cuda.Stream(device=dev)
    down = d2h_stream or torch.cuda.Stream(device=dev)
    check(lib().lsa_prefill_host(_ptr(hQ), _ptr(hK), _ptr(hV), _ptr(hO), _ptr(Q), _ptr(K), _ptr(V), _ptr(O), T, hq,
                                 hkv, _ptr(W_k), _ptr(W_q), ctypes.byref(cfg.c()), ctypes.byref(cache.c),
                                 ctypes.byref(tree.t) if tree is not None else None, chunk, _ptr(ws), ws.numel(),
                                 _stream(stream), _stream(up), _stream(down)), "lsa_prefill_host")
    return hO


class Decode:
    """Batched decode state (lsa_decode): `batch` requests of `cap` tokens,
    K/V pools [batch, cap, hkv, 128], a cache whose heads are
    (request, kv-head) pairs, the per-request block ring, and (tree mode) the
    tree.  `load` installs a prompt, `step` decodes one token per request."""

    def __init__(self, batch: int, hkv: int, hq: int, cap: int, cfg: Config, device="cuda", shared=None,
                 fp8: bool = False):
        """`shared`: optional (K_shared, V_shared) [shared_len, hkv, 128], a
        prefix every request starts with (shared_len a multiple of 512); the
        pools then hold each request's tokens from shared_len on.  `fp8`: the
        cache keeps FP8 centroids and the flat search scores those."""
        if cap % 512:
            raise ValueError("cap must be a multiple of 512")
        self.cfg = cfg
        z = dict(device=device)
        self.shared = shared
        sl = 0 if shared is None else int(shared[0].shape[0])
        self.shared_len = sl
        self.K = torch.zeros((batch, cap - sl, hkv, 128), dtype=torch.bfloat16, **z)
        self.V = torch.zeros((batch, cap - sl, hkv, 128), dtype=torch.bfloat16, **z)
        self.U_blk = torch.zeros((batch * hkv, 128, 64), dtype=torch.float64, **z)
        self.cache = Cache(batch * hkv, cap, cfg, device=device, with_units=False, fp8=fp8)
        self.tree = Tree(self.cache, device=device) if cfg.mode == 1 else None
        d = _lib.lsa_decode()
        d.batch, d.hkv, d.hq, d.cap = batch, hkv, hq, cap
        d.K, d.V, d.U_blk = self.K.data_ptr(), self.V.data_ptr(), self.U_blk.data_ptr()
        if shared is not None:
            _spec(shared[0], "K_shared", BF16, (None, hkv, 128))
            _spec(shared[1], "V_shared", BF16, tuple(shared[0].shape))
            _need_cuda(*shared)
            d.K_shared, d.V_shared, d.shared_len = shared[0].data_ptr(), shared[1].data_ptr(), sl
        d.cache = self.cache.c
        if self.tree is not None:
            d.tree = self.tree.t
        self.d = d
        need = int(lib().lsa_decode_workspace_bytes(ctypes.byref(cfg.c()), ctypes.byref(d)))
        if need == 0:
            check(_lib.LSA_EINVAL, "lsa_decode_workspace_bytes")
        self.ws = torch.empty(need, dtype=torch.uint8, **z)

    @property
    def len(self):
        return [int(self.d.len[i]) for i in range(self.d.batch)]

    def load(self, r: int, K: torch.Tensor, V: torch.Tensor, W_k: torch.Tensor, stream=None):
        """Install a prompt as request r: K/V [n, hkv, 128], or with a shared
        prefix the prompt's tokens after it (the prompt holds shared_len + n)."""
        hkv = self.K.shape[2]
        _spec(K, "K", BF16, (None, hkv, 128))
        _spec(V, "V", BF16, tuple(K.shape))
        _spec(W_k, "W_k", F32, W_SHAPE)
        _need_cuda(W_k)
        n = K.shape[0]
        self.K[r, :n].copy_(K)
        self.V[r, :n].copy_(V)
        check(lib().lsa_decode_load(ctypes.byref(self.d), r, self.shared_len + n, _ptr(W_k),
                                    ctypes.byref(self.cfg.c()), _ptr(self.ws), self.ws.numel(), _stream(stream)),
              "lsa_decode_load")

    def step(self, q, k, v, W_k, W_q, o=None, idx_out=None, stream=None):
        """One token per request: q [batch, hq, 128], k/v [batch, hkv, 128]."""
        b, hkv, hq = int(self.d.batch), int(self.d.hkv), int(self.d.hq)
        _spec(q, "q", BF16, (b, hq, 128))
        _spec(k, "k", BF16, (b, hkv, 128))
        _spec(v, "v", BF16, (b, hkv, 128))
        _spec(W_k, "W_k", F32, W_SHAPE)
        _spec(W_q, "W_q", F32, W_SHAPE)
        _spec(o, "o", BF16, (b, hq, 128))
        _spec(idx_out, "idx_out", I32, (b, hkv, self.cfg.row))
        _need_cuda(q, k, v, W_k, W_q, o, idx_out)
        if o is None:
            o = torch.empty_like(q)
        check(lib().lsa_decode_step(ctypes.byref(self.d), _ptr(q), _ptr(k), _ptr(v), _ptr(W_k), _ptr(W_q),
                                    ctypes.byref(self.cfg.c()), _ptr(o), _ptr(idx_out), _ptr(self.ws),
                                    self.ws.numel(), _stream(stream)), "lsa_decode_step")
        return o


# ------------------------------------------------ sequence-sharded layer

def shard_cand_cap(cfg: Config) -> int:
    """lsa_shard_cand_cap: records per (query, kv-head) row."""
    return int(lib().lsa_shard_cand_cap(ctypes.byref(cfg.c())))


def shard_build_buckets(K: torch.Tensor, W_k: torch.Tensor, cfg: Config, p0: int, cache: Cache, stream=None):
    """lsa_shard_build_buckets: the cache of a shard's keys K [n, hkv, 128]
    (global positions p0 ..)."""
    _spec(K, "K", BF16, (None, None, 128))
    _spec(W_k, "W_k", F32, W_SHAPE)
    _need_cuda(K, W_k)
    n, hkv, _ = K.shape
    check(lib().lsa_shard_build_buckets(_ptr(K), n, hkv, _ptr(W_k), ctypes.byref(cfg.c()), p0,
                                        ctypes.byref(cache.c), _stream(stream)), "lsa_shard_build_buckets")
    return cache


def shard_candidates(Q: torch.Tensor, t0: int, W_q: torch.Tensor, cache: Cache, p0: int, cfg: Config,
                     rec=None, rec_n=None, ws=None, stream=None):
    """lsa_shard_candidates: the shard's own fill as records.  Returns (rec
    int32 [nq, hkv, cap, 4] -- each record's 16 bytes: id, taken, fp64
    score --, rec_n int32 [nq, hkv])."""
    _spec(Q, "Q", BF16, (None, None, 128))
    _spec(W_q, "W_q", F32, W_SHAPE)
    nq, hq, _ = Q.shape
    cap = shard_cand_cap(cfg)
    _spec(rec, "rec", I32, (nq, cache.hkv, cap, 4))
    _spec(rec_n, "rec_n", I32, (nq, cache.hkv))
    _need_cuda(Q, W_q, rec, rec_n, ws)
    if rec is None:
        rec = torch.empty((nq, cache.hkv, cap, 4), dtype=I32, device=Q.device)
    if rec_n is None:
        rec_n = torch.empty((nq, cache.hkv), dtype=I32, device=Q.device)
    need = select_workspace_bytes(cfg, nq, hq, cache)
    if ws is None or ws.numel() < need:
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=Q.device)
    check(lib().lsa_shard_candidates(_ptr(Q), t0, nq, hq, _ptr(W_q), ctypes.byref(cache.c), p0,
                                     ctypes.byref(cfg.c()), _ptr(rec), _ptr(rec_n), _ptr(ws), ws.numel(),
                                     _stream(stream)), "lsa_shard_candidates")
    return rec, rec_n


def shard_merge(rec_all: torch.Tensor, rec_n_all: torch.Tensor, rank: int, t0: int, cache: Cache, p0: int,
                cfg: Config, idx=None, stream=None) -> torch.Tensor:
    """lsa_shard_merge: shard `rank`'s part of the index rows [nq, hkv, S+k+W]
    from every shard's records (rec_all [world, nq, hkv, cap, 4], rec_n_all
    [world, nq, hkv])."""
    _spec(rec_all, "rec_all", I32, (None, None, cache.hkv, shard_cand_cap(cfg), 4))
    world, nq = int(rec_all.shape[0]), int(rec_all.shape[1])
    _spec(rec_n_all, "rec_n_all", I32, (world, nq, cache.hkv))
    _spec(idx, "idx", I32, (nq, cache.hkv, cfg.row))
    _need_cuda(rec_all, rec_n_all, idx)
    if idx is None:
        idx = torch.empty((nq, cache.hkv, cfg.row), dtype=I32, device=rec_all.device)
    check(lib().lsa_shard_merge(_ptr(rec_all), _ptr(rec_n_all), world, rank, t0, nq, ctypes.byref(cache.c), p0,
                                ctypes.byref(cfg.c()), _ptr(idx), _stream(stream)), "lsa_shard_merge")
    return idx


def sparse_attn_partial(Q, K, V, idx, p0: int, O_part=None, lse=None, stream=None):
    """lsa_sparse_attn_partial: (O_part fp32 [nq, hq, 128], lse fp32 [nq, hq])
    over a shard's entries (global positions p0 .. p0 + K.shape[0] - 1)."""
    _spec(Q, "Q", BF16, (None, None, 128))
    _spec(K, "K", BF16, (None, None, 128))
    _spec(V, "V", BF16, tuple(K.shape))
    nq, hq, _ = Q.shape
    hkv = K.shape[1]
    _spec(idx, "idx", I32, (nq, hkv, None))
    _spec(O_part, "O_part", F32, (nq, hq, 128))
    _spec(lse, "lse", F32, (nq, hq))
    _need_cuda(Q, K, V, idx, O_part, lse)
    if O_part is None:
        O_part = torch.empty((nq, hq, 128), dtype=F32, device=Q.device)
    if lse is None:
        lse = torch.empty((nq, hq), dtype=F32, device=Q.device)
    check(lib().lsa_sparse_attn_partial(_ptr(Q), _ptr(K), _ptr(V), _ptr(idx), nq, hq, hkv, idx.shape[2], p0,
                                        K.shape[0], _ptr(O_part), _ptr(lse), _stream(stream)),
          "lsa_sparse_attn_partial")
    return O_part, lse


def lse_combine(O_parts, lse_parts, O=None, stream=None) -> torch.Tensor:
    """lsa_lse_combine: bf16 O [nq, hq, 128] from every shard's (O_r, L_r)."""
    _spec(O_parts, "O_parts", F32, (None, None, None, 128))
    world, nq, hq, _ = O_parts.shape
    _spec(lse_parts, "lse_parts", F32, (world, nq, hq))
    _spec(O, "O", BF16, (nq, hq, 128))
    _need_cuda(O_parts, lse_parts, O)
    if O is None:
        O = torch.empty((nq, hq, 128), dtype=BF16, device=O_parts.device)
    check(lib().lsa_lse_combine(_ptr(O_parts), _ptr(lse_parts), world, nq, hq, _ptr(O), _stream(stream)),
          "lsa_lse_combine")
    return O


class KernelTimer:
    """Context manager around lsa_timing_begin / lsa_timing_end; get(name)
    returns (total ms, launches) of one kernel recorded inside it."""

    def __enter__(self):
        lib().lsa_timing_begin()
        return self

    def __exit__(self, *exc):
        lib().lsa_timing_end()
        return False

    @staticmethod
    def get(name: str):
        ms, n = ctypes.c_double(0.0), ctypes.c_int64(0)
        check(lib().lsa_timing_get(name.encode(), ctypes.byref(ms), ctypes.byref(n)), "lsa_timing_get")
        return ms.value, n.value
