"""ctypes view of liblsa.so (the C ABI declared in include/lsa.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Loading fails loudly when the shared library has not been built;
there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(HERE, "liblsa.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "lsa.h")

LSA_OK, LSA_EINVAL, LSA_EUNSUPPORTED, LSA_ECUDA, LSA_ENOSPACE, LSA_EDEVICE = range(6)
STATUS_NAMES = {0: "LSA_OK", 1: "LSA_EINVAL", 2: "LSA_EUNSUPPORTED", 3: "LSA_ECUDA",
                4: "LSA_ENOSPACE", 5: "LSA_EDEVICE"}
MAX_LEVELS = 48

i32, i64, vp, sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t


class lsa_cfg(ctypes.Structure):
    _fields_ = [(n, i32) for n in ("d_head", "d_latent", "pool", "block", "bucket_mean",
                                   "bucket_max", "k", "sinks", "window", "beam", "mode", "agg")]


class lsa_cache(ctypes.Structure):
    _fields_ = [("hkv", i32), ("n_tokens", i64), ("cap_units", i64), ("cap_buckets", i64),
                ("U", vp), ("bucket_of_unit", vp), ("members", vp), ("offsets", vp),
                ("cnt_lr", vp), ("minlr", vp), ("maxpos", vp), ("sum", vp), ("cent", vp),
                ("units", vp), ("cent8", vp)]


class lsa_tree(ctypes.Structure):
    _fields_ = [("levels", i32), ("level_n", i64 * MAX_LEVELS), ("level_off", i64 * MAX_LEVELS),
                ("n_nodes", i64), ("sum", vp), ("minlr", vp), ("cent", vp)]


MAX_BATCH = 128


class lsa_decode(ctypes.Structure):
    _fields_ = [("batch", i32), ("hkv", i32), ("hq", i32), ("cap", i64), ("K", vp), ("V", vp),
                ("U_blk", vp), ("cache", lsa_cache), ("tree", lsa_tree), ("len", i64 * MAX_BATCH),
                ("K_shared", vp), ("V_shared", vp), ("shared_len", i64)]


class LSAError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


_lib = None


def lib():
    """The loaded library (raises if liblsa.so is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(SO):
            raise RuntimeError(
                f"{SO} is not built; run `python -m clustered_key_indexing_b200.build` "
                "(the LSA path has no CPU fallback)")
        L = ctypes.CDLL(SO)
        P = ctypes.POINTER
        L.lsa_last_error.restype = ctypes.c_char_p
        L.lsa_version.restype = ctypes.c_char_p
        L.lsa_launch_count.restype = i64
        L.lsa_fallback_rows.restype = i64
        L.lsa_cfg_default.argtypes = [P(lsa_cfg)]
        L.lsa_cfg_check.argtypes = [P(lsa_cfg)]
        L.lsa_cache_units.argtypes = [P(lsa_cfg), i64]
        L.lsa_cache_units.restype = i64
        L.lsa_cache_buckets.argtypes = [P(lsa_cfg), i64]
        L.lsa_cache_buckets.restype = i64
        L.lsa_tree_layout.argtypes = [i64, P(lsa_tree)]
        L.lsa_build_buckets.argtypes = [vp, i64, i32, vp, P(lsa_cfg), P(lsa_cache), vp]
        L.lsa_build_tree.argtypes = [P(lsa_cache), P(lsa_cfg), P(lsa_tree), vp]
        L.lsa_query_latent.argtypes = [vp, i64, i32, i32, vp, P(lsa_cfg), vp, vp]
        L.lsa_select_workspace_bytes.argtypes = [P(lsa_cfg), i64, i32, P(lsa_cache)]
        L.lsa_select_workspace_bytes.restype = sz
        L.lsa_select.argtypes = [vp, i64, i64, i32, vp, P(lsa_cache), P(lsa_tree), P(lsa_cfg),
                                 vp, vp, vp, sz, vp]
        L.lsa_select_noalloc.argtypes = [vp, i64, i64, i32, vp, P(lsa_cache), P(lsa_tree),
                                         P(lsa_cfg), vp, vp]
        L.lsa_select_noalloc_scratch_bytes.restype = sz
        L.lsa_sparse_attn.argtypes = [vp, vp, vp, vp, i64, i32, i32, i32, i64, vp, vp]
        L.lsa_select_attn_workspace_bytes.argtypes = [i64, i32]
        L.lsa_select_attn_workspace_bytes.restype = sz
        L.lsa_select_attn.argtypes = [vp, vp, vp, vp, i64, i64, i32, i32, i64, P(lsa_cfg), vp, vp, sz, vp]
        L.lsa_timing_get.argtypes = [ctypes.c_char_p, P(ctypes.c_double), P(i64)]
        L.lsa_prefill_chunk.argtypes = [P(lsa_cfg), i64, i32, i32, i64]
        L.lsa_prefill_chunk.restype = i64
        L.lsa_decode_workspace_bytes.argtypes = [P(lsa_cfg), P(lsa_decode)]
        L.lsa_decode_workspace_bytes.restype = sz
        L.lsa_decode_load.argtypes = [P(lsa_decode), i32, i64, vp, P(lsa_cfg), vp, sz, vp]
        L.lsa_decode_step.argtypes = [P(lsa_decode), vp, vp, vp, vp, vp, P(lsa_cfg), vp, vp, vp, sz, vp]
        L.lsa_prefill_workspace_bytes.argtypes = [P(lsa_cfg), i64, i32, i32, i64]
        L.lsa_prefill_workspace_bytes.restype = sz
        L.lsa_prefill.argtypes = [vp, vp, vp, i64, i32, i32, vp, vp, P(lsa_cfg), P(lsa_cache),
                                  P(lsa_tree), vp, i64, vp, sz, vp]
        L.lsa_prefill_host.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i64, i32, i32, vp, vp, P(lsa_cfg),
                                       P(lsa_cache), P(lsa_tree), i64, vp, sz, vp, vp, vp]
        L.lsa_fit_pca_workspace_bytes.argtypes = [i64, i32]
        L.lsa_fit_pca_workspace_bytes.restype = sz
        L.lsa_fit_pca.argtypes = [vp, i64, i32, i32, vp, vp, vp, sz, vp]
        L.lsa_l2_read_sink_bytes.argtypes = [i32]
        L.lsa_l2_read_sink_bytes.restype = sz
        L.lsa_l2_read_bytes.argtypes = [sz, i32]
        L.lsa_l2_read_bytes.restype = i64
        L.lsa_l2_read.argtypes = [vp, sz, i32, i32, vp, vp]
        L.lsa_shard_cand_cap.argtypes = [P(lsa_cfg)]
        L.lsa_shard_cand_cap.restype = i32
        L.lsa_shard_build_buckets.argtypes = [vp, i64, i32, vp, P(lsa_cfg), i64, P(lsa_cache), vp]
        L.lsa_shard_candidates.argtypes = [vp, i64, i64, i32, vp, P(lsa_cache), i64, P(lsa_cfg), vp, vp, vp, sz, vp]
        L.lsa_shard_merge.argtypes = [vp, vp, i32, i32, i64, i64, P(lsa_cache), i64, P(lsa_cfg), vp, vp]
        L.lsa_sparse_attn_partial.argtypes = [vp, vp, vp, vp, i64, i32, i32, i32, i64, i64, vp, vp, vp]
        L.lsa_lse_combine.argtypes = [vp, vp, i32, i64, i32, vp, vp]
        L.lsa_attn_backward.argtypes = [vp, vp, vp, vp, vp, vp, i64, i32, i32, i32, i64, vp, vp, vp, vp]
        for name in exported_names():
            if getattr(L, name).restype is ctypes.c_int:
                getattr(L, name).restype = i32
        _lib = L
    return _lib


def exported_names() -> list[str]:
    """Function names declared in include/lsa.h."""
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lsa_[a-z_0-9]+)\s*\(", src)))


def check(status: int, what: str = ""):
    if status != LSA_OK:
        msg = lib().lsa_last_error().decode(errors="replace")
        raise LSAError(status, f"{what}: {msg}" if what else msg)
