"""Seeded synthetic inputs for the LSA path.

This module only draws inputs; it holds none of the method's arithmetic.  It
is the one piece the CUDA library's tests / benchmark and the CPU oracle both
use.  Recipe (a stand-in for the long-context prefill/decode workloads the
LSA pages measure on real models, whose weights and datasets are not used):

* centres: ``n_centres`` unit vectors (normalised N(0, I_d));
* keys:    k_{t,h} = 4 * mu_{c} + N(0, I_d), c uniform per (token, kv-head);
* queries: q_{t,h} = mu_{c'} + N(0, I_d), c' uniform per (token, q-head);
* values:  N(0, 1);
* W_k, W_q: independent random orthonormal d x d_latent matrices (QR of a
  Gaussian, signs fixed so diag(R) > 0), fp32;
* everything drawn in fp32 and rounded to bf16 (ties to even).

Streams are numpy PCG64 generators keyed by (seed, tensor tag), so any tensor
can be regenerated alone and in token chunks.
"""
from __future__ import annotations

import numpy as np

# The five workloads (shapes of the pages' single-layer prefill / decode
# measurements).  T = context tokens, hkv / hq = KV / query heads.
CONFIGS = {
    "prefill-4k": dict(T=4096, hkv=1, hq=4, d=128, dl=64, n_centres=32, k=512,
                       sinks=4, window=256, mode=0, agg=0, beam=2),
    "prefill-128k": dict(T=131072, hkv=8, hq=32, d=128, dl=64, n_centres=1024,
                         k=2048, sinks=4, window=1024, mode=0, agg=0, beam=2),
    "prefill-1m": dict(T=1 << 20, hkv=8, hq=32, d=128, dl=64, n_centres=8192,
                       k=2048, sinks=4, window=1024, mode=0, agg=0, beam=2),
    "decode-32x1m": dict(T=1 << 20, batch=32, hkv=8, hq=32, d=128, dl=64,
                         n_centres=8192, k=2048, sinks=4, window=1024, mode=0,
                         agg=0, beam=2),
    "decode-small": dict(T=4096, batch=3, hkv=2, hq=8, d=128, dl=64, n_centres=64, k=256,
                         sinks=4, window=600, mode=0, agg=0, beam=2),
    "decode-4x10m": dict(T=10_000_000, batch=4, hkv=8, hq=32, d=128, dl=64,
                         n_centres=65536, k=2048, sinks=4, window=1024, mode=0,
                         agg=0, beam=2, shared_prefix=True),
}

_TAGS = {"centres": 1, "kc": 2, "kn": 3, "qc": 4, "qn": 5, "v": 6, "wk": 7, "wq": 8}


def _rng(seed: int, tag: str, chunk: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, _TAGS[tag], chunk])))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def centres(seed: int, n: int, d: int) -> np.ndarray:
    c = _rng(seed, "centres").standard_normal((n, d), dtype=np.float32)
    c /= np.linalg.norm(c, axis=1, keepdims=True)
    return c


def orthonormal(seed: int, tag: str, d: int, dl: int) -> np.ndarray:
    g = _rng(seed, tag).standard_normal((d, dl))
    q, r = np.linalg.qr(g)
    q = q * np.sign(np.diag(r))[None, :]
    return np.ascontiguousarray(q, dtype=np.float32)


def projections(seed: int = 0, d: int = 128, dl: int = 64):
    """(W_k, W_q), fp32 [d, dl] row-major."""
    return orthonormal(seed, "wk", d, dl), orthonormal(seed, "wq", d, dl)


_CHUNK = 8192  # tokens per generator chunk (tensors are drawn chunk by chunk)


def _tokens(seed, kind, t0, t1, heads, d, mu, scale):
    """bf16 bits [t1 - t0, heads, d] of `scale * mu_c + N(0, I)` (kind k/q)
    or N(0, 1) (kind v), drawn chunk-wise so any token range is reproducible."""
    out = np.empty((t1 - t0, heads, d), np.uint16)
    c0 = t0 // _CHUNK
    c1 = (t1 + _CHUNK - 1) // _CHUNK
    for c in range(c0, c1):
        a, b = c * _CHUNK, (c + 1) * _CHUNK
        if kind == "v":
            x = _rng(seed, "v", c).standard_normal((_CHUNK, heads, d), dtype=np.float32)
        else:
            ci = _rng(seed, kind + "c", c).integers(0, mu.shape[0], size=(_CHUNK, heads))
            x = _rng(seed, kind + "n", c).standard_normal((_CHUNK, heads, d), dtype=np.float32)
            x += np.float32(scale) * mu[ci]
        lo, hi = max(a, t0), min(b, t1)
        out[lo - t0:hi - t0] = f32_to_bf16_bits(x[lo - a:hi - a])
    return out


def layer_inputs(name: str = "prefill-4k", seed: int = 0, T: int | None = None,
                 parts=("Q", "K", "V"), hkv: int | None = None) -> dict:
    """Q [T, hq, d], K/V [T, hkv, d] as bf16 bits, W_k/W_q fp32 [d, dl].
    `T` overrides the configuration's length (a prefix of the same stream);
    `hkv` draws that many kv-heads (and their hkv * hq / hkv query heads) of
    the same recipe instead (another stream than the full layer's)."""
    c = CONFIGS[name]
    if hkv is not None:
        c = dict(c, hkv=hkv, hq=hkv * (c["hq"] // c["hkv"]))
    T = c["T"] if T is None else T
    mu = centres(seed, c["n_centres"], c["d"])
    Wk, Wq = projections(seed, c["d"], c["dl"])
    out = dict(Wk=Wk, Wq=Wq, cfg=dict(c, T=T))
    if "K" in parts:
        out["K"] = _tokens(seed, "k", 0, T, c["hkv"], c["d"], mu, 4.0)
    if "V" in parts:
        out["V"] = _tokens(seed, "v", 0, T, c["hkv"], c["d"], mu, 0.0)
    if "Q" in parts:
        out["Q"] = _tokens(seed, "q", 0, T, c["hq"], c["d"], mu, 1.0)
    return out


def query_rows(name: str, tpos, seed: int = 0) -> np.ndarray:
    """The Q rows at positions `tpos` (same values as layer_inputs' Q)."""
    c = CONFIGS[name]
    mu = centres(seed, c["n_centres"], c["d"])
    tpos = np.asarray(tpos, np.int64)
    out = np.empty((tpos.size, c["hq"], c["d"]), np.uint16)
    for i, t in enumerate(tpos):
        out[i] = _tokens(seed, "q", int(t), int(t) + 1, c["hq"], c["d"], mu, 1.0)[0]
    return out


# ----------------------------------------------------- device-drawn inputs
#
# The 1M-token and decode workloads are too large to draw on the host; they
# use the same recipe with torch's seeded device generator (another random
# stream than the host tensors above).  Both the benchmark and the full-size
# tests draw through these two functions, so they see identical bytes.

def device_tokens(n, heads, d, mu, scale, gen, device, out=None, chunk=65536):
    """bf16 [n, heads, d] of scale * mu_c + N(0, I) (scale 0: N(0, 1)), c
    uniform per (token, head), drawn by the seeded device generator `gen`."""
    import torch
    if out is None:
        out = torch.empty((n, heads, d), dtype=torch.bfloat16, device=device)
    for t0 in range(0, n, chunk):
        t1 = min(n, t0 + chunk)
        x = torch.randn((t1 - t0, heads, d), generator=gen, device=device, dtype=torch.float32)
        if scale != 0.0:
            ci = torch.randint(0, mu.shape[0], (t1 - t0, heads), generator=gen, device=device)
            x += scale * mu[ci]
        out[t0:t1] = x.to(torch.bfloat16)
    return out


def device_layer(c: dict, seed: int, device):
    """(Q [T, hq, d], K/V [T, hkv, d]) bf16 on `device` for configuration `c`."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    mu = torch.from_numpy(centres(seed, c["n_centres"], c["d"])).to(device)
    K = device_tokens(c["T"], c["hkv"], c["d"], mu, 4.0, gen, device)
    V = device_tokens(c["T"], c["hkv"], c["d"], mu, 0.0, gen, device)
    Q = device_tokens(c["T"], c["hq"], c["d"], mu, 1.0, gen, device)
    return Q, K, V


def device_decode(c: dict, seed: int, device, n0: int, steps: int, K_out, V_out):
    """Decode inputs: prompts of n0 tokens per request written into
    K_out[r, :n0] / V_out[r, :n0], then (q, k, v) for `steps` steps,
    [steps, batch, heads, d] each."""
    import torch
    B, hkv, hq, d = c["batch"], c["hkv"], c["hq"], c["d"]
    gen = torch.Generator(device=device)
    gen.manual_seed(1000 * seed)
    mu = torch.from_numpy(centres(seed, c["n_centres"], d)).to(device)
    for r in range(B):
        device_tokens(n0, hkv, d, mu, 4.0, gen, device, out=K_out[r, :n0])
        device_tokens(n0, hkv, d, mu, 0.0, gen, device, out=V_out[r, :n0])
    q = device_tokens(steps * B, hq, d, mu, 1.0, gen, device).view(steps, B, hq, d)
    k = device_tokens(steps * B, hkv, d, mu, 4.0, gen, device).view(steps, B, hkv, d)
    v = device_tokens(steps * B, hkv, d, mu, 0.0, gen, device).view(steps, B, hkv, d)
    return q, k, v


def device_shared_prefix(c: dict, seed: int, device, shared_len: int):
    """K/V [shared_len, hkv, d] of a prefix every decode request shares."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(1000 * seed + 1)
    mu = torch.from_numpy(centres(seed, c["n_centres"], c["d"])).to(device)
    Ks = device_tokens(shared_len, c["hkv"], c["d"], mu, 4.0, gen, device)
    Vs = device_tokens(shared_len, c["hkv"], c["d"], mu, 0.0, gen, device)
    return Ks, Vs


def device_decode_tails(c: dict, seed: int, device, shared_len: int, n0: int, steps: int, K_tail, V_tail):
    """Each request's prompt tokens shared_len .. n0 - 1 written into
    K_tail[r] / V_tail[r] (rows from 0), then (q, k, v) for `steps` steps,
    [steps, batch, heads, d] each."""
    import torch
    B, hkv, hq, d = c["batch"], c["hkv"], c["hq"], c["d"]
    gen = torch.Generator(device=device)
    gen.manual_seed(1000 * seed + 2)
    mu = torch.from_numpy(centres(seed, c["n_centres"], d)).to(device)
    for r in range(B):
        device_tokens(n0 - shared_len, hkv, d, mu, 4.0, gen, device, out=K_tail[r, :n0 - shared_len])
        device_tokens(n0 - shared_len, hkv, d, mu, 0.0, gen, device, out=V_tail[r, :n0 - shared_len])
    q = device_tokens(steps * B, hq, d, mu, 1.0, gen, device).view(steps, B, hq, d)
    k = device_tokens(steps * B, hkv, d, mu, 4.0, gen, device).view(steps, B, hkv, d)
    v = device_tokens(steps * B, hkv, d, mu, 0.0, gen, device).view(steps, B, hkv, d)
    return q, k, v


def pca_keys(seed: int, T: int, hkv: int, d: int = 128, decay: float = 0.97) -> np.ndarray:
    """bf16 bits [T, hkv, d] of keys with a known, well-separated spectrum:
    k = R (s * g) + m, with R a random orthogonal d x d matrix, s_i =
    4 * decay^i, g ~ N(0, I) and a fixed offset m (the principal directions
    are R's columns in order)."""
    rng = _rng(seed, "kn", 7777)
    R = orthonormal(seed, "wk", d, d)
    s = (4.0 * decay ** np.arange(d)).astype(np.float32)
    g = rng.standard_normal((T * hkv, d), dtype=np.float32)
    m = rng.standard_normal(d, dtype=np.float32)
    x = (g * s[None, :]) @ R.T + m[None, :]
    return f32_to_bf16_bits(x.astype(np.float32)).reshape(T, hkv, d)
