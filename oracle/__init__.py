"""CPU oracle for the batch-1 quantized-weight decode path (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It wraps ``libntx_oracle.so`` (plain C,
fp64, see ``ntx_oracle.c`` for the definitions and the passages they follow)
and composes the per-token model step from the oracle's own embed / layer /
head functions.  It shares no code with the CUDA path or the input generator.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(HERE, "libntx_oracle.so")

F32, F16, Q4_0, Q8_0, Q4_K, Q5_K, Q6_K = 0, 1, 2, 8, 12, 13, 14
MATS = ("wq", "wk", "wv", "wo", "wg", "wu", "wd")


def build(force: bool = False) -> None:
    src = os.path.join(HERE, "ntx_oracle.c")
    if force or not os.path.exists(SO) or os.path.getmtime(SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-pthread",
                               "-o", SO, src, "-lm"])


class Config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("n_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("ffn", ctypes.c_int32), ("vocab", ctypes.c_int32),
                ("n_layers", ctypes.c_int32), ("eps", ctypes.c_double), ("theta", ctypes.c_double),
                ("max_ctx", ctypes.c_int32)]


class LayerWeights(ctypes.Structure):
    _fields_ = [("qt", ctypes.c_int32 * 7)] + [(n, ctypes.c_void_p) for n in
                                                ("wq", "wk", "wv", "wo", "wg", "wu", "wd", "attn_norm", "ffn_norm")]


def mat_types(qtype) -> list:
    """Block type of each of wq..wd: one type for all, or a sequence of seven
    (mixed models such as Q4_K_M), or a dict keyed by matrix name."""
    if isinstance(qtype, dict):
        return [int(qtype[k]) for k in MATS]
    if isinstance(qtype, (list, tuple)):
        assert len(qtype) == 7
        return [int(t) for t in qtype]
    return [int(qtype)] * 7


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(SO):
            build()
        L = ctypes.CDLL(SO)
        vp, i64, dbl, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_double, ctypes.c_int
        L.orc_half.argtypes = [ctypes.c_uint16]
        L.orc_half.restype = dbl
        L.orc_to_half.argtypes = [dbl]
        L.orc_to_half.restype = ctypes.c_uint16
        L.orc_dequant.argtypes = [i32, vp, i64, vp]
        L.orc_dequant.restype = i32
        L.orc_gemv.argtypes = [i32, vp, i64, i64, vp, vp, vp, i32]
        L.orc_gemv.restype = i32
        L.orc_rmsnorm.argtypes = [vp, vp, i64, dbl, vp]
        L.orc_rope.argtypes = [vp, i32, i32, i32, dbl]
        L.orc_attention.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, vp, vp]
        L.orc_attention.restype = i32
        L.orc_swiglu.argtypes = [vp, vp, i64, vp]
        L.orc_cosine.argtypes = [vp, vp, i64]
        L.orc_cosine.restype = dbl
        L.orc_argmax.argtypes = [vp, i64]
        L.orc_argmax.restype = i64
        L.orc_layer.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(LayerWeights), vp, vp, vp, i32, vp, vp, i32]
        L.orc_layer.restype = i32
        L.orc_embed.argtypes = [vp, i64, i64, vp]
        L.orc_head.argtypes = [ctypes.POINTER(Config), i32, vp, vp, vp, vp, i32]
        L.orc_head.restype = i32
        _lib = L
    return _lib


def _nt(n):
    return n if n else (os.cpu_count() or 1)


def _d(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def half_to_double(h: int) -> float:
    return lib().orc_half(h)


def double_to_half(v: float) -> int:
    return int(lib().orc_to_half(v))


def dequant(qtype: int, blocks: np.ndarray, n: int) -> np.ndarray:
    blocks = np.ascontiguousarray(blocks, dtype=np.uint8)
    out = np.empty(n, dtype=np.float64)
    if lib().orc_dequant(qtype, blocks.ctypes.data, n, out.ctypes.data) != 0:
        raise ValueError("orc_dequant: bad qtype or n")
    return out


def gemv(qtype: int, W: np.ndarray, M: int, K: int, x, nthreads: int | None = None):
    """Returns (y, b): y = W_deq x and b = sum_j |w_ij x_j|, both fp64."""
    W = np.ascontiguousarray(W, dtype=np.uint8)
    x = _d(x)
    y = np.empty(M, dtype=np.float64)
    b = np.empty(M, dtype=np.float64)
    if lib().orc_gemv(qtype, W.ctypes.data, M, K, x.ctypes.data, y.ctypes.data, b.ctypes.data, _nt(nthreads)) != 0:
        raise ValueError("orc_gemv: bad arguments")
    return y, b


def rmsnorm(x, w, eps):
    x, w = _d(x), _d(w)
    y = np.empty_like(x)
    lib().orc_rmsnorm(x.ctypes.data, w.ctypes.data, x.size, eps, y.ctypes.data)
    return y


def rope(v, n_heads, head_dim, pos, theta):
    v = _d(v).copy()
    lib().orc_rope(v.ctypes.data, n_heads, head_dim, pos, theta)
    return v


def attention(q, k_cache, v_cache, n_q_heads, n_kv_heads, head_dim, n_ctx, max_ctx):
    """Returns (out, bound) for fp16-bit-pattern caches [n_kv_heads][max_ctx][head_dim]."""
    q = _d(q)
    kc = np.ascontiguousarray(k_cache, dtype=np.uint16)
    vc = np.ascontiguousarray(v_cache, dtype=np.uint16)
    out = np.empty(n_q_heads * head_dim, dtype=np.float64)
    bound = np.empty_like(out)
    rc = lib().orc_attention(q.ctypes.data, kc.ctypes.data, vc.ctypes.data, n_q_heads, n_kv_heads, head_dim, n_ctx,
                             max_ctx, out.ctypes.data, bound.ctypes.data)
    if rc != 0:
        raise ValueError("orc_attention: bad arguments")
    return out, bound


def swiglu(g, u):
    g, u = _d(g), _d(u)
    out = np.empty_like(g)
    lib().orc_swiglu(g.ctypes.data, u.ctypes.data, g.size, out.ctypes.data)
    return out


def cosine(a, b):
    a, b = _d(a), _d(b)
    return lib().orc_cosine(a.ctypes.data, b.ctypes.data, a.size)


def argmax(v):
    v = _d(v)
    return int(lib().orc_argmax(v.ctypes.data, v.size))


def make_config(hidden, n_heads, n_kv_heads, head_dim, ffn, vocab, n_layers, eps, theta, max_ctx) -> Config:
    return Config(hidden, n_heads, n_kv_heads, head_dim, ffn, vocab, n_layers, eps, theta, max_ctx)


def layer(cfg: Config, qtype: int, mats: dict, attn_norm, ffn_norm, k_cache, v_cache, h_in, pos,
          nthreads: int | None = None):
    """One decode layer.  ``mats`` maps wq..wd to uint8 block arrays (and may
    carry "qtypes", the seven matrices' block types, which then replace
    ``qtype``); the fp16 caches (uint16 numpy arrays) are updated in place.
    Returns (h_out, cos)."""
    keep = {k: np.ascontiguousarray(mats[k], dtype=np.uint8) for k in MATS}
    an = np.ascontiguousarray(attn_norm, dtype=np.float32)
    fn = np.ascontiguousarray(ffn_norm, dtype=np.float32)
    L = LayerWeights((ctypes.c_int32 * 7)(*mat_types(mats.get("qtypes", qtype))),
                     *[keep[k].ctypes.data for k in MATS], an.ctypes.data, fn.ctypes.data)
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    assert k_cache.dtype == np.uint16 and v_cache.dtype == np.uint16
    h = _d(h_in)
    out = np.empty_like(h)
    c = ctypes.c_double()
    rc = lib().orc_layer(ctypes.byref(cfg), ctypes.byref(L), k_cache.ctypes.data, v_cache.ctypes.data, h.ctypes.data,
                         pos, out.ctypes.data, ctypes.byref(c), _nt(nthreads))
    if rc != 0:
        raise ValueError("orc_layer: bad arguments")
    return out, c.value


def embed(table_f16: np.ndarray, hidden: int, token: int):
    t = np.ascontiguousarray(table_f16, dtype=np.uint16)
    out = np.empty(hidden, dtype=np.float64)
    lib().orc_embed(t.ctypes.data, hidden, token, out.ctypes.data)
    return out


def head(cfg: Config, head_qtype: int, W_head: np.ndarray, final_norm, h, nthreads: int | None = None):
    W = np.ascontiguousarray(W_head, dtype=np.uint8)
    fn = np.ascontiguousarray(final_norm, dtype=np.float32)
    h = _d(h)
    logits = np.empty(cfg.vocab, dtype=np.float64)
    rc = lib().orc_head(ctypes.byref(cfg), head_qtype, W.ctypes.data, fn.ctypes.data, h.ctypes.data,
                        logits.ctypes.data, _nt(nthreads))
    if rc != 0:
        raise ValueError("orc_head: bad arguments")
    return logits


def model_step(cfg: Config, qtype: int, layers, head_qtype: int, W_head, final_norm, embed_table, k_caches, v_caches,
               token: int, pos: int, skip=None, nthreads: int | None = None):
    """One decode step of the whole model: embed -> layers -> final norm -> head.

    ``layers`` is a sequence of dicts with keys wq..wd, attn_norm, ffn_norm (or
    a callable l -> dict, so layers can be fetched one at a time).  Layers with
    ``skip[l]`` true are not computed and do not append to their KV cache.
    Returns (logits, cos per layer (nan where skipped))."""
    h = embed(embed_table, cfg.hidden, token)
    cos = np.full(cfg.n_layers, np.nan)
    for l in range(cfg.n_layers):
        if skip is not None and skip[l]:
            continue
        Lw = layers(l) if callable(layers) else layers[l]
        h, cos[l] = layer(cfg, qtype, Lw, Lw["attn_norm"], Lw["ffn_norm"], k_caches[l], v_caches[l], h, pos, nthreads)
    logits = head(cfg, head_qtype, W_head, final_norm, h, nthreads)
    return logits, cos
