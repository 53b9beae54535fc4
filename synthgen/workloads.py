"""Named synthetic workloads: model shapes, seeds, tensor names and layer blobs.

Input-generation infrastructure shared by the tests and the benchmark.  Holds
no arithmetic of the method: it only decides which seeded stream fills which
tensor and where each tensor sits in a layer blob.  The blob layout rule is
written out here on its own (consecutive matrices wq, wk, wv, wo, wg, wu, wd
then the two fp32 norm vectors, each start rounded up to 256 bytes); a test
checks it against the library's ``ntx_layer_layout``.

Workloads (numbering of the configuration list they come from):
  1  Q8_0 GEMV 4096 x 4096
  2  Q4_0 GEMV sweep 4096x4096, 1024x4096, 14336x4096, 4096x14336
  3  one 8B-shaped Q8_0 decode layer, 1024 prior KV positions, token at 1024
  4  32-layer 8B-shaped Q8_0 model, 16-token prompt + 128 greedy steps
  5  80-layer 70B-shaped Q6_K model, 2048 prior KV positions, (a) resident,
     (b) layers 40-79 in pinned host memory; the same shapes as Q4_K_M
"""
from __future__ import annotations

import numpy as np

from . import (BLOCK_BYTES, BLOCK_ELEMS, Q4_0, Q4_K, Q6_K, Q8_0, SEED_BASE, dev_fill_f16, dev_fill_f32,
               dev_quant_rows, fill_f16, fill_f32, quant_rows)

MODEL_8B = dict(hidden=4096, n_heads=32, n_kv_heads=8, head_dim=128, ffn=14336, vocab=128256, n_layers=32,
                eps=1e-5, theta=500000.0)
MODEL_70B = dict(hidden=8192, n_heads=64, n_kv_heads=8, head_dim=128, ffn=28672, vocab=128256, n_layers=80,
                 eps=1e-5, theta=500000.0)

Q4_0_SWEEP = [(4096, 4096), (1024, 4096), (14336, 4096), (4096, 14336)]

W_SIGMA = 0.02     # linear weights ~ N(0, 0.02)
NORM_SIGMA = 0.02  # norm weights ~ 1 + N(0, 0.02)
EMB_SIGMA = 0.02   # embeddings ~ N(0, 0.02)

MATS = ("wq", "wk", "wv", "wo", "wg", "wu", "wd")

# Q4_K_M ("Q4_K super-blocks, mixed"): every matrix Q4_K except the down
# projection, which is Q6_K; the output head is Q6_K too.
Q4_K_M = (Q4_K, Q4_K, Q4_K, Q4_K, Q4_K, Q4_K, Q6_K)
Q4_K_M_HEAD = Q6_K


def mat_types(qtype) -> tuple:
    """Block type of each of wq..wd: one type for all, or a sequence of seven."""
    if isinstance(qtype, (list, tuple)):
        assert len(qtype) == 7
        return tuple(int(t) for t in qtype)
    return (int(qtype),) * 7


def seed(workload: int) -> int:
    return SEED_BASE + workload


def mat_shapes(d: dict) -> dict:
    H, F = d["hidden"], d["ffn"]
    Q, KV = d["n_heads"] * d["head_dim"], d["n_kv_heads"] * d["head_dim"]
    return {"wq": (Q, H), "wk": (KV, H), "wv": (KV, H), "wo": (H, Q), "wg": (F, H), "wu": (F, H), "wd": (H, F)}


def mat_bytes(qtype: int, M: int, K: int) -> int:
    return M * (K // BLOCK_ELEMS[qtype]) * BLOCK_BYTES[qtype]


def _up256(v: int) -> int:
    return (v + 255) // 256 * 256


def layer_layout(d: dict, qtype) -> tuple[int, dict]:
    """(blob bytes, {name: byte offset}) for wq..wd, attn_norm, ffn_norm;
    qtype is one block type or the seven matrices' types."""
    offs, o = {}, 0
    for (name, (M, K)), qt in zip(mat_shapes(d).items(), mat_types(qtype)):
        offs[name] = o
        o = _up256(o + mat_bytes(qt, M, K))
    for name in ("attn_norm", "ffn_norm"):
        offs[name] = o
        o = _up256(o + 4 * d["hidden"])
    return o, offs


def layer_weight_bytes(d: dict, qtype) -> int:
    return sum(mat_bytes(qt, M, K) for (M, K), qt in zip(mat_shapes(d).values(), mat_types(qtype)))


def bytes_per_token(d: dict, qtype, head_qtype: int, n_ctx: int, layers: int | None = None) -> int:
    """Algorithmic HBM bytes of one decode step: every weight byte once, the KV
    cache rows 0..n_ctx-1 of K and V (fp16) read once per computed layer, the
    new k, v row written, norms read; the head and the embedding row."""
    L = d["n_layers"] if layers is None else layers
    H, D, Hkv = d["hidden"], d["head_dim"], d["n_kv_heads"]
    per_layer = layer_weight_bytes(d, qtype) + 2 * Hkv * D * 2 * n_ctx + 2 * 4 * H
    head = mat_bytes(head_qtype, d["vocab"], H) + 4 * H
    return L * per_layer + head + 2 * H


def tensor_name(layer: int, what: str) -> str:
    return f"layer.{layer}.{what}"


# ------------------------------------------------------------ host (small sizes)
def host_layer(d: dict, qtype, sd: int, layer: int, nthreads=None) -> dict:
    """numpy tensors of one layer: wq..wd block matrices, attn_norm, ffn_norm
    (and "qtypes", the seven matrices' block types)."""
    out = {}
    for (name, (M, K)), qt in zip(mat_shapes(d).items(), mat_types(qtype)):
        out[name] = quant_rows(qt, sd, tensor_name(layer, name), M, K, sigma=W_SIGMA, nthreads=nthreads)
    out["qtypes"] = list(mat_types(qtype))
    for name in ("attn_norm", "ffn_norm"):
        out[name] = fill_f32(sd, tensor_name(layer, name), d["hidden"], mean=1.0, sigma=NORM_SIGMA)
    return out


def host_layer_blob(d: dict, qtype: int, sd: int, layer: int, nthreads=None):
    """(uint8 blob in the canonical layout, tensors dict)."""
    n, offs = layer_layout(d, qtype)
    t = host_layer(d, qtype, sd, layer, nthreads)
    blob = np.zeros(n, dtype=np.uint8)
    for name, o in offs.items():
        b = np.asarray(t[name]).view(np.uint8).ravel()
        blob[o:o + b.size] = b
    return blob, t


def tensors_from_blob(blob: np.ndarray, d: dict, qtype) -> dict:
    """Views of the tensors inside a canonical blob (for the oracle), with
    "qtypes", the seven matrices' block types."""
    _, offs = layer_layout(d, qtype)
    out = {"qtypes": list(mat_types(qtype))}
    for (name, (M, K)), qt in zip(mat_shapes(d).items(), mat_types(qtype)):
        out[name] = blob[offs[name]:offs[name] + mat_bytes(qt, M, K)].reshape(M, -1)
    for name in ("attn_norm", "ffn_norm"):
        out[name] = blob[offs[name]:offs[name] + 4 * d["hidden"]].view(np.float32)
    return out


def host_kv_prior(d: dict, sd: int, layer: int, max_ctx: int, n_prior: int):
    """fp16 bit patterns [Hkv][max_ctx][D] with rows < n_prior ~ N(0,1), rest 0."""
    Hkv, D = d["n_kv_heads"], d["head_dim"]
    k = np.zeros((Hkv, max_ctx, D), dtype=np.uint16)
    v = np.zeros_like(k)
    if n_prior:
        kp = fill_f16(sd, tensor_name(layer, "k_prior"), Hkv * max_ctx * D).reshape(Hkv, max_ctx, D)
        vp = fill_f16(sd, tensor_name(layer, "v_prior"), Hkv * max_ctx * D).reshape(Hkv, max_ctx, D)
        k[:, :n_prior] = kp[:, :n_prior]
        v[:, :n_prior] = vp[:, :n_prior]
    return k, v


# ------------------------------------------------------------ device (full sizes)
def dev_layer_blob(d: dict, qtype, sd: int, layer: int, base_ptr: int, stream=0) -> None:
    """Fill a canonical layer blob at device address base_ptr with the GPU twin."""
    _, offs = layer_layout(d, qtype)
    for (name, (M, K)), qt in zip(mat_shapes(d).items(), mat_types(qtype)):
        dev_quant_rows(qt, sd, tensor_name(layer, name), M, K, base_ptr + offs[name], sigma=W_SIGMA,
                       stream=stream)
    for name in ("attn_norm", "ffn_norm"):
        dev_fill_f32(sd, tensor_name(layer, name), d["hidden"], 1.0, NORM_SIGMA, base_ptr + offs[name], stream)


def dev_kv_prior(d: dict, sd: int, layer: int, max_ctx: int, k_ptr: int, v_ptr: int, stream=0) -> None:
    """Fill whole [Hkv][max_ctx][D] caches with the prior stream (rows at or
    beyond the prior length are overwritten by decoding before being read)."""
    n = d["n_kv_heads"] * max_ctx * d["head_dim"]
    dev_fill_f16(sd, tensor_name(layer, "k_prior"), n, 0.0, 1.0, k_ptr, stream)
    dev_fill_f16(sd, tensor_name(layer, "v_prior"), n, 0.0, 1.0, v_ptr, stream)
