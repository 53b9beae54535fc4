"""Python binding of libntx (batch-1 decode over GGUF block-quantized weights, sm_100a).

Argument marshalling only: every function below forwards to the extern "C"
entry point of the same name in ``libntx.so`` (declared in ``include/ntx.h``).
Pointer arguments accept an int address or anything with ``data_ptr()`` (a
torch tensor); stream arguments accept an int handle, ``None`` (legacy default
stream) or a ``torch.cuda.Stream``.  A non-zero status raises ``NtxError``
carrying ``ntx_last_error()``.  There is no fallback: if the shared library is
missing, loading raises.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# NTX_LIB selects another build of the library (the bounds-checked one, for tests)
LIB_PATH = os.environ.get("NTX_LIB") or os.path.join(HERE, "libntx.so")

NTX_OK = 0
NTX_ERR_INVALID_ARG = -1
NTX_ERR_SHAPE = -2
NTX_ERR_QTYPE = -3
NTX_ERR_ALIGN = -4
NTX_ERR_CUDA = -5
NTX_ERR_TIMEOUT = -6
NTX_ERR_NOMEM = -7

NTX_F32, NTX_F16, NTX_Q4_0, NTX_Q8_0, NTX_Q4_K, NTX_Q5_K, NTX_Q6_K = 0, 1, 2, 8, 12, 13, 14
NTX_MIXED = -1
NTX_CALIBRATE_SKIP, NTX_USE_SKIP, NTX_NO_GRAPH, NTX_NO_PERSIST = 1, 2, 4, 8

BLOCK_ELEMS = {NTX_F32: 1, NTX_F16: 1, NTX_Q4_0: 32, NTX_Q8_0: 32, NTX_Q4_K: 256, NTX_Q5_K: 256, NTX_Q6_K: 256}
BLOCK_BYTES = {NTX_F32: 4, NTX_F16: 2, NTX_Q4_0: 18, NTX_Q8_0: 34, NTX_Q4_K: 144, NTX_Q5_K: 176, NTX_Q6_K: 210}

# Symbols exported by libntx (all declared in include/ntx.h).
EXPORTS = (
    "ntx_last_error", "ntx_version", "ntx_device_status", "ntx_sm_count", "ntx_set_gemv_ctas_per_sm", "ntx_set_gemv_pdl",
    "ntx_dequant", "ntx_gemv_q", "ntx_rmsnorm", "ntx_rope", "ntx_attn_workspace_bytes", "ntx_attn_decode",
    "ntx_swiglu", "ntx_layer_layout", "ntx_layer_workspace_bytes", "ntx_decode_layer", "ntx_engine_workspace_bytes",
    "ntx_engine_create", "ntx_decode_step", "ntx_engine_skip_mask", "ntx_engine_destroy", "ntx_engine_set_probe",
    "ntx_engine_launches_per_step", "ntx_attn_decode_static", "ntx_engine_set_phase_probe",
    "ntx_persistent_plan", "ntx_layer_layout_mixed", "ntx_engine_device_bytes", "ntx_auto_tier_map",
    "ntx_memory_budget", "ntx_set_host_wait_limit", "ntx_engine_set_fault", "ntx_decode_spec",
    "ntx_set_persist_two_types", "ntx_check_enabled", "ntx_check_report", "ntx_hbm_read_probe",
)


class NtxError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"libntx error {code}: {msg}")
        self.code = code


class ntx_model_config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("n_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("ffn", ctypes.c_int32), ("vocab", ctypes.c_int32),
                ("n_layers", ctypes.c_int32), ("eps", ctypes.c_float), ("theta", ctypes.c_float),
                ("max_ctx", ctypes.c_int32), ("skip_threshold", ctypes.c_float)]


class ntx_layer_weights(ctypes.Structure):
    _fields_ = [("qtype", ctypes.c_int32), ("base", ctypes.c_void_p)] + [
        (n, ctypes.c_uint64) for n in ("off_wq", "off_wk", "off_wv", "off_wo", "off_wg", "off_wu", "off_wd",
                                       "off_attn_norm", "off_ffn_norm")] + [("mat_qtype", ctypes.c_int32 * 7)]


_lib = None


def lib():
    """The loaded libntx.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libntx.so not found at {LIB_PATH}; build it with "
                               "`python -m quantized_weight_gemv_dequant_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, sz, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
        P = ctypes.POINTER
        sig = {
            "ntx_last_error": ([], ctypes.c_char_p),
            "ntx_version": ([], i32),
            "ntx_device_status": ([P(ctypes.c_int)], i32),
            "ntx_check_enabled": ([], i32),
            "ntx_check_report": ([P(ctypes.c_int), P(ctypes.c_longlong)], i32),
            "ntx_sm_count": ([], i32),
            "ntx_hbm_read_probe": ([vp, ctypes.c_uint64, vp, vp], i32),
            "ntx_set_gemv_ctas_per_sm": ([i32], i32),
            "ntx_set_gemv_pdl": ([i32], i32),
            "ntx_dequant": ([i32, vp, vp, i64, vp], i32),
            "ntx_gemv_q": ([i32, vp, i64, i64, vp, vp, vp, vp], i32),
            "ntx_rmsnorm": ([vp, vp, vp, i64, f32, vp], i32),
            "ntx_rope": ([vp, vp, i32, i32, i32, i32, f32, vp], i32),
            "ntx_attn_workspace_bytes": ([i32, i32, i32, i32], sz),
            "ntx_attn_decode": ([vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, sz, vp], i32),
            "ntx_swiglu": ([vp, vp, vp, i64, vp], i32),
            "ntx_layer_layout": ([P(ntx_model_config), i32, P(ntx_layer_weights)], ctypes.c_uint64),
            "ntx_layer_layout_mixed": ([P(ntx_model_config), P(ctypes.c_int32), P(ntx_layer_weights)],
                                       ctypes.c_uint64),
            "ntx_layer_workspace_bytes": ([P(ntx_model_config)], sz),
            "ntx_decode_layer": ([P(ntx_model_config), P(ntx_layer_weights), vp, vp, vp, i32, vp, vp, sz, vp], i32),
            "ntx_engine_workspace_bytes": ([P(ntx_model_config)], sz),
            "ntx_engine_create": ([P(ntx_model_config), P(ntx_layer_weights), vp, vp, vp, sz, vp, vp, vp, i32, vp,
                                   vp, vp, sz, vp, vp, P(vp)], i32),
            "ntx_decode_step": ([vp, ctypes.c_int32, i32, vp, vp, i32, vp], i32),
            "ntx_engine_skip_mask": ([vp, vp], i32),
            "ntx_decode_spec": ([vp, ctypes.c_int32, i32, i32, P(ctypes.c_int32), P(i32), i32], i32),
            "ntx_engine_destroy": ([vp], i32),
            "ntx_set_host_wait_limit": ([ctypes.c_uint64], i32),
            "ntx_set_persist_two_types": ([i32], i32),
            "ntx_engine_set_fault": ([vp, i32, ctypes.c_uint64], i32),
            "ntx_engine_set_probe": ([vp, vp, vp, i32], i32),
            "ntx_engine_launches_per_step": ([vp], i32),
            "ntx_attn_decode_static": ([vp, vp, vp, vp, i32, i32, i32, i32, i32, vp], i32),
            "ntx_engine_set_phase_probe": ([vp, vp, sz], i32),
            "ntx_persistent_plan": ([P(ntx_model_config), i32, P(i32), P(i32), P(sz), P(i32)], i32),
            "ntx_engine_device_bytes": ([P(ntx_model_config), i32], ctypes.c_uint64),
            "ntx_auto_tier_map": ([P(ntx_model_config), ctypes.c_uint64, i32, ctypes.c_uint64, ctypes.c_uint64,
                                   ctypes.c_uint64, ctypes.c_uint64, P(ctypes.c_int8), P(i32)], i32),
            "ntx_memory_budget": ([P(ctypes.c_uint64), P(ctypes.c_uint64), P(ctypes.c_uint64), ctypes.c_char_p],
                                  i32),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def _p(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if isinstance(x, ctypes.c_void_p):
        return x.value
    raise TypeError(f"cannot take a pointer from {type(x).__name__}")


def _s(stream):
    if stream is None:
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc):
    if rc != NTX_OK:
        raise NtxError(rc, lib().ntx_last_error().decode(errors="replace"))
    return rc


# ---------------------------------------------------------------- per-op calls
def ntx_last_error() -> str:
    return lib().ntx_last_error().decode(errors="replace")


def ntx_version() -> int:
    return lib().ntx_version()


def ntx_device_status() -> int:
    code = ctypes.c_int(0)
    _check(lib().ntx_device_status(ctypes.byref(code)))
    return code.value


def ntx_check_enabled() -> int:
    return lib().ntx_check_enabled()


def ntx_check_report() -> tuple:
    """(site, index) of the first failed bounds check of the debug build; (0, 0) if none."""
    site, index = ctypes.c_int(0), ctypes.c_longlong(0)
    _check(lib().ntx_check_report(ctypes.byref(site), ctypes.byref(index)))
    return site.value, index.value


def ntx_sm_count() -> int:
    return lib().ntx_sm_count()


def ntx_hbm_read_probe(buf, nbytes, sum_out, stream=None):
    """Read buf (device, nbytes) once; *sum_out (device uint32) = sum of its 32-bit words mod 2^32."""
    _check(lib().ntx_hbm_read_probe(_p(buf), nbytes, _p(sum_out), _s(stream)))


def ntx_set_gemv_ctas_per_sm(cps: int) -> None:
    _check(lib().ntx_set_gemv_ctas_per_sm(cps))


def ntx_set_gemv_pdl(on: int) -> None:
    _check(lib().ntx_set_gemv_pdl(on))


def ntx_dequant(qtype, blocks, out, n, stream=None):
    _check(lib().ntx_dequant(qtype, _p(blocks), _p(out), n, _s(stream)))


def ntx_gemv_q(qtype, W, M, K, x, y, residual=None, stream=None):
    _check(lib().ntx_gemv_q(qtype, _p(W), M, K, _p(x), _p(y), _p(residual), _s(stream)))


def ntx_rmsnorm(x, w, y, n, eps, stream=None):
    _check(lib().ntx_rmsnorm(_p(x), _p(w), _p(y), n, eps, _s(stream)))


def ntx_rope(q, k, n_q_heads, n_kv_heads, head_dim, pos, theta, stream=None):
    _check(lib().ntx_rope(_p(q), _p(k), n_q_heads, n_kv_heads, head_dim, pos, theta, _s(stream)))


def ntx_attn_workspace_bytes(n_q_heads, n_kv_heads, head_dim, max_ctx) -> int:
    return lib().ntx_attn_workspace_bytes(n_q_heads, n_kv_heads, head_dim, max_ctx)


def ntx_attn_decode(q, k_cache, v_cache, out, n_q_heads, n_kv_heads, head_dim, n_ctx, max_ctx, workspace, ws_bytes,
                    stream=None):
    _check(lib().ntx_attn_decode(_p(q), _p(k_cache), _p(v_cache), _p(out), n_q_heads, n_kv_heads, head_dim, n_ctx,
                                 max_ctx, _p(workspace), ws_bytes, _s(stream)))


def ntx_attn_decode_static(q, k_cache, v_cache, out, n_q_heads, n_kv_heads, head_dim, n_ctx, max_ctx, stream=None):
    """ntx_attn_decode without a workspace (partials in libntx's static device array)."""
    _check(lib().ntx_attn_decode_static(_p(q), _p(k_cache), _p(v_cache), _p(out), n_q_heads, n_kv_heads, head_dim,
                                        n_ctx, max_ctx, _s(stream)))


def ntx_swiglu(gate, up, out, n, stream=None):
    _check(lib().ntx_swiglu(_p(gate), _p(up), _p(out), n, _s(stream)))


# ---------------------------------------------------------------- layer / model
def make_config(hidden, n_heads, n_kv_heads, head_dim, ffn, vocab, n_layers, eps, theta, max_ctx,
                skip_threshold=0.98) -> ntx_model_config:
    return ntx_model_config(hidden, n_heads, n_kv_heads, head_dim, ffn, vocab, n_layers, eps, theta, max_ctx,
                            skip_threshold)


def ntx_layer_layout(cfg: ntx_model_config, qtype: int):
    """Returns (blob_bytes, ntx_layer_weights with base NULL)."""
    w = ntx_layer_weights()
    n = lib().ntx_layer_layout(ctypes.byref(cfg), qtype, ctypes.byref(w))
    if n == 0:
        raise NtxError(NTX_ERR_INVALID_ARG, "ntx_layer_layout: bad config or type")
    return int(n), w


def ntx_layer_layout_mixed(cfg: ntx_model_config, qtypes):
    """qtypes: the seven block types of wq, wk, wv, wo, wg, wu, wd.  Returns
    (blob_bytes, ntx_layer_weights with base NULL and qtype NTX_MIXED)."""
    w = ntx_layer_weights()
    t = (ctypes.c_int32 * 7)(*qtypes)
    n = lib().ntx_layer_layout_mixed(ctypes.byref(cfg), t, ctypes.byref(w))
    if n == 0:
        raise NtxError(NTX_ERR_INVALID_ARG, "ntx_layer_layout_mixed: bad config or types")
    return int(n), w


def ntx_layer_workspace_bytes(cfg: ntx_model_config) -> int:
    return lib().ntx_layer_workspace_bytes(ctypes.byref(cfg))


def ntx_decode_layer(cfg, weights: ntx_layer_weights, k_cache, v_cache, hidden, pos, cos_out, workspace, ws_bytes,
                     stream=None):
    _check(lib().ntx_decode_layer(ctypes.byref(cfg), ctypes.byref(weights), _p(k_cache), _p(v_cache), _p(hidden),
                                  pos, _p(cos_out), _p(workspace), ws_bytes, _s(stream)))


def ntx_engine_workspace_bytes(cfg: ntx_model_config) -> int:
    return lib().ntx_engine_workspace_bytes(ctypes.byref(cfg))


def ntx_engine_create(cfg, layers, tier_map, slot0, slot1, slot_bytes, embed, final_norm, head, head_qtype,
                      k_caches, v_caches, workspace, ws_bytes, compute_stream, copy_stream=None):
    """layers: sequence of ntx_layer_weights; tier_map: sequence of 0/1 or None;
    k_caches / v_caches: sequences of device pointers.  Returns the engine handle."""
    n = len(layers)
    arr = (ntx_layer_weights * max(n, 1))(*layers)
    tm = (ctypes.c_int8 * max(n, 1))(*(tier_map if tier_map is not None else [0] * n))
    kc = (ctypes.c_void_p * max(n, 1))(*[_p(k) for k in k_caches])
    vc = (ctypes.c_void_p * max(n, 1))(*[_p(v) for v in v_caches])
    h = ctypes.c_void_p()
    _check(lib().ntx_engine_create(ctypes.byref(cfg), arr, tm, _p(slot0), _p(slot1), slot_bytes, _p(embed),
                                   _p(final_norm), _p(head), head_qtype, kc, vc, _p(workspace), ws_bytes,
                                   _s(compute_stream), _s(copy_stream), ctypes.byref(h)))
    return h


def ntx_decode_step(engine, token, pos, logits=None, next_token=None, flags=0, cos_out=None):
    _check(lib().ntx_decode_step(engine, token, pos, _p(logits), _p(next_token), flags, _p(cos_out)))


def ntx_decode_spec(engine, token, pos, draft_k, flags=0):
    """Self-speculative step; returns the emitted greedy tokens (a list of 1 .. draft_k + 1)."""
    out = (ctypes.c_int32 * (draft_k + 1))()
    n = ctypes.c_int(0)
    _check(lib().ntx_decode_spec(engine, token, pos, draft_k, out, ctypes.byref(n), flags))
    return [int(t) for t in out[:n.value]]


def ntx_engine_skip_mask(engine, n_layers):
    mask = (ctypes.c_uint8 * max(n_layers, 1))()
    rc = lib().ntx_engine_skip_mask(engine, mask)
    if rc < 0:
        _check(rc)
    return [int(m) for m in mask[:n_layers]]


def ntx_engine_destroy(engine):
    _check(lib().ntx_engine_destroy(engine))


def ntx_set_persist_two_types(on: int) -> None:
    _check(lib().ntx_set_persist_two_types(on))


def ntx_set_host_wait_limit(ms: int) -> None:
    _check(lib().ntx_set_host_wait_limit(ms))


def ntx_engine_set_fault(engine, stall_cta: int, wait_ns: int = 0) -> None:
    _check(lib().ntx_engine_set_fault(engine, stall_cta, wait_ns))


def ntx_engine_set_probe(engine, begin_events, end_events):
    """begin_events / end_events: sequences of raw cudaEvent_t handles (ints)."""
    n = len(begin_events)
    b = (ctypes.c_void_p * max(n, 1))(*begin_events)
    e = (ctypes.c_void_p * max(n, 1))(*end_events)
    _check(lib().ntx_engine_set_probe(engine, b, e, n))


def ntx_engine_set_phase_probe(engine, dev_ts, n_words: int) -> int:
    """dev_ts: device buffer of n_words uint64 (a torch tensor or pointer) or
    None.  Returns the persistent kernel's grid size (0 if not used)."""
    rc = lib().ntx_engine_set_phase_probe(engine, _p(dev_ts) if dev_ts is not None else None, n_words)
    if rc < 0:
        _check(rc)
    return rc


def ntx_persistent_plan(cfg: ntx_model_config, qtype: int) -> dict:
    """The persistent decode kernel's plan: slot_bytes, n_slots, smem_bytes and
    rows per slot for the qkv, o, gu, down and head phases."""
    zb, ns = ctypes.c_int(), ctypes.c_int()
    smem = ctypes.c_size_t()
    rows = (ctypes.c_int * 5)()
    _check(lib().ntx_persistent_plan(ctypes.byref(cfg), qtype, ctypes.byref(zb), ctypes.byref(ns), ctypes.byref(smem),
                                     rows))
    return {"slot_bytes": zb.value, "n_slots": ns.value, "smem_bytes": smem.value,
            "rows": dict(zip(["qkv", "o", "gu", "down", "head"], list(rows)))}


def ntx_engine_launches_per_step(engine) -> int:
    rc = lib().ntx_engine_launches_per_step(engine)
    if rc < 0:
        _check(rc)
    return rc


# ---------------------------------------------------------------- tier sizing
def ntx_engine_device_bytes(cfg: ntx_model_config, head_qtype: int) -> int:
    return int(lib().ntx_engine_device_bytes(ctypes.byref(cfg), head_qtype))


def ntx_auto_tier_map(cfg: ntx_model_config, layer_bytes: int, head_qtype: int, device_free: int,
                      device_reserve: int, host_available: int, host_reserve: int):
    """Returns (tier_map list of 0/1, number of resident layers)."""
    n = cfg.n_layers
    tm = (ctypes.c_int8 * max(n, 1))()
    nres = ctypes.c_int(0)
    _check(lib().ntx_auto_tier_map(ctypes.byref(cfg), layer_bytes, head_qtype, device_free, device_reserve,
                                   host_available, host_reserve, tm, ctypes.byref(nres)))
    return [int(t) for t in tm[:n]], nres.value


def ntx_memory_budget(device=True, meminfo_path=None):
    """Returns (device_free, device_total, host_available) in bytes; the device
    figures are None when device is False."""
    f, t, h = ctypes.c_uint64(0), ctypes.c_uint64(0), ctypes.c_uint64(0)
    _check(lib().ntx_memory_budget(ctypes.byref(f) if device else None, ctypes.byref(t) if device else None,
                                   ctypes.byref(h), meminfo_path.encode() if meminfo_path else None))
    return (f.value if device else None), (t.value if device else None), h.value
