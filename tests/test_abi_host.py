"""Host-side checks of the C ABI: the library loads, exports every function
include/ntx.h declares, lays out layer blobs as documented, and rejects bad
arguments with the documented codes before any device work.  CPU only: no
call here reaches a kernel launch."""
import ctypes
import os
import re

import pytest

import quantized_weight_gemv_dequant_b200 as ntx
from synthgen import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "ntx.h"), encoding="utf-8").read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ntx_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module", autouse=True)
def built():
    from quantized_weight_gemv_dequant_b200 import build
    build.build()


def test_library_exports_every_declared_function():
    names = _declared_functions()
    assert len(names) >= 20
    L = ctypes.CDLL(ntx.LIB_PATH)
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(ntx.EXPORTS)


def test_version():
    assert ntx.ntx_version() >= 100


def _cfg(d, max_ctx=2048, layers=None):
    return ntx.make_config(d["hidden"], d["n_heads"], d["n_kv_heads"], d["head_dim"], d["ffn"], d["vocab"],
                           d["n_layers"] if layers is None else layers, d["eps"], d["theta"], max_ctx)


@pytest.mark.parametrize("d,qt,weights", [(wl.MODEL_8B, ntx.NTX_Q8_0, 231735296),
                                           (wl.MODEL_70B, ntx.NTX_Q6_K, 701890560)])
def test_layer_layout_matches_closed_forms(d, qt, weights):
    n, w = ntx.ntx_layer_layout(_cfg(d), qt)
    n2, offs = wl.layer_layout(d, qt)
    assert n == n2
    for k in wl.MATS + ("attn_norm", "ffn_norm"):
        assert getattr(w, "off_" + k) == offs[k]
        assert offs[k] % 256 == 0
    assert wl.layer_weight_bytes(d, qt) == weights
    assert weights < n < weights + 9 * 256 + 8 * d["hidden"]


def test_bytes_per_token_closed_form_8b():
    # 32 layers x 231,735,296 + Q8_0 head 128256 x 4096 (558,170,112) = 7,973,699,584 weight bytes
    d = wl.MODEL_8B
    assert 32 * wl.layer_weight_bytes(d, ntx.NTX_Q8_0) + wl.mat_bytes(ntx.NTX_Q8_0, 128256, 4096) == 7973699584
    b1 = wl.bytes_per_token(d, ntx.NTX_Q8_0, ntx.NTX_Q8_0, 1)
    b2 = wl.bytes_per_token(d, ntx.NTX_Q8_0, ntx.NTX_Q8_0, 2)
    assert b2 - b1 == 32 * 2 * 8 * 128 * 2  # 131,072 bytes per extra context position


def _rc(fn, *args):
    try:
        fn(*args)
    except ntx.NtxError as e:
        return e.code
    return 0


FAKE = 0x7F0000000000  # never dereferenced: every call below fails its argument check


def test_gemv_argument_errors():
    assert _rc(ntx.ntx_gemv_q, 99, FAKE, 16, 256, FAKE + 0x100000, FAKE + 0x200000) == ntx.NTX_ERR_QTYPE
    assert _rc(ntx.ntx_gemv_q, ntx.NTX_Q8_0, FAKE, 16, 33, FAKE + 0x100000, FAKE + 0x200000) == ntx.NTX_ERR_SHAPE
    assert _rc(ntx.ntx_gemv_q, ntx.NTX_Q6_K, FAKE, 16, 128, FAKE + 0x100000, FAKE + 0x200000) == ntx.NTX_ERR_SHAPE
    assert _rc(ntx.ntx_gemv_q, ntx.NTX_Q8_0, FAKE, 0, 256, FAKE + 0x100000, FAKE + 0x200000) == ntx.NTX_ERR_SHAPE
    assert _rc(ntx.ntx_gemv_q, ntx.NTX_Q8_0, None, 16, 256, FAKE + 0x100000, FAKE + 0x200000) == ntx.NTX_ERR_INVALID_ARG
    assert _rc(ntx.ntx_gemv_q, ntx.NTX_Q8_0, FAKE + 2, 16, 256, FAKE + 0x100000, FAKE + 0x200000) == ntx.NTX_ERR_ALIGN
    assert _rc(ntx.ntx_gemv_q, ntx.NTX_Q8_0, FAKE, 16, 256, FAKE + 0x100004, FAKE + 0x200000) == ntx.NTX_ERR_ALIGN
    # y overlapping x
    assert _rc(ntx.ntx_gemv_q, ntx.NTX_Q8_0, FAKE, 16, 256, FAKE + 0x100000, FAKE + 0x100010) == \
        ntx.NTX_ERR_INVALID_ARG
    assert "overlaps" in ntx.ntx_last_error()


def test_tuning_switch_argument_errors():
    L = ntx.lib()
    assert L.ntx_set_gemv_pdl(2) == ntx.NTX_ERR_INVALID_ARG
    assert L.ntx_set_gemv_pdl(-1) == ntx.NTX_ERR_INVALID_ARG
    assert L.ntx_set_gemv_pdl(0) == ntx.NTX_OK
    assert L.ntx_set_gemv_ctas_per_sm(0) == ntx.NTX_ERR_INVALID_ARG
    assert L.ntx_set_gemv_ctas_per_sm(5) == ntx.NTX_ERR_INVALID_ARG
    assert L.ntx_set_gemv_ctas_per_sm(1) == ntx.NTX_OK
    assert L.ntx_set_persist_two_types(2) == ntx.NTX_ERR_INVALID_ARG
    assert L.ntx_set_persist_two_types(-1) == ntx.NTX_ERR_INVALID_ARG
    assert L.ntx_set_persist_two_types(0) == ntx.NTX_OK
    # the release build reports no bounds checks; the report call checks its arguments first
    assert L.ntx_check_enabled() == 0
    assert L.ntx_check_report(None, None) == ntx.NTX_ERR_INVALID_ARG


def test_small_op_argument_errors():
    assert _rc(ntx.ntx_dequant, ntx.NTX_Q4_0, FAKE, FAKE + 0x1000, 33) == ntx.NTX_ERR_SHAPE
    assert _rc(ntx.ntx_dequant, 3, FAKE, FAKE + 0x1000, 32) == ntx.NTX_ERR_QTYPE
    assert _rc(ntx.ntx_rmsnorm, FAKE, FAKE, FAKE, 0, 1e-5) == ntx.NTX_ERR_SHAPE
    assert _rc(ntx.ntx_rmsnorm, None, FAKE, FAKE, 16, 1e-5) == ntx.NTX_ERR_INVALID_ARG
    assert _rc(ntx.ntx_rope, FAKE, FAKE, 4, 2, 127, 0, 5e5) == ntx.NTX_ERR_SHAPE
    assert _rc(ntx.ntx_rope, FAKE, None, 4, 2, 128, 0, 5e5) == ntx.NTX_ERR_INVALID_ARG
    assert _rc(ntx.ntx_rope, FAKE, FAKE, 4, 2, 128, -1, 5e5) == ntx.NTX_ERR_INVALID_ARG
    assert _rc(ntx.ntx_swiglu, FAKE, FAKE, FAKE, -1) == ntx.NTX_ERR_SHAPE
    # the HBM read probe checks pointers and alignment before any CUDA call
    assert _rc(ntx.ntx_hbm_read_probe, FAKE, 1 << 20, None) == ntx.NTX_ERR_INVALID_ARG
    assert _rc(ntx.ntx_hbm_read_probe, None, 1 << 20, FAKE) == ntx.NTX_ERR_INVALID_ARG
    assert _rc(ntx.ntx_hbm_read_probe, FAKE + 4, 1 << 20, FAKE + 0x1000) == ntx.NTX_ERR_ALIGN
    assert _rc(ntx.ntx_hbm_read_probe, FAKE, (1 << 20) + 8, FAKE + 0x1000) == ntx.NTX_ERR_ALIGN
    # attention
    args = [FAKE, FAKE + 0x10000, FAKE + 0x20000, FAKE + 0x30000]
    assert _rc(ntx.ntx_attn_decode, *args, 32, 8, 64, 10, 100, FAKE + 0x40000, 1 << 30) == ntx.NTX_ERR_SHAPE
    assert _rc(ntx.ntx_attn_decode, *args, 32, 6, 128, 10, 100, FAKE + 0x40000, 1 << 30) == ntx.NTX_ERR_SHAPE
    assert _rc(ntx.ntx_attn_decode, *args, 48, 3, 128, 10, 100, FAKE + 0x40000, 1 << 30) == ntx.NTX_ERR_SHAPE
    assert _rc(ntx.ntx_attn_decode, *args, 32, 8, 128, 0, 100, FAKE + 0x40000, 1 << 30) == ntx.NTX_ERR_SHAPE
    assert _rc(ntx.ntx_attn_decode, *args, 32, 8, 128, 101, 100, FAKE + 0x40000, 1 << 30) == ntx.NTX_ERR_SHAPE
    assert _rc(ntx.ntx_attn_decode, *args, 32, 8, 128, 10, 100, FAKE + 0x40000, 16) == ntx.NTX_ERR_NOMEM


def test_layer_and_engine_argument_errors():
    d = wl.MODEL_8B
    cfg = _cfg(d, layers=1)
    n, w = ntx.ntx_layer_layout(cfg, ntx.NTX_Q8_0)
    w.base = FAKE
    ws = ntx.ntx_layer_workspace_bytes(cfg)
    assert ws > 0
    assert _rc(ntx.ntx_decode_layer, cfg, w, FAKE, FAKE, FAKE, 2048, None, FAKE, ws) == ntx.NTX_ERR_SHAPE
    assert _rc(ntx.ntx_decode_layer, cfg, w, FAKE, FAKE, FAKE, 0, None, FAKE, ws - 256) == ntx.NTX_ERR_NOMEM
    assert _rc(ntx.ntx_decode_layer, cfg, w, FAKE, FAKE, FAKE, 0, None, FAKE + 16, ws) == ntx.NTX_ERR_ALIGN
    bad = ntx.make_config(4096, 32, 8, 64, 14336, 128256, 1, 1e-5, 5e5, 2048)
    assert _rc(ntx.ntx_decode_layer, bad, w, FAKE, FAKE, FAKE, 0, None, FAKE, ws) == ntx.NTX_ERR_SHAPE
    w.off_wk += 8
    assert _rc(ntx.ntx_decode_layer, cfg, w, FAKE, FAKE, FAKE, 0, None, FAKE, ws) == ntx.NTX_ERR_ALIGN
    w2 = ntx.ntx_layer_weights()
    w2.qtype = 5
    assert _rc(ntx.ntx_decode_layer, cfg, w2, FAKE, FAKE, FAKE, 0, None, FAKE, ws) == ntx.NTX_ERR_QTYPE
    # engine
    _, lw = ntx.ntx_layer_layout(cfg, ntx.NTX_Q8_0)
    lw.base = FAKE
    ews = ntx.ntx_engine_workspace_bytes(cfg)
    common = dict(slot0=None, slot1=None, slot_bytes=0, embed=FAKE, final_norm=FAKE, head=FAKE,
                  head_qtype=ntx.NTX_Q8_0, k_caches=[FAKE], v_caches=[FAKE], workspace=FAKE, ws_bytes=ews)
    assert _rc(ntx.ntx_engine_create, cfg, [lw], [2], *common.values(), 1) == ntx.NTX_ERR_INVALID_ARG
    assert _rc(ntx.ntx_engine_create, cfg, [lw], [0], *common.values(), None) == ntx.NTX_ERR_INVALID_ARG
    # a host-tier layer without slots / copy stream
    assert _rc(ntx.ntx_engine_create, cfg, [lw], [1], *common.values(), 1, None) == ntx.NTX_ERR_INVALID_ARG
    assert _rc(ntx.ntx_decode_step, None, 0, 0) == ntx.NTX_ERR_INVALID_ARG


def test_static_attention_refuses_oversize_before_any_cuda_call():
    """The no-workspace attention checks its size against the 2 MiB static
    array before touching the device.  Run only where no GPU is visible, so the
    made-up addresses can never reach a kernel; the GPU suite repeats this with
    real buffers."""
    try:
        import torch
        if torch.cuda.is_available():
            pytest.skip("covered with real device buffers by the GPU suite")
    except ImportError:
        pass
    # 64 query heads over 8 KV heads at 20000 positions: 79 splits x 64 x 130 floats > 524,288
    args = [FAKE, FAKE + 0x10000000, FAKE + 0x20000000, FAKE + 0x30000000]
    assert _rc(ntx.ntx_attn_decode_static, *args, 64, 8, 128, 20000, 20000) == ntx.NTX_ERR_NOMEM
    assert "2 MiB" in ntx.ntx_last_error()
    # shape and pointer checks come first
    assert _rc(ntx.ntx_attn_decode_static, *args, 64, 8, 64, 100, 100) == ntx.NTX_ERR_SHAPE
    assert _rc(ntx.ntx_attn_decode_static, None, *args[1:], 64, 8, 128, 100, 100) == ntx.NTX_ERR_INVALID_ARG
    assert _rc(ntx.ntx_attn_decode_static, FAKE + 4, *args[1:], 64, 8, 128, 100, 100) == ntx.NTX_ERR_ALIGN


def test_mixed_layer_layout_and_type_rules():
    d = dict(hidden=2048, n_heads=16, n_kv_heads=4, head_dim=128, ffn=4096, vocab=1000, n_layers=1, eps=1e-5,
             theta=500000.0)
    cfg = _cfg(d, max_ctx=16, layers=1)
    q4km = wl.Q4_K_M
    n, w = ntx.ntx_layer_layout_mixed(cfg, q4km)
    n2, offs = wl.layer_layout(d, q4km)
    assert n == n2 and w.qtype == ntx.NTX_MIXED and list(w.mat_qtype) == list(q4km)
    for k in wl.MATS + ("attn_norm", "ffn_norm"):
        assert getattr(w, "off_" + k) == offs[k]
    # one type: the same offsets as the uniform call
    n3, w3 = ntx.ntx_layer_layout(cfg, ntx.NTX_Q4_K)
    n4, w4 = ntx.ntx_layer_layout_mixed(cfg, [ntx.NTX_Q4_K] * 7)
    assert n3 == n4 and w3.qtype == ntx.NTX_Q4_K and w4.qtype == ntx.NTX_MIXED
    # wq, wk, wv (and wg, wu) are one fused GEMV each: one type per group
    ws = ntx.ntx_layer_workspace_bytes(cfg)
    for bad in ((12, 12, 14, 12, 12, 12, 14), (12, 12, 12, 12, 12, 13, 14)):
        _, wb = ntx.ntx_layer_layout_mixed(cfg, bad)
        wb.base = FAKE
        assert _rc(ntx.ntx_decode_layer, cfg, wb, FAKE, FAKE, FAKE, 0, None, FAKE, ws) == ntx.NTX_ERR_QTYPE
    # Q6_K needs input lengths that are multiples of 2048
    small = ntx.make_config(1024, 8, 2, 128, 3072, 1000, 1, 1e-5, 5e5, 16)
    _, wq6 = ntx.ntx_layer_layout(small, ntx.NTX_Q6_K)
    wq6.base = FAKE
    assert _rc(ntx.ntx_decode_layer, small, wq6, FAKE, FAKE, FAKE, 0, None, FAKE,
               ntx.ntx_layer_workspace_bytes(small)) == ntx.NTX_ERR_SHAPE
    with pytest.raises(ntx.NtxError):
        ntx.ntx_layer_layout_mixed(cfg, [99] * 7)


def test_new_formats_argument_checks():
    for qt in (ntx.NTX_Q4_K, ntx.NTX_Q5_K):
        assert _rc(ntx.ntx_gemv_q, qt, FAKE, 16, 128, FAKE + 0x100000, FAKE + 0x200000) == ntx.NTX_ERR_SHAPE
        assert _rc(ntx.ntx_dequant, qt, FAKE, FAKE + 0x1000, 255) == ntx.NTX_ERR_SHAPE
    assert _rc(ntx.ntx_gemv_q, ntx.NTX_MIXED, FAKE, 16, 256, FAKE + 0x100000, FAKE + 0x200000) == ntx.NTX_ERR_QTYPE
    assert _rc(ntx.ntx_dequant, 3, FAKE, FAKE + 0x1000, 256) == ntx.NTX_ERR_QTYPE


def test_injected_pinned_alloc_failure_enqueues_nothing(monkeypatch):
    """NTX_FAULT=pinned_alloc: ntx_engine_create fails with NTX_ERR_NOMEM at its
    first allocation, before any stream work (the made-up addresses are never
    touched: the call returns before enqueuing)."""
    d = wl.MODEL_8B
    cfg = _cfg(d, layers=1)
    _, lw = ntx.ntx_layer_layout(cfg, ntx.NTX_Q8_0)
    lw.base = FAKE
    ews = ntx.ntx_engine_workspace_bytes(cfg)
    monkeypatch.setenv("NTX_FAULT", "host_wait,pinned_alloc")
    rc = _rc(ntx.ntx_engine_create, cfg, [lw], [0], None, None, 0, FAKE, FAKE, FAKE, ntx.NTX_Q8_0, [FAKE], [FAKE],
             FAKE, ews, 1, None)
    assert rc == ntx.NTX_ERR_NOMEM and "injected" in ntx.ntx_last_error()


def test_host_wait_limit_argument():
    assert ntx.lib().ntx_set_host_wait_limit(0) == ntx.NTX_ERR_INVALID_ARG
    assert ntx.lib().ntx_set_host_wait_limit(60000) == ntx.NTX_OK
    assert ntx.lib().ntx_engine_set_fault(None, -1, 0) == ntx.NTX_ERR_INVALID_ARG
