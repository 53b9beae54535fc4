"""Automatic tier sizing on the host (no GPU): the resident / pinned-host split
follows the device and host budgets, the two streaming slots are charged only
when some layer is streamed, and a model needing a third tier is refused.
The budgets are made-up numbers and a made-up meminfo file, as the rule is a
pure function of them."""
import os

import pytest

import quantized_weight_gemv_dequant_b200 as ntx
from synthgen import workloads as wl

GiB = 1 << 30


@pytest.fixture(scope="module", autouse=True)
def built():
    from quantized_weight_gemv_dequant_b200 import build
    build.build()


def _cfg(d, max_ctx):
    return ntx.make_config(d["hidden"], d["n_heads"], d["n_kv_heads"], d["head_dim"], d["ffn"], d["vocab"],
                           d["n_layers"], d["eps"], d["theta"], max_ctx)


def test_engine_device_bytes_closed_form():
    d = wl.MODEL_70B
    cfg = _cfg(d, 2080)
    V, H, L = d["vocab"], d["hidden"], d["n_layers"]
    kv = 2 * L * 8 * 2080 * 128 * 2
    want = V * H * 2 + 4 * H + wl.mat_bytes(ntx.NTX_Q6_K, V, H) + kv + ntx.ntx_engine_workspace_bytes(cfg)
    assert ntx.ntx_engine_device_bytes(cfg, ntx.NTX_Q6_K) == want


@pytest.mark.parametrize("qt,head", [(ntx.NTX_Q6_K, ntx.NTX_Q6_K), (wl.Q4_K_M, wl.Q4_K_M_HEAD)])
def test_split_follows_device_budget(qt, head):
    d = wl.MODEL_70B
    cfg = _cfg(d, 2080)
    LB = (ntx.ntx_layer_layout_mixed(cfg, qt) if isinstance(qt, tuple) else ntx.ntx_layer_layout(cfg, qt))[0]
    fixed = ntx.ntx_engine_device_bytes(cfg, head)
    reserve = 2 * GiB
    for n_want in (0, 1, 26, 36, 40, 77):  # 78, 79 cannot happen: 80 blobs need less room than 78 + 2 slots
        free = reserve + fixed + (n_want + 2) * LB + LB // 2  # room for n_want layers and the two slots
        tm, n = ntx.ntx_auto_tier_map(cfg, LB, head, free, reserve, 1 << 50, 0)
        assert n == n_want
        assert tm == [0] * n_want + [1] * (80 - n_want)
    # everything fits: no slots are charged
    tm, n = ntx.ntx_auto_tier_map(cfg, LB, head, reserve + fixed + 80 * LB, reserve, 0, 0)
    assert n == 80 and tm == [0] * 80
    # one byte less: the two slots now cost room, so 77 stay resident
    tm, n = ntx.ntx_auto_tier_map(cfg, LB, head, reserve + fixed + 80 * LB - 1, reserve, 1 << 50, 0)
    assert n == 77


def test_refusals():
    d = wl.MODEL_70B
    cfg = _cfg(d, 2080)
    LB = ntx.ntx_layer_layout(cfg, ntx.NTX_Q6_K)[0]
    fixed = ntx.ntx_engine_device_bytes(cfg, ntx.NTX_Q6_K)
    with pytest.raises(ntx.NtxError) as e:  # non-layer buffers alone do not fit
        ntx.ntx_auto_tier_map(cfg, LB, ntx.NTX_Q6_K, fixed - 1, 0, 1 << 50, 0)
    assert e.value.code == ntx.NTX_ERR_NOMEM
    with pytest.raises(ntx.NtxError) as e:  # no room for two slots
        ntx.ntx_auto_tier_map(cfg, LB, ntx.NTX_Q6_K, fixed + LB, 0, 1 << 50, 0)
    assert e.value.code == ntx.NTX_ERR_NOMEM
    with pytest.raises(ntx.NtxError) as e:  # 40 streamed layers do not fit 30 layers' worth of host memory
        ntx.ntx_auto_tier_map(cfg, LB, ntx.NTX_Q6_K, fixed + 42 * LB, 0, 31 * LB, LB)
    assert e.value.code == ntx.NTX_ERR_NOMEM and "third tier" in ntx.ntx_last_error()
    tm, n = ntx.ntx_auto_tier_map(cfg, LB, ntx.NTX_Q6_K, fixed + 42 * LB, 0, 41 * LB, LB)
    assert n == 40
    with pytest.raises(ntx.NtxError):
        ntx.ntx_auto_tier_map(cfg, 0, ntx.NTX_Q6_K, 1 << 50, 0, 1 << 50, 0)


def test_memory_budget_reads_meminfo(tmp_path):
    p = tmp_path / "meminfo"
    p.write_text("MemTotal:       1000000 kB\nMemFree:         200000 kB\nMemAvailable:    123456 kB\n")
    _, _, host = ntx.ntx_memory_budget(device=False, meminfo_path=str(p))
    assert host == 123456 * 1024
    (tmp_path / "bad").write_text("MemTotal: 1 kB\n")
    with pytest.raises(ntx.NtxError):
        ntx.ntx_memory_budget(device=False, meminfo_path=str(tmp_path / "bad"))
    if os.path.exists("/proc/meminfo"):
        _, _, h = ntx.ntx_memory_budget(device=False)
        assert h > 0
