"""Host-side checks of the persistent decode kernel's plan (ntx_persistent_plan;
no GPU): the ring fits the shared memory a CTA may use, every phase's slot
holds whole rows (an even count where the epilogue pairs rows), every phase can
keep all its row-group warps busy, and for Q6_K -- whose phases are paced by the
consumer warps' dot products -- a slot's rows split evenly over each phase's
row groups."""
import pytest

import quantized_weight_gemv_dequant_b200 as ntx
from synthgen import workloads as wl

SMEM_MAX = 227 * 1024
CONSUMERS = 14
SLICE = 2048
BLOCK = {ntx.NTX_Q8_0: (32, 34), ntx.NTX_Q4_0: (32, 18), ntx.NTX_Q6_K: (256, 210), ntx.NTX_Q4_K: (256, 144),
         ntx.NTX_Q5_K: (256, 176)}
PHASES = ["qkv", "o", "gu", "down", "head"]
PAIRED = {"qkv", "gu"}


@pytest.fixture(scope="module", autouse=True)
def built():
    from quantized_weight_gemv_dequant_b200 import build
    build.build()


def _cfg(d, max_ctx):
    return ntx.make_config(d["hidden"], d["n_heads"], d["n_kv_heads"], d["head_dim"], d["ffn"], d["vocab"],
                           d["n_layers"], d["eps"], d["theta"], max_ctx)


def _phase_K(d):
    H, Q, F = d["hidden"], d["n_heads"] * d["head_dim"], d["ffn"]
    return {"qkv": H, "o": Q, "gu": H, "down": F, "head": H}


TINY_Q6 = dict(hidden=2048, n_heads=16, n_kv_heads=2, head_dim=128, ffn=4096, vocab=1000, n_layers=3, eps=1e-5,
               theta=500000.0)
CASES = [
    ("llama8b", wl.MODEL_8B, ntx.NTX_Q8_0, 144),
    ("llama8b-q4_0", wl.MODEL_8B, ntx.NTX_Q4_0, 144),
    ("llama70b", wl.MODEL_70B, ntx.NTX_Q6_K, 2080),
    ("tiny-q6_k", TINY_Q6, ntx.NTX_Q6_K, 64),
    ("llama70b-q4_k", wl.MODEL_70B, ntx.NTX_Q4_K, 2080),
    ("llama70b-q5_k", wl.MODEL_70B, ntx.NTX_Q5_K, 2080),
    ("llama8b-q4_k", wl.MODEL_8B, ntx.NTX_Q4_K, 144),
]


@pytest.mark.parametrize("name,d,qt,max_ctx", CASES, ids=[c[0] for c in CASES])
def test_plan_invariants(name, d, qt, max_ctx):
    plan = ntx.ntx_persistent_plan(_cfg(d, max_ctx), qt)
    be, bb = BLOCK[qt]
    assert plan["smem_bytes"] <= SMEM_MAX
    assert plan["n_slots"] >= 3
    for ph, K in _phase_K(d).items():
        rows = plan["rows"][ph]
        row_bytes = K // be * bb
        assert rows >= 1 and rows * row_bytes <= plan["slot_bytes"], ph
        assert (rows + 1) * row_bytes > plan["slot_bytes"] or rows == 32 or (ph in PAIRED and rows % 2 == 0), ph
        if ph in PAIRED:
            assert rows % 2 == 0, ph
        n_slices = -(-K // SLICE)
        groups = max(1, CONSUMERS // n_slices)
        assert rows >= groups, (ph, rows, groups)  # every row-group warp gets a row
        if qt == ntx.NTX_Q6_K:
            assert rows % groups == 0, (ph, rows, groups)


def test_plan_of_the_bench_models():
    """The plans the measured numbers were taken with."""
    p8 = ntx.ntx_persistent_plan(_cfg(wl.MODEL_8B, 144), ntx.NTX_Q8_0)
    assert (p8["slot_bytes"], p8["n_slots"]) == (60928, 3)
    assert [p8["rows"][k] for k in PHASES] == [14, 14, 14, 4, 14]  # two rows for every row-group warp
    p70 = ntx.ntx_persistent_plan(_cfg(wl.MODEL_70B, 2080), ntx.NTX_Q6_K)
    assert (p70["slot_bytes"], p70["n_slots"]) == (40320, 4)
    assert [p70["rows"][k] for k in PHASES] == [6, 6, 6, 1, 6]


def test_plan_argument_errors():
    L = ntx.lib()
    cfg = _cfg(wl.MODEL_8B, 144)
    assert L.ntx_persistent_plan(None, ntx.NTX_Q8_0, None, None, None, None) == ntx.NTX_ERR_INVALID_ARG
    # F16 / F32 layers run on the per-op chain only
    assert L.ntx_persistent_plan(cfg, ntx.NTX_F16, None, None, None, None) == ntx.NTX_ERR_SHAPE
    assert L.ntx_persistent_plan(cfg, 99, None, None, None, None) == ntx.NTX_ERR_QTYPE
    bad = dict(wl.MODEL_8B, head_dim=64)  # the persistent kernel takes head_dim 128 only
    assert L.ntx_persistent_plan(_cfg(bad, 144), ntx.NTX_Q8_0, None, None, None, None) == ntx.NTX_ERR_SHAPE
    bad = dict(wl.MODEL_8B, n_heads=12)  # query group 12 / 8 is not whole
    assert L.ntx_persistent_plan(_cfg(bad, 144), ntx.NTX_Q8_0, None, None, None, None) == ntx.NTX_ERR_SHAPE
    bad = dict(wl.MODEL_8B, hidden=0)
    assert L.ntx_persistent_plan(_cfg(bad, 144), ntx.NTX_Q8_0, None, None, None, None) == ntx.NTX_ERR_INVALID_ARG
