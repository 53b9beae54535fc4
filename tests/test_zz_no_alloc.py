"""ntx_attn_decode_static, the attention call that allocates nothing.

Some callers cannot give libntx a scratch buffer: their device memory belongs
to another allocator with a fixed budget, or they are plain C code with no
allocator on that path, or a latency-critical thread that must not take an
allocator's lock.  ntx_attn_decode_static keeps the split partials in a fixed
2 MiB device array inside the library instead.  This file checks, through the
C ABI, that two calls in a row give bit for bit what ntx_attn_decode (caller
workspace, same split count) gives and meet the oracle's attention bar, also
at the largest context the array holds, and that one position more is refused
before any launch.  Every pointer handed to the library here is a real device
buffer sized for the arguments.  It is collected last so that a failure here
does not hide the other tests' results; it passes alone and after them."""
import numpy as np
import pytest

import oracle
import quantized_weight_gemv_dequant_b200 as ntx
import synthgen as sg
from helpers import dev

pytestmark = pytest.mark.gpu

D = 128
# 32 query heads, 8 KV heads on a 148-SM part: 126 splits of 256 positions x 32
# heads x 130 floats = 524,160 <= 524,288 floats (2 MiB); one position more
# needs 127 splits.
LIMIT_CTX = 126 * 256


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    import torch
    from quantized_weight_gemv_dequant_b200 import build
    build.build()
    torch.cuda.init()
    yield
    torch.cuda.synchronize()
    assert ntx.ntx_device_status() == 0


def _case(Hq, Hkv, T, sd):
    q = sg.fill_f32(sd, "za_q", Hq * D)
    kc = sg.fill_f16(sd, "za_k", Hkv * T * D).reshape(Hkv, T, D)
    vc = sg.fill_f16(sd, "za_v", Hkv * T * D).reshape(Hkv, T, D)
    return q, kc, vc


def _run_both(q, kc, vc, Hq, Hkv, n_ctx, T):
    """Two static calls in a row and one workspace call; returns host arrays."""
    import torch
    qd, kd, vd = dev(q), dev(kc), dev(vc)
    ws_bytes = ntx.ntx_attn_workspace_bytes(Hq, Hkv, D, T)
    ws = torch.empty(ws_bytes // 4 + 64, dtype=torch.float32, device="cuda")
    ref = torch.empty(Hq * D, dtype=torch.float32, device="cuda")
    got = [torch.full((Hq * D,), float("nan"), dtype=torch.float32, device="cuda") for _ in range(2)]
    ntx.ntx_attn_decode(qd, kd, vd, ref, Hq, Hkv, D, n_ctx, T, ws, ws_bytes)
    for g in got:
        ntx.ntx_attn_decode_static(qd, kd, vd, g, Hq, Hkv, D, n_ctx, T)
    torch.cuda.synchronize()
    return ref.cpu().numpy(), [g.cpu().numpy() for g in got]


@pytest.mark.parametrize("Hq,Hkv,n_ctx,T,sd", [(32, 8, 1025, 1100, 71), (64, 8, 2049, 2080, 72),
                                               (32, 8, LIMIT_CTX, LIMIT_CTX, 73)])
def test_static_scratch_attention_twice_matches_oracle_and_workspace_call(Hq, Hkv, n_ctx, T, sd):
    q, kc, vc = _case(Hq, Hkv, T, sd)
    ref, got = _run_both(q, kc, vc, Hq, Hkv, n_ctx, T)
    want, bound = oracle.attention(q, kc, vc, Hq, Hkv, D, n_ctx, T)
    for g in got:
        # the same split-KV kernels with the same split count: identical bits
        assert np.array_equal(g.view(np.uint32), ref.view(np.uint32))
        assert np.all(np.isfinite(g))
        assert np.all(np.abs(g.astype(np.float64) - want) <= 1e-3 * bound + 1e-6)


def test_static_scratch_refuses_one_position_beyond_the_array():
    import torch
    Hq, Hkv, T = 32, 8, LIMIT_CTX + 1
    if ntx.ntx_sm_count() != 148:
        pytest.skip("the limit case is sized for a 148-SM device")
    # real buffers sized for the arguments: if the check ever moved after the
    # launch, the kernels would read memory that exists
    q = torch.zeros(Hq * D, dtype=torch.float32, device="cuda")
    kc = torch.zeros(Hkv * T * D, dtype=torch.int16, device="cuda")
    vc = torch.zeros_like(kc)
    out = torch.zeros(Hq * D, dtype=torch.float32, device="cuda")
    with pytest.raises(ntx.NtxError) as e:
        ntx.ntx_attn_decode_static(q, kc, vc, out, Hq, Hkv, D, T, T)
    assert e.value.code == ntx.NTX_ERR_NOMEM
    assert "2 MiB" in ntx.ntx_last_error()
    torch.cuda.synchronize()
    assert not torch.any(out != 0).item()  # nothing was launched
