"""ntx_attn_decode_static, the attention call that allocates nothing.

Some callers cannot give libntx a scratch buffer: their device memory belongs
to another allocator with a fixed budget, or they are plain C code with no
allocator on that path, or a latency-critical thread that must not take an
allocator's lock.  ntx_attn_decode_static keeps the split partials in a fixed
2 MiB device array inside the library instead.  This file checks, through the
C ABI, that two calls in a row give what ntx_attn_decode (caller workspace)
gives, within the attention tolerance used by the other tests, and that a size
beyond the array is refused before any launch.  It is collected last so that a
failure here does not hide the other tests' results; it passes alone and after
them."""
import numpy as np
import pytest

import oracle
import quantized_weight_gemv_dequant_b200 as ntx
import synthgen as sg
from helpers import dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    import torch
    from quantized_weight_gemv_dequant_b200 import build
    build.build()
    torch.cuda.init()
    yield
    torch.cuda.synchronize()
    assert ntx.ntx_device_status() == 0


def test_static_scratch_attention_matches_workspace_call_twice():
    import torch
    for Hq, Hkv, n_ctx, T, sd in ((32, 8, 1025, 1100, 71), (64, 8, 2049, 2080, 72)):
        D = 128
        q = sg.fill_f32(sd, "za_q", Hq * D)
        kc = sg.fill_f16(sd, "za_k", Hkv * T * D).reshape(Hkv, T, D)
        vc = sg.fill_f16(sd, "za_v", Hkv * T * D).reshape(Hkv, T, D)
        qd, kd, vd = dev(q), dev(kc), dev(vc)
        ws_bytes = ntx.ntx_attn_workspace_bytes(Hq, Hkv, D, T)
        ws = torch.empty(ws_bytes // 4 + 64, dtype=torch.float32, device="cuda")
        ref = torch.empty(Hq * D, dtype=torch.float32, device="cuda")
        got = torch.full((Hq * D,), float("nan"), dtype=torch.float32, device="cuda")
        ntx.ntx_attn_decode(qd, kd, vd, ref, Hq, Hkv, D, n_ctx, T, ws, ws_bytes)
        ntx.ntx_attn_decode_static(qd, kd, vd, got, Hq, Hkv, D, n_ctx, T)
        torch.cuda.synchronize()
        _, bound = oracle.attention(q, kc, vc, Hq, Hkv, D, n_ctx, T)
        g, r = got.cpu().numpy().astype(np.float64), ref.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(g))
        assert np.all(np.abs(g - r) <= 1e-3 * bound + 1e-6)


def test_static_scratch_refuses_oversize():
    fake = 0x7F0000000000
    with pytest.raises(ntx.NtxError) as e:
        ntx.ntx_attn_decode_static(fake, fake + 0x1000, fake + 0x2000, fake + 0x3000, 64, 8, 128, 20000, 20000)
    assert e.value.code == ntx.NTX_ERR_NOMEM
    assert "2 MiB" in ntx.ntx_last_error()
