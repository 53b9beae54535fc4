"""GPU parity of ntx_decode_layer (one pre-norm Llama decode layer) against
the oracle's layer, on small shapes for every weight format and on the full
8B-shaped Q8_0 layer with 1024 prior KV positions.

Bars: layer output max|diff| <= 2e-3 * RMS(ref); the appended k, v rows
within 2e-3 * RMS of the oracle's (fp16 rounding of values that are fp32 on the
GPU and fp64 in the oracle may differ by one fp16 ulp); every other cache row
bit-identical; cosine |diff| <= 1e-5."""
import numpy as np
import pytest

import oracle
import quantized_weight_gemv_dequant_b200 as ntx
import synthgen as sg
from helpers import dev
from synthgen import workloads as wl

pytestmark = pytest.mark.gpu

SMALL = dict(hidden=512, n_heads=8, n_kv_heads=2, head_dim=128, ffn=1536, vocab=1000, n_layers=1, eps=1e-5,
             theta=500000.0)
SMALL_G8 = dict(hidden=1024, n_heads=16, n_kv_heads=2, head_dim=128, ffn=2816, vocab=1000, n_layers=1, eps=1e-5,
                theta=500000.0)
SMALL_Q6K = dict(hidden=2048, n_heads=16, n_kv_heads=2, head_dim=128, ffn=4096, vocab=1000, n_layers=1, eps=1e-5,
                 theta=500000.0)


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    import torch
    from quantized_weight_gemv_dequant_b200 import build
    build.build()
    torch.cuda.init()
    yield
    torch.cuda.synchronize()
    assert ntx.ntx_device_status() == 0


def _cfg(d, max_ctx, layers=1):
    return ntx.make_config(d["hidden"], d["n_heads"], d["n_kv_heads"], d["head_dim"], d["ffn"], d["vocab"], layers,
                           d["eps"], d["theta"], max_ctx)


def _ocfg(d, max_ctx, layers=1):
    return oracle.make_config(d["hidden"], d["n_heads"], d["n_kv_heads"], d["head_dim"], d["ffn"], d["vocab"], layers,
                              d["eps"], d["theta"], max_ctx)


def run_layer_case(d, qtype, sd, pos, max_ctx, blob=None, tensors=None):
    import torch
    if blob is None:
        blob, tensors = wl.host_layer_blob(d, qtype, sd, 0)
    kc, vc = wl.host_kv_prior(d, sd, 0, max_ctx, pos)
    h = sg.fill_f32(sd, "hidden", d["hidden"])
    cfg = _cfg(d, max_ctx)
    _, lw = ntx.ntx_layer_layout(cfg, qtype)
    blob_d = dev(blob)
    lw.base = blob_d.data_ptr()
    kc_d, vc_d, h_d = dev(kc), dev(vc), dev(h)
    ws_bytes = ntx.ntx_layer_workspace_bytes(cfg)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    cos_d = torch.zeros(4, dtype=torch.float32, device="cuda")
    ntx.ntx_decode_layer(cfg, lw, kc_d, vc_d, h_d, pos, cos_d, ws, ws_bytes)
    torch.cuda.synchronize()
    got_h = h_d.cpu().numpy().astype(np.float64)
    got_k, got_v = kc_d.cpu().numpy(), vc_d.cpu().numpy()
    got_cos = float(cos_d[0].item())

    kc_o, vc_o = kc.copy(), vc.copy()
    ref_h, ref_cos = oracle.layer(_ocfg(d, max_ctx), qtype, tensors, tensors["attn_norm"], tensors["ffn_norm"],
                                  kc_o, vc_o, h, pos)
    rms = np.sqrt(np.mean(ref_h ** 2))
    assert np.max(np.abs(got_h - ref_h)) <= 2e-3 * rms, np.max(np.abs(got_h - ref_h)) / rms
    assert abs(got_cos - ref_cos) <= 1e-5, (got_cos, ref_cos)
    # appended rows close, all other rows untouched
    for got, ref, orig in ((got_k, kc_o, kc), (got_v, vc_o, vc)):
        g = got[:, pos].view(np.float16).astype(np.float64)
        r = ref[:, pos].view(np.float16).astype(np.float64)
        assert np.max(np.abs(g - r)) <= 2e-3 * np.sqrt(np.mean(r ** 2)) + 1e-6
        mask = np.ones(max_ctx, dtype=bool)
        mask[pos] = False
        assert np.array_equal(got[:, mask], orig[:, mask])
    return got_h, ref_h


@pytest.mark.parametrize("qtype", [ntx.NTX_Q8_0, ntx.NTX_Q4_0])
@pytest.mark.parametrize("pos", [0, 1, 37, 300])
def test_layer_small(qtype, pos):
    run_layer_case(SMALL, qtype, 1000 + pos, pos, 320)


@pytest.mark.parametrize("pos", [0, 5, 129])
def test_layer_small_group8(pos):
    run_layer_case(SMALL_G8, ntx.NTX_Q8_0, 2000 + pos, pos, 160)


@pytest.mark.parametrize("pos", [0, 63, 511])
def test_layer_small_q6_k(pos):
    run_layer_case(SMALL_Q6K, ntx.NTX_Q6_K, 3000 + pos, pos, 512)


@pytest.mark.parametrize("pos", [7, 4100, 4499])
def test_layer_long_context_split_combine_path(pos):
    """A cache longer than 16 clusters x 256 positions takes the split +
    combine attention kernels instead of the cluster-fused one."""
    run_layer_case(SMALL, ntx.NTX_Q8_0, 4000 + pos, pos, 4500)


def test_layer_llama8b_q8_0_pos1024():
    """Config 3: the 8B-shaped Q8_0 layer, 1024 prior positions, token at 1024.
    Also checks that the device generator writes this layer bit-identically."""
    import torch
    d = dict(wl.MODEL_8B)
    sd = wl.seed(3)
    blob, tensors = wl.host_layer_blob(d, ntx.NTX_Q8_0, sd, 0)
    blob_dev = torch.zeros(blob.size, dtype=torch.uint8, device="cuda")
    wl.dev_layer_blob(d, ntx.NTX_Q8_0, sd, 0, blob_dev.data_ptr())
    torch.cuda.synchronize()
    assert np.array_equal(blob_dev.cpu().numpy(), blob)
    run_layer_case(d, ntx.NTX_Q8_0, sd, 1024, 1025, blob=blob, tensors=tensors)
