"""Config 5: the 80-layer Llama-3-70B-shaped Q6_K model, 2048 prior KV
positions, (a) fully resident and (b) tiered with layers 40-79 in pinned host
memory streamed through two device slots, each with the cosine layer skip at
threshold 0.98 calibrated on the first decode step.

Checks (teacher-forced, 2 steps -- the oracle takes ~10 s per step here):
logits within 2e-2 * RMS of the oracle's; calibration cosines within 1e-5;
skip decisions equal wherever |cos - 0.98| > 1e-4; the tiered run's logits and
skip set bit-identical to the resident run's.  The model is made by the
generator's CUDA twin; sampled rows of every matrix are checked bit-identical
to the host generator first."""
import os

import numpy as np
import pytest

import oracle
import quantized_weight_gemv_dequant_b200 as ntx
import synthgen as sg
from synthgen import workloads as wl
from synthgen.devmodel import DeviceModel
from test_gpu_engine import Engine, check_logits

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    import torch
    from quantized_weight_gemv_dequant_b200 import build
    build.build()
    torch.cuda.init()
    yield
    torch.cuda.synchronize()
    assert ntx.ntx_device_status() == 0


def test_engine_config_5_llama70b_q6_k_resident_and_tiered_with_skip():
    d = dict(wl.MODEL_70B)
    L = d["n_layers"]
    sd = wl.seed(5)
    tiers = [0] * 40 + [1] * 40
    m = DeviceModel(d, ntx.NTX_Q6_K, ntx.NTX_Q6_K, sd, max_ctx=2080, n_prior=2048, tier_map=tiers, source="device",
                    keep_resident_copy=True)
    rs = np.random.RandomState(5)
    for l in list(range(0, L, 7)) + [L - 1]:
        t = m.host_layer_tensors(l)
        for name, (M, K) in wl.mat_shapes(d).items():
            r = int(rs.randint(0, M))
            ref = sg.quant_rows(ntx.NTX_Q6_K, sd, wl.tensor_name(l, name), M, K, sigma=wl.W_SIGMA, row0=r, nrows=1)
            assert np.array_equal(t[name][r], ref[0]), (l, name, r)

    prompt = [int(sg.tokens(sd, "prompt", 1, d["vocab"])[0])]
    # (a) resident
    m.reset_kv()
    ea = Engine(m, tau=0.98, use_resident_copy=True)
    lg_a0, fed_a0, nx_a0, cos_a = ea.run(prompt, pos0=2048, flags=ntx.NTX_CALIBRATE_SKIP, collect_cos=True)
    mask_a = ntx.ntx_engine_skip_mask(ea.h, L)
    lg_a1, fed_a1, nx_a1, _ = ea.run([-1], pos0=2049, flags=ntx.NTX_USE_SKIP)
    ea.close()
    # (b) tiered
    m.reset_kv()
    eb = Engine(m, tau=0.98)
    lg_b0, _, _, _ = eb.run(prompt, pos0=2048, flags=ntx.NTX_CALIBRATE_SKIP, collect_cos=True)
    mask_b = ntx.ntx_engine_skip_mask(eb.h, L)
    lg_b1, _, _, _ = eb.run([-1], pos0=2049, flags=ntx.NTX_USE_SKIP)
    eb.close()
    assert mask_a == mask_b
    assert np.array_equal(lg_a0, lg_b0) and np.array_equal(lg_a1, lg_b1)

    fed = fed_a0 + fed_a1
    ocfg = oracle.make_config(d["hidden"], d["n_heads"], d["n_kv_heads"], d["head_dim"], d["ffn"], d["vocab"], L,
                              d["eps"], d["theta"], 2080)
    kcs, vcs = zip(*[m.host_kv(l) for l in range(L)])
    kcs, vcs = [k.copy() for k in kcs], [v.copy() for v in vcs]
    emb, fn, head = m.host_embed(), m.host_final_norm(), m.host_head()
    nt = os.cpu_count()
    ref0, cos0 = oracle.model_step(ocfg, ntx.NTX_Q6_K, m.host_layer_tensors, ntx.NTX_Q6_K, head, fn, emb, kcs, vcs,
                                   fed[0], 2048, nthreads=nt)
    for l in range(L):
        assert abs(cos_a[0][l] - cos0[l]) <= 1e-5, (l, cos_a[0][l], cos0[l])
        if abs(cos0[l] - 0.98) > 1e-4:
            assert mask_a[l] == (1 if cos0[l] >= 0.98 else 0), l
    check_logits(lg_a0[0], ref0, int(nx_a0[0]), 0)
    ref1, _ = oracle.model_step(ocfg, ntx.NTX_Q6_K, m.host_layer_tensors, ntx.NTX_Q6_K, head, fn, emb, kcs, vcs,
                                fed[1], 2049, skip=mask_a, nthreads=nt)
    check_logits(lg_a1[0], ref1, int(nx_a1[0]), 1)
    print(f"skipped {sum(mask_a)}/{L} layers at tau 0.98")
