"""Config 5: the 80-layer Llama-3-70B-shaped Q6_K model, 2048 prior KV
positions, (a) fully resident and (b) tiered with layers 40-79 in pinned host
memory streamed through two device slots, each with the cosine layer skip at
threshold 0.98 calibrated on the first decode step.

The resident run is one persistent kernel per step; the tiered run is the
per-op kernel chain with the copy stream.  Checks on each (teacher-forced, 2
steps -- the oracle takes ~10 s per step here): logits within 2e-2 * RMS of the
oracle's; calibration cosines within 1e-5; skip decisions equal wherever
|cos - 0.98| > 1e-4.  The model is made by the generator's CUDA twin; sampled
rows of every matrix are checked bit-identical to the host generator first."""
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


def test_engine_llama70b_q6_k_resident_and_tiered_with_skip():
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
    runs = {}
    for name, kw in (("resident", dict(use_resident_copy=True)), ("tiered", {})):
        m.reset_kv()
        e = Engine(m, tau=0.98, **kw)
        lg0, fed0, nx0, cos0 = e.run(prompt, pos0=2048, flags=ntx.NTX_CALIBRATE_SKIP, collect_cos=True)
        mask = ntx.ntx_engine_skip_mask(e.h, L)
        lg1, fed1, nx1, _ = e.run([-1], pos0=2049, flags=ntx.NTX_USE_SKIP)
        launches = ntx.ntx_engine_launches_per_step(e.h)
        e.close()
        runs[name] = (lg0, fed0 + fed1, nx0, cos0, mask, lg1, nx1, launches)
    assert runs["resident"][7] == 1

    ocfg = oracle.make_config(d["hidden"], d["n_heads"], d["n_kv_heads"], d["head_dim"], d["ffn"], d["vocab"], L,
                              d["eps"], d["theta"], 2080)
    emb, fn, head = m.host_embed(), m.host_final_norm(), m.host_head()
    nt = os.cpu_count()
    refs = {}
    for name, (lg0, fed, nx0, cos0, mask, lg1, nx1, _) in runs.items():
        kcs, vcs = zip(*[m.host_kv(l) for l in range(L)])
        kcs, vcs = [k.copy() for k in kcs], [v.copy() for v in vcs]
        key0 = fed[0]
        if key0 not in refs:
            refs[key0] = oracle.model_step(ocfg, ntx.NTX_Q6_K, m.host_layer_tensors, ntx.NTX_Q6_K, head, fn, emb, kcs,
                                           vcs, fed[0], 2048, nthreads=nt)
        else:
            # the oracle's caches must still take the calibration step's k, v
            oracle.model_step(ocfg, ntx.NTX_Q6_K, m.host_layer_tensors, ntx.NTX_Q6_K, head, fn, emb, kcs, vcs,
                              fed[0], 2048, nthreads=nt)
        ref0, cref = refs[key0]
        for l in range(L):
            assert abs(cos0[0][l] - cref[l]) <= 1e-5, (name, l, cos0[0][l], cref[l])
            if abs(cref[l] - 0.98) > 1e-4:
                assert mask[l] == (1 if cref[l] >= 0.98 else 0), (name, l)
        check_logits(lg0[0], ref0, int(nx0[0]), 0)
        ref1, _ = oracle.model_step(ocfg, ntx.NTX_Q6_K, m.host_layer_tensors, ntx.NTX_Q6_K, head, fn, emb, kcs, vcs,
                                    fed[1], 2049, skip=mask, nthreads=nt)
        check_logits(lg1[0], ref1, int(nx1[0]), 1)
        print(f"{name}: skipped {sum(mask)}/{L} layers at tau 0.98")


def test_engine_llama70b_q4_k_m_resident_persistent():
    """The 70B shapes as Q4_K_M (Q4_K matrices, Q6_K down projections and head):
    the persistent kernel with two block types (opted in; the default for
    two-type steps is the per-op chain) (Q4_K phases over 4 K-slices,
    the Q6_K down projection over 14), checked teacher-forced for 2 steps."""
    d = dict(wl.MODEL_70B)
    L = d["n_layers"]
    sd = wl.seed(5)
    m = DeviceModel(d, wl.Q4_K_M, wl.Q4_K_M_HEAD, sd, max_ctx=2080, n_prior=2048, source="device")
    for l in (0, L - 1):
        t = m.host_layer_tensors(l)
        for (name, (M, K)), qt in zip(wl.mat_shapes(d).items(), wl.Q4_K_M):
            ref = sg.quant_rows(qt, sd, wl.tensor_name(l, name), M, K, sigma=wl.W_SIGMA, row0=7, nrows=1)
            assert np.array_equal(t[name][7], ref[0]), (l, name)
    prompt = [int(sg.tokens(sd, "prompt", 1, d["vocab"])[0])]
    ntx.ntx_set_persist_two_types(1)  # opt in: two-type steps default to the per-op chain
    try:
        e = Engine(m)
    finally:
        ntx.ntx_set_persist_two_types(0)
    lg, fed, nx, _ = e.run(prompt + [-1], pos0=2048)
    launches = ntx.ntx_engine_launches_per_step(e.h)
    e.close()
    assert launches == 1
    ocfg = oracle.make_config(d["hidden"], d["n_heads"], d["n_kv_heads"], d["head_dim"], d["ffn"], d["vocab"], L,
                              d["eps"], d["theta"], 2080)
    emb, fn, head = m.host_embed(), m.host_final_norm(), m.host_head()
    kcs, vcs = zip(*[m.host_kv(l) for l in range(L)])
    kcs, vcs = [k.copy() for k in kcs], [v.copy() for v in vcs]
    for s in range(2):
        ref, _ = oracle.model_step(ocfg, wl.Q4_K_M, m.host_layer_tensors, wl.Q4_K_M_HEAD, head, fn, emb, kcs, vcs,
                                   fed[s], 2048 + s, nthreads=os.cpu_count())
        check_logits(lg[s], ref, int(nx[s]), s)
