"""Self-speculative decoding (ntx_decode_spec): the resident layers draft
draft_k tokens, the whole model verifies them in one layer-by-layer pass.

The emitted tokens must be exactly the greedy continuation an ordinary decode
gives (same engine layout, same kernels), for any acceptance pattern:
* host layers with random weights (the draft often disagrees), and
* host layers made the identity (their O and down projections zeroed), where
  the draft is the whole model and every proposal should be accepted;
and the oracle, teacher-forced on the emitted sequence, agrees with the
greedy choice wherever its top two logits are clearly apart."""
import numpy as np
import pytest

import quantized_weight_gemv_dequant_b200 as ntx
import synthgen as sg
from synthgen import workloads as wl
from synthgen.devmodel import DeviceModel
from test_gpu_engine import TINY, Engine, oracle_run

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


def _greedy(m, prompt, n):
    """Ordinary decode: the prompt, then n greedy tokens."""
    m.reset_kv()
    e = Engine(m)
    _, fed, nx, _ = e.run(list(prompt) + [-1] * (n - 1))
    e.close()
    return [int(t) for t in nx[len(prompt) - 1:]]


def _spec(m, prompt, n, k, flags=0):
    m.reset_kv()
    e = Engine(m)
    e.run(list(prompt[:-1]))  # positions 0 .. len-2
    tok, pos = int(prompt[-1]), len(prompt) - 1
    out, accepted = [], []
    while len(out) < n:
        got = ntx.ntx_decode_spec(e.h, tok, pos, k, flags)
        assert 1 <= len(got) <= k + 1
        accepted.append(len(got) - 1)
        out += got
        pos += len(got)
        tok = got[-1]
    e.close()
    return out[:n], accepted


def _zero_matrix(m, layer, name):
    """Zero a host-tier layer's matrix in its pinned blob (all block scales 0)."""
    d = m.d
    M, K = wl.mat_shapes(d)[name]
    off = m.offsets[name]
    m.layers[layer][off:off + wl.mat_bytes(m.qtype, M, K)].zero_()


@pytest.mark.parametrize("k", [1, 3, 7])
def test_spec_equals_greedy_random_host_layers(k):
    m = DeviceModel(TINY, ntx.NTX_Q8_0, ntx.NTX_Q8_0, 71, max_ctx=48, n_prior=0, tier_map=[0, 0, 1, 1],
                    source="host")
    prompt = [int(t) for t in sg.tokens(71, "prompt", 4, TINY["vocab"])]
    n = 20
    ref = _greedy(m, prompt, n)
    got, acc = _spec(m, prompt, n, k)
    assert got == ref, (got, ref)
    # the oracle agrees on the emitted sequence (teacher-forced)
    logits, _ = oracle_run(m, prompt + got[:-1])
    for s in range(len(prompt) - 1, len(prompt) + len(got) - 1):
        top2 = np.sort(logits[s])[-2:]
        if top2[1] - top2[0] > 4e-2 * np.sqrt(np.mean(logits[s] ** 2)):
            assert got[s - len(prompt) + 1] == int(np.argmax(logits[s]))


def test_spec_identity_host_layers_accepts_drafts():
    m = DeviceModel(TINY, ntx.NTX_Q8_0, ntx.NTX_Q8_0, 72, max_ctx=48, n_prior=0, tier_map=[0, 0, 1, 1],
                    source="host")
    for l in (2, 3):
        _zero_matrix(m, l, "wo")
        _zero_matrix(m, l, "wd")
    prompt = [int(t) for t in sg.tokens(72, "prompt", 3, TINY["vocab"])]
    n, k = 24, 3
    ref = _greedy(m, prompt, n)
    got, acc = _spec(m, prompt, n, k)
    assert got == ref
    # the draft is the whole model here: (nearly) every proposal is accepted
    assert np.mean(acc) >= 0.8 * k, acc
    # with the persistent kernel off for the draft, the same tokens
    got2, _ = _spec(m, prompt, n, k, ntx.NTX_NO_PERSIST)
    assert got2 == ref


def test_spec_argument_checks():
    m = DeviceModel(TINY, ntx.NTX_Q8_0, ntx.NTX_Q8_0, 73, max_ctx=16, n_prior=0, source="host")
    e = Engine(m)  # all resident: nothing to verify against
    with pytest.raises(ntx.NtxError) as err:
        ntx.ntx_decode_spec(e.h, 1, 0, 3)
    assert err.value.code == ntx.NTX_ERR_INVALID_ARG
    e.close()
    m2 = DeviceModel(TINY, ntx.NTX_Q8_0, ntx.NTX_Q8_0, 73, max_ctx=16, n_prior=0, tier_map=[0, 1, 1, 1],
                     source="host")
    e2 = Engine(m2)
    for args, code in (((1, 0, 0), ntx.NTX_ERR_INVALID_ARG), ((1, 0, 8), ntx.NTX_ERR_INVALID_ARG),
                       ((1, 13, 3), ntx.NTX_ERR_SHAPE), ((-1, 0, 3), ntx.NTX_ERR_INVALID_ARG)):
        with pytest.raises(ntx.NtxError) as err:
            ntx.ntx_decode_spec(e2.h, *args)
        assert err.value.code == code, args
    e2.close()
