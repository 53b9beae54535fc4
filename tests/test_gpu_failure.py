"""Failure detection on the GPU without a fault: bounded waits that run out
report a status the host reads, and injected host-side failures enqueue
nothing.  Nothing here traps, faults or waits without a limit: the stalled
step's waits are cut to 1 ms, every other wait keeps its limit.

* A CTA of the persistent decode kernel withholds its first publication: the
  other CTAs give up after 1 ms, the kernel returns, ntx_device_status reads
  4 (grid barrier ran out), and the next ordinary step matches the oracle.
* NTX_FAULT=h2d_submit on a tiered engine: the step fails before enqueuing
  anything (the logits buffer keeps its canary), and a later step works.
* NTX_FAULT=host_wait: the calibration read-back and ntx_engine_destroy report
  NTX_ERR_TIMEOUT; without the fault destroy then succeeds."""
import numpy as np
import pytest

import quantized_weight_gemv_dequant_b200 as ntx
import synthgen as sg
from synthgen.devmodel import DeviceModel
from test_gpu_engine import TINY, Engine, check_logits, oracle_run

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


def test_stalled_cta_makes_grid_waits_run_out_and_report():
    import torch
    m = DeviceModel(TINY, ntx.NTX_Q8_0, ntx.NTX_Q8_0, 61, max_ctx=16, n_prior=0, source="host")
    e = Engine(m)
    assert ntx.ntx_engine_set_phase_probe(e.h, None, 0) > 3  # the persistent kernel runs this engine
    prompt = [int(t) for t in sg.tokens(61, "prompt", 2, TINY["vocab"])]
    e.run(prompt[:1], flags=ntx.NTX_NO_GRAPH)
    assert ntx.ntx_device_status() == 0
    ntx.ntx_engine_set_fault(e.h, 3, 1000000)  # CTA 3 withholds its embed publication; waits give up after 1 ms
    e.logits.fill_(float("nan"))
    with torch.cuda.stream(e.cs):
        ntx.ntx_decode_step(e.h, prompt[1], 1, e.logits, e.next_tok, ntx.NTX_NO_GRAPH, None)
    e.cs.synchronize()  # returns: no CTA is left waiting
    assert ntx.ntx_device_status() == 4  # a grid-wide wait ran out (and the word is cleared by the read)
    ntx.ntx_engine_set_fault(e.h, -1, 0)
    lg, fed, nx, _ = e.run(prompt[1:2], pos0=1, flags=ntx.NTX_NO_GRAPH)
    e.close()
    assert ntx.ntx_device_status() == 0
    ref, _ = oracle_run(m, prompt[:2])
    check_logits(lg[0], ref[1], int(nx[0]), 1)


def test_injected_h2d_submit_failure_enqueues_nothing(monkeypatch):
    import torch
    m = DeviceModel(TINY, ntx.NTX_Q8_0, ntx.NTX_Q8_0, 62, max_ctx=16, n_prior=0, tier_map=[0, 1, 0, 1],
                    source="host", keep_resident_copy=True)
    e = Engine(m)
    e.logits.fill_(float("nan"))
    monkeypatch.setenv("NTX_FAULT", "h2d_submit")
    with pytest.raises(ntx.NtxError) as err:
        ntx.ntx_decode_step(e.h, 5, 0, e.logits, e.next_tok, 0, None)
    assert err.value.code == ntx.NTX_ERR_CUDA and "injected" in ntx.ntx_last_error()
    e.cs.synchronize()
    assert torch.isnan(e.logits).all().item()  # nothing ran
    monkeypatch.delenv("NTX_FAULT")
    lg, fed, nx, _ = e.run([5])
    e.close()
    ref, _ = oracle_run(m, fed)
    check_logits(lg[0], ref[0], int(nx[0]), 0)


def test_injected_host_wait_timeouts(monkeypatch):
    m = DeviceModel(TINY, ntx.NTX_Q8_0, ntx.NTX_Q8_0, 63, max_ctx=16, n_prior=0, source="host")
    e = Engine(m)
    monkeypatch.setenv("NTX_FAULT", "host_wait")
    with pytest.raises(ntx.NtxError) as err:
        ntx.ntx_decode_step(e.h, 7, 0, e.logits, e.next_tok, ntx.NTX_CALIBRATE_SKIP, None)
    assert err.value.code == ntx.NTX_ERR_TIMEOUT
    with pytest.raises(ntx.NtxError) as err:
        ntx.ntx_engine_destroy(e.h)
    assert err.value.code == ntx.NTX_ERR_TIMEOUT
    monkeypatch.delenv("NTX_FAULT")
    ntx.ntx_engine_destroy(e.h)  # kept on timeout; now freed
    assert ntx.ntx_device_status() == 0
