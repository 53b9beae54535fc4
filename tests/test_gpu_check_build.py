"""The bounds-checked debug build (NTX_CHECK, see ntx_check_report) on the GPU.

check_build_run.py runs one fixed set of calls -- persistent-kernel decodes
(one split and several splits per KV head), the per-op chain, per-op GEMVs of
every quantized type -- once against the release library and once against
libntx_check.so, each in its own process.  In the checked run every index
check must pass (report site 0) with the device status 0, and every output
must equal the release build's bit for bit: the checks observe, they do not
change the arithmetic."""
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def _run(lib: str, out: str) -> dict:
    env = dict(os.environ, NTX_LIB=lib)
    r = subprocess.run([sys.executable, os.path.join(HERE, "check_build_run.py"), out], env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    z = np.load(out)
    return {k: z[k] for k in z.files}


def test_check_build_passes_and_matches_release(tmp_path):
    from quantized_weight_gemv_dequant_b200 import build
    rel = _run(build.build(), str(tmp_path / "release.npz"))
    chk = _run(build.build_check(), str(tmp_path / "check.npz"))
    assert int(rel["check_enabled"][0]) == 0 and int(chk["check_enabled"][0]) == 1
    assert int(chk["check_site"][0]) == 0, (int(chk["check_site"][0]), int(chk["check_index"][0]))
    assert int(chk["status"][0]) == 0 and int(rel["status"][0]) == 0
    keys = [k for k in rel if k not in ("check_enabled", "check_site", "check_index", "status")]
    assert len(keys) >= 10
    for k in keys:
        a, b = rel[k], chk[k]
        assert a.shape == b.shape, k
        if a.dtype == np.float32:
            assert np.array_equal(a.view(np.uint32), b.view(np.uint32)), k
        else:
            assert np.array_equal(a, b), k
