"""One fixed set of decode and GEMV calls, run in its own process against the
library NTX_LIB names; its outputs, the bounds-check report and the device
status go to an .npz file (argv[1]).  test_gpu_check_build.py runs it once with
the release library and once with the bounds-checked one and compares.

Covered: the persistent kernel on a Q8_0 model (one split per KV head) and on
Q6_K and Q4_0 models whose contexts give several splits per KV head (split
merge), the per-op chain of the same Q8_0 model, and per-op GEMVs of every
quantized block type."""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
for p in (ROOT, HERE):
    if p not in sys.path:
        sys.path.insert(0, p)


def main(out_path: str) -> None:
    import numpy as np
    import torch

    import quantized_weight_gemv_dequant_b200 as ntx
    import synthgen as sg
    from synthgen.devmodel import DeviceModel
    from test_gpu_engine import TINY, Engine

    torch.cuda.init()
    res = {"check_enabled": np.array([ntx.ntx_check_enabled()])}
    models = [
        ("q8_0", ntx.NTX_Q8_0, TINY, 32, 0),
        ("q6_k_splits", ntx.NTX_Q6_K, dict(TINY, hidden=2048, n_heads=16, n_kv_heads=8, ffn=6144, n_layers=2),
         300, 290),
        ("q4_0_splits", ntx.NTX_Q4_0, dict(TINY, n_heads=4, n_kv_heads=4, n_layers=2), 600, 590),
    ]
    for name, qt, d, max_ctx, n_prior in models:
        m = DeviceModel(d, qt, qt, 61, max_ctx=max_ctx, n_prior=n_prior, source="host")
        toks = list(sg.tokens(61, "prompt", 3, d["vocab"])) + [-1] * 3
        for flags, tag in ((0, "persistent"), (ntx.NTX_NO_PERSIST, "chain")):
            if tag == "chain" and name != "q8_0":
                continue
            m.reset_kv()
            e = Engine(m)
            lg, _, nx, _ = e.run(toks, pos0=n_prior, flags=flags)
            e.close()
            res[f"{name}_{tag}_logits"] = lg
            res[f"{name}_{tag}_tokens"] = nx
    M, K = 640, 4096
    x = torch.from_numpy(sg.fill_f32(62, "x", K)).cuda()
    for qt in (ntx.NTX_Q8_0, ntx.NTX_Q4_0, ntx.NTX_Q4_K, ntx.NTX_Q5_K, ntx.NTX_Q6_K):
        W = torch.from_numpy(sg.quant_rows(qt, 62, f"w{qt}", M, K).ravel()).cuda()
        y = torch.empty(M, dtype=torch.float32, device="cuda")
        ntx.ntx_gemv_q(qt, W, M, K, x, y)
        torch.cuda.synchronize()
        res[f"gemv_{qt}"] = y.cpu().numpy()
    site, index = ntx.ntx_check_report()
    res["check_site"] = np.array([site])
    res["check_index"] = np.array([index])
    res["status"] = np.array([ntx.ntx_device_status()])
    np.savez(out_path, **res)


if __name__ == "__main__":
    main(sys.argv[1])
