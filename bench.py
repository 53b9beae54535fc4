#!/usr/bin/env python
"""Batch-1 decode benchmark of libntx on B200.

Default workload: the 32-layer Llama-3-8B-shaped Q8_0 model, all layers
resident in HBM, 16-token prompt then greedy decode with the fp16 KV cache
growing to 144 positions (positions 16..143 are reused cyclically when more
steps are timed).  A step is one token through the whole hot path: embed, 32 x
(RMSNorm + QKV GEMV + RoPE + KV append, split-KV GQA attention, O GEMV +
residual, RMSNorm + gate/up GEMV + SwiGLU, down GEMV + residual + cosine
statistics), final RMSNorm + head GEMV, argmax.  Weights (7.97 GB) are far
larger than the 126 MB L2, so no flush is needed between steps.

Prints one JSON line.  Under torchrun each rank runs an independent replica
on its own GPU (the path has no data-path collective); value = tokens of all
ranks / the slowest rank's device time.

--impl reference times the CPU oracle (fp64, tests' reference implementation)
on the same workload: each step is one layer of the model plus 1/32 of the
head, scaled to a whole token.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "batch-1 decode tok/s; quantized GEMV achieved HBM GB/s vs B200 peak"
# DRAM bytes read + written per algorithmic byte by the persistent decode
# kernel, from one ncu capture (--set full) per instantiation of a cut-down
# case that fits the capture size rule: Q8_0, 4 layers of the 8B shapes,
# 1,485,809,408 + 4,275,456 bytes against 1,485,578,240 algorithmic bytes;
# Q6_K, 2 layers of the 70B shapes, 2,282,932,224 + 4,280,064 bytes against
# 2,282,651,648.  The kernel streams every weight byte once, so a full
# launch's traffic is this ratio times its algorithmic bytes.
PERSIST_TRAFFIC_RATIO = {8: 1490084864 / 1485578240, 14: 2287212288 / 2282651648}
FALLBACK_HBM_GBS = 6650.0


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "of measured"
    except Exception:
        return FALLBACK_HBM_GBS, "of fallback"


WORKLOADS = {
    "llama8b-q8_0": dict(desc="Llama-3-8B-shaped 32-layer Q8_0 model (Q8_0 head, fp16 embeddings), resident in HBM; "
                              "16-token prompt then greedy batch-1 decode, KV cache 17..144 positions",
                         model="MODEL_8B", qtype=8, head_qtype=8, workload_id=4, max_ctx=144, n_prior=0,
                         prompt=16, tiers=None),
    "llama70b-q6_k": dict(desc="Llama-3-70B-shaped 80-layer Q6_K model, resident in HBM; 2048 prior KV positions, "
                               "greedy batch-1 decode from position 2048",
                          model="MODEL_70B", qtype=14, head_qtype=14, workload_id=5, max_ctx=2080, n_prior=2048,
                          prompt=1, tiers=None),
    "llama70b-q6_k-tiered": dict(desc="Llama-3-70B-shaped 80-layer Q6_K model, layers 40-79 in pinned host RAM "
                                      "streamed through two device slots; 2048 prior KV positions",
                                 model="MODEL_70B", qtype=14, head_qtype=14, workload_id=5, max_ctx=2080,
                                 n_prior=2048, prompt=1, tiers="40-79"),
}


# ---------------------------------------------------------------- distributed
class Dist:
    """One process per GPU (torchrun env): barrier and max over ranks.  NCCL on
    GPUs; gloo (CPU tensors) where asked -- the CPU tests use it."""

    def __init__(self, n_gpus, backend=None):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        if n_gpus != self.world:
            raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={self.world}: launch one process per GPU "
                             f"(python -m torch.distributed.run --nproc-per-node {n_gpus} bench.py ...)")
        self.pg = None
        self.backend = backend or "nccl"
        if self.world > 1:
            import datetime
            import torch
            import torch.distributed as dist
            kw = {}
            if self.backend == "nccl":
                torch.cuda.set_device(self.local)
                kw["device_id"] = torch.device("cuda", self.local)
            dist.init_process_group(self.backend, timeout=datetime.timedelta(seconds=600), **kw)
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, v: float) -> float:
        if not self.pg:
            return v
        import torch
        t = torch.tensor([v], dtype=torch.float64, device="cuda" if self.backend == "nccl" else "cpu")
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.barrier()
            self.pg.destroy_process_group()
            self.pg = None


def whole_job_rate(world: int, steps: int, ms_max: float) -> float:
    """Tokens per second of the whole job: every rank decodes `steps` tokens of
    its own replica; the time is the slowest rank's (weak scaling)."""
    return world * steps / (ms_max / 1e3)


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                       "-lms", "100", "-i", str(self.gpu)], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None
        time.sleep(0.15)

    def stop(self):
        if self.p is None:
            return None
        time.sleep(0.15)
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except Exception:
            self.p.kill()
        self.f.flush()
        rows = []
        with open(self.f.name) as fh:
            for line in fh:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.f.name)
        if not rows:
            return None
        try:
            sm = [float(r[1]) for r in rows]
            mx = max(float(r[2]) for r in rows)
        except ValueError:
            return None
        load = [s for s, r in zip(sm, rows) if float(r[3] or 0) > 200.0] or sm
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(rows)}


# ---------------------------------------------------------------- ntx arm
def run_ntx(args, dist: Dist):
    import numpy as np
    import torch

    import quantized_weight_gemv_dequant_b200 as ntx
    import synthgen as sg
    from synthgen import workloads as wl
    from synthgen.devmodel import DeviceModel

    wk = WORKLOADS[args.workload]
    d = dict(getattr(wl, wk["model"]))
    if args.layers is not None:
        d["n_layers"] = args.layers
    L = d["n_layers"]
    qt, hqt = wk["qtype"], wk["head_qtype"]
    sd = wl.seed(wk["workload_id"])
    torch.cuda.init()
    dev_index = torch.cuda.current_device()
    tier_map = [0] * L
    if wk["tiers"]:
        a, b = (int(t) for t in wk["tiers"].split("-"))
        for l in range(a, min(b + 1, L)):
            tier_map[l] = 1
    m = DeviceModel(d, qt, hqt, sd, wk["max_ctx"], wk["n_prior"], tier_map=tier_map, source="device")
    cfg = ntx.make_config(d["hidden"], d["n_heads"], d["n_kv_heads"], d["head_dim"], d["ffn"], d["vocab"], L,
                          d["eps"], d["theta"], wk["max_ctx"], 0.98)
    layers = []
    for l in range(L):
        _, lw = ntx.ntx_layer_layout(cfg, qt)
        lw.base = m.layers[l].data_ptr()
        layers.append(lw)
    ws_bytes = ntx.ntx_engine_workspace_bytes(cfg)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    cs = torch.cuda.Stream()
    xs = torch.cuda.Stream() if any(tier_map) else None
    eng = ntx.ntx_engine_create(cfg, layers, tier_map, m.slots[0], m.slots[1], m.blob_bytes, m.embed, m.final_norm,
                                m.head, hqt, m.k_caches, m.v_caches, ws, ws_bytes, cs, xs)
    next_tok = torch.zeros(1, dtype=torch.int32, device="cuda")
    prompt = sg.tokens(sd, "prompt", wk["prompt"], d["vocab"])
    p0 = wk["n_prior"]
    p_first = p0 + wk["prompt"]
    span = wk["max_ctx"] - p_first

    def pos_of(i):  # i-th decode step after the prompt
        return p_first + (i % span)

    with torch.cuda.stream(cs):
        for s, t in enumerate(prompt):
            ntx.ntx_decode_step(eng, int(t), p0 + s, None, next_tok, 0, None)
        for i in range(args.warmup):
            ntx.ntx_decode_step(eng, -1, pos_of(i), None, next_tok, 0, None)
    cs.synchronize()
    launches = ntx.ntx_engine_launches_per_step(eng)

    # ------------------------------------------------------------ timed region
    clocks = ClockSampler(dev_index)
    clocks.start()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(cs):
        ev0.record(cs)
        for i in range(args.steps):
            ntx.ntx_decode_step(eng, -1, pos_of(args.warmup + i), None, next_tok, 0, None)
        ev1.record(cs)
    torch.cuda.synchronize()
    dist.barrier()
    ms_local = ev0.elapsed_time(ev1)
    clk = clocks.stop()
    ms_total = dist.max(ms_local)
    status = ntx.ntx_device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")
    ms_step = ms_total / args.steps
    value = whole_job_rate(dist.world, args.steps, ms_total)

    persistent = launches <= 2  # one persistent kernel (+ cosine finalisation when asked)

    def probe(flags, n_ev, n_steps, pos_base):
        """Kernel-by-kernel steps with probe events; returns (durations ms, ms/step)."""
        ev_b = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(n_steps)]
        ev_e = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(n_steps)]
        with torch.cuda.stream(cs):
            for row in ev_b + ev_e:
                for ev in row:
                    ev.record(cs)  # creates the CUDA events
        cs.synchronize()
        p0_, p1_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(cs):
            p0_.record(cs)
            for i in range(n_steps):
                ntx.ntx_engine_set_probe(eng, [e.cuda_event for e in ev_b[i]], [e.cuda_event for e in ev_e[i]])
                ntx.ntx_decode_step(eng, -1, pos_of(pos_base + i), None, next_tok, flags | ntx.NTX_NO_GRAPH, None)
            p1_.record(cs)
            ntx.ntx_engine_set_probe(eng, [], [])
        cs.synchronize()
        durs = [ev_b[i][k].elapsed_time(ev_e[i][k]) for i in range(n_steps) for k in range(n_ev)]
        return durs, p0_.elapsed_time(p1_) / n_steps

    # ------------------------------------------------ dominant kernel (probe)
    n_probe = min(args.steps, 24)
    pos_base = args.warmup + args.steps
    H, F = d["hidden"], d["ffn"]
    peak, peak_kind = measured_peaks()
    if persistent:
        durs, probe_ms_step = probe(0, 1, n_probe, pos_base)
        k_ms = statistics.mean(durs)
        n_ctx_mean = statistics.mean(pos_of(pos_base + i) + 1 for i in range(n_probe))
        k_bytes = wl.bytes_per_token(d, qt, hqt, int(round(n_ctx_mean)))
        roof = {"bound": "hbm", "kernel": "persistent decode-step kernel (one launch per token)",
                "achieved": round(k_bytes / (k_ms * 1e-3) / 1e9, 1), "peak": peak, "peak_kind": peak_kind,
                "unit": "GB/s", "frac": round(k_bytes / (k_ms * 1e-3) / 1e9 / peak, 4),
                "traffic": args.traffic if args.traffic is not None else (
                    round(PERSIST_TRAFFIC_RATIO[qt] * k_bytes) if qt in PERSIST_TRAFFIC_RATIO else None),
                "traffic_note": ("ncu dram__bytes_read.sum + dram__bytes_write.sum of a "
                                 + ("4-layer" if qt == 8 else "2-layer")
                                 + " case of the same kernel, scaled to this launch's algorithmic bytes")
                                if qt in PERSIST_TRAFFIC_RATIO else "no capture of this instantiation",
                "bytes_per_launch": k_bytes, "avg_launch_us": round(k_ms * 1e3, 3),
                "timing": f"CUDA events on the compute stream around each of {n_probe} kernel launches "
                          f"(uncaptured steps right after the timed region, {round(probe_ms_step, 4)} ms/step there)"}
    pos_base += n_probe

    # --------------------------- GEMV phases inside the step (persistent kernel)
    in_step = None
    if persistent:
        n_ph = 2 + 5 * L
        grid = ntx.ntx_engine_set_phase_probe(eng, None, 0)
        ts = torch.zeros((1 + n_ph) * grid, dtype=torch.int64, device="cuda")
        ntx.ntx_engine_set_phase_probe(eng, ts, ts.numel())
        spans = []
        n_phase_steps = min(args.steps, 8)
        for i in range(n_phase_steps):
            with torch.cuda.stream(cs):
                ntx.ntx_decode_step(eng, -1, pos_of(pos_base + i), None, next_tok, ntx.NTX_NO_GRAPH, None)
            cs.synchronize()
            t = ts.cpu().numpy().reshape(1 + n_ph, grid)
            done = t[1:].max(axis=1)  # phase p complete when its last CTA published it
            spans.append(np.diff(np.concatenate([[t[0].min()], done])) / 1e3)  # us per phase
        ntx.ntx_engine_set_phase_probe(eng, None, 0)
        pos_base += n_phase_steps
        spans = np.array(spans)  # [steps][phases]
        H, F, Hq, Hkv, D = d["hidden"], d["ffn"], d["n_heads"], d["n_kv_heads"], d["head_dim"]
        kinds = {"q/k/v (RMSNorm, RoPE, KV append)": (0, (Hq + 2 * Hkv) * D, H),
                 "o (+ residual)": (2, H, Hq * D),
                 "gate/up (RMSNorm, SwiGLU)": (3, 2 * F, H),
                 "down (+ residual, cosine statistics)": (4, H, F)}
        in_step = []
        for name, (j, M, K) in kinds.items():
            us = float(spans[:, [1 + 5 * k + j for k in range(L)]].mean())
            by = wl.mat_bytes(qt, M, K)
            in_step.append({"phase": name, "M": M, "K": K, "weight_bytes": by, "us": round(us, 3),
                            "GBs": round(by / (us * 1e-6) / 1e9, 1), "frac": round(by / (us * 1e-6) / 1e9 / peak, 4)})
        us = float(spans[:, 1 + 5 * L].mean())
        by = wl.mat_bytes(hqt, d["vocab"], H)
        in_step.append({"phase": "head (final RMSNorm, argmax)", "M": d["vocab"], "K": H, "weight_bytes": by,
                        "us": round(us, 3), "GBs": round(by / (us * 1e-6) / 1e9, 1),
                        "frac": round(by / (us * 1e-6) / 1e9 / peak, 4)})
        in_step = {"phases": in_step,
                   "attention_us": round(float(spans[:, [2 + 5 * k for k in range(L)]].mean()), 3),
                   "embed_us": round(float(spans[:, 0].mean()), 3),
                   "timing": f"%globaltimer per CTA at each phase's publication, {n_phase_steps} uncaptured steps; "
                             "a phase's time runs from the previous phase's last publication to its own last one "
                             "(grid barrier, x staging and the epilogue tail included)"}

    # ------------------------------------------- the per-op kernel chain, for comparison
    chain = None
    if not args.no_chain:
        n_chain = min(args.steps, 256)
        with torch.cuda.stream(cs):
            for i in range(3):
                ntx.ntx_decode_step(eng, -1, pos_of(pos_base + i), None, next_tok, ntx.NTX_NO_PERSIST, None)
        pos_base += 3
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(cs):
            c0.record(cs)
            for i in range(n_chain):
                ntx.ntx_decode_step(eng, -1, pos_of(pos_base + i), None, next_tok, ntx.NTX_NO_PERSIST, None)
            c1.record(cs)
        cs.synchronize()
        pos_base += n_chain
        chain_launches = ntx.ntx_engine_launches_per_step(eng)
        gdurs, gprobe_ms = probe(ntx.NTX_NO_PERSIST, L, n_probe, pos_base)
        pos_base += n_probe
        gu_ms = statistics.mean(gdurs)
        gu_bytes = 2 * wl.mat_bytes(qt, F, H) + 2 * 4 * H + 4 * F + 4 * 4 * 148  # weights, h1 + norm, u, stats
        chain = {"tok_s": round(n_chain / (c0.elapsed_time(c1) / 1e3), 3), "steps": n_chain,
                 "launches_per_step": chain_launches,
                 "gate_up_gemv": {"achieved": round(gu_bytes / (gu_ms * 1e-3) / 1e9, 1),
                                  "frac": round(gu_bytes / (gu_ms * 1e-3) / 1e9 / peak, 4),
                                  "bytes_per_launch": gu_bytes, "avg_launch_us": round(gu_ms * 1e3, 3),
                                  "timing": f"CUDA events around every gate/up launch of {n_probe} kernel-by-kernel "
                                            f"steps ({round(gprobe_ms, 4)} ms/step there)"}}
        if not persistent:
            roof = {"bound": "hbm", "kernel": "gate/up GEMV (RMSNorm prologue + SwiGLU epilogue)",
                    "achieved": chain["gate_up_gemv"]["achieved"], "peak": peak, "peak_kind": peak_kind,
                    "unit": "GB/s", "frac": chain["gate_up_gemv"]["frac"], "traffic": args.traffic,
                    "bytes_per_launch": gu_bytes, "avg_launch_us": round(gu_ms * 1e3, 3),
                    "timing": chain["gate_up_gemv"]["timing"]}
    elif not persistent:
        raise SystemExit("--no-chain needs the persistent kernel (all layers resident)")

    # ------------------------------------------------------------ e2e
    host_tok = torch.zeros(1, dtype=torch.int32, pin_memory=True)
    n_e2e = min(args.steps, 256)
    tok = int(prompt[-1])
    dist.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    with torch.cuda.stream(cs):
        for i in range(n_e2e):
            ntx.ntx_decode_step(eng, tok, pos_of(pos_base + i), None, next_tok, 0, None)
            host_tok.copy_(next_tok, non_blocking=True)
            cs.synchronize()
            tok = int(host_tok[0])
    e2e_s = dist.max(time.perf_counter() - t0)
    e2e_value = dist.world * n_e2e / e2e_s

    # ------------------------------------------------------------ GEMV sweep
    gemv = [] if args.no_gemv else gemv_sweep(ntx, sg, wl, torch, peak)

    # ------------------------------------------------------------ CPU baseline
    cpu = None
    if not args.no_cpu_baseline and dist.rank == 0 and dist.world == 1:
        cpu = cpu_baseline_from_model(m, wk, d, pos_of(0))

    bpt = wl.bytes_per_token(d, qt, hqt, p_first + span // 2)
    # ------------------------------------------------- host link (tier-B layers)
    host_link = None
    if any(tier_map):
        streamed = sum(tier_map) * m.blob_bytes  # every host layer crosses the link once per step (no skip set)
        link_peak = h2d_peak_gbs(torch)
        link_gbs = streamed / (ms_step * 1e-3) / 1e9
        host_link = {"streamed_bytes_per_step": streamed, "h2d_gbs": round(link_gbs, 1),
                     "peak_gbs": round(link_peak, 1), "frac": round(link_gbs / link_peak, 4),
                     "timing": "streamed bytes over the whole step time: a lower bound on the copy stream's rate "
                               "(the step is bound by its copies; the compute stream waits on them)",
                     "peak_how": "pinned host -> device cudaMemcpyAsync of 1 GiB on its own stream, best of 10, "
                                 "CUDA events"}
    ntx.ntx_engine_destroy(eng)
    torch.cuda.synchronize()
    desc = wk["desc"] if args.layers is None else f"{wk['desc']} -- layer count overridden to {L} (profiling only)"
    out = {
        "metric": METRIC, "value": round(value, 3), "unit": "tok/s", "n_gpus": dist.world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded; random-init weights of the named shapes)",
        "config": {"workload": desc, "weights": {8: "Q8_0", 14: "Q6_K", 2: "Q4_0"}[qt], "layers": L,
                   "hidden": d["hidden"], "ffn": d["ffn"], "vocab": d["vocab"], "batch": 1,
                   "parallelism": f"replicas x{dist.world}" if dist.world > 1 else "single GPU",
                   "l2": "weights per step >> 126 MB L2 (inputs larger than L2; no flush)",
                   "graph": ("one CUDA graph per step: parameter copy, sync-word reset, one persistent kernel"
                             if persistent else "one CUDA graph per step, PDL between kernels")},
        "roofline": roof,
        "decode_roofline": {"bytes_per_token": bpt, "peak": peak, "unit": "GB/s",
                            "roofline_tok_s": round(peak * 1e9 / bpt, 2),
                            "frac": round(value / dist.world / (peak * 1e9 / bpt), 4),
                            "achieved_gbs": round(bpt * value / dist.world / 1e9, 1)},
        "e2e": {"value": round(e2e_value, 3), "unit": "tok/s", "h2d_bytes_per_step": 8, "d2h_bytes_per_step": 4,
                "steps": n_e2e, "how": "ntx_decode_step with the token passed from the host each step (pinned H2D "
                                      "of position+token), next token read back to pinned host memory and "
                                      "synchronised before the next step"},
        "gpu_launches": launches * args.steps,
        "launches_per_step": launches,
        "clocks": clk,
        "gemv": gemv,
        "gemv_in_step": in_step,
        "chain": chain,
        "host_link": host_link,
        "cpu_baseline": cpu,
    }
    return out


def h2d_peak_gbs(torch, nbytes=1 << 30, reps=10):
    """Host-link peak: one pinned-host -> device copy of nbytes on a stream of
    its own, the best of reps, timed with CUDA events on that stream."""
    src = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    dst = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    best = float("inf")
    with torch.cuda.stream(s):
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            dst.copy_(src, non_blocking=True)
            e1.record(s)
            e1.synchronize()
            best = min(best, e0.elapsed_time(e1))
    del src, dst
    return nbytes / (best * 1e-3) / 1e9


def time_gemv(ntx, sg, wl, torch, qt, M, K, reps=40, pdl=False):
    """Device time of one GEMV: `n` back-to-back launches over rotating weight
    copies (more than 3x L2 in total) captured in one CUDA graph, replayed, so
    the host's per-call cost does not set the pace.  pdl: launches made with
    programmatic dependent launch (ntx_set_gemv_pdl), so each GEMV starts
    streaming its weights while the previous one drains."""
    L2 = 126 * 2 ** 20
    wbytes = wl.mat_bytes(qt, M, K)
    ncopy = max(2, (3 * L2) // wbytes + 1)
    n = max(reps, ncopy)
    Ws = []
    for i in range(ncopy):
        w = torch.empty(wbytes, dtype=torch.uint8, device="cuda")
        sg.dev_quant_rows(qt, 99, f"bench{i}", M, K, w.data_ptr())
        Ws.append(w)
    x = torch.randn(K, device="cuda")
    y = torch.empty(M, device="cuda")
    s = torch.cuda.current_stream()
    torch.cuda.synchronize()
    ntx.ntx_set_gemv_pdl(1 if pdl else 0)
    try:
        for i in range(4):
            ntx.ntx_gemv_q(qt, Ws[i % ncopy], M, K, x, y, None, s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            cap = torch.cuda.current_stream()
            for i in range(n):
                ntx.ntx_gemv_q(qt, Ws[i % ncopy], M, K, x, y, None, cap)
    finally:
        ntx.ntx_set_gemv_pdl(0)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    replays = 3
    e0.record(s)
    for _ in range(replays):
        g.replay()
    e1.record(s)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / (replays * n)
    del g, Ws
    torch.cuda.empty_cache()
    return ms, wbytes + 4 * K + 4 * M, ncopy


def gemv_sweep(ntx, sg, wl, torch, peak):
    shapes = [(8, 4096, 4096, "Q8_0 GEMV 4096x4096, batch 1")] + [(2, M, K, "Q4_0 GEMV sweep over Llama-3-8B projection shapes, batch 1") for M, K in wl.Q4_0_SWEEP]
    out = []
    for qt, M, K, name in shapes:
        ms, nbytes, ncopy = time_gemv(ntx, sg, wl, torch, qt, M, K, pdl=True)
        ms_s, _, _ = time_gemv(ntx, sg, wl, torch, qt, M, K, pdl=False)
        gbs = nbytes / (ms * 1e-3) / 1e9
        gbs_s = nbytes / (ms_s * 1e-3) / 1e9
        out.append({"workload": name, "qtype": {8: "Q8_0", 2: "Q4_0"}[qt], "M": M, "K": K, "us": round(ms * 1e3, 3),
                    "GBs": round(gbs, 1), "frac": round(gbs / peak, 4),
                    "launch": "programmatic dependent launch (ntx_set_gemv_pdl(1))",
                    "us_serial": round(ms_s * 1e3, 3), "frac_serial": round(gbs_s / peak, 4),
                    "rotation": f"{ncopy} weight copies (>3x L2), back-to-back launches in one CUDA graph"})
    return out


# ---------------------------------------------------------------- CPU oracle
def oracle_sample_step(orc, m_host_layer, d, qt, hqt, head_rows, final_norm, emb, pos, nthreads, max_ctx):
    """One layer of the oracle at position pos plus the head over head_rows rows."""
    import numpy as np
    ocfg = orc.make_config(d["hidden"], d["n_heads"], d["n_kv_heads"], d["head_dim"], d["ffn"], d["vocab"], 1,
                           d["eps"], d["theta"], max_ctx)
    kc = np.zeros((d["n_kv_heads"], max_ctx, d["head_dim"]), dtype=np.uint16)
    vc = np.zeros_like(kc)
    h = orc.embed(emb, d["hidden"], 1)
    t0 = time.perf_counter()
    h2, _ = orc.layer(ocfg, qt, m_host_layer, m_host_layer["attn_norm"], m_host_layer["ffn_norm"], kc, vc, h, pos,
                      nthreads)
    hc = orc.make_config(d["hidden"], d["n_heads"], d["n_kv_heads"], d["head_dim"], d["ffn"], head_rows.shape[0], 1,
                         d["eps"], d["theta"], max_ctx)
    orc.head(hc, hqt, head_rows, final_norm, h2, nthreads)
    return time.perf_counter() - t0


def cpu_baseline_from_model(m, wk, d, pos):
    """The oracle as it stands on the host cores, on one sample: layer 0 plus
    1/32 of the head rows at a decode position, scaled to one whole token."""
    import oracle as orc
    L = d["n_layers"]
    cores = os.cpu_count() or 1
    lt = m.host_layer_tensors(0)
    head = m.host_head()
    rows = head[: max(1, d["vocab"] // L)]
    emb = m.host_embed()[: 4 * d["hidden"]]
    fn = m.host_final_norm()
    t = oracle_sample_step(orc, lt, d, wk["qtype"], wk["head_qtype"], rows, fn, emb, pos, cores, wk["max_ctx"])
    per_token = t * L
    return {"value": round(1.0 / per_token, 5), "unit": "tok/s", "cores": cores, "kind": "oracle",
            "sample": f"one decode layer (layer 0, position {pos}) + 1/{L} of the head rows, timed once on "
                      f"{cores} threads and scaled x{L} to a whole token ({t:.3f} s per sample)"}


def run_reference(args, dist: Dist):
    """The CPU oracle as the reference arm (rank 0 only)."""
    import oracle as orc
    import synthgen as sg
    from synthgen import workloads as wl

    wk = WORKLOADS[args.workload]
    d = dict(getattr(wl, wk["model"]))
    if args.layers is not None:
        d["n_layers"] = args.layers
    L = d["n_layers"]
    qt, hqt = wk["qtype"], wk["head_qtype"]
    sd = wl.seed(wk["workload_id"])
    cores = os.cpu_count() or 1
    lt = wl.host_layer(d, qt, sd, 0, nthreads=cores)
    nrows = max(1, d["vocab"] // L)
    head_rows = sg.quant_rows(hqt, sd, "head", d["vocab"], d["hidden"], sigma=wl.W_SIGMA, row0=0, nrows=nrows,
                              nthreads=cores)
    fn = sg.fill_f32(sd, "final_norm", d["hidden"], mean=1.0, sigma=wl.NORM_SIGMA)
    emb = sg.fill_f16(sd, "embed", 4 * d["hidden"], 0.0, wl.EMB_SIGMA)
    p_first = wk["n_prior"] + wk["prompt"]
    span = wk["max_ctx"] - p_first
    times = []
    for i in range(args.warmup + args.steps):
        pos = p_first + (i % span)
        t = oracle_sample_step(orc, lt, d, qt, hqt, head_rows, fn, emb, pos, cores, wk["max_ctx"])
        if i >= args.warmup:
            times.append(t * L)
    total = sum(times)
    value = args.steps / total
    return {"metric": METRIC, "value": round(value, 5), "unit": "tok/s", "n_gpus": dist.world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * total / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded; random-init weights of the named shapes)",
            "config": {"workload": wk["desc"], "weights": {8: "Q8_0", 14: "Q6_K", 2: "Q4_0"}[qt], "layers": L,
                       "hidden": d["hidden"], "ffn": d["ffn"], "vocab": d["vocab"], "batch": 1},
            "impl": "reference",
            "cpu_baseline": {"value": round(value, 5), "unit": "tok/s", "cores": cores, "kind": "oracle",
                             "sample": f"each step: one decode layer + 1/{L} of the head rows on {cores} threads, "
                                       f"scaled x{L} to a whole token"},
            "e2e": {"value": round(value, 5), "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1024)
    ap.add_argument("--warmup", type=int, default=16)
    ap.add_argument("--impl", choices=["ntx", "reference"], default="ntx")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="llama8b-q8_0")
    ap.add_argument("--no-gemv", action="store_true", help="skip the standalone Q8_0 / Q4_0 GEMV sweep")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-chain", action="store_true", help="skip timing the per-op kernel chain for comparison")
    ap.add_argument("--layers", type=int, default=None,
                    help="profiling only: run the workload's model with this many layers (the line then describes "
                         "that smaller model and is not a benchmark of the named workload)")
    ap.add_argument("--traffic", type=float, default=None,
                    help="DRAM bytes per launch of the dominant kernel from an ncu capture (reported as is)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return 0
        out = run_reference(args, type("D", (), {"world": world})())
        print(json.dumps(out), flush=True)
        return 0
    dist = Dist(args.gpus)
    try:
        out = run_ntx(args, dist)
        if dist.rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        dist.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
