#!/usr/bin/env python
"""Batch-1 decode benchmark of libntx on B200.

Headline workload (value, e2e, roofline): the 32-layer Llama-3-8B-shaped Q8_0
model, all layers resident in HBM, 16-token prompt then greedy decode with the
fp16 KV cache growing to 144 positions (positions 16..143 are reused
cyclically when more steps are timed).  A step is one token through the whole
hot path: embed, 32 x (RMSNorm + QKV GEMV + RoPE + KV append, split-KV GQA
attention, O GEMV + residual, RMSNorm + gate/up GEMV + SwiGLU, down GEMV +
residual + cosine statistics), final RMSNorm + head GEMV, argmax.  Weights
(7.97 GB) are far larger than the 126 MB L2, so no flush is needed between
steps.

The same JSON line also carries, under "configs", the 80-layer
Llama-3-70B-shaped Q6_K model with 2048 prior KV positions: resident (5a) and
tiered with layers 40-79 in pinned host memory streamed through two device
slots (5b), each without and with the cosine layer skip at 0.98, and the
tiered run's host-link figures; under "gemv", standalone quantized GEMVs.

Timed region of the headline: K kernel-by-kernel steps (no graph), CUDA events
on the compute stream around the whole region and around the persistent kernel
of every step, so the kernel time and the step time come from the same region
(a graph-replayed region of the same length is reported beside it).

Prints one JSON line.  Under torchrun each rank runs an independent replica
on its own GPU (the path has no data-path collective); value = tokens of all
ranks / the slowest rank's device time.

--impl reference times the CPU oracle (fp64, the tests' reference
implementation) on the headline workload: each step is one whole token
through every layer and the head, on all host cores, the prompt fed first and
the oracle's own greedy tokens after it.
"""
from __future__ import annotations

import argparse
import json
import os
import platform
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
# 1,485,863,680 + 4,421,632 bytes against 1,485,578,240 algorithmic bytes;
# Q6_K, 2 layers of the 70B shapes, 2,283,495,936 + 4,485,632 bytes against
# 2,282,659,840.  The kernel streams every weight byte once, so a full
# launch's traffic is this ratio times its algorithmic bytes.
PERSIST_TRAFFIC_RATIO = {8: (1485863680 + 4421632) / 1485578240, 14: (2283495936 + 4485632) / 2282659840}
FALLBACK_HBM_GBS = 6650.0


SPEC_HBM_GBS = 8000.0  # the ~8 TB/s HBM3e figure decode rooflines are usually quoted against


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
                         prompt=16),
    "llama70b-q6_k": dict(desc="Llama-3-70B-shaped 80-layer Q6_K model (Q6_K head), 2048 prior KV positions, "
                               "greedy batch-1 decode from position 2048; resident, and tiered with layers 40-79 in "
                               "pinned host RAM streamed through two device slots",
                          model="MODEL_70B", qtype=14, head_qtype=14, workload_id=5, max_ctx=2080, n_prior=2048,
                          prompt=1),
    "llama70b-q4_k_m": dict(desc="Llama-3-70B-shaped 80-layer Q4_K_M model (Q4_K matrices, Q6_K down projections "
                                 "and head), 2048 prior KV positions, greedy batch-1 decode from position 2048, "
                                 "resident",
                            model="MODEL_70B", qtype=(12, 12, 12, 12, 12, 12, 14), head_qtype=14, workload_id=5,
                            max_ctx=2080, n_prior=2048, prompt=1),
}
QNAME = {8: "Q8_0", 14: "Q6_K", 2: "Q4_0", 12: "Q4_K", 13: "Q5_K", 1: "F16", 0: "F32"}


def qname(qt) -> str:
    """Name of one block type, or of a per-matrix mix (wq..wd)."""
    if isinstance(qt, (list, tuple)):
        return "Q4_K_M" if tuple(qt) == (12, 12, 12, 12, 12, 12, 14) else "/".join(QNAME[t] for t in qt)
    return QNAME[qt]


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


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ---------------------------------------------------------------- engine runs
class Run:
    """An engine over a DeviceModel on its own compute stream (plus a copy
    stream when some layer lives in pinned host memory)."""

    def __init__(self, ntx, torch, m, d, L, qt, hqt, max_ctx, tier_map, resident_layers=False):
        self.ntx, self.torch = ntx, torch
        self.cfg = ntx.make_config(d["hidden"], d["n_heads"], d["n_kv_heads"], d["head_dim"], d["ffn"], d["vocab"],
                                   L, d["eps"], d["theta"], max_ctx, 0.98)
        layers = []
        for l in range(L):
            _, lw = (ntx.ntx_layer_layout_mixed(self.cfg, qt) if isinstance(qt, (list, tuple))
                     else ntx.ntx_layer_layout(self.cfg, qt))
            src = m.resident_copy[l] if (resident_layers or tier_map[l] == 0) else m.layers[l]
            lw.base = src.data_ptr()
            layers.append(lw)
        self.tier_map = [0] * L if resident_layers else list(tier_map)
        self.ws_bytes = ntx.ntx_engine_workspace_bytes(self.cfg)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device="cuda")
        self.cs = torch.cuda.Stream()
        self.xs = torch.cuda.Stream() if any(self.tier_map) else None
        self.eng = ntx.ntx_engine_create(self.cfg, layers, self.tier_map, m.slots[0], m.slots[1], m.blob_bytes,
                                         m.embed, m.final_norm, m.head, hqt, m.k_caches, m.v_caches, self.ws,
                                         self.ws_bytes, self.cs, self.xs)
        self.next_tok = torch.zeros(1, dtype=torch.int32, device="cuda")

    def steps(self, tokens, positions, flags=0):
        with self.torch.cuda.stream(self.cs):
            for t, p in zip(tokens, positions):
                self.ntx.ntx_decode_step(self.eng, int(t), int(p), None, self.next_tok, flags, None)

    def timed(self, positions, flags=0, kernel_events=True):
        """Kernel-by-kernel steps (token -1 = the previous greedy token) with
        CUDA events on the compute stream around the region and, when the step
        is one persistent kernel, around that kernel in every step.  Returns
        (region ms, [kernel ms per step] or None)."""
        torch, ntx = self.torch, self.ntx
        n = len(positions)
        ev = (lambda: torch.cuda.Event(enable_timing=True))
        kb = [ev() for _ in range(n)] if kernel_events else []
        ke = [ev() for _ in range(n)] if kernel_events else []
        with torch.cuda.stream(self.cs):
            for e in kb + ke:
                e.record(self.cs)  # creates the CUDA events before the region
        self.cs.synchronize()
        e0, e1 = ev(), ev()
        with torch.cuda.stream(self.cs):
            e0.record(self.cs)
            for i, p in enumerate(positions):
                if kernel_events:
                    ntx.ntx_engine_set_probe(self.eng, [kb[i].cuda_event], [ke[i].cuda_event])
                ntx.ntx_decode_step(self.eng, -1, int(p), None, self.next_tok, flags | ntx.NTX_NO_GRAPH, None)
            e1.record(self.cs)
            if kernel_events:
                ntx.ntx_engine_set_probe(self.eng, [], [])
        self.cs.synchronize()
        ks = [kb[i].elapsed_time(ke[i]) for i in range(n)] if kernel_events else None
        return e0.elapsed_time(e1), ks

    def graph_timed(self, positions, flags=0):
        """The same steps replayed from the engine's captured CUDA graph."""
        torch = self.torch
        with torch.cuda.stream(self.cs):
            self.ntx.ntx_decode_step(self.eng, -1, int(positions[0]), None, self.next_tok, flags, None)  # capture
        self.cs.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(self.cs):
            e0.record(self.cs)
            for p in positions:
                self.ntx.ntx_decode_step(self.eng, -1, int(p), None, self.next_tok, flags, None)
            e1.record(self.cs)
        self.cs.synchronize()
        return e0.elapsed_time(e1)

    def e2e(self, first_token, positions, flags=0):
        """Through the public API as a user calls it: the token goes from the
        host each step (pinned H2D of position + token inside the call), the
        next token is read back to pinned host memory and synchronised on."""
        torch, ntx = self.torch, self.ntx
        host_tok = torch.zeros(1, dtype=torch.int32, pin_memory=True)
        tok = int(first_token)
        with torch.cuda.stream(self.cs):
            ntx.ntx_decode_step(self.eng, tok, int(positions[0]), None, self.next_tok, flags, None)  # capture
        self.cs.synchronize()
        t0 = time.perf_counter()
        with torch.cuda.stream(self.cs):
            for p in positions:
                ntx.ntx_decode_step(self.eng, tok, int(p), None, self.next_tok, flags, None)
                host_tok.copy_(self.next_tok, non_blocking=True)
                self.cs.synchronize()
                tok = int(host_tok[0])
        return time.perf_counter() - t0

    def phases(self, positions, L_run, d, qt, hqt, peak, flags=0):
        """Per-phase times of the persistent kernel from its %globaltimer probe."""
        import numpy as np
        torch, ntx = self.torch, self.ntx
        grid = ntx.ntx_engine_set_phase_probe(self.eng, None, 0)
        if grid <= 0:
            return None
        n_ph = 2 + 5 * L_run
        ts = torch.zeros((1 + n_ph) * grid, dtype=torch.int64, device="cuda")
        ntx.ntx_engine_set_phase_probe(self.eng, ts, ts.numel())
        spans = []
        for p in positions:
            with torch.cuda.stream(self.cs):
                ntx.ntx_decode_step(self.eng, -1, int(p), None, self.next_tok, flags | ntx.NTX_NO_GRAPH, None)
            self.cs.synchronize()
            t = ts.cpu().numpy().reshape(1 + n_ph, grid)
            done = t[1:].max(axis=1)  # phase p complete when its last CTA published it
            spans.append(np.diff(np.concatenate([[t[0].min()], done])) / 1e3)  # us per phase
        ntx.ntx_engine_set_phase_probe(self.eng, None, 0)
        spans = np.array(spans)
        H, F, Hq, Hkv, D = d["hidden"], d["ffn"], d["n_heads"], d["n_kv_heads"], d["head_dim"]
        from synthgen import workloads as wl
        kinds = {"q/k/v (RMSNorm, RoPE, KV append)": (0, (Hq + 2 * Hkv) * D, H, 0),
                 "o (+ residual)": (2, H, Hq * D, 3),
                 "gate/up (RMSNorm, SwiGLU)": (3, 2 * F, H, 4),
                 "down (+ residual, cosine statistics)": (4, H, F, 6)}
        out = []
        for name, (j, M, K, mi) in kinds.items():
            us = float(spans[:, [1 + 5 * k + j for k in range(L_run)]].mean())
            by = wl.mat_bytes(wl.mat_types(qt)[mi], M, K)
            out.append({"phase": name, "M": M, "K": K, "weight_bytes": by, "us": round(us, 3),
                        "GBs": round(by / (us * 1e-6) / 1e9, 1), "frac": round(by / (us * 1e-6) / 1e9 / peak, 4)})
        us = float(spans[:, 1 + 5 * L_run].mean())
        by = wl.mat_bytes(hqt, d["vocab"], H)
        out.append({"phase": "head (final RMSNorm, argmax)", "M": d["vocab"], "K": H, "weight_bytes": by,
                    "us": round(us, 3), "GBs": round(by / (us * 1e-6) / 1e9, 1),
                    "frac": round(by / (us * 1e-6) / 1e9 / peak, 4)})
        return {"phases": out,
                "attention_us": round(float(spans[:, [2 + 5 * k for k in range(L_run)]].mean()), 3),
                "embed_us": round(float(spans[:, 0].mean()), 3),
                "timing": f"%globaltimer per CTA at each phase's publication, {len(positions)} uncaptured steps; "
                          "a phase's time runs from the previous phase's last publication to its own last one "
                          "(grid barrier, x staging and the epilogue tail included)"}

    def close(self):
        self.ntx.ntx_engine_destroy(self.eng)
        self.torch.cuda.synchronize()


def roofline(k_ms_list, k_bytes, peak, peak_kind, qt, traffic_arg, region_ms_step, what):
    k_ms = statistics.mean(k_ms_list)
    gbs = k_bytes / (k_ms * 1e-3) / 1e9
    if k_ms > region_ms_step * (1 + 1e-9):
        raise RuntimeError(f"kernel time {k_ms} ms exceeds the step time {region_ms_step} ms of the same region")
    return {"bound": "hbm", "kernel": "persistent decode-step kernel (one launch per token)",
            "achieved": round(gbs, 1), "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
            "frac": round(gbs / peak, 4),
            "traffic": traffic_arg if traffic_arg is not None else (
                round(PERSIST_TRAFFIC_RATIO[qt] * k_bytes) if qt in PERSIST_TRAFFIC_RATIO else None),
            "traffic_note": ("ncu dram__bytes_read.sum + dram__bytes_write.sum of a "
                             + ("4-layer" if qt == 8 else "2-layer")
                             + " case of the same kernel, scaled to this launch's algorithmic bytes")
                            if qt in PERSIST_TRAFFIC_RATIO else "no capture of this instantiation",
            "bytes_per_launch": k_bytes, "avg_launch_us": round(k_ms * 1e3, 3),
            "timing": f"CUDA events on the compute stream around the kernel of each of the {len(k_ms_list)} steps "
                      f"of {what} (step time there {round(region_ms_step * 1e3, 3)} us)"}


# ---------------------------------------------------------------- headline (8B)
def run_ntx(args, dist: Dist):
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
    m = DeviceModel(d, qt, hqt, sd, wk["max_ctx"], wk["n_prior"], source="device")
    if args.persist_two:
        ntx.ntx_set_persist_two_types(1)  # read when the engine is created
    try:
        r = Run(ntx, torch, m, d, L, qt, hqt, wk["max_ctx"], [0] * L)
    finally:
        ntx.ntx_set_persist_two_types(0)
    prompt = sg.tokens(sd, "prompt", wk["prompt"], d["vocab"])
    p_first = wk["n_prior"] + wk["prompt"]
    span = wk["max_ctx"] - p_first

    def pos_of(i):  # i-th decode step after the prompt
        return p_first + (i % span)

    r.steps(prompt, range(wk["n_prior"], p_first))
    r.steps([-1] * args.warmup, [pos_of(i) for i in range(args.warmup)])
    r.cs.synchronize()
    launches = ntx.ntx_engine_launches_per_step(r.eng)
    persistent = launches <= 2  # one persistent kernel (+ cosine finalisation when asked)
    peak, peak_kind = measured_peaks()

    # ------------------------------------------------------------ timed region
    positions = [pos_of(args.warmup + i) for i in range(args.steps)]
    clocks = ClockSampler(dev_index)
    clocks.start()
    dist.barrier()
    torch.cuda.synchronize()
    ms_local, kms = r.timed(positions, kernel_events=persistent)
    torch.cuda.synchronize()
    dist.barrier()
    clk = clocks.stop()
    ms_total = dist.max(ms_local)
    status = ntx.ntx_device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")
    ms_step = ms_total / args.steps
    value = whole_job_rate(dist.world, args.steps, ms_total)
    pos_base = args.warmup + args.steps

    roof = None
    if persistent:
        n_ctx_mean = statistics.mean(p + 1 for p in positions)
        k_bytes = wl.bytes_per_token(d, qt, hqt, int(round(n_ctx_mean)))
        roof = roofline(kms, k_bytes, peak, peak_kind, qt, args.traffic, ms_local / args.steps, "the timed region")
        # the same achieved rate against the three denominators: the copy peak above, the ~8 TB/s HBM3e
        # figure, and the read-only bandwidth measured here
        rp = hbm_read_peak(ntx, torch)
        roof["denominators"] = {
            "copy": {"gbs": peak, "kind": peak_kind, "frac": roof["frac"]},
            "spec": {"gbs": SPEC_HBM_GBS, "frac": round(roof["achieved"] / SPEC_HBM_GBS, 4)},
            "read_probe": dict(rp, frac=round(roof["achieved"] / rp["median_gbs"], 4))}

    # the same number of steps replayed from the captured graph, for comparison
    g_positions = [pos_of(pos_base + i) for i in range(args.steps)]
    g_ms = r.graph_timed(g_positions)
    pos_base += args.steps + 1

    in_step = None
    if persistent:
        n_ph = min(args.steps, 8)
        in_step = r.phases([pos_of(pos_base + i) for i in range(n_ph)], L, d, qt, hqt, peak)
        pos_base += n_ph

    # ------------------------------------------- the per-op kernel chain, for comparison
    chain = None
    if not args.no_chain:
        n_chain = min(args.steps, 256)
        r.steps([-1] * 3, [pos_of(pos_base + i) for i in range(3)], ntx.NTX_NO_PERSIST)
        pos_base += 3
        c_ms, _ = r.timed([pos_of(pos_base + i) for i in range(n_chain)], ntx.NTX_NO_PERSIST, kernel_events=False)
        pos_base += n_chain
        chain = {"tok_s": round(n_chain / (c_ms / 1e3), 3), "steps": n_chain,
                 "launches_per_step": ntx.ntx_engine_launches_per_step(r.eng),
                 "timing": "CUDA events around kernel-by-kernel steps of the per-op chain (NTX_NO_PERSIST)"}
        r.steps([-1], [pos_of(pos_base)])  # leave the engine's last step on the persistent kernel
        pos_base += 1

    # ------------------------------------------------------------ e2e
    n_e2e = min(args.steps, 256)
    dist.barrier()
    torch.cuda.synchronize()
    e2e_s = dist.max(r.e2e(prompt[-1], [pos_of(pos_base + i) for i in range(n_e2e)]))
    e2e_value = dist.world * n_e2e / e2e_s
    pos_base += n_e2e + 1

    # ------------------------------------------------------------ CPU baseline
    cpu = None
    if not args.no_cpu_baseline and dist.rank == 0 and dist.world == 1:
        cpu = cpu_baseline_8b(m, d, wk, prompt)
    r.close()
    del r, m
    torch.cuda.empty_cache()

    # ------------------------------------------------------------ GEMV sweep
    gemv = [] if args.no_gemv else gemv_sweep(ntx, sg, wl, torch, peak)

    # ------------------------------------------------------------ 70B configs
    configs = None
    if not args.no_70b and args.layers is None and dist.world == 1 and args.workload == "llama8b-q8_0":
        configs = run_70b(args, dist, ntx, torch, sg, wl, peak, peak_kind, dev_index)

    bpt = wl.bytes_per_token(d, qt, hqt, p_first + span // 2)
    desc = wk["desc"] if args.layers is None else f"{wk['desc']} -- layer count overridden to {L} (profiling only)"
    out = {
        "metric": METRIC, "value": round(value, 3), "unit": "tok/s", "n_gpus": dist.world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded; random-init weights of the named shapes)",
        "config": {"workload": desc, "weights": qname(qt), "layers": L, "hidden": d["hidden"], "ffn": d["ffn"],
                   "vocab": d["vocab"], "batch": 1, "persist_two_types": bool(args.persist_two),
                   "parallelism": f"replicas x{dist.world}" if dist.world > 1 else "single GPU",
                   "l2": "weights per step >> 126 MB L2 (inputs larger than L2; no flush)",
                   "graph": ("kernel-by-kernel steps: parameter copy, sync-word reset, one persistent kernel "
                             "bracketed by CUDA events" if persistent else
                             "kernel-by-kernel steps of the per-op chain, PDL between kernels")},
        "roofline": roof,
        "graph_replay": {"tok_s": round(dist.world * args.steps / (dist.max(g_ms) / 1e3), 3), "steps": args.steps,
                         "how": "the same step count replayed from the engine's captured CUDA graph"},
        "decode_roofline": {"bytes_per_token": bpt, "peak": peak, "unit": "GB/s",
                            "roofline_tok_s": round(peak * 1e9 / bpt, 2),
                            "frac": round(value / dist.world / (peak * 1e9 / bpt), 4),
                            "achieved_gbs": round(bpt * value / dist.world / 1e9, 1)},
        "e2e": {"value": round(e2e_value, 3), "unit": "tok/s", "h2d_bytes_per_step": 8, "d2h_bytes_per_step": 4,
                "steps": n_e2e, "how": "ntx_decode_step (graph replay) with the token passed from the host each "
                                      "step (pinned H2D of position+token), next token read back to pinned host "
                                      "memory and synchronised before the next step; host wall clock"},
        "gpu_launches": launches * args.steps,
        "launches_per_step": launches,
        "clocks": clk,
        "gemv": gemv,
        "gemv_in_step": in_step,
        "chain": chain,
        "configs": configs,
        "cpu_baseline": cpu,
    }
    return out


# ---------------------------------------------------------------- 70B (configs 5a / 5b)
def run_70b(args, dist, ntx, torch, sg, wl, peak, peak_kind, dev_index):
    """Config 5: the 80-layer 70B-shaped Q6_K model with 2048 prior KV
    positions.  5a: every layer resident (one persistent kernel per step).
    5b: layers 40-79 in pinned host memory, streamed through two device slots
    on a copy stream (per-op kernel chain).  Each without and with the cosine
    skip set calibrated on the first decode step (tau 0.98)."""
    from synthgen.devmodel import DeviceModel
    wk = WORKLOADS["llama70b-q6_k"]
    d = dict(wl.MODEL_70B)
    L = d["n_layers"]
    qt, hqt = wk["qtype"], wk["head_qtype"]
    sd = wl.seed(wk["workload_id"])
    tiers = [0] * 40 + [1] * 40
    t0 = time.perf_counter()
    m = DeviceModel(d, qt, hqt, sd, wk["max_ctx"], wk["n_prior"], tier_map=tiers, source="device",
                    keep_resident_copy=True)
    gen_s = time.perf_counter() - t0
    start = int(sg.tokens(sd, "prompt", 1, d["vocab"])[0])
    p0 = wk["n_prior"]
    span = wk["max_ctx"] - p0 - 1

    def pos_of(i):
        return p0 + 1 + (i % span)

    n_a = min(args.steps, 32)
    n_b = min(args.steps, 4)
    res = {"workload": wk["desc"], "generation_s": round(gen_s, 1)}

    # ---- 5a: resident
    ra = Run(ntx, torch, m, d, L, qt, hqt, wk["max_ctx"], tiers, resident_layers=True)
    ra.steps([start], [p0])
    ra.steps([-1] * args.warmup, [pos_of(i) for i in range(args.warmup)])
    pos = [pos_of(args.warmup + i) for i in range(n_a)]
    clocks = ClockSampler(dev_index)
    clocks.start()
    ms, kms = ra.timed(pos)
    clk = clocks.stop()
    launches = ntx.ntx_engine_launches_per_step(ra.eng)
    n_ctx = int(round(statistics.mean(p + 1 for p in pos)))
    k_bytes = wl.bytes_per_token(d, qt, hqt, n_ctx)
    a = {"value": round(n_a / (ms / 1e3), 3), "unit": "tok/s", "steps": n_a, "ms_per_step": round(ms / n_a, 4),
         "launches_per_step": launches, "clocks": clk,
         "roofline": roofline(kms, k_bytes, peak, peak_kind, qt, None, ms / n_a, "5a's timed region"),
         "decode_roofline": {"bytes_per_token": k_bytes, "roofline_tok_s": round(peak * 1e9 / k_bytes, 2),
                             "frac": round((n_a / (ms / 1e3)) / (peak * 1e9 / k_bytes), 4)}}
    a["gemv_in_step"] = ra.phases([pos_of(args.warmup + n_a + i) for i in range(4)], L, d, qt, hqt, peak)
    n_e = min(args.steps, 16)
    e_s = ra.e2e(start, [pos_of(i) for i in range(n_e)])
    a["e2e"] = {"value": round(n_e / e_s, 3), "unit": "tok/s", "h2d_bytes_per_step": 8, "d2h_bytes_per_step": 4,
                "steps": n_e}
    # calibrated skip set (first decode step, every layer computed)
    ra.steps([start], [p0], ntx.NTX_CALIBRATE_SKIP)
    mask = ntx.ntx_engine_skip_mask(ra.eng, L)
    executed = [l for l in range(L) if not mask[l]]
    ra.steps([-1] * 3, [pos_of(i) for i in range(3)], ntx.NTX_USE_SKIP)
    ms_s, kms_s = ra.timed([pos_of(3 + i) for i in range(n_a)], ntx.NTX_USE_SKIP)
    sk_bytes = wl.bytes_per_token(d, qt, hqt, n_ctx, layers=len(executed))
    a["with_skip"] = {"value": round(n_a / (ms_s / 1e3), 3), "unit": "tok/s", "steps": n_a,
                      "skipped_layers": L - len(executed), "skip_set": [l for l in range(L) if mask[l]],
                      "bytes_per_token": sk_bytes,
                      "roofline": roofline(kms_s, sk_bytes, peak, peak_kind, qt, None, ms_s / n_a,
                                           "5a+skip's timed region")}
    ra.close()
    del ra
    res["5a_resident"] = a

    # ---- 5b: tiered
    m.reset_kv()
    rb = Run(ntx, torch, m, d, L, qt, hqt, wk["max_ctx"], tiers)
    rb.steps([start], [p0])
    rb.steps([-1] * 3, [pos_of(i) for i in range(3)])
    clocks = ClockSampler(dev_index)
    clocks.start()
    ms_b, _ = rb.timed([pos_of(3 + i) for i in range(n_b)], kernel_events=False)
    clk_b = clocks.stop()
    streamed = 40 * m.blob_bytes  # every host layer crosses the link once per step (no skip set)
    link_peak = h2d_peak_gbs(torch)
    link_gbs = streamed / (ms_b / n_b * 1e-3) / 1e9
    b = {"value": round(n_b / (ms_b / 1e3), 3), "unit": "tok/s", "steps": n_b, "ms_per_step": round(ms_b / n_b, 3),
         "launches_per_step": ntx.ntx_engine_launches_per_step(rb.eng), "clocks": clk_b,
         "host_link": {"streamed_bytes_per_step": streamed, "h2d_gbs": round(link_gbs, 1),
                       "peak_gbs": round(link_peak, 1), "frac": round(link_gbs / link_peak, 4),
                       "timing": "streamed bytes over the whole step time: a lower bound on the copy stream's rate "
                                 "(the step is bound by its copies; the compute stream waits on them)",
                       "peak_how": "pinned host -> device cudaMemcpyAsync of 1 GiB on its own stream, best of 10, "
                                   "CUDA events"},
         "roofline_tok_s": round(link_peak * 1e9 / streamed, 3)}
    rb.steps([start], [p0], ntx.NTX_CALIBRATE_SKIP)
    mask_b = ntx.ntx_engine_skip_mask(rb.eng, L)
    host_run = [l for l in range(40, L) if not mask_b[l]]
    rb.steps([-1] * 3, [pos_of(i) for i in range(3)], ntx.NTX_USE_SKIP)
    n_bs = n_a if not host_run else n_b
    ms_bs, kms_bs = rb.timed([pos_of(3 + i) for i in range(n_bs)], ntx.NTX_USE_SKIP,
                             kernel_events=not host_run)
    b["with_skip"] = {"value": round(n_bs / (ms_bs / 1e3), 3), "unit": "tok/s", "steps": n_bs,
                      "skipped_layers": sum(mask_b), "host_layers_streamed": len(host_run),
                      "streamed_bytes_per_step": len(host_run) * m.blob_bytes,
                      "launches_per_step": ntx.ntx_engine_launches_per_step(rb.eng),
                      "note": ("every host layer is skipped: nothing crosses the link and the step runs as one "
                               "persistent kernel over the resident executed layers") if not host_run else
                              "the executed host layers stream through the slots"}
    # self-speculative decoding on the tiered engine: the resident layers 0-39 draft 3 tokens, the whole
    # model verifies the 4 in one pass that streams layers 40-79 once
    rb.steps([start], [p0])
    rb.cs.synchronize()
    n_calls, k = min(args.steps, 4), 3
    tok, pos, emitted, acc = start, p0 + 1, 0, []
    t0 = time.perf_counter()
    for _ in range(n_calls):
        got = ntx.ntx_decode_spec(rb.eng, tok, pos, k)
        acc.append(len(got) - 1)
        emitted += len(got)
        pos += len(got)
        tok = got[-1]
    spec_s = time.perf_counter() - t0
    b["self_spec"] = {"value": round(emitted / spec_s, 3), "unit": "tok/s", "draft_k": k, "calls": n_calls,
                      "tokens": emitted, "accepted_per_call": acc,
                      "how": "ntx_decode_spec on the tiered engine (draft = resident layers 0-39 + head, "
                             "verification streams layers 40-79 once per call); host wall clock, the call "
                             "waits for its tokens",
                      "note": "random-init weights: the draft rarely agrees with the whole model"}
    # the same after making layers 40-79 the identity (their O and down projections zeroed in the pinned
    # blobs): the draft is then the whole model, every proposal is accepted, and one verification pass's
    # stream of the host layers serves k + 1 tokens -- the other end of the acceptance range
    for l in range(40, L):
        for name in ("wo", "wd"):
            M_, K_ = wl.mat_shapes(d)[name]
            off = m.offsets[name]
            m.layers[l][off:off + wl.mat_bytes(qt, M_, K_)].zero_()
    rb.steps([start], [p0])
    rb.cs.synchronize()
    tok, pos, emitted_i, acc_i = start, p0 + 1, 0, []
    t0 = time.perf_counter()
    for _ in range(n_calls):
        got = ntx.ntx_decode_spec(rb.eng, tok, pos, k)
        acc_i.append(len(got) - 1)
        emitted_i += len(got)
        pos += len(got)
        tok = got[-1]
    spec_i = time.perf_counter() - t0
    b["self_spec"]["identity_host_layers"] = {
        "value": round(emitted_i / spec_i, 3), "unit": "tok/s", "calls": n_calls, "tokens": emitted_i,
        "accepted_per_call": acc_i,
        "how": "layers 40-79 made the identity (O and down projections zeroed), same engine and calls; plain "
               "decode streams the same bytes per token as above"}
    rb.close()
    del rb
    res["5b_tiered"] = b

    if not args.no_cpu_baseline and dist.rank == 0 and dist.world == 1:
        res["cpu_baseline"] = cpu_baseline_70b(m, d, wk, start)
    del m
    torch.cuda.empty_cache()

    # ---- 5c: the same shapes as Q4_K_M (Q4_K matrices, Q6_K down projections and head), resident
    qm = wl.Q4_K_M
    m = DeviceModel(d, qm, wl.Q4_K_M_HEAD, sd, wk["max_ctx"], wk["n_prior"], source="device")
    rc = Run(ntx, torch, m, d, L, qm, wl.Q4_K_M_HEAD, wk["max_ctx"], [0] * L)
    rc.steps([start], [p0])
    rc.steps([-1] * args.warmup, [pos_of(i) for i in range(args.warmup)])
    launches_c = ntx.ntx_engine_launches_per_step(rc.eng)
    persistent_c = launches_c <= 2
    ms_c, kms_c = rc.timed([pos_of(args.warmup + i) for i in range(n_a)], kernel_events=persistent_c)
    c_bytes = wl.bytes_per_token(d, qm, wl.Q4_K_M_HEAD, n_ctx)
    res["5c_q4_k_m_resident"] = {
        "value": round(n_a / (ms_c / 1e3), 3), "unit": "tok/s", "steps": n_a, "ms_per_step": round(ms_c / n_a, 4),
        "weights": "Q4_K (wq wk wv wo wg wu), Q6_K (wd, head)",
        "path": "persistent decode kernel" if persistent_c else
                "per-op kernel chain (the engine's default for two block types)",
        "launches_per_step": launches_c,
        "roofline": roofline(kms_c, c_bytes, peak, peak_kind, 12, None, ms_c / n_a, "5c's timed region")
                    if persistent_c else None,
        "decode_roofline": {"bytes_per_token": c_bytes, "roofline_tok_s": round(peak * 1e9 / c_bytes, 2),
                            "frac": round((n_a / (ms_c / 1e3)) / (peak * 1e9 / c_bytes), 4)}}
    rc.close()
    del rc
    # the two-type persistent kernel (opt-in), for comparison
    ntx.ntx_set_persist_two_types(1)
    try:
        rc = Run(ntx, torch, m, d, L, qm, wl.Q4_K_M_HEAD, wk["max_ctx"], [0] * L)
    finally:
        ntx.ntx_set_persist_two_types(0)
    rc.steps([-1] * args.warmup, [pos_of(i) for i in range(args.warmup)])
    ms_p, _ = rc.timed([pos_of(args.warmup + i) for i in range(n_a)], kernel_events=False)
    res["5c_q4_k_m_resident"]["two_type_persistent"] = {
        "value": round(n_a / (ms_p / 1e3), 3), "unit": "tok/s", "steps": n_a,
        "launches_per_step": ntx.ntx_engine_launches_per_step(rc.eng),
        "how": "ntx_set_persist_two_types(1): one persistent kernel with Q4_K and Q6_K row decoders",
        "gemv_in_step": rc.phases([pos_of(args.warmup + n_a + i) for i in range(4)], L, d, qm, wl.Q4_K_M_HEAD,
                                  peak)}
    rc.close()
    del rc, m
    torch.cuda.empty_cache()
    return res


def hbm_read_peak(ntx, torch, nbytes=4 << 30, reps=10):
    """Read-only HBM bandwidth measured here: ntx_hbm_read_probe over a
    buffer of ones 32x the L2, each launch timed with CUDA events on the
    current stream after two untimed ones; the probe's word sum is checked."""
    buf = torch.ones(nbytes // 4, dtype=torch.int32, device="cuda")
    out = torch.zeros(1, dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream()
    times = []
    for i in range(reps + 2):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        ntx.ntx_hbm_read_probe(buf, nbytes, out, s)
        e1.record(s)
        e1.synchronize()
        if i >= 2:
            times.append(e0.elapsed_time(e1))
    if int(out.item()) & 0xFFFFFFFF != (nbytes // 4) % (1 << 32):
        raise RuntimeError("HBM read probe: wrong word sum")
    del buf, out
    torch.cuda.empty_cache()
    return {"median_gbs": round(nbytes / (statistics.median(times) * 1e-3) / 1e9, 1),
            "best_gbs": round(nbytes / (min(times) * 1e-3) / 1e9, 1), "bytes": nbytes, "launches": reps,
            "how": "ntx_hbm_read_probe (streaming 16-byte loads, 8 x 256-thread CTAs per SM) over 4 GiB, "
                   "CUDA events per launch"}


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


GEMV_SHAPES = [(8, 4096, 4096, "Q8_0 GEMV 4096x4096, batch 1")] + \
    [(2, M, K, "Q4_0 GEMV sweep over Llama-3-8B projection shapes, batch 1") for M, K in
     ((4096, 4096), (1024, 4096), (14336, 4096), (4096, 14336))] + \
    [(14, M, K, "Q6_K GEMV over Llama-3-70B projection shapes, batch 1") for M, K in
     ((8192, 8192), (28672, 8192), (8192, 28672))] + \
    [(12, M, K, "Q4_K GEMV over Llama-3-70B projection shapes, batch 1") for M, K in
     ((8192, 8192), (28672, 8192), (8192, 28672))] + \
    [(13, 8192, 8192, "Q5_K GEMV 8192x8192, batch 1"), (1, 4096, 4096, "F16 GEMV 4096x4096, batch 1")]


def gemv_sweep(ntx, sg, wl, torch, peak):
    out = []
    for qt, M, K, name in GEMV_SHAPES:
        ms, nbytes, ncopy = time_gemv(ntx, sg, wl, torch, qt, M, K, pdl=True)
        ms_s, _, _ = time_gemv(ntx, sg, wl, torch, qt, M, K, pdl=False)
        gbs = nbytes / (ms * 1e-3) / 1e9
        gbs_s = nbytes / (ms_s * 1e-3) / 1e9
        out.append({"workload": name, "qtype": QNAME[qt], "M": M, "K": K, "bytes_per_launch": nbytes,
                    "us": round(ms * 1e3, 3), "GBs": round(gbs, 1), "frac": round(gbs / peak, 4),
                    "launch": "programmatic dependent launch (ntx_set_gemv_pdl(1))",
                    "us_serial": round(ms_s * 1e3, 3), "frac_serial": round(gbs_s / peak, 4),
                    "rotation": f"{ncopy} weight copies (>3x L2), back-to-back launches in one CUDA graph"})
    return out


# ---------------------------------------------------------------- CPU oracle
class _Pinned:
    """Runs the enclosed block with this process pinned to one core."""

    def __enter__(self):
        self.old = os.sched_getaffinity(0)
        os.sched_setaffinity(0, {min(self.old)})
        return self

    def __exit__(self, *exc):
        os.sched_setaffinity(0, self.old)


def oracle_tokens(orc, d, qt, hqt, layer_fn, head, final_norm, embed_tab, kcs, vcs, tokens, positions, nthreads,
                  max_ctx, greedy_after=None):
    """Whole teacher-forced oracle steps (embed, every layer, final norm, head)
    at the given positions; a token of -1 takes the previous step's argmax.
    Returns (seconds per step, fed tokens)."""
    ocfg = orc.make_config(d["hidden"], d["n_heads"], d["n_kv_heads"], d["head_dim"], d["ffn"], d["vocab"],
                           d["n_layers"], d["eps"], d["theta"], max_ctx)
    times, fed, prev = [], [], None
    for t, p in zip(tokens, positions):
        tok = prev if t < 0 else int(t)
        t0 = time.perf_counter()
        logits, _ = orc.model_step(ocfg, qt, layer_fn, hqt, head, final_norm, embed_tab, kcs, vcs, tok, p,
                                   nthreads=nthreads)
        times.append(time.perf_counter() - t0)
        prev = orc.argmax(logits)
        fed.append(tok)
    return times, fed


def cpu_baseline_8b(m, d, wk, prompt):
    """The oracle as it stands on the host cores: two whole tokens of the
    workload (the first two prompt tokens at positions 0 and 1, each through
    all 32 layers and the head, the oracle keeping its own KV cache), on one
    pinned core and on all cores."""
    import oracle as orc
    L = d["n_layers"]
    tensors = [m.host_layer_tensors(l) for l in range(L)]
    head, fn, emb = m.host_head(), m.host_final_norm(), m.host_embed()

    def caches():
        kv = [m.host_kv(l) for l in range(L)]
        return [k.copy() for k, _ in kv], [v.copy() for _, v in kv]

    cores = host_cores()
    k1, v1 = caches()
    with _Pinned():
        t1, _ = oracle_tokens(orc, d, wk["qtype"], wk["head_qtype"], tensors, head, fn, emb, k1, v1, prompt[:2],
                              [0, 1], 1, wk["max_ctx"])
    kn, vn = caches()
    tn, _ = oracle_tokens(orc, d, wk["qtype"], wk["head_qtype"], tensors, head, fn, emb, kn, vn, prompt[:2], [0, 1],
                          cores, wk["max_ctx"])
    v_all = len(tn) / sum(tn)
    return {"value": round(v_all, 5), "unit": "tok/s", "cores": cores, "kind": "oracle",
            "sample": f"2 whole tokens of the workload (prompt tokens at positions 0 and 1: embed, {L} layers, head; "
                      f"the oracle's own fp16 KV cache), timed per token on {cores} threads",
            "one_core": {"value": round(len(t1) / sum(t1), 5), "unit": "tok/s", "cores": 1,
                         "s_per_token": [round(t, 3) for t in t1]},
            "all_cores_s_per_token": [round(t, 3) for t in tn], "cpu": cpu_model(), "nproc": os.cpu_count()}


def cpu_baseline_70b(m, d, wk, start):
    """One whole oracle token of the 70B workload (position 2048 over the
    generator's 2048 prior KV rows, every layer fetched from the device model
    one at a time), on all host cores."""
    import oracle as orc
    L = d["n_layers"]
    kv = [m.host_kv(l) for l in range(L)]
    kcs, vcs = [k.copy() for k, _ in kv], [v.copy() for _, v in kv]
    cores = host_cores()
    t, _ = oracle_tokens(orc, d, wk["qtype"], wk["head_qtype"], m.host_layer_tensors, m.host_head(),
                         m.host_final_norm(), m.host_embed(), kcs, vcs, [start], [wk["n_prior"]], cores,
                         wk["max_ctx"])
    return {"value": round(1.0 / t[0], 5), "unit": "tok/s", "cores": cores, "kind": "oracle",
            "sample": f"1 whole token at position {wk['n_prior']} ({L} layers + head; layer weights copied back "
                      f"from the device one layer at a time inside the timed step) on {cores} threads",
            "cpu": cpu_model()}


def run_reference(args, world):
    """The CPU oracle as the reference arm (rank 0 only): whole tokens of the
    headline workload on all host cores."""
    import numpy as np

    import oracle as orc
    import synthgen as sg
    from synthgen import workloads as wl

    wk = WORKLOADS["llama8b-q8_0"]
    d = dict(wl.MODEL_8B)
    if args.layers is not None:
        d["n_layers"] = args.layers
    L = d["n_layers"]
    qt, hqt = wk["qtype"], wk["head_qtype"]
    sd = wl.seed(wk["workload_id"])
    cores = host_cores()
    H, V = d["hidden"], d["vocab"]
    t0 = time.perf_counter()
    use_dev = False
    try:
        import torch
        use_dev = torch.cuda.is_available()
    except ImportError:
        pass
    if use_dev:  # the generator's CUDA twin writes the same bytes as the host build, much faster
        from synthgen.devmodel import DeviceModel
        m = DeviceModel(d, qt, hqt, sd, wk["max_ctx"], 0, source="device")
        tensors = [m.host_layer_tensors(l) for l in range(L)]
        head, fn, emb = m.host_head(), m.host_final_norm(), m.host_embed()
        del m
    else:
        tensors = [wl.host_layer(d, qt, sd, l, nthreads=cores) for l in range(L)]
        head = sg.quant_rows(hqt, sd, "head", V, H, sigma=wl.W_SIGMA, nthreads=cores)
        fn = sg.fill_f32(sd, "final_norm", H, mean=1.0, sigma=wl.NORM_SIGMA)
        emb = sg.fill_f16(sd, "embed", V * H, 0.0, wl.EMB_SIGMA, nthreads=cores)
    gen_s = time.perf_counter() - t0
    Hkv, D = d["n_kv_heads"], d["head_dim"]
    kcs = [np.zeros((Hkv, wk["max_ctx"], D), dtype=np.uint16) for _ in range(L)]
    vcs = [np.zeros_like(k) for k in kcs]
    prompt = [int(t) for t in sg.tokens(sd, "prompt", wk["prompt"], V)]
    n = args.warmup + args.steps
    toks = [prompt[i] if i < len(prompt) else -1 for i in range(n)]
    span = wk["max_ctx"] - len(prompt)  # decode positions 16..143 are reused cyclically, as in the GPU arm
    positions = [i if i < len(prompt) else len(prompt) + (i - len(prompt)) % span for i in range(n)]
    times, _ = oracle_tokens(orc, d, qt, hqt, tensors, head, fn, emb, kcs, vcs, toks, positions, cores,
                             wk["max_ctx"])
    total = sum(times[args.warmup:])
    value = args.steps / total
    desc = wk["desc"] if args.layers is None else f"{wk['desc']} -- layer count overridden to {L} (test only)"
    return {"metric": METRIC, "value": round(value, 5), "unit": "tok/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * total / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded; random-init weights of the named shapes)",
            "config": {"workload": desc, "weights": qname(qt), "layers": L, "hidden": H, "ffn": d["ffn"],
                       "vocab": V, "batch": 1, "parallelism": "single process, host threads",
                       "l2": "n/a (host)", "graph": "n/a (host)"},
            "impl": "reference",
            "cpu_baseline": {"value": round(value, 5), "unit": "tok/s", "cores": cores, "kind": "oracle",
                             "sample": f"each step one whole token (embed, {L} layers, head) at the workload's positions "
                                       f"(steps {args.warmup}..{n - 1} after {args.warmup} untimed ones), the prompt fed "
                                       f"first and the oracle's own greedy tokens after it, on {cores} threads",
                             "cpu": cpu_model(), "input_generation_s": round(gen_s, 1)},
            "e2e": {"value": round(value, 5), "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=128)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", choices=["ntx", "reference"], default="ntx")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="llama8b-q8_0",
                    help="the model of the headline line (profiling: the 70B models with --layers); the 70B "
                         "configurations are added only to the default workload's line")
    ap.add_argument("--no-gemv", action="store_true", help="skip the standalone quantized GEMV sweep")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-chain", action="store_true", help="skip timing the per-op kernel chain for comparison")
    ap.add_argument("--no-70b", action="store_true", help="skip the 70B configurations (5a resident, 5b tiered)")
    ap.add_argument("--layers", type=int, default=None,
                    help="profiling and tests only: run the headline model with this many layers (the line then "
                         "describes that smaller model and is not a benchmark of the named workload)")
    ap.add_argument("--persist-two", action="store_true",
                    help="run a two-block-type model (llama70b-q4_k_m) on the two-type persistent kernel "
                         "(ntx_set_persist_two_types(1)) instead of the per-op chain that is the default for it")
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
        out = run_reference(args, world)
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
