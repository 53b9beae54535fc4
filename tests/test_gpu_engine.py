"""GPU parity of the decode engine (ntx_engine_create / ntx_decode_step).

* Teacher-forced logits: the oracle runs the model on the token sequence the
  GPU produced (prompt, then the GPU's greedy choices) with its own fp16 KV
  cache; every step's logits must satisfy max|diff| <= 2e-2 * RMS(ref), and the
  GPU's greedy token must be the oracle's argmax wherever the oracle's top two
  logits are more than twice that tolerance apart.
* CUDA-graph replay and kernel-by-kernel launch give bit-identical logits;
  tiered (pinned-host layers streamed through two slots) and resident runs of
  the per-op kernel chain give bit-identical logits.
* The persistent decode kernel (the default for all-resident models) and the
  per-op kernel chain each match the oracle; one launch per step.  A long
  context with query group 8 makes more attention units than CTAs.
* Cosine skip: calibration cosines within 1e-5 of the oracle's, skip
  decisions equal wherever |cos - tau| > 1e-4, and later steps with the skip set
  applied match the oracle run with the same set.
* Config 4: the full 32-layer 8B-shaped Q8_0 model, 16-token prompt plus 128
  greedy steps, checked teacher-forced over all 144 steps."""
import os
import time

import numpy as np
import pytest

import oracle
import quantized_weight_gemv_dequant_b200 as ntx
import synthgen as sg
from synthgen import workloads as wl
from synthgen.devmodel import DeviceModel

pytestmark = pytest.mark.gpu

TINY = dict(hidden=512, n_heads=8, n_kv_heads=2, head_dim=128, ffn=1536, vocab=1000, n_layers=4, eps=1e-5,
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


class Engine:
    """An engine over a DeviceModel plus the buffers a run reads back."""

    def __init__(self, m: DeviceModel, tau=0.98, tier_map=None, use_resident_copy=False):
        import torch
        d = m.d
        self.m = m
        self.cfg = ntx.make_config(d["hidden"], d["n_heads"], d["n_kv_heads"], d["head_dim"], d["ffn"], d["vocab"],
                                   d["n_layers"], d["eps"], d["theta"], m.max_ctx, tau)
        tmap = list(m.tier_map) if tier_map is None else list(tier_map)
        layers = []
        for l in range(d["n_layers"]):
            _, lw = (ntx.ntx_layer_layout_mixed(self.cfg, m.qtype) if isinstance(m.qtype, (list, tuple))
                     else ntx.ntx_layer_layout(self.cfg, m.qtype))
            src = m.resident_copy[l] if (use_resident_copy or tmap[l] == 0) else m.layers[l]
            lw.base = src.data_ptr()
            layers.append(lw)
        if use_resident_copy:
            tmap = [0] * d["n_layers"]
        self.ws_bytes = ntx.ntx_engine_workspace_bytes(self.cfg)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device="cuda")
        self.cs = torch.cuda.Stream()
        self.xs = torch.cuda.Stream() if any(tmap) else None
        self.h = ntx.ntx_engine_create(self.cfg, layers, tmap, m.slots[0], m.slots[1], m.blob_bytes, m.embed,
                                       m.final_norm, m.head, m.head_qtype, m.k_caches, m.v_caches, self.ws,
                                       self.ws_bytes, self.cs, self.xs)
        self.logits = torch.zeros(d["vocab"], dtype=torch.float32, device="cuda")
        self.next_tok = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.cos = torch.full((d["n_layers"],), float("nan"), dtype=torch.float32, device="cuda")
        self.prev = None  # greedy token of the last step run

    def run(self, tokens_in, pos0=0, flags=0, n_steps=None, collect_cos=False):
        """Feed tokens_in[s] (or -1 = previous greedy token) at positions pos0+s.
        Returns (logits [steps, V], fed token per step, greedy token per step, cos)."""
        import torch
        n = len(tokens_in) if n_steps is None else n_steps
        V = self.m.d["vocab"]
        out = torch.empty((n, V), dtype=torch.float32, device="cuda")
        nxt = torch.empty(n, dtype=torch.int32, device="cuda")
        coss = []
        with torch.cuda.stream(self.cs):
            for s in range(n):
                ntx.ntx_decode_step(self.h, int(tokens_in[s]), pos0 + s, self.logits, self.next_tok, flags,
                                    self.cos if collect_cos else None)
                out[s].copy_(self.logits)
                nxt[s:s + 1].copy_(self.next_tok)
                if collect_cos:
                    coss.append(self.cos.clone())
        self.cs.synchronize()
        nxt_h = nxt.cpu().numpy()
        fed = []
        for s in range(n):
            if tokens_in[s] >= 0:
                fed.append(int(tokens_in[s]))
            else:
                fed.append(int(nxt_h[s - 1]) if s > 0 else int(self.prev))
        self.prev = int(nxt_h[-1])
        cos = torch.stack(coss).cpu().numpy() if coss else None
        return out.cpu().numpy(), fed, nxt_h, cos

    def close(self):
        ntx.ntx_engine_destroy(self.h)


def oracle_run(m: DeviceModel, fed, pos0=0, skip=None, tensors=None, nthreads=None, check=None):
    """Teacher-forced oracle over the fed tokens; returns (logits, cos) per step."""
    d = m.d
    ocfg = oracle.make_config(d["hidden"], d["n_heads"], d["n_kv_heads"], d["head_dim"], d["ffn"], d["vocab"],
                              d["n_layers"], d["eps"], d["theta"], m.max_ctx)
    if tensors is None:
        tensors = [m.host_layer_tensors(l) for l in range(d["n_layers"])]
    kcs, vcs = [], []
    for l in range(d["n_layers"]):
        k, v = m.host_kv(l)
        kcs.append(k)
        vcs.append(v)
    emb, fn, head = m.host_embed(), m.host_final_norm(), m.host_head()
    logits, coss = [], []
    for s, tok in enumerate(fed):
        sk = skip[s] if skip is not None else None
        lg, cs = oracle.model_step(ocfg, m.qtype, tensors, m.head_qtype, head, fn, emb, kcs, vcs, tok, pos0 + s,
                                   skip=sk, nthreads=nthreads)
        if check is not None:
            check(s, lg)
        logits.append(lg)
        coss.append(cs)
    return np.array(logits), np.array(coss)


def check_logits(got, ref, greedy, step):
    rms = np.sqrt(np.mean(ref ** 2))
    tol = 2e-2 * rms
    err = np.max(np.abs(got.astype(np.float64) - ref))
    assert err <= tol, f"step {step}: max|diff| {err:.3e} > {tol:.3e}"
    top2 = np.sort(ref)[-2:]
    if top2[1] - top2[0] > 2 * tol:
        assert greedy == int(np.argmax(ref)), f"step {step}: greedy {greedy} vs oracle {int(np.argmax(ref))}"


@pytest.mark.parametrize("chain", [False, True], ids=["persistent", "per_op_chain"])
def test_engine_tiny_teacher_forced_graph_and_nograph(chain):
    m = DeviceModel(TINY, ntx.NTX_Q8_0, ntx.NTX_Q8_0, 41, max_ctx=32, n_prior=0, source="host")
    prompt = sg.tokens(41, "prompt", 6, TINY["vocab"])
    toks = list(prompt) + [-1] * 10
    f = ntx.NTX_NO_PERSIST if chain else 0
    e = Engine(m)
    lg_g, fed, nxt, _ = e.run(toks, flags=f)
    launches = ntx.ntx_engine_launches_per_step(e.h)
    m.reset_kv()
    lg_n, fed_n, _, _ = e.run(toks, flags=f | ntx.NTX_NO_GRAPH)
    e.close()
    assert launches == (1 + 5 * TINY["n_layers"] + 2 if chain else 1)
    assert fed == fed_n
    assert np.array_equal(lg_g, lg_n)
    ref, _ = oracle_run(m, fed)
    for s in range(len(fed)):
        check_logits(lg_g[s], ref[s], int(nxt[s]), s)


@pytest.mark.parametrize("qtype,d,max_ctx,n_prior", [
    (ntx.NTX_Q8_0, dict(TINY, n_heads=16, n_kv_heads=2, n_layers=2), 20000, 19990),
    (ntx.NTX_Q4_0, dict(TINY, n_heads=4, n_kv_heads=4, n_layers=2), 600, 590),
    (ntx.NTX_Q6_K, dict(TINY, hidden=2048, n_heads=16, n_kv_heads=8, ffn=6144, n_layers=2), 300, 290),
    (ntx.NTX_Q8_0, dict(TINY, n_heads=8, n_kv_heads=1, n_layers=2), 20000, 19990),
], ids=["q8_0_g8_ctx20000", "q4_0_g1_ctx600", "q6_k_g2_ctx300", "q8_0_one_kv_head_ctx20000"])
def test_engine_persistent_long_context(qtype, d, max_ctx, n_prior):
    """Persistent kernel at contexts where a (KV head, split) unit holds many
    positions, and where the splits of one KV head are many: 74 per KV head
    (first case), one per CTA for a single KV head (last case), so that each
    split merges a few outputs over every split in several rounds of loads."""
    m = DeviceModel(d, qtype, qtype, 49, max_ctx=max_ctx, n_prior=n_prior, source="host")
    toks = list(sg.tokens(49, "prompt", 2, d["vocab"])) + [-1] * 2
    e = Engine(m)
    lg, fed, nxt, _ = e.run(toks, pos0=n_prior)
    assert ntx.ntx_engine_launches_per_step(e.h) == 1
    e.close()
    ref, _ = oracle_run(m, fed, pos0=n_prior, nthreads=os.cpu_count())
    for s in range(len(fed)):
        check_logits(lg[s], ref[s], int(nxt[s]), s)


@pytest.mark.parametrize("qtype,d", [(ntx.NTX_Q4_0, TINY),
                                     (ntx.NTX_Q6_K, dict(TINY, hidden=2048, n_heads=16, ffn=4096, n_layers=3))])
def test_engine_tiny_other_formats(qtype, d):
    m = DeviceModel(d, qtype, qtype, 43, max_ctx=24, n_prior=7, source="host")
    toks = list(sg.tokens(43, "prompt", 3, d["vocab"])) + [-1] * 5
    e = Engine(m)
    lg, fed, nxt, _ = e.run(toks, pos0=7)
    e.close()
    ref, _ = oracle_run(m, fed, pos0=7)
    for s in range(len(fed)):
        check_logits(lg[s], ref[s], int(nxt[s]), s)


def test_engine_tiered_equals_resident():
    d = dict(TINY, n_layers=5)
    m = DeviceModel(d, ntx.NTX_Q8_0, ntx.NTX_Q8_0, 45, max_ctx=32, n_prior=3, tier_map=[0, 1, 1, 0, 1],
                    source="host", keep_resident_copy=True)
    toks = list(sg.tokens(45, "prompt", 4, d["vocab"])) + [-1] * 6
    et = Engine(m)
    lg_t, fed_t, _, _ = et.run(toks, pos0=3)
    m.reset_kv()
    lg_tn, _, _, _ = et.run(toks, pos0=3, flags=ntx.NTX_NO_GRAPH)
    et.close()
    m.reset_kv()
    er = Engine(m, use_resident_copy=True)
    lg_r, fed_r, _, _ = er.run(toks, pos0=3, flags=ntx.NTX_NO_PERSIST)
    m.reset_kv()
    lg_p, fed_p, nxt_p, _ = er.run(toks, pos0=3)  # the persistent kernel
    er.close()
    assert fed_t == fed_r
    assert np.array_equal(lg_t, lg_r)
    assert np.array_equal(lg_tn, lg_r)
    m.reset_kv()
    ref, _ = oracle_run(m, fed_p, pos0=3)
    for s in range(len(fed_p)):
        check_logits(lg_p[s], ref[s], int(nxt_p[s]), s)


def test_engine_cosine_skip_calibration():
    d = dict(TINY, n_layers=6)
    m = DeviceModel(d, ntx.NTX_Q8_0, ntx.NTX_Q8_0, 47, max_ctx=32, n_prior=0, source="host")
    prompt = list(sg.tokens(47, "prompt", 5, d["vocab"]))
    # oracle cosines at the calibration step decide a threshold that splits the layers
    e0 = Engine(m)
    _, fed0, _, _ = e0.run(prompt + [-1], n_steps=6)
    e0.close()
    m.reset_kv()
    _, cos_ref0 = oracle_run(m, fed0)
    c = np.sort(cos_ref0[5])
    tau = float((c[2] + c[3]) / 2)
    e = Engine(m, tau=tau)
    lg_a, fed_a, nxt_a, cos_a = e.run(prompt, collect_cos=True)
    lg_c, fed_c, nxt_c, cos_c = e.run([-1], pos0=5, flags=ntx.NTX_CALIBRATE_SKIP, collect_cos=True)
    mask = ntx.ntx_engine_skip_mask(e.h, d["n_layers"])
    lg_s, fed_s, nxt_s, _ = e.run([-1] * 4, pos0=6, flags=ntx.NTX_USE_SKIP)
    e.close()
    assert fed_c == [int(nxt_a[-1])]
    assert fed_s == [int(nxt_c[0])] + [int(t) for t in nxt_s[:-1]]
    fed_all = fed_a + fed_c + fed_s
    m.reset_kv()
    skip_sets = [None] * 6 + [mask] * 4
    ref, cos_ref = oracle_run(m, fed_all, skip=skip_sets)
    for l in range(d["n_layers"]):
        assert abs(cos_c[0][l] - cos_ref[5][l]) <= 1e-5, (l, cos_c[0][l], cos_ref[5][l])
        if abs(cos_ref[5][l] - tau) > 1e-4:
            assert mask[l] == (1 if cos_ref[5][l] >= tau else 0)
    assert 0 < sum(mask) < d["n_layers"]
    lg_all = np.concatenate([lg_a, lg_c, lg_s])
    greedy = list(nxt_a) + list(nxt_c) + list(nxt_s)
    for s in range(len(fed_all)):
        check_logits(lg_all[s], ref[s], int(greedy[s]), s)


@pytest.mark.slow
def test_engine_llama8b_q8_0_144_steps():
    """Config 4: 32-layer 8B-shaped Q8_0 model, 16-token prompt + 128 greedy
    steps (KV grows to 144), checked teacher-forced over all 144 steps.  The
    model is made by the generator's CUDA twin; sampled rows of every tensor are
    first checked bit-identical to the host generator."""
    d = dict(wl.MODEL_8B)
    sd = wl.seed(4)
    m = DeviceModel(d, ntx.NTX_Q8_0, ntx.NTX_Q8_0, sd, max_ctx=144, n_prior=0, source="device")
    # device generator == host generator on sampled rows of every matrix
    rs = np.random.RandomState(4)
    shapes = wl.mat_shapes(d)
    for l in range(d["n_layers"]):
        t = m.host_layer_tensors(l)
        for name, (M, K) in shapes.items():
            for r in rs.randint(0, M, size=2):
                ref = sg.quant_rows(ntx.NTX_Q8_0, sd, wl.tensor_name(l, name), M, K, sigma=wl.W_SIGMA, row0=int(r),
                                    nrows=1)
                assert np.array_equal(t[name][r], ref[0]), (l, name, r)
    head = m.host_head()
    for r in rs.randint(0, d["vocab"], size=8):
        ref = sg.quant_rows(ntx.NTX_Q8_0, sd, "head", d["vocab"], d["hidden"], sigma=wl.W_SIGMA, row0=int(r), nrows=1)
        assert np.array_equal(head[r], ref[0])
    emb = m.host_embed()
    assert np.array_equal(emb[:4096 * 3], sg.fill_f16(sd, "embed", 4096 * 3, 0.0, wl.EMB_SIGMA))

    prompt = sg.tokens(sd, "prompt", 16, d["vocab"])
    toks = list(prompt) + [-1] * 128
    e = Engine(m)
    lg, fed, nxt, _ = e.run(toks)
    e.close()
    tensors = [m.host_layer_tensors(l) for l in range(d["n_layers"])]
    t0 = time.time()
    oracle_run(m, fed, tensors=tensors, nthreads=os.cpu_count(),
               check=lambda s, ref: check_logits(lg[s], ref, int(nxt[s]), s))
    print(f"oracle teacher-forced 144 steps: {time.time() - t0:.1f} s")


def test_engine_phase_probe_records_every_phase_in_order():
    import torch
    m = DeviceModel(TINY, ntx.NTX_Q8_0, ntx.NTX_Q8_0, 51, max_ctx=16, n_prior=0, source="host")
    e = Engine(m)
    grid = ntx.ntx_engine_set_phase_probe(e.h, None, 0)
    assert grid == ntx.ntx_sm_count()
    n_ph = 2 + 5 * TINY["n_layers"]
    ts = torch.zeros((1 + n_ph) * grid, dtype=torch.int64, device="cuda")
    assert ntx.ntx_engine_set_phase_probe(e.h, ts, ts.numel()) == grid
    e.run([3], flags=ntx.NTX_NO_GRAPH)
    t = ts.cpu().numpy().reshape(1 + n_ph, grid)
    assert (t > 0).all()  # every CTA stamped its start and every phase
    done = t[1:].max(axis=1)
    assert (done[1:] >= done[:-1]).all()  # phases complete in order
    assert (t[1:].min(axis=1) >= t[0].min()).all()
    # graph replays record nothing; a cleared probe records nothing
    ts.zero_()
    e.run([-1], pos0=1)
    assert int(ts.abs().sum()) == 0
    ntx.ntx_engine_set_phase_probe(e.h, None, 0)
    e.run([-1], pos0=2, flags=ntx.NTX_NO_GRAPH)
    assert int(ts.abs().sum()) == 0
    e.close()


def test_engine_skip_every_layer_and_none():
    """Degenerate skip sets on the persistent kernel: tau -1 skips every layer
    (embed feeds the head directly), tau 2 skips none."""
    d = dict(TINY, n_layers=3)
    m = DeviceModel(d, ntx.NTX_Q8_0, ntx.NTX_Q8_0, 53, max_ctx=16, n_prior=0, source="host")
    prompt = list(sg.tokens(53, "prompt", 2, d["vocab"]))
    for tau, n_skip in ((-1.0, d["n_layers"]), (2.0, 0)):
        m.reset_kv()
        e = Engine(m, tau=tau)
        lg_a, fed_a, nxt_a, _ = e.run(prompt[:1])
        lg_c, fed_c, nxt_c, _ = e.run(prompt[1:], pos0=1, flags=ntx.NTX_CALIBRATE_SKIP)
        mask = ntx.ntx_engine_skip_mask(e.h, d["n_layers"])
        lg_s, fed_s, nxt_s, _ = e.run([-1, -1], pos0=2, flags=ntx.NTX_USE_SKIP)
        assert ntx.ntx_engine_launches_per_step(e.h) == 1
        e.close()
        assert sum(mask) == n_skip
        m.reset_kv()
        fed = fed_a + fed_c + fed_s
        ref, _ = oracle_run(m, fed, skip=[None, None, mask, mask])
        lg = np.concatenate([lg_a, lg_c, lg_s])
        greedy = list(nxt_a) + list(nxt_c) + list(nxt_s)
        for s in range(len(fed)):
            check_logits(lg[s], ref[s], int(greedy[s]), s)


def test_engine_falls_back_to_chain_beyond_persistent_limits():
    """FFN 30720 needs 15 slices of 2048 columns, one more than the persistent
    kernel's consumer warps: the engine runs the per-op chain, same results."""
    d = dict(TINY, ffn=30720, n_layers=1)
    m = DeviceModel(d, ntx.NTX_Q8_0, ntx.NTX_Q8_0, 55, max_ctx=8, n_prior=0, source="host")
    toks = list(sg.tokens(55, "prompt", 2, d["vocab"])) + [-1]
    e = Engine(m)
    lg, fed, nxt, _ = e.run(toks)
    assert ntx.ntx_engine_launches_per_step(e.h) > 1
    assert ntx.ntx_engine_set_phase_probe(e.h, None, 0) == 0  # no persistent kernel
    e.close()
    ref, _ = oracle_run(m, fed)
    for s in range(len(fed)):
        check_logits(lg[s], ref[s], int(nxt[s]), s)
