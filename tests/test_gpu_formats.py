"""GPU parity of the K-quant and float weight formats (Q4_K, Q5_K, F16, F32),
of mixed-type (Q4_K_M) layers, and of every format's GEMV on adversarial
inputs, against the CPU oracle.

Bars: dequantisation bit-exact against the oracle's exact value rounded once
to fp32 (uint32 compare); GEMV |y - y_ref| <= 1e-3 * sum_j |w_ij x_j| + 1e-6;
a layer max|diff| <= 2e-3 * RMS(ref) and its cosine within 1e-5.  Adversarial
inputs: raw random block bytes (every code, negative and subnormal scales,
Q8_0 code -128, Q6_K scale -128) and heavy-tailed x (one channel per 32 at
1e3 and 1e6 times the rest; magnitudes spread over 2^-20..2^20)."""
import numpy as np
import pytest

import oracle
import quantized_weight_gemv_dequant_b200 as ntx
import synthgen as sg
from helpers import body, check_guards, dev, f32_bits, guarded_f32
from synthgen import workloads as wl

pytestmark = pytest.mark.gpu

Q4_0, Q8_0, Q6_K = ntx.NTX_Q4_0, ntx.NTX_Q8_0, ntx.NTX_Q6_K
Q4_K, Q5_K, F16, F32 = ntx.NTX_Q4_K, ntx.NTX_Q5_K, ntx.NTX_F16, ntx.NTX_F32
ALL = [Q8_0, Q4_0, Q6_K, Q4_K, Q5_K, F16, F32]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    import torch
    from quantized_weight_gemv_dequant_b200 import build
    build.build()
    torch.cuda.init()
    yield
    torch.cuda.synchronize()
    assert ntx.ntx_device_status() == 0


def _sync():
    import torch
    torch.cuda.synchronize()


def _finite_half(hi):
    """High byte of an fp16 with exponent 31 (inf/nan) moved to exponent 15."""
    return np.where((hi & 0x7C) == 0x7C, hi & 0xBF, hi)


def random_blocks(qtype, nblk, seed, small_exp=False):
    """Arbitrary block bytes with finite fp16 scales.  small_exp: scales and
    float weights kept below 2^10 in magnitude (no fp32 overflow in a GEMV)."""
    rs = np.random.RandomState(seed)
    bb = sg.BLOCK_BYTES[qtype]
    raw = rs.randint(0, 256, size=(nblk, bb)).astype(np.uint8)
    if qtype == F32:
        f = (rs.randn(nblk) * np.exp2(rs.uniform(-30 if small_exp else -120, 10 if small_exp else 120, nblk)))
        return f.astype(np.float32).view(np.uint8).reshape(nblk, 4)
    if qtype == F16:
        raw[:, 1] = _finite_half(raw[:, 1])
        if small_exp:
            raw[:, 1] = np.minimum(raw[:, 1] & 0x7F, 0x63) | (raw[:, 1] & 0x80)  # |w| < 2^10
        return raw
    half_pos = [208] if qtype == Q6_K else ([0, 2] if qtype in (Q4_K, Q5_K) else [0])
    for p in half_pos:
        raw[:, p + 1] = _finite_half(raw[:, p + 1])
        if small_exp:
            raw[:, p + 1] = np.minimum(raw[:, p + 1] & 0x7F, 0x4F) | (raw[:, p + 1] & 0x80)  # |d| < 2^5
    return raw


# ------------------------------------------------------------------ dequant
@pytest.mark.parametrize("qtype", [Q4_K, Q5_K, F16, F32])
@pytest.mark.parametrize("nblk", [1, 7, 1000, 4099])
def test_dequant_bit_exact_random_blocks(qtype, nblk):
    blocks = random_blocks(qtype, nblk, 300 + nblk + qtype)
    n = nblk * sg.BLOCK_ELEMS[qtype]
    ref = oracle.dequant(qtype, blocks, n).astype(np.float32)  # the exact value rounded once
    buf, off = guarded_f32(n)
    ntx.ntx_dequant(qtype, dev(blocks), body(buf, off, n), n)
    _sync()
    check_guards(buf, off, n)
    got = body(buf, off, n).cpu().numpy()
    assert np.array_equal(f32_bits(got), f32_bits(ref))


@pytest.mark.parametrize("qtype", [Q4_K, Q5_K, F16, F32])
def test_dequant_generator_blocks_bit_exact(qtype):
    W = sg.quant_rows(qtype, wl.seed(6), "dq", 64, 2048)
    ref = oracle.dequant(qtype, W, 64 * 2048).astype(np.float32)
    out = dev(np.zeros(64 * 2048, dtype=np.float32))
    ntx.ntx_dequant(qtype, dev(W), out, 64 * 2048)
    _sync()
    assert np.array_equal(f32_bits(out.cpu().numpy()), f32_bits(ref))


# ------------------------------------------------------------------ GEMV
def gemv_check(qtype, W, M, K, x):
    buf, off = guarded_f32(M)
    y = body(buf, off, M)
    ntx.ntx_gemv_q(qtype, dev(np.ascontiguousarray(W)), M, K, dev(x.astype(np.float32)), y, None)
    _sync()
    check_guards(buf, off, M)
    got = y.cpu().numpy().astype(np.float64)
    ref, b = oracle.gemv(qtype, W, M, K, x.astype(np.float32).astype(np.float64))
    err = np.abs(got - ref)
    tol = 1e-3 * b + 1e-6
    bad = np.nonzero(err > tol)[0]
    assert bad.size == 0, f"{bad.size} rows over tolerance, first {bad[:5]}, excess {np.max(err - tol)}"
    return got, ref


SHAPES = [(1, 256), (3, 512), (37, 2048), (300, 4096), (129, 6400), (70, 8192), (5, 14336)]


@pytest.mark.parametrize("qtype", [Q4_K, Q5_K, F16, F32])
@pytest.mark.parametrize("M,K", SHAPES)
def test_gemv_shapes(qtype, M, K):
    W = sg.quant_rows(qtype, wl.seed(6), f"g{M}x{K}", M, K)
    x = sg.fill_f32(wl.seed(6), f"x{K}", K)
    gemv_check(qtype, W, M, K, x)


@pytest.mark.parametrize("qtype", [Q4_K, Q5_K, F16])
def test_gemv_generic_path_odd_k(qtype):
    """K not a multiple of 256 (or a misaligned row) takes the generic kernel."""
    K = 2 * sg.BLOCK_ELEMS[qtype] * 3 if qtype != F16 else 200
    M = 19
    W = sg.quant_rows(qtype, 8, "odd", M, K)
    x = sg.fill_f32(8, "oddx", K)
    gemv_check(qtype, W, M, K, x)


@pytest.mark.parametrize("M,K", [(8192, 8192), (1024, 8192), (28672, 8192), (8192, 28672)])
def test_gemv_q4_k_llama70b_projection_shapes(M, K):
    W = sg.quant_rows(Q4_K, wl.seed(5), f"K4W{M}x{K}", M, K)
    x = sg.fill_f32(wl.seed(5), f"x{K}", K)
    gemv_check(Q4_K, W, M, K, x)


@pytest.mark.parametrize("qtype", ALL)
def test_gemv_raw_random_blocks(qtype):
    """Arbitrary block bytes: every code (Q8_0 -128, Q6_K scale -128),
    negative and subnormal fp16 scales."""
    M, K = 96, 4096
    nb = K // sg.BLOCK_ELEMS[qtype]
    W = random_blocks(qtype, M * nb, 500 + qtype, small_exp=True).reshape(M, -1)
    if qtype == Q8_0:
        W.reshape(M, nb, 34)[:, ::5, 2 + 7] = 0x80  # q = -128 in every fifth block
    if qtype == Q6_K:
        W.reshape(M, nb, 210)[:, :, 192] = 0x80      # sub-block scale -128
    if qtype not in (F16, F32):
        hpos = 208 if qtype == Q6_K else 0
        Wb = W.reshape(M, nb, -1)
        Wb[::3, :, hpos], Wb[::3, :, hpos + 1] = 0x05, 0x80  # d = -5 * 2^-24, subnormal and negative
    x = sg.fill_f32(9, "rawx", K)
    gemv_check(qtype, W, M, K, x)


def _heavy_x(K, kind, seed):
    rs = np.random.RandomState(seed)
    x = rs.randn(K).astype(np.float64)
    if kind == "outlier1e3":
        x[rs.randint(0, 32) + 32 * np.arange(K // 32)] *= 1e3
    elif kind == "outlier1e6":
        x[rs.randint(0, 32) + 32 * np.arange(K // 32)] *= 1e6
    elif kind == "single1e6":
        x[rs.randint(0, K)] *= 1e6
    else:  # magnitudes log-uniform over 2^-20 .. 2^20
        x = np.sign(x) * np.exp2(rs.uniform(-20, 20, K))
    return x.astype(np.float32)


@pytest.mark.parametrize("qtype", ALL)
@pytest.mark.parametrize("kind", ["outlier1e3", "outlier1e6", "single1e6", "span2e20"])
def test_gemv_heavy_tailed_x(qtype, kind):
    M, K = 128, 8192
    W = sg.quant_rows(qtype, 12, "heavy", M, K)
    x = _heavy_x(K, kind, 40 + qtype)
    gemv_check(qtype, W, M, K, x)


# ------------------------------------------------------------------ mixed layer
MIX_D = dict(hidden=2048, n_heads=16, n_kv_heads=4, head_dim=128, ffn=4096, vocab=1000, n_layers=1, eps=1e-5,
             theta=500000.0)


@pytest.mark.parametrize("types", [wl.Q4_K_M, (Q5_K,) * 6 + (Q6_K,), (Q4_K,) * 3 + (Q5_K, F16, F16, Q4_K),
                                   (F32,) * 7])
def test_decode_layer_mixed_types(types):
    """One Q4_K_M-style (and other mixed) layer through ntx_decode_layer."""
    import torch
    d = MIX_D
    sd = 77
    T, pos = 40, 31
    cfg = ntx.make_config(d["hidden"], d["n_heads"], d["n_kv_heads"], d["head_dim"], d["ffn"], d["vocab"], 1,
                          d["eps"], d["theta"], T)
    blob, t = wl.host_layer_blob(d, types, sd, 0)
    n, w = ntx.ntx_layer_layout_mixed(cfg, types)
    assert n == blob.size and w.qtype == ntx.NTX_MIXED and list(w.mat_qtype) == list(types)
    bd = dev(blob)
    w.base = bd.data_ptr()
    kc, vc = wl.host_kv_prior(d, sd, 0, T, pos)
    kd, vd = dev(kc.view(np.int16)), dev(vc.view(np.int16))
    h = sg.fill_f32(sd, "h", d["hidden"])
    hd = dev(h)
    cos = torch.zeros(1, dtype=torch.float32, device="cuda")
    ws_bytes = ntx.ntx_layer_workspace_bytes(cfg)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    ntx.ntx_decode_layer(cfg, w, kd, vd, hd, pos, cos, ws, ws_bytes)
    _sync()
    ocfg = oracle.make_config(d["hidden"], d["n_heads"], d["n_kv_heads"], d["head_dim"], d["ffn"], d["vocab"], 1,
                              d["eps"], d["theta"], T)
    ref, cref = oracle.layer(ocfg, types[0], t, t["attn_norm"], t["ffn_norm"], kc, vc, h, pos)
    got = hd.cpu().numpy().astype(np.float64)
    rms = np.sqrt(np.mean(ref ** 2))
    assert np.max(np.abs(got - ref)) <= 2e-3 * rms
    assert abs(float(cos.item()) - cref) <= 1e-5


@pytest.mark.parametrize("types,head", [(wl.Q4_K_M, wl.Q4_K_M_HEAD), ((Q5_K,) * 6 + (Q6_K,), Q6_K),
                                        ((Q4_K,) * 7, Q4_K)], ids=["q4_k_m", "q5_k_q6_k", "q4_k"])
def test_engine_k_quant_models_persistent_and_chain(types, head):
    """4-layer K-quant models (Q4_K_M: Q4_K matrices, Q6_K down projections and
    head) through the engine, as the persistent kernel (one launch per step,
    per-phase block types; opted in for two-type models), as the engine's
    default (the chain for two-type models) and as the per-op chain: every step's logits within
    2e-2 * RMS of the oracle's, teacher-forced on the GPU's tokens, greedy
    token where the gap allows."""
    from synthgen.devmodel import DeviceModel
    from test_gpu_engine import Engine, check_logits, oracle_run
    d = dict(MIX_D, n_layers=4)
    m = DeviceModel(d, types, head, 91, max_ctx=24, n_prior=0, source="host")
    prompt = [int(t) for t in sg.tokens(91, "prompt", 3, d["vocab"])]
    two = len(set(types) | {head}) > 1
    # persistent (two-type kernels are opt-in), the engine's default, the chain
    for opt_in, flags in ((1, 0), (0, 0), (0, ntx.NTX_NO_PERSIST)):
        if opt_in == 0 and flags == 0 and not two:
            continue  # a one-type model's default is the persistent case above
        m.reset_kv()
        ntx.ntx_set_persist_two_types(opt_in)
        try:
            e = Engine(m)
        finally:
            ntx.ntx_set_persist_two_types(0)
        lg, fed, nx, _ = e.run(prompt + [-1] * 3, flags=flags)
        launches = ntx.ntx_engine_launches_per_step(e.h)
        e.close()
        assert (launches == 1) == (flags == 0 and (opt_in == 1 or not two)), launches
        refs, _ = oracle_run(m, fed)
        for s in range(len(fed)):
            check_logits(lg[s], refs[s], int(nx[s]), s)
