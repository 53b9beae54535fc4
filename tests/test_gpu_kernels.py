"""GPU parity of the per-op C-ABI calls against the CPU oracle.

Bars: dequantisation bit-exact (uint32 compare); GEMV |y - y_ref| <= 1e-3 *
sum_j |w_ij x_j| + 1e-6; RMSNorm / RoPE / SwiGLU |diff| <= 1e-5 * max(1,
|ref|); attention |diff| <= 1e-3 * sum_p p_p |v_p| + 1e-6.  Every output sits
between canary guard bands that must survive the call."""
import numpy as np
import pytest

import oracle
import quantized_weight_gemv_dequant_b200 as ntx
import synthgen as sg
from helpers import body, check_guards, dev, f32_bits, guarded_f32
from synthgen import workloads as wl

pytestmark = pytest.mark.gpu

Q4_0, Q8_0, Q6_K = ntx.NTX_Q4_0, ntx.NTX_Q8_0, ntx.NTX_Q6_K


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


# ------------------------------------------------------------------ dequant
def _random_blocks(qtype, nblk, seed):
    """Arbitrary block bytes with a finite fp16 scale (every q pattern)."""
    rs = np.random.RandomState(seed)
    bb = sg.BLOCK_BYTES[qtype]
    raw = rs.randint(0, 256, size=(nblk, bb)).astype(np.uint8)
    dpos = 208 if qtype == Q6_K else 0
    hi = raw[:, dpos + 1]
    raw[:, dpos + 1] = np.where((hi & 0x7C) == 0x7C, hi & 0xBF, hi)  # exponent 31 -> 15: no inf/nan
    return raw


@pytest.mark.parametrize("qtype", [Q8_0, Q4_0, Q6_K])
@pytest.mark.parametrize("nblk", [1, 7, 1000, 4099])
def test_dequant_bit_exact(qtype, nblk):
    blocks = _random_blocks(qtype, nblk, 100 + nblk + qtype)
    n = nblk * sg.BLOCK_ELEMS[qtype]
    ref = oracle.dequant(qtype, blocks, n).astype(np.float32)  # exact values, exact cast
    buf, off = guarded_f32(n)
    ntx.ntx_dequant(qtype, dev(blocks), body(buf, off, n), n)
    _sync()
    check_guards(buf, off, n)
    got = body(buf, off, n).cpu().numpy()
    assert np.array_equal(f32_bits(got), f32_bits(ref))


def test_dequant_generator_blocks_bit_exact():
    for qtype in (Q8_0, Q4_0, Q6_K):
        W = sg.quant_rows(qtype, wl.seed(1), "dq", 64, 2048)
        ref = oracle.dequant(qtype, W, 64 * 2048).astype(np.float32)
        out = dev(np.zeros(64 * 2048, dtype=np.float32))
        ntx.ntx_dequant(qtype, dev(W), out, 64 * 2048)
        _sync()
        assert np.array_equal(f32_bits(out.cpu().numpy()), f32_bits(ref))


# ------------------------------------------------------------------ GEMV
def gemv_check(qtype, W, M, K, x, resid=None, in_place=False):
    buf, off = guarded_f32(M)
    y = body(buf, off, M)
    r = None
    if resid is not None:
        if in_place:
            y.copy_(dev(resid.astype(np.float32)))
            r = y
        else:
            r = dev(resid.astype(np.float32))
    ntx.ntx_gemv_q(qtype, dev(W), M, K, dev(x.astype(np.float32)), y, r)
    _sync()
    check_guards(buf, off, M)
    got = y.cpu().numpy().astype(np.float64)
    ref, b = oracle.gemv(qtype, W, M, K, x.astype(np.float32).astype(np.float64))
    if resid is not None:
        ref = ref + resid.astype(np.float32)
        b = b + np.abs(resid.astype(np.float32))
    err = np.abs(got - ref)
    tol = 1e-3 * b + 1e-6
    bad = np.nonzero(err > tol)[0]
    assert bad.size == 0, f"{bad.size} rows over tolerance, first {bad[:5]}, excess {np.max(err - tol)}"
    return got, ref


SHAPES_32 = [(1, 256), (3, 256), (7, 2304), (37, 4096), (300, 6400), (129, 8704), (5, 288), (9, 32), (70, 1056)]
SHAPES_256 = [(1, 2048), (5, 4096), (37, 6144), (130, 2048), (3, 256), (7, 768), (11, 2304)]


@pytest.mark.parametrize("qtype", [Q8_0, Q4_0])
@pytest.mark.parametrize("M,K", SHAPES_32)
def test_gemv_shapes_32(qtype, M, K):
    W = sg.quant_rows(qtype, wl.seed(2), f"g{M}x{K}", M, K)
    x = sg.fill_f32(wl.seed(2), f"x{K}", K)
    gemv_check(qtype, W, M, K, x)


@pytest.mark.parametrize("M,K", SHAPES_256)
def test_gemv_shapes_q6_k(M, K):
    W = sg.quant_rows(Q6_K, wl.seed(5), f"g{M}x{K}", M, K)
    x = sg.fill_f32(wl.seed(5), f"x{K}", K)
    gemv_check(Q6_K, W, M, K, x)


@pytest.mark.parametrize("qtype", [Q8_0, Q4_0, Q6_K])
def test_gemv_residual_and_in_place(qtype):
    M, K = 77, 4096
    W = sg.quant_rows(qtype, 3, "res", M, K)
    x = sg.fill_f32(3, "resx", K)
    r = sg.fill_f32(3, "resr", M)
    gemv_check(qtype, W, M, K, x, resid=r)
    gemv_check(qtype, W, M, K, x, resid=r, in_place=True)


@pytest.mark.parametrize("qtype", [Q8_0, Q4_0, Q6_K])
def test_gemv_exact_on_grid(qtype):
    """Small-integer x and grid weights: fp32 sums are exact, GPU == oracle."""
    M, K = 24, 4096
    rs = np.random.RandomState(qtype)
    W = sg.quant_rows(qtype, 4, "exact", M, K)
    # overwrite scales with 2^-4 so every product is a small dyadic number
    bb, be = sg.BLOCK_BYTES[qtype], sg.BLOCK_ELEMS[qtype]
    blk = W.reshape(M, K // be, bb)
    dpos = 208 if qtype == Q6_K else 0
    blk[..., dpos], blk[..., dpos + 1] = 0x00, 0x2C  # 0x2C00 = 2^-4
    if qtype == Q6_K:
        blk[..., 192:208] = rs.randint(-3, 4, size=blk[..., 192:208].shape).astype(np.int8).view(np.uint8)
    x = rs.randint(-3, 4, size=K).astype(np.float32)
    got, ref = gemv_check(qtype, W, M, K, x)
    assert np.array_equal(got, ref)


def test_gemv_q8_0_4096x4096():
    M = K = 4096
    W = sg.quant_rows(Q8_0, wl.seed(1), "W", M, K)
    x = sg.fill_f32(wl.seed(1), "x", K)
    gemv_check(Q8_0, W, M, K, x)


@pytest.mark.parametrize("M,K", wl.Q4_0_SWEEP)
def test_gemv_q4_0_llama8b_projection_shapes(M, K):
    W = sg.quant_rows(Q4_0, wl.seed(2), f"W{M}x{K}", M, K)
    x = sg.fill_f32(wl.seed(2), f"x{K}", K)
    gemv_check(Q4_0, W, M, K, x)


@pytest.mark.parametrize("cps", [2, 3, 4])
def test_gemv_ctas_per_sm_same_result(cps):
    M, K = 4096, 4096
    W = sg.quant_rows(Q8_0, 7, "cps", M, K)
    x = sg.fill_f32(7, "cpsx", K)
    Wd, xd = dev(W), dev(x)
    y1 = dev(np.zeros(M, dtype=np.float32))
    y2 = dev(np.zeros(M, dtype=np.float32))
    ntx.ntx_gemv_q(Q8_0, Wd, M, K, xd, y1)
    ntx.ntx_set_gemv_ctas_per_sm(cps)
    try:
        ntx.ntx_gemv_q(Q8_0, Wd, M, K, xd, y2)
    finally:
        ntx.ntx_set_gemv_ctas_per_sm(1)
    _sync()
    assert np.array_equal(y1.cpu().numpy(), y2.cpu().numpy())  # each row is one warp's sum either way


def test_gemv_pdl_back_to_back_matches_oracle():
    """Programmatic launch on: a chain of GEMVs on one stream, each reading the
    previous one's output as x (the dependent reads wait for it), every y
    checked against the oracle."""
    M = K = 4096
    Ws = [sg.quant_rows(q, 11, f"pdl{i}", M, K) for i, q in enumerate([Q8_0, Q4_0, Q6_K, Q8_0])]
    qts = [Q8_0, Q4_0, Q6_K, Q8_0]
    x0 = sg.fill_f32(11, "pdlx", K)
    Wd = [dev(w) for w in Ws]
    ys = [dev(np.zeros(M, dtype=np.float32)) for _ in Ws]
    _sync()
    ntx.ntx_set_gemv_pdl(1)
    try:
        xin = dev(x0)
        for q, w, y in zip(qts, Wd, ys):
            ntx.ntx_gemv_q(q, w, M, K, xin, y)
            xin = y
        _sync()
    finally:
        ntx.ntx_set_gemv_pdl(0)
    x = x0.astype(np.float64)
    for q, w, y in zip(qts, Ws, ys):
        got = y.cpu().numpy()
        ref, b = oracle.gemv(q, w, M, K, x.astype(np.float32).astype(np.float64))
        assert np.all(np.abs(got.astype(np.float64) - ref) <= 1e-3 * b + 1e-6)
        x = got.astype(np.float64)


# ------------------------------------------------------------------ small ops
def _rel_ok(got, ref, rel=1e-5):
    err = np.abs(got.astype(np.float64) - ref)
    return np.all(err <= rel * np.maximum(1.0, np.abs(ref))), np.max(err)


@pytest.mark.parametrize("n", [1, 100, 4096, 8192, 14336])
def test_rmsnorm(n):
    x = sg.fill_f32(11, f"rx{n}", n)
    w = sg.fill_f32(11, f"rw{n}", n, mean=1.0, sigma=0.02)
    buf, off = guarded_f32(n)
    ntx.ntx_rmsnorm(dev(x), dev(w), body(buf, off, n), n, 1e-5)
    _sync()
    check_guards(buf, off, n)
    ok, e = _rel_ok(body(buf, off, n).cpu().numpy(), oracle.rmsnorm(x, w, 1e-5))
    assert ok, e


@pytest.mark.parametrize("pos", [0, 1, 1024, 2048, 131071])
def test_rope(pos):
    Hq, Hkv, D = 32, 8, 128
    q = sg.fill_f32(12, "rq", Hq * D)
    k = sg.fill_f32(12, "rk", Hkv * D)
    qd, kd = dev(q), dev(k)
    ntx.ntx_rope(qd, kd, Hq, Hkv, D, pos, 500000.0)
    _sync()
    ok, e = _rel_ok(qd.cpu().numpy(), oracle.rope(q, Hq, D, pos, 500000.0))
    assert ok, e
    ok, e = _rel_ok(kd.cpu().numpy(), oracle.rope(k, Hkv, D, pos, 500000.0))
    assert ok, e


def test_swiglu():
    n = 14336 + 5
    g = sg.fill_f32(13, "g", n, sigma=3.0)
    u = sg.fill_f32(13, "u", n)
    buf, off = guarded_f32(n)
    ntx.ntx_swiglu(dev(g), dev(u), body(buf, off, n), n)
    _sync()
    check_guards(buf, off, n)
    ok, e = _rel_ok(body(buf, off, n).cpu().numpy(), oracle.swiglu(g, u))
    assert ok, e


@pytest.mark.parametrize("nbytes", [0, 16, 16 * 7, (1 << 20) + 48, (64 << 20) + 16 * 1001])
def test_hbm_read_probe_reads_every_word(nbytes):
    """The read probe bench.py times for the read-only HBM peak: its sum of
    32-bit words modulo 2^32 equals the host's, so every word was read once."""
    import torch
    rs = np.random.RandomState(nbytes % 1000 + 7)
    words = rs.randint(0, 1 << 32, size=nbytes // 4, dtype=np.uint64).astype(np.uint32)
    buf = torch.from_numpy(words.view(np.int32)).cuda() if nbytes else torch.empty(4, dtype=torch.int32).cuda()
    out = torch.full((4,), 0x5A5A5A5A, dtype=torch.int32, device="cuda")
    ntx.ntx_hbm_read_probe(buf.data_ptr(), nbytes, out[1:].data_ptr())
    _sync()
    got = out.cpu().numpy().view(np.uint32)
    assert int(got[1]) == int(words.astype(np.uint64).sum() % (1 << 32))
    assert got[0] == 0x5A5A5A5A and got[2] == 0x5A5A5A5A and got[3] == 0x5A5A5A5A


@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (64, 8), (8, 8), (16, 8), (4, 2)])
@pytest.mark.parametrize("n_ctx", [1, 2, 17, 300, 1025])
def test_attention(Hq, Hkv, n_ctx):
    D, T = 128, 1100
    q = sg.fill_f32(14, "aq", Hq * D)
    kc = sg.fill_f16(14, "ak", Hkv * T * D).reshape(Hkv, T, D)
    vc = sg.fill_f16(14, "av", Hkv * T * D).reshape(Hkv, T, D)
    ws_bytes = ntx.ntx_attn_workspace_bytes(Hq, Hkv, D, T)
    import torch
    ws = torch.empty(ws_bytes // 4 + 64, dtype=torch.float32, device="cuda")
    buf, off = guarded_f32(Hq * D)
    ntx.ntx_attn_decode(dev(q), dev(kc), dev(vc), body(buf, off, Hq * D), Hq, Hkv, D, n_ctx, T, ws, ws_bytes)
    _sync()
    check_guards(buf, off, Hq * D)
    ref, bound = oracle.attention(q, kc, vc, Hq, Hkv, D, n_ctx, T)
    got = body(buf, off, Hq * D).cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    assert np.all(err <= 1e-3 * bound + 1e-6), np.max(err - 1e-3 * bound)
