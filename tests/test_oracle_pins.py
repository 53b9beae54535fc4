"""Pins for the CPU oracle against facts fixed outside the oracle itself:
worked examples from the format descriptions (golden fixtures), closed forms,
invariants, brute force on tiny exact inputs, and library routines.  CPU only."""
import math

import numpy as np
import pytest

import oracle
import synthgen as sg
from conftest import read_golden

Q4_0, Q8_0, Q6_K = oracle.Q4_0, oracle.Q8_0, oracle.Q6_K


# ----------------------------------------------------------------- binary16
def test_half_decode_known_values_and_exhaustive():
    assert oracle.half_to_double(0x3C00) == 1.0
    assert oracle.half_to_double(0xC000) == -2.0
    assert oracle.half_to_double(0x7BFF) == 65504.0
    assert oracle.half_to_double(0x0001) == 2.0 ** -24
    assert oracle.half_to_double(0x0400) == 2.0 ** -14
    assert oracle.half_to_double(0x3555) == 0.333251953125
    allh = np.arange(0, 1 << 16, dtype=np.uint16)
    ref = allh.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(h)) for h in allh])
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isnan(got), np.isnan(ref))


@pytest.mark.filterwarnings("ignore:overflow")
def test_half_encode_matches_numpy_rne():
    rs = np.random.RandomState(3)
    v = np.concatenate([rs.randn(30000) * 10.0 ** rs.uniform(-9, 5.5, 30000),
                        [0.5 + 2 ** -12, 1 + 2 ** -11, 1 + 3 * 2 ** -11, 2 ** -25, 3 * 2 ** -25, 65519.0, 65520.0,
                         -65520.0, 2 ** -24 * 1.5]])
    got = np.array([oracle.double_to_half(float(x)) for x in v], dtype=np.uint16)
    assert np.array_equal(got, v.astype(np.float16).view(np.uint16))


# ----------------------------------------------------------------- dequant
def _golden_blocks(name):
    rows = read_golden(name)
    out = []
    for i in range(0, len(rows), 2):
        assert rows[i][0] == "block" and rows[i + 1][0] == "expect"
        out.append((np.array([int(t, 16) for t in rows[i][1:]], dtype=np.uint8),
                    np.array([float(t) for t in rows[i + 1][1:]])))
    return out


def test_q8_0_worked_examples():
    for blk, exp in _golden_blocks("q8_0_blocks.txt"):
        assert blk.size == 34
        assert np.array_equal(oracle.dequant(Q8_0, blk, 32), exp)


def test_q4_0_worked_example():
    for blk, exp in _golden_blocks("q4_0_blocks.txt"):
        assert blk.size == 18
        assert np.array_equal(oracle.dequant(Q4_0, blk, 32), exp)


def _q6k_base():
    b = np.zeros(210, dtype=np.uint8)
    b[192:208] = 1            # all sub-block scales 1
    b[208], b[209] = 0x00, 0x3C  # d = 1.0
    return b


def test_q6_k_bit_positions_from_fixture():
    base = oracle.dequant(Q6_K, _q6k_base(), 256)
    assert np.array_equal(base, np.full(256, -32.0))
    for field, byte, part, elem in read_golden("q6_k_onehot.txt"):
        b = _q6k_base()
        byte, elem = int(byte), int(elem)
        if field == "ql":
            b[byte] = 0x01 if part == "lo" else 0x10
            want = -31.0
        else:
            b[128 + byte] = 1 << (2 * int(part))
            want = -16.0
        w = oracle.dequant(Q6_K, b, 256)
        changed = np.nonzero(w != -32.0)[0]
        assert list(changed) == [elem], (field, byte, part)
        assert w[elem] == want


def test_q6_k_every_bit_reaches_exactly_one_element():
    """Bijection: the 4 low bits x 256 and 2 high bits x 256 land on distinct elements."""
    seen_low, seen_high = set(), set()
    for byte in range(128):
        for part, val in (("lo", 0x01), ("hi", 0x10)):
            b = _q6k_base()
            b[byte] = val
            ch = np.nonzero(oracle.dequant(Q6_K, b, 256) != -32.0)[0]
            assert len(ch) == 1
            seen_low.add(int(ch[0]))
    for byte in range(64):
        for pair in range(4):
            b = _q6k_base()
            b[128 + byte] = 1 << (2 * pair)
            ch = np.nonzero(oracle.dequant(Q6_K, b, 256) != -32.0)[0]
            assert len(ch) == 1
            seen_high.add(int(ch[0]))
    assert seen_low == set(range(256)) and seen_high == set(range(256))


def test_q6_k_scale_index_and_sign():
    for s in range(16):
        b = _q6k_base()
        b[192 + s] = 0xFD  # int8 -3
        w = oracle.dequant(Q6_K, b, 256)
        exp = np.full(256, -32.0)
        exp[16 * s:16 * s + 16] = 96.0
        assert np.array_equal(w, exp)
    b = _q6k_base()
    b[208], b[209] = 0x00, 0xB8  # d = -0.5
    b[0] = 0x0F                  # element 0: low nibble 15
    b[128] = 0x03                # element 0: high bits 3 -> q = 63
    w = oracle.dequant(Q6_K, b, 256)
    assert w[0] == -0.5 * 31 and w[1] == -0.5 * -32


@pytest.mark.parametrize("qtype", [Q8_0, Q4_0, Q6_K])
def test_dequant_inverts_independent_packer_on_grid(qtype):
    """Values already on the quantization grid survive the generator's packer
    (an independent implementation of the same byte layout) unchanged."""
    rs = np.random.RandomState(qtype)
    nblk = 12
    if qtype == Q8_0:
        d = np.float32(2.0 ** -7)
        q = rs.randint(-127, 128, size=(nblk, 32))
        q[:, 0] = 127                          # pins amax -> d = amax / 127 exactly
        w = (q * d).astype(np.float32)
    elif qtype == Q4_0:
        d = np.float32(2.0 ** -6)
        q = rs.randint(0, 16, size=(nblk, 32))
        q[:, 3] = 0                            # the max-|w| element (w = -8 d) ...
        w = ((q - 8) * -d).astype(np.float32)  # ... with d' = m/-8 = d
    else:
        # per super-block: integer sub-block scales with one at magnitude 128
        d = np.float32(2.0 ** -10)
        w = np.zeros((nblk, 256), dtype=np.float32)
        for b in range(nblk):
            sc = rs.randint(1, 128, size=16)
            sc[0] = 128
            for j in range(16):
                qq = rs.randint(0, 64, size=16)
                qq[0] = 0                      # the sub-block's max-|w| element at q = 0
                # w = d sc (q - 32); the recipe stores d' = -d and scales -sc (sc = 128 -> -128)
                w[b, 16 * j:16 * j + 16] = sc[j] * d * (qq - 32)
    blocks = sg.quantize(qtype, w)
    got = oracle.dequant(qtype, blocks, w.size)
    assert np.array_equal(got, w.astype(np.float64).ravel())


# ----------------------------------------------------------------- GEMV
def _pack_q8(d_bits, q):
    nb = q.shape[-1] // 32
    out = np.zeros(q.shape[:-1] + (nb, 34), dtype=np.uint8)
    out[..., 0] = d_bits & 0xFF
    out[..., 1] = d_bits >> 8
    out[..., 2:] = q.reshape(q.shape[:-1] + (nb, 32)).astype(np.int8).view(np.uint8)
    return out.reshape(q.shape[:-1] + (-1,))


@pytest.mark.parametrize("M,nb", [(1, 1), (2, 3), (3, 2), (3, 3)])
def test_gemv_q8_0_brute_force_exact(M, nb):
    """Weights on the grid (d = 0.25), x small integers: every product and sum
    is exact in double, so the oracle must equal the integer matmul."""
    rs = np.random.RandomState(M * 10 + nb)
    K = 32 * nb
    q = rs.randint(-127, 128, size=(M, K))
    x = rs.randint(-9, 10, size=K)
    W = _pack_q8(0x3400, q)  # 0x3400 = 0.25
    y, b = oracle.gemv(Q8_0, W, M, K, x.astype(np.float64))
    assert np.array_equal(y, (q @ x) * 0.25)
    assert np.array_equal(b, (np.abs(q) @ np.abs(x)) * 0.25)


@pytest.mark.parametrize("M,nb", [(1, 1), (2, 3), (3, 2)])
def test_gemv_q4_0_brute_force_exact(M, nb):
    rs = np.random.RandomState(M * 7 + nb)
    K = 32 * nb
    q = rs.randint(0, 16, size=(M, K))
    x = rs.randint(-9, 10, size=K)
    blk = np.zeros((M, nb, 18), dtype=np.uint8)
    blk[..., 0], blk[..., 1] = 0x00, 0xC0  # d = -2.0
    qb = q.reshape(M, nb, 32)
    blk[..., 2:] = (qb[..., :16] | (qb[..., 16:] << 4)).astype(np.uint8)
    y, _ = oracle.gemv(Q4_0, blk.reshape(M, -1), M, K, x.astype(np.float64))
    assert np.array_equal(y, ((q - 8) @ x) * -2.0)


def test_gemv_q6_k_brute_force_exact():
    rs = np.random.RandomState(5)
    M, K = 3, 512
    Wf = np.zeros((M, K), dtype=np.float32)
    d = 2.0 ** -8
    for r in range(M):
        for s in range(K // 256):
            blk = Wf[r, 256 * s: 256 * s + 256]
            sc = rs.randint(1, 100, size=16)
            sc[5] = 128
            for j in range(16):
                qq = rs.randint(0, 64, size=16)
                qq[2] = 0
                blk[16 * j:16 * j + 16] = sc[j] * d * (qq - 32)
    W = sg.quantize(Q6_K, Wf).reshape(M, -1)
    assert np.array_equal(oracle.dequant(Q6_K, W, M * K), Wf.ravel().astype(np.float64))
    x = rs.randint(-5, 6, size=K)
    y, _ = oracle.gemv(Q6_K, W, M, K, x.astype(np.float64))
    assert np.array_equal(y, Wf.astype(np.float64) @ x)


@pytest.mark.parametrize("qtype", [Q8_0, Q4_0, Q6_K])
def test_gemv_one_hot_selects_dequant_column(qtype):
    M, K = 5, 512
    W = sg.quant_rows(qtype, 1, "onehot", M, K)
    full = oracle.dequant(qtype, W, M * K).reshape(M, K)
    for j in (0, 17, 255, 256, 511):
        x = np.zeros(K)
        x[j] = 1.0
        y, b = oracle.gemv(qtype, W, M, K, x)
        assert np.array_equal(y, full[:, j])
        assert np.array_equal(b, np.abs(full[:, j]))


def test_gemv_thread_count_invariant():
    W = sg.quant_rows(Q8_0, 2, "t", 97, 1024)
    x = sg.fill_f32(2, "tx", 1024).astype(np.float64)
    y1, b1 = oracle.gemv(Q8_0, W, 97, 1024, x, nthreads=1)
    y8, b8 = oracle.gemv(Q8_0, W, 97, 1024, x, nthreads=8)
    assert y1.tobytes() == y8.tobytes() and b1.tobytes() == b8.tobytes()


# ----------------------------------------------------------------- RMSNorm
def test_rmsnorm_constant_vector_closed_form():
    n, eps = 4096, 1e-5
    y = oracle.rmsnorm(np.ones(n), np.ones(n), eps)
    assert np.allclose(y, 1.0 / math.sqrt(1.0 + 1e-5), rtol=1e-15, atol=0)
    c, w = -3.0, np.linspace(0.5, 1.5, n)
    y = oracle.rmsnorm(np.full(n, c), w, eps)
    assert np.allclose(y, w * c / math.sqrt(c * c + eps), rtol=1e-14, atol=0)


def test_rmsnorm_eps_inside_root_and_scale_invariance():
    y = oracle.rmsnorm(np.zeros(8), np.ones(8), 1e-5)
    assert np.array_equal(y, np.zeros(8))
    x = np.array([1e-3, -2e-3, 0.0, 4e-3])
    y = oracle.rmsnorm(x, np.ones(4), 1e-5)  # eps dominates: y = x / sqrt(mean x^2 + eps)
    assert np.allclose(y, x / math.sqrt(np.mean(x ** 2) + 1e-5), rtol=1e-14)
    rs = np.random.RandomState(0)
    x = rs.randn(1000) * 10
    a = oracle.rmsnorm(x, np.ones(1000), 0.0)
    b = oracle.rmsnorm(7.5 * x, np.ones(1000), 0.0)
    assert np.allclose(a, b, rtol=1e-13)
    assert abs(np.sqrt(np.mean(a ** 2)) - 1.0) < 1e-13


# ----------------------------------------------------------------- RoPE
def test_rope_adjacent_pairs_closed_form():
    D, theta, pos = 128, 500000.0, 37
    for i in (0, 1, 5, 63):
        v = np.zeros(D)
        v[2 * i] = 1.0
        r = oracle.rope(v, 1, D, pos, theta)
        ang = pos * theta ** (-2.0 * i / D)
        exp = np.zeros(D)
        exp[2 * i], exp[2 * i + 1] = math.cos(ang), math.sin(ang)
        assert np.allclose(r, exp, atol=1e-15)
        v = np.zeros(D)
        v[2 * i + 1] = 1.0
        r = oracle.rope(v, 1, D, pos, theta)
        exp = np.zeros(D)
        exp[2 * i], exp[2 * i + 1] = -math.sin(ang), math.cos(ang)
        assert np.allclose(r, exp, atol=1e-15)


def test_rope_invariants():
    rs = np.random.RandomState(1)
    D, H, theta = 128, 4, 500000.0
    q = rs.randn(H * D)
    assert np.array_equal(oracle.rope(q, H, D, 0, theta), q)  # pos 0 is the identity
    r = oracle.rope(q, H, D, 1234, theta)
    pq, pr = q.reshape(-1, 2), r.reshape(-1, 2)
    assert np.allclose(np.hypot(pr[:, 0], pr[:, 1]), np.hypot(pq[:, 0], pq[:, 1]), rtol=1e-13)
    k = rs.randn(D)
    # <R_p q, R_r k> depends only on p - r
    d1 = oracle.rope(q[:D], 1, D, 100, theta) @ oracle.rope(k, 1, D, 60, theta)
    d2 = oracle.rope(q[:D], 1, D, 1040, theta) @ oracle.rope(k, 1, D, 1000, theta)
    assert abs(d1 - d2) < 1e-11 * (np.abs(q[:D]).sum() * np.abs(k).max())
    # heads are rotated independently with the same angles
    assert np.allclose(r[D:2 * D], oracle.rope(q[D:2 * D], 1, D, 1234, theta), rtol=0, atol=0)


# ----------------------------------------------------------------- attention
def _f16(a):
    return np.asarray(a, dtype=np.float16).view(np.uint16)


def test_attention_single_position_returns_v0():
    rs = np.random.RandomState(2)
    Hq, Hkv, D, T = 8, 2, 16, 5
    kc = _f16(rs.randn(Hkv, T, D))
    vc = _f16(rs.randn(Hkv, T, D))
    out, _ = oracle.attention(rs.randn(Hq * D), kc, vc, Hq, Hkv, D, 1, T)
    vf = vc.view(np.float16).astype(np.float64)
    for h in range(Hq):
        assert np.allclose(out[h * D:(h + 1) * D], vf[h // 4, 0], rtol=0, atol=1e-15)


def test_attention_weights_sum_to_one_and_equal_keys_average():
    rs = np.random.RandomState(3)
    Hq, Hkv, D, T = 4, 1, 32, 50
    kc = _f16(rs.randn(Hkv, T, D))
    ones = _f16(np.ones((Hkv, T, D)))
    out, _ = oracle.attention(rs.randn(Hq * D) * 3, kc, ones, Hq, Hkv, D, 37, T)
    assert np.allclose(out, 1.0, rtol=0, atol=1e-14)
    same = _f16(np.broadcast_to(rs.randn(1, 1, D), (Hkv, T, D)))
    vc = _f16(rs.randn(Hkv, T, D))
    out, _ = oracle.attention(rs.randn(Hq * D), same, vc, Hq, Hkv, D, 20, T)
    mean_v = vc.view(np.float16).astype(np.float64)[0, :20].mean(axis=0)
    for h in range(Hq):
        assert np.allclose(out[h * D:(h + 1) * D], mean_v, atol=1e-14)


def test_attention_dominant_score_and_causality():
    Hq, Hkv, D, T = 2, 1, 8, 10
    k = np.zeros((Hkv, T, D))
    k[0, 6, 0] = 30.0  # q . k_6 / sqrt(8) = 30 * 3 / 2.83 -> weight ~1
    v = np.arange(T * D, dtype=np.float64).reshape(1, T, D) / 64
    q = np.zeros(Hq * D)
    q[0] = q[D] = 3.0
    out, _ = oracle.attention(q, _f16(k), _f16(v), Hq, Hkv, D, 8, T)
    assert np.allclose(out[:D], v[0, 6], atol=1e-9)
    # positions >= n_ctx are never read
    k2, v2 = k.copy(), v.copy()
    k2[0, 8:] = 99.0
    v2[0, 8:] = -99.0
    out2, _ = oracle.attention(q, _f16(k2), _f16(v2), Hq, Hkv, D, 8, T)
    assert np.array_equal(out, out2)


def test_attention_gqa_head_mapping():
    Hq, Hkv, D, T = 8, 4, 4, 3
    v = np.zeros((Hkv, T, D))
    for g in range(Hkv):
        v[g] = g + 1
    rs = np.random.RandomState(4)
    out, _ = oracle.attention(rs.randn(Hq * D), _f16(rs.randn(Hkv, T, D)), _f16(v), Hq, Hkv, D, 3, T)
    for h in range(Hq):
        assert np.allclose(out[h * D:(h + 1) * D], h // 2 + 1, atol=1e-14)


def test_attention_matches_scipy_softmax():
    from scipy.special import softmax
    rs = np.random.RandomState(6)
    Hq, Hkv, D, T, n = 4, 2, 16, 12, 9
    kc, vc = _f16(rs.randn(Hkv, T, D)), _f16(rs.randn(Hkv, T, D))
    q = rs.randn(Hq * D)
    out, bound = oracle.attention(q, kc, vc, Hq, Hkv, D, n, T)
    kf, vf = kc.view(np.float16).astype(np.float64), vc.view(np.float16).astype(np.float64)
    for h in range(Hq):
        p = softmax(kf[h // 2, :n] @ q[h * D:(h + 1) * D] / math.sqrt(D))
        assert np.allclose(out[h * D:(h + 1) * D], p @ vf[h // 2, :n], atol=1e-13)
        assert np.allclose(bound[h * D:(h + 1) * D], p @ np.abs(vf[h // 2, :n]), atol=1e-13)


# ----------------------------------------------------------------- SwiGLU
def test_swiglu_closed_forms():
    g = np.array([0.0, 1.0, -1.0, 50.0, -50.0, 2.5])
    u = np.array([3.0, 2.0, 2.0, 0.5, 7.0, -1.0])
    out = oracle.swiglu(g, u)
    assert out[0] == 0.0
    assert abs(out[1] - 2.0 * 0.7310585786300049) < 1e-15
    assert abs(out[2] - 2.0 * -0.2689414213699951) < 1e-15
    assert abs(out[3] - 25.0) < 1e-12
    assert abs(out[4]) < 1e-18
    from scipy.special import expit
    assert abs(out[5] - 2.5 * expit(2.5) * -1.0) < 1e-15


# ----------------------------------------------------------------- cosine / argmax
def test_cosine_invariants():
    rs = np.random.RandomState(7)
    x = rs.randn(4096)
    assert abs(oracle.cosine(x, x) - 1.0) < 1e-15
    assert abs(oracle.cosine(x, -x) + 1.0) < 1e-15
    a, b = np.zeros(4), np.zeros(4)
    a[0], b[1] = 1, 1
    assert oracle.cosine(a, b) == 0.0
    y = rs.randn(4096)
    assert abs(oracle.cosine(x, y) - oracle.cosine(3 * x, 0.1 * y)) < 1e-15
    assert abs(oracle.cosine(x, y) - x @ y / (np.linalg.norm(x) * np.linalg.norm(y))) < 1e-15


def test_argmax_ties_lowest_index():
    v = np.array([1.0, 5.0, 2.0, 5.0, 5.0])
    assert oracle.argmax(v) == 1
    assert oracle.argmax(np.array([-3.0])) == 0


# ----------------------------------------------------------------- layer
def _tiny_cfg(H=64, Hq=4, Hkv=2, D=16, F=96, T=8):
    return oracle.make_config(H, Hq, Hkv, D, F, 100, 1, 1e-5, 500000.0, T)


def _layer_mats(cfg, qtype, seed, zero=()):
    H, Q, KV, F = cfg.hidden, cfg.n_heads * cfg.head_dim, cfg.n_kv_heads * cfg.head_dim, cfg.ffn
    shapes = {"wq": (Q, H), "wk": (KV, H), "wv": (KV, H), "wo": (H, Q), "wg": (F, H), "wu": (F, H), "wd": (H, F)}
    m = {}
    for k, (M, K) in shapes.items():
        m[k] = sg.quant_rows(qtype, seed, k, M, K, sigma=0.0 if k in zero else 0.02)
    m["attn_norm"] = sg.fill_f32(seed, "an", H, mean=1.0, sigma=0.02)
    m["ffn_norm"] = sg.fill_f32(seed, "fn", H, mean=1.0, sigma=0.02)
    return m


def test_layer_zero_weights_is_identity():
    cfg = _tiny_cfg(D=32, F=64)
    m = _layer_mats(cfg, Q8_0, 1, zero=("wq", "wk", "wv", "wo", "wg", "wu", "wd"))
    kc = np.full((2, 8, 32), 0x3C00, dtype=np.uint16)
    vc = kc.copy()
    h = np.random.RandomState(0).randn(64)
    out, c = oracle.layer(cfg, Q8_0, m, m["attn_norm"], m["ffn_norm"], kc, vc, h, 3)
    assert np.array_equal(out, h)
    assert abs(c - 1.0) < 1e-15
    assert np.all((kc[:, 3] & 0x7FFF) == 0) and np.all((vc[:, 3] & 0x7FFF) == 0)  # k = v = +-0 appended at pos
    assert np.all(kc[:, [0, 1, 2, 4, 5, 6, 7]] == 0x3C00)           # other rows untouched


def test_layer_attention_only_path_with_zero_ffn():
    """With Wd = 0 the FFN adds nothing: h_out = h + Wo attn(...).  Rebuild that
    from the oracle's separately pinned parts."""
    cfg = _tiny_cfg(D=32, F=64)
    m = _layer_mats(cfg, Q8_0, 2, zero=("wd",))
    rs = np.random.RandomState(1)
    kc = _f16(rs.randn(2, 8, 32))
    vc = _f16(rs.randn(2, 8, 32))
    h = rs.randn(64)
    kc0, vc0 = kc.copy(), vc.copy()
    out, _ = oracle.layer(cfg, Q8_0, m, m["attn_norm"], m["ffn_norm"], kc, vc, h, 5)
    n1 = oracle.rmsnorm(h, m["attn_norm"].astype(np.float64), 1e-5)
    q, _ = oracle.gemv(Q8_0, m["wq"], 4 * 32, 64, n1)
    k, _ = oracle.gemv(Q8_0, m["wk"], 2 * 32, 64, n1)
    v, _ = oracle.gemv(Q8_0, m["wv"], 2 * 32, 64, n1)
    q = oracle.rope(q, 4, 32, 5, 500000.0)
    k = oracle.rope(k, 2, 32, 5, 500000.0)
    kc0[:, 5] = np.array([oracle.double_to_half(t) for t in k], dtype=np.uint16).reshape(2, 32)
    vc0[:, 5] = np.array([oracle.double_to_half(t) for t in v], dtype=np.uint16).reshape(2, 32)
    assert np.array_equal(kc, kc0) and np.array_equal(vc, vc0)
    a, _ = oracle.attention(q, kc0, vc0, 4, 2, 32, 6, 8)
    o, _ = oracle.gemv(Q8_0, m["wo"], 64, 4 * 32, a)
    assert np.allclose(out, h + o, rtol=0, atol=1e-14)


def test_layer_is_causal_in_cache():
    cfg = _tiny_cfg()
    m = _layer_mats(cfg, Q8_0, 3)
    rs = np.random.RandomState(2)
    kc, vc = _f16(rs.randn(2, 8, 16)), _f16(rs.randn(2, 8, 16))
    kc2, vc2 = kc.copy(), vc.copy()
    kc2[:, 5:] = 0x5000
    vc2[:, 5:] = 0xD000
    h = rs.randn(64)
    o1, c1 = oracle.layer(cfg, Q8_0, m, m["attn_norm"], m["ffn_norm"], kc, vc, h, 4)
    o2, c2 = oracle.layer(cfg, Q8_0, m, m["attn_norm"], m["ffn_norm"], kc2, vc2, h, 4)
    assert np.array_equal(o1, o2) and c1 == c2
    assert abs(c1 - oracle.cosine(h, o1)) < 1e-15


def test_layer_ffn_only_path_with_zero_attention_output():
    """With Wo = 0 attention adds nothing: h_out = h + Wd (silu(Wg n) * Wu n),
    n = RMSNorm(h) w_ffn.  Rebuild that from the oracle's separately pinned parts."""
    cfg = _tiny_cfg(D=32, F=64)
    m = _layer_mats(cfg, Q8_0, 4, zero=("wo",))
    rs = np.random.RandomState(3)
    kc, vc = _f16(rs.randn(2, 8, 32)), _f16(rs.randn(2, 8, 32))
    h = rs.randn(64)
    out, c = oracle.layer(cfg, Q8_0, m, m["attn_norm"], m["ffn_norm"], kc, vc, h, 2)
    n2 = oracle.rmsnorm(h, m["ffn_norm"].astype(np.float64), 1e-5)
    g, _ = oracle.gemv(Q8_0, m["wg"], 64, 64, n2)
    u, _ = oracle.gemv(Q8_0, m["wu"], 64, 64, n2)
    d, _ = oracle.gemv(Q8_0, m["wd"], 64, 64, oracle.swiglu(g, u))
    assert np.allclose(out, h + d, rtol=0, atol=1e-14)
    assert abs(c - oracle.cosine(h, out)) < 1e-15


# ----------------------------------------------------------------- embed / head / model step
def test_embed_is_the_fp16_row():
    t = _f16(np.random.RandomState(7).randn(5, 48))
    for tok in (0, 3, 4):
        assert np.array_equal(oracle.embed(t, 48, tok), t[tok].view(np.float16).astype(np.float64))


def test_head_applies_the_final_norm():
    """Logits are the head GEMV of RMSNorm(h) w_final: equal to the pinned GEMV of
    the pinned RMSNorm, and blind to the scale of h up to eps."""
    cfg = oracle.make_config(64, 4, 2, 16, 96, 40, 1, 1e-5, 500000.0, 8)
    W = sg.quant_rows(Q8_0, 5, "head", 40, 64)
    fn = sg.fill_f32(5, "fn", 64, mean=1.0, sigma=0.02)
    h = np.random.RandomState(4).randn(64)
    logits = oracle.head(cfg, Q8_0, W, fn, h)
    ref, _ = oracle.gemv(Q8_0, W, 40, 64, oracle.rmsnorm(h, fn.astype(np.float64), 1e-5))
    assert np.array_equal(logits, ref)
    # eps = 1e-5 against mean(h^2) ~ 1 shifts the scale by at most ~5e-6
    assert np.allclose(oracle.head(cfg, Q8_0, W, fn, 1000.0 * h), logits, rtol=1e-5, atol=0)
    assert not np.allclose(1000.0 * logits, logits)


def _tiny_model(L, seed, zero_layers):
    cfg = oracle.make_config(64, 4, 2, 16, 96, 40, L, 1e-5, 500000.0, 8)
    names = ("wq", "wk", "wv", "wo", "wg", "wu", "wd")
    layers = [_layer_mats(cfg, Q8_0, seed + l, zero=names if zero_layers else ()) for l in range(L)]
    W = sg.quant_rows(Q8_0, seed, "head", 40, 64)
    fn = sg.fill_f32(seed, "fn", 64, mean=1.0, sigma=0.02)
    emb = sg.fill_f16(seed, "emb", 40 * 64, sigma=0.5).reshape(40, 64)
    return cfg, layers, W, fn, emb


def _caches(L, seed):
    rs = np.random.RandomState(seed)
    return [_f16(rs.randn(2, 8, 16)) for _ in range(L)], [_f16(rs.randn(2, 8, 16)) for _ in range(L)]


def test_model_step_with_every_layer_skipped_is_head_of_embedding():
    """Skipped layers are neither computed nor appended to their cache."""
    cfg, layers, W, fn, emb = _tiny_model(3, 11, zero_layers=False)
    kcs, vcs = _caches(3, 1)
    k0, v0 = [k.copy() for k in kcs], [v.copy() for v in vcs]
    logits, cos = oracle.model_step(cfg, Q8_0, layers, Q8_0, W, fn, emb, kcs, vcs, 9, 4, skip=[1, 1, 1])
    assert np.array_equal(logits, oracle.head(cfg, Q8_0, W, fn, oracle.embed(emb, 64, 9)))
    assert np.all(np.isnan(cos))
    assert all(np.array_equal(a, b) for a, b in zip(kcs + vcs, k0 + v0))


def test_model_step_skip_changes_only_the_skipped_layer():
    cfg, layers, W, fn, emb = _tiny_model(3, 12, zero_layers=False)
    kcs, vcs = _caches(3, 2)
    k0, v0 = [k.copy() for k in kcs], [v.copy() for v in vcs]
    _, cos = oracle.model_step(cfg, Q8_0, layers, Q8_0, W, fn, emb, kcs, vcs, 3, 5, skip=[0, 1, 0])
    assert np.isnan(cos[1]) and not np.isnan(cos[0]) and not np.isnan(cos[2])
    assert np.array_equal(kcs[1], k0[1]) and np.array_equal(vcs[1], v0[1])
    assert not np.array_equal(kcs[0][:, 5], k0[0][:, 5]) and not np.array_equal(kcs[2][:, 5], k0[2][:, 5])
    rows = [p for p in range(8) if p != 5]
    assert np.array_equal(kcs[0][:, rows], k0[0][:, rows]) and np.array_equal(vcs[2][:, rows], v0[2][:, rows])


def test_model_step_of_identity_layers():
    """All-zero projection weights make every layer the identity (cosine 1), so
    the logits are the head of the embedding row and the token picks the row."""
    cfg, layers, W, fn, emb = _tiny_model(2, 13, zero_layers=True)
    for tok in (0, 17, 39):
        kcs, vcs = _caches(2, 3)
        logits, cos = oracle.model_step(cfg, Q8_0, layers, Q8_0, W, fn, emb, kcs, vcs, tok, 6)
        assert np.array_equal(logits, oracle.head(cfg, Q8_0, W, fn, oracle.embed(emb, 64, tok)))
        assert np.allclose(cos, 1.0, rtol=0, atol=1e-15)
