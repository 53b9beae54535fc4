"""Pins for the oracle's Q4_K, Q5_K, F16 and F32 weight formats against facts
fixed outside the oracle: the format table's sizes, a hand-derived map of
every packed scale/min bit (golden fixture), one-hot code positions written
from the layout statement, values on the quantisation grid through the
generator's independent packer, numpy's binary16/binary32 decoding, and
brute-force GEMVs on exact integer inputs.  CPU only.

Layout reading (GGUF's; the pages give the sizes only): Q4_K = fp16 d | fp16
dmin | 12 scale bytes | qs[128] (144 B); Q5_K = the same plus qh[32] before
qs (176 B); element n = 64c + 32h + l takes nibble h of qs[32c + l] and, for
Q5_K, bit 2c + h of qh[l] as its fifth bit; w = d sc_j q - dmin m_j with
j = n / 32."""
import numpy as np
import pytest

import oracle
import synthgen as sg
from conftest import read_golden

Q4_K, Q5_K, F16, F32 = oracle.Q4_K, oracle.Q5_K, oracle.F16, oracle.F32
NBYTES = {Q4_K: 144, Q5_K: 176}
QS_OFF = {Q4_K: 16, Q5_K: 48}


def _blk(qt, d=0x3C00, dmin=0x3C00):
    b = np.zeros(NBYTES[qt], dtype=np.uint8)
    b[0], b[1] = d & 0xFF, d >> 8
    b[2], b[3] = dmin & 0xFF, dmin >> 8
    return b


def _all_scales_one(b):
    """sc_j = 1, m_j = 0 for every sub-block (bytes 0-3 and the low nibbles of 8-11)."""
    b[4:8] = 1
    b[12:16] = 0x01
    return b


@pytest.mark.parametrize("qt", [Q4_K, Q5_K])
def test_every_scale_and_min_bit_from_fixture(qt):
    rows = read_golden("k_quant_scale_bits.txt")
    assert len(rows) == 96
    seen = set()
    for field, j, bit, byte, pos in rows:
        j, bit, byte, pos = int(j), int(bit), int(byte), int(pos)
        b = _blk(qt)  # d = dmin = 1
        b[QS_OFF[qt]:QS_OFF[qt] + 128] = 0x11  # every low code 1 (Q5_K fifth bits 0): q = 1
        b[4 + byte] = 1 << pos
        w = oracle.dequant(qt, b, 256)
        exp = np.zeros(256)
        exp[32 * j:32 * j + 32] = (2.0 ** bit) if field == "sc" else -(2.0 ** bit)
        assert np.array_equal(w, exp), (field, j, bit, byte, pos)
        seen.add((byte, pos))
    assert len(seen) == 96  # 12 bytes x 8 bits, each used exactly once


@pytest.mark.parametrize("qt", [Q4_K, Q5_K])
def test_every_code_nibble_reaches_its_element(qt):
    for i in range(128):
        for h in range(2):
            b = _all_scales_one(_blk(qt, dmin=0))
            b[QS_OFF[qt] + i] = 1 << (4 * h)
            w = oracle.dequant(qt, b, 256)
            exp = np.zeros(256)
            exp[64 * (i // 32) + 32 * h + i % 32] = 1.0
            assert np.array_equal(w, exp), (i, h)


def test_q5_k_every_fifth_bit_reaches_its_element():
    seen = set()
    for l in range(32):
        for bit in range(8):
            b = _all_scales_one(_blk(Q5_K, dmin=0))
            b[16 + l] = 1 << bit
            w = oracle.dequant(Q5_K, b, 256)
            n = 64 * (bit // 2) + 32 * (bit % 2) + l
            exp = np.zeros(256)
            exp[n] = 16.0
            assert np.array_equal(w, exp), (l, bit)
            seen.add(n)
    assert seen == set(range(256))


@pytest.mark.parametrize("qt", [Q4_K, Q5_K])
def test_scale_min_formula_and_signs(qt):
    b = _blk(qt, d=0xB800, dmin=0x4000)  # d = -0.5, dmin = 2
    b[4 + 0] = 63          # sc_0 = 63
    b[4 + 4] = 5           # m_0 = 5
    b[QS_OFF[qt]] = 0x0F   # element 0: low code 15
    if qt == Q5_K:
        b[16] = 0x01       # element 0: fifth bit -> q = 31
    w = oracle.dequant(qt, b, 256)
    q0 = 31 if qt == Q5_K else 15
    assert w[0] == -0.5 * 63 * q0 - 2.0 * 5
    assert w[1] == -2.0 * 5          # q = 0
    assert np.all(w[32:] == 0.0)     # sc = m = 0 elsewhere


@pytest.mark.parametrize("qt", [Q4_K, Q5_K])
def test_dequant_inverts_independent_packer_on_grid(qt):
    """Values on the grid w = d sc q - dmin m (d, dmin powers of two; in each
    super-block one scale and one min at 63; in each sub-block a code 0 and a
    code n_max) come back unchanged through the generator's packer."""
    rs = np.random.RandomState(qt)
    nmax = 31 if qt == Q5_K else 15
    d, dmin = np.float32(2.0 ** -10), np.float32(2.0 ** -9)
    nblk = 10
    w = np.zeros((nblk, 256), dtype=np.float32)
    for bi in range(nblk):
        sc = rs.randint(1, 64, size=8)
        mi = rs.randint(0, 64, size=8)
        sc[rs.randint(8)] = 63
        mi[rs.randint(8)] = 63
        for j in range(8):
            q = rs.randint(0, nmax + 1, size=32)
            q[0], q[1] = 0, nmax
            w[bi, 32 * j:32 * j + 32] = d * sc[j] * q - dmin * mi[j]
    blocks = sg.quantize(qt, w)
    assert blocks.size == nblk * NBYTES[qt]
    got = oracle.dequant(qt, blocks, w.size)
    assert np.array_equal(got, w.astype(np.float64).ravel())


def test_f16_and_f32_are_ieee_values():
    rs = np.random.RandomState(9)
    h = rs.randint(0, 1 << 16, size=4096).astype(np.uint16)
    ref = h.view(np.float16).astype(np.float64)
    got = oracle.dequant(F16, h.view(np.uint8), h.size)
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin], ref[fin])
    f = (rs.randn(1000) * 10.0 ** rs.uniform(-30, 30, 1000)).astype(np.float32)
    assert np.array_equal(oracle.dequant(F32, f.view(np.uint8), f.size), f.astype(np.float64))


@pytest.mark.parametrize("qt", [Q4_K, Q5_K])
def test_gemv_brute_force_exact(qt):
    """Integer codes, d = 1/4, dmin = 1/8, integer x: every product and sum is
    exact in double, so the oracle equals the integer matmul of the closed form."""
    rs = np.random.RandomState(100 + qt)
    M, K = 3, 512
    nmax = 31 if qt == Q5_K else 15
    q = rs.randint(0, nmax + 1, size=(M, K))
    sc = rs.randint(0, 64, size=(M, K // 32))
    mi = rs.randint(0, 64, size=(M, K // 32))
    W = np.zeros((M, K // 256, NBYTES[qt]), dtype=np.uint8)
    W[..., 0], W[..., 1] = 0x00, 0x34  # d = 0.25
    W[..., 2], W[..., 3] = 0x00, 0x30  # dmin = 0.125
    for r in range(M):
        for s in range(K // 256):
            p = W[r, s, 4:16]
            S, Mn = sc[r, 8 * s:8 * s + 8], mi[r, 8 * s:8 * s + 8]
            for j in range(4):  # the packing of the fixture's map, written out
                p[j] = (S[j] & 63) | ((S[j + 4] >> 4) << 6)
                p[j + 4] = (Mn[j] & 63) | ((Mn[j + 4] >> 4) << 6)
                p[j + 8] = (S[j + 4] & 15) | ((Mn[j + 4] & 15) << 4)
            qq = q[r, 256 * s:256 * s + 256]
            for n in range(256):
                c, h, l = n // 64, (n % 64) // 32, n % 32
                W[r, s, QS_OFF[qt] + 32 * c + l] |= (qq[n] & 15) << (4 * h)
                if qt == Q5_K:
                    W[r, s, 16 + l] |= ((qq[n] >> 4) & 1) << (2 * c + h)
    Wd = 0.25 * np.repeat(sc, 32, axis=1) * q - 0.125 * np.repeat(mi, 32, axis=1)
    x = rs.randint(-7, 8, size=K)
    y, b = oracle.gemv(qt, W.reshape(M, -1), M, K, x.astype(np.float64))
    assert np.array_equal(y, Wd @ x)
    assert np.array_equal(b, np.abs(Wd) @ np.abs(x))
    assert np.array_equal(oracle.dequant(qt, W.reshape(-1), M * K), Wd.ravel())


@pytest.mark.parametrize("qt", [F16, F32])
def test_gemv_float_formats_brute_force(qt):
    rs = np.random.RandomState(qt)
    M, K = 4, 96
    Wf = (rs.randint(-64, 65, size=(M, K)) / 64.0).astype(np.float16 if qt == F16 else np.float32)
    x = rs.randint(-9, 10, size=K).astype(np.float64)
    y, _ = oracle.gemv(qt, Wf.view(np.uint8).reshape(M, -1), M, K, x)
    assert np.array_equal(y, Wf.astype(np.float64) @ x)


def test_layer_per_matrix_types_match_uniform_dequantised_layer():
    """A mixed-type layer equals the same layer with every matrix re-encoded
    as F32 (its dequantised values, exact), the oracle's per-matrix type
    dispatch being the only difference."""
    d = dict(hidden=256, n_heads=2, n_kv_heads=1, head_dim=128, ffn=512, vocab=16, n_layers=1, eps=1e-5,
             theta=500000.0)
    shapes = {"wq": (256, 256), "wk": (128, 256), "wv": (128, 256), "wo": (256, 256), "wg": (512, 256),
              "wu": (512, 256), "wd": (256, 512)}
    types = [Q4_K, Q4_K, Q5_K, Q4_K, Q5_K, Q5_K, oracle.Q6_K]
    mats, f32 = {}, {}
    for (name, (M, K)), qt in zip(shapes.items(), types):
        mats[name] = sg.quant_rows(qt, 11, "mix." + name, M, K)
        deq = oracle.dequant(qt, mats[name], M * K)
        assert np.array_equal(deq, deq.astype(np.float32))  # exact in fp32, so the F32 copy is the same matrix
        f32[name] = deq.astype(np.float32).view(np.uint8).reshape(M, -1)
    mats["qtypes"] = types
    an = sg.fill_f32(11, "an", 256, mean=1.0, sigma=0.02)
    fn = sg.fill_f32(11, "fn", 256, mean=1.0, sigma=0.02)
    cfg = oracle.make_config(256, 2, 1, 128, 512, 16, 1, 1e-5, 500000.0, 8)
    h = sg.fill_f32(11, "h", 256).astype(np.float64)
    outs = []
    for m, qt in ((mats, Q4_K), (f32, F32)):
        kc = np.zeros((1, 8, 128), np.uint16)
        vc = np.zeros_like(kc)
        outs.append(oracle.layer(cfg, qt, m, an, fn, kc, vc, h, 3)[0])
    assert np.array_equal(outs[0], outs[1])
