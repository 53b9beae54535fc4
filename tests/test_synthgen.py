"""Pins for the seeded input generator (host build).  CPU only."""
import math

import numpy as np
import pytest

import synthgen as sg
from conftest import read_golden


def test_philox_known_answers():
    rows = read_golden("philox4x32_10_kat.txt")
    assert len(rows) == 3
    for r in rows:
        v = [int(t, 16) for t in r]
        assert sg.philox(v[0:4], v[4:6]) == v[6:10]


def test_ln_series_matches_libm():
    rs = np.random.RandomState(1)
    for s in list(rs.uniform(1e-12, 1.0, 2000)) + [0.5, 2.0 ** -64, 0.999999999, 1e-300]:
        got = sg.host_lib().sg_ln(float(s))
        assert abs(got - math.log(s)) <= 4e-16 * max(1.0, abs(math.log(s)))


def test_normal_distribution_moments():
    x = sg.fill_f32(7, "moments", 400000).astype(np.float64)
    assert abs(x.mean()) < 0.01
    assert abs(x.std() - 1.0) < 0.01
    # fraction inside one and two standard deviations of N(0,1)
    assert abs(np.mean(np.abs(x) < 1.0) - 0.682689) < 0.004
    assert abs(np.mean(np.abs(x) < 2.0) - 0.954500) < 0.002
    # Kolmogorov-Smirnov distance against the normal CDF
    from scipy.stats import kstest
    assert kstest(x[:50000], "norm").statistic < 0.01


def test_scaled_streams_and_determinism():
    a = sg.fill_f32(3, "w", 1000, mean=0.0, sigma=0.02, nthreads=1)
    b = sg.fill_f32(3, "w", 1000, mean=0.0, sigma=0.02, nthreads=7)
    assert a.tobytes() == b.tobytes()
    z = np.array([sg.normal_at(3, "w", i) for i in range(1000)])
    assert np.array_equal(a, (0.0 + 0.02 * z).astype(np.float32))
    c = sg.fill_f32(3, "other", 1000, sigma=0.02)
    assert not np.array_equal(a, c)
    n = sg.fill_f32(3, "norm", 1000, mean=1.0, sigma=0.02)
    assert abs(n.mean() - 1.0) < 0.005


@pytest.mark.filterwarnings("ignore:overflow")
def test_half_conversion_matches_ieee():
    rs = np.random.RandomState(2)
    vals = np.concatenate([rs.randn(20000) * 10.0 ** rs.uniform(-9, 5, 20000),
                           np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e9, -1e9, 2.0 ** -24, 2.0 ** -25,
                                     3 * 2.0 ** -26, 2.0 ** -14, 6.1e-5])]).astype(np.float32)
    got = np.array([sg.half_from_float(float(v)) for v in vals], dtype=np.uint16)
    assert np.array_equal(got, vals.astype(np.float16).view(np.uint16))  # numpy rounds to nearest even


def test_token_range_and_uniformity():
    t = sg.tokens(11, "prompt", 100000, 128256)
    assert t.min() >= 0 and t.max() < 128256
    hist = np.bincount(t * 16 // 128256, minlength=16)
    assert hist.min() > 0.9 * len(t) / 16


@pytest.mark.parametrize("qtype", [sg.Q8_0, sg.Q4_0, sg.Q6_K])
def test_quant_rows_thread_invariant(qtype):
    a = sg.quant_rows(qtype, 5, "m", 16, 512, nthreads=1)
    b = sg.quant_rows(qtype, 5, "m", 16, 512, nthreads=6)
    assert a.tobytes() == b.tobytes()
    part = sg.quant_rows(qtype, 5, "m", 16, 512, row0=5, nrows=3, nthreads=2)
    assert part.tobytes() == a[5:8].tobytes()


def test_q8_0_recipe():
    """d = fp16(max|w|/127), q = round(w/d) with the largest |w| at |q| = 127."""
    w = sg.fill_f32(9, "q8", 32 * 64, sigma=0.02)
    blk = sg.quantize(sg.Q8_0, w).reshape(64, 34)
    for b in range(64):
        wb = w[32 * b: 32 * b + 32]
        d32 = np.float32(np.abs(wb).max()) / np.float32(127.0)
        assert int(blk[b, 0]) | (int(blk[b, 1]) << 8) == np.float16(d32).view(np.uint16)
        q = blk[b, 2:].view(np.int8).astype(int)
        assert np.abs(q).max() == 127
        assert q[np.argmax(np.abs(wb))] == np.sign(wb[np.argmax(np.abs(wb))]) * 127


def test_q4_0_recipe():
    """d = (signed max-|w| element)/-8 ; that element quantizes to 0 (w = 8 d)."""
    w = sg.fill_f32(9, "q4", 32 * 64, sigma=0.02)
    blk = sg.quantize(sg.Q4_0, w).reshape(64, 18)
    for b in range(64):
        wb = w[32 * b: 32 * b + 32]
        m = wb[np.argmax(np.abs(wb))]
        assert int(blk[b, 0]) | (int(blk[b, 1]) << 8) == np.float16(np.float32(m) / np.float32(-8.0)).view(np.uint16)
        j = int(np.argmax(np.abs(wb)))
        byte = blk[b, 2 + (j % 16)]
        q = (byte & 15) if j < 16 else (byte >> 4)
        assert q == 0


def test_block_sizes_reproduce_printed_bits_per_weight():
    rows = read_golden("format_sizes.txt")
    for r in rows:
        if r[0] == "layer70b_mib":
            continue
        qt, be, bpw, tol = int(r[0]), int(r[1]), float(r[2]), float(r[3])
        assert sg.BLOCK_ELEMS[qt] == be
        assert abs(8.0 * sg.BLOCK_BYTES[qt] / be - bpw) <= tol + 1e-12
    mib, tol = [(float(r[1]), float(r[2])) for r in rows if r[0] == "layer70b_mib"][0]
    H, Q, KV, F = 8192, 64 * 128, 8 * 128, 28672
    weights = H * Q + 2 * H * KV + Q * H + 3 * H * F
    layer_bytes = weights // 256 * 210
    assert layer_bytes == 701890560
    assert abs(layer_bytes / 2 ** 20 - mib) <= tol
