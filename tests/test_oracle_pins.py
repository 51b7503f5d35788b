"""Pins for the fp64 oracle's single ops: closed forms, invariants, special
cases and exhaustive comparisons against independent library routines.

Each test names the passage or mathematical fact it checks.  The ops are the
instruction set listed in paperfeed "RightNow-AI/AutoMegaKernel", "How it
works" (GEMV tiles, attention tile, RMSNorm, RoPE, SwiGLU, dequant).
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle as orc

BF16_ONE = 0x3F80
BF16_TWO = 0x4000


# ---- number formats --------------------------------------------------------

def test_bf16_decode_known_patterns():
    assert orc.bf16_to_double(0x3F80) == 1.0
    assert orc.bf16_to_double(0xC000) == -2.0
    assert orc.bf16_to_double(0x3F00) == 0.5
    assert orc.bf16_to_double(0x0001) == 2.0 ** -133  # smallest subnormal
    assert orc.bf16_to_double(0x7F80) == math.inf
    assert orc.bf16_to_double(0x4049) == 3.140625


def test_fp16_decode_exhaustive_against_numpy():
    # every non-NaN binary16 pattern, against numpy's float16 (a library
    # decoder written independently of the oracle)
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([orc.fp16_to_double(int(b)) for b in bits])
    ok = np.isnan(ref)
    assert np.array_equal(np.isnan(got), ok)
    assert np.array_equal(got[~ok], ref[~ok])


def _bf16_exact_round(v: float) -> Fraction:
    """Nearest 8-significant-bit value to v with ties to even, by exact
    rational arithmetic over the two candidate neighbours."""
    x = Fraction(v)
    if x == 0:
        return Fraction(0)
    e = math.frexp(v)[1] - 1          # 2**e <= |v| < 2**(e+1)
    step = Fraction(2) ** (e - 7)
    lo = (x / step).__floor__() * step
    hi = lo + step
    dlo, dhi = x - lo, hi - x
    if dlo < dhi:
        return lo
    if dhi < dlo:
        return hi
    return lo if ((lo / step) % 2 == 0) else hi


def test_double_to_bf16_ties_and_random():
    # ties: halfway cases round to the even significand
    assert orc.double_to_bf16(1.0 + 2.0 ** -8) == 0x3F80
    assert orc.double_to_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82
    assert orc.double_to_bf16(-(1.0 + 2.0 ** -8)) == 0xBF80
    assert orc.double_to_bf16(0.0) == 0
    rng = np.random.default_rng(123)
    vals = np.concatenate([rng.standard_normal(3000) * 10.0 ** rng.integers(-6, 6, 3000),
                           rng.integers(-300, 300, 200) / 64.0])
    for v in vals:
        b = orc.double_to_bf16(float(v))
        got = Fraction(orc.bf16_to_double(b))
        assert got == _bf16_exact_round(float(v)), v


# ---- RMSNorm ---------------------------------------------------------------

def test_rmsnorm_closed_form():
    # x = (3, 4): mean square 12.5; with eps = 0 and unit gains the output is
    # x / sqrt(12.5)
    out = orc.rmsnorm([3.0, 4.0], [BF16_ONE, BF16_ONE], 0.0)
    assert np.allclose(out, np.array([3.0, 4.0]) / math.sqrt(12.5), rtol=0, atol=1e-15)


def test_rmsnorm_unit_rms_before_gain_and_eps_term():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(257) * 0.1
    ms = float(np.mean(x * x))
    eps = 1e-5
    out = orc.rmsnorm(x, np.full(257, BF16_ONE, np.uint16), eps)
    rms = math.sqrt(float(np.mean(out * out)))
    assert rms == pytest.approx(math.sqrt(ms / (ms + eps)), rel=1e-13)


def test_rmsnorm_scale_invariance_and_gain():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(64)
    g1 = np.full(64, BF16_ONE, np.uint16)
    a = orc.rmsnorm(x, g1, 0.0)
    b = orc.rmsnorm(7.5 * x, g1, 0.0)
    assert np.allclose(a, b, rtol=1e-14, atol=0)
    c = orc.rmsnorm(x, np.full(64, BF16_TWO, np.uint16), 0.0)
    assert np.allclose(c, 2 * a, rtol=1e-15, atol=0)
    # per-element gain: gains are applied element-wise, not summed or shifted
    g = np.full(64, BF16_ONE, np.uint16)
    g[5] = BF16_TWO
    d = orc.rmsnorm(x, g, 0.0)
    assert d[5] == pytest.approx(2 * a[5], rel=1e-15)
    assert np.allclose(np.delete(d, 5), np.delete(a, 5), rtol=1e-15, atol=0)


# ---- GEMV / dequant ----------------------------------------------------------

def test_matvec_identity_and_one_hot():
    n = 12
    eye = np.zeros((n, n), np.uint16)
    eye[np.arange(n), np.arange(n)] = BF16_ONE
    x = np.arange(1, n + 1, dtype=np.float64) * 0.25
    assert np.array_equal(orc.matvec(eye, x), x)
    # a rectangular W (rows != cols) against a one-hot x picks one column,
    # so a transposed operand would be caught
    rng = np.random.default_rng(2)
    W = rng.integers(0x3C00, 0x4100, size=(5, 9)).astype(np.uint16)
    for k in range(9):
        e = np.zeros(9)
        e[k] = 1.0
        col = np.array([orc.bf16_to_double(int(b)) for b in W[:, k]])
        assert np.array_equal(orc.matvec(W, e), col)


def test_matvec_int8_row_scales():
    # y_j = s_j * sum_k q_jk x_k, fp16 scales 0.5 (0x3800) and 2.0 (0x4000)
    q = np.array([[1, -2, 3], [127, -127, 0]], dtype=np.int8)
    s = np.array([0x3800, 0x4000], dtype=np.uint16)
    x = np.array([1.0, 2.0, 4.0])
    y = orc.matvec(q, x, scale_bits=s)
    assert y[0] == 0.5 * (1 - 4 + 12)
    assert y[1] == 2.0 * (127 - 254)


def test_matvec_int4_nibble_order_and_sign():
    """Packed int4 row, scale 1.0 (fp16 0x3C00): input 2i sits in the low
    nibble of byte i, input 2i + 1 in the high nibble, 4-bit two's
    complement.  Bytes 0x8F, 0x70, 0x21 hold the codes -1, -8, 0, 7, 1, 2,
    read off one by one with one-hot inputs."""
    W = np.array([[0x8F, 0x70, 0x21]], dtype=np.uint8)
    s = np.array([[0x3C00]], dtype=np.uint16)
    want = [-1, -8, 0, 7, 1, 2]
    for k, v in enumerate(want):
        e = np.zeros(6)
        e[k] = 1.0
        assert orc.matvec(W, e, scale_bits=s)[0] == v


def test_matvec_int4_group_scales_ragged_closed_form():
    """576 inputs = four groups of 128 and a last group of 64.  Every code 1
    (byte 0x11) in row 0 and -1 (0xFF) in row 1, group g scaled by 2**g
    (fp16 1, 2, 4, 8, 16), x all ones: y = +-(128 (1 + 2 + 4 + 8) + 64 * 16)
    = +-2944.  A scale indexed per 64 inputs, or the last group taken as
    full, gives another sum."""
    W = np.empty((2, 288), dtype=np.uint8)
    W[0] = 0x11
    W[1] = 0xFF
    s = np.array([[0x3C00, 0x4000, 0x4400, 0x4800, 0x4C00]] * 2, dtype=np.uint16)
    y = orc.matvec(W, np.ones(576), scale_bits=s)
    assert y[0] == 2944.0 and y[1] == -2944.0
    # one input at a time: its group's scale times its code
    for k in (0, 127, 128, 511, 512, 575):
        e = np.zeros(576)
        e[k] = 3.0
        assert orc.matvec(W, e, scale_bits=s)[0] == 3.0 * 2 ** (k // 128)


# ---- RoPE --------------------------------------------------------------------

def test_rope_position_zero_is_identity():
    x = np.random.default_rng(3).standard_normal(16)
    assert np.array_equal(orc.rope(x, 0, 1e4), x)


def test_rope_hd2_closed_form():
    # head_dim 2: a single pair at frequency theta^0 = 1, so the angle is pos
    x0, x1, p = 0.3, -1.7, 5
    y = orc.rope([x0, x1], p, 1e4)
    assert y[0] == pytest.approx(x0 * math.cos(p) - x1 * math.sin(p), abs=1e-15)
    assert y[1] == pytest.approx(x1 * math.cos(p) + x0 * math.sin(p), abs=1e-15)


def test_rope_hd4_pairs_and_frequencies():
    # head_dim 4: pairs (0, 2) at frequency 1 and (1, 3) at theta^(-1/2)
    theta, p = 1e4, 3
    x = np.array([1.0, 0.0, 0.0, 0.0])
    y = orc.rope(x, p, theta)
    assert np.allclose(y, [math.cos(p), 0, math.sin(p), 0], atol=1e-15)
    x = np.array([0.0, 1.0, 0.0, 0.0])
    y = orc.rope(x, p, theta)
    a = p * theta ** -0.5
    assert np.allclose(y, [0, math.cos(a), 0, math.sin(a)], atol=1e-15)


def test_rope_norm_preserving_and_relative():
    rng = np.random.default_rng(4)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    for p in (1, 17, 1000):
        assert np.linalg.norm(orc.rope(q, p, 1e4)) == pytest.approx(np.linalg.norm(q), rel=1e-14)
    # <R_a q, R_b k> depends only on a - b
    d1 = np.dot(orc.rope(q, 10, 1e4), orc.rope(k, 3, 1e4))
    d2 = np.dot(orc.rope(q, 107, 1e4), orc.rope(k, 100, 1e4))
    assert d1 == pytest.approx(d2, rel=1e-10)


# ---- attention -----------------------------------------------------------------

def _bits(vals):
    return np.array([[orc.double_to_bf16(v) for v in row] for row in vals], np.uint16)


def test_attention_single_position_returns_v0():
    K = _bits([[0.5, -1.0, 2.0, 0.25]])
    V = _bits([[1.5, -0.75, 3.0, 8.0]])
    out, p = orc.attention_head(np.array([9.0, -3.0, 1.0, 4.0]), K, V)
    assert np.array_equal(out, [1.5, -0.75, 3.0, 8.0])
    assert p.tolist() == [1.0]


def test_attention_constant_scores_give_mean_of_v():
    rng = np.random.default_rng(5)
    K = _bits(rng.standard_normal((7, 8)))
    Vf = rng.standard_normal((7, 8))
    V = _bits(Vf)
    out, p = orc.attention_head(np.zeros(8), K, V)
    Vd = np.array([[orc.bf16_to_double(int(b)) for b in r] for r in V])
    assert np.allclose(out, Vd.mean(axis=0), rtol=1e-14, atol=1e-15)
    assert np.allclose(p, 1 / 7)


def test_attention_two_positions_closed_form():
    # hd = 2, scale 1/sqrt(2): scores s0 = q.k0/sqrt2, s1 = q.k1/sqrt2
    K = _bits([[1.0, 0.0], [0.0, 1.0]])
    V = _bits([[2.0, 0.0], [0.0, 4.0]])
    q = np.array([math.sqrt(2) * 1.0, 0.0])
    out, p = orc.attention_head(q, K, V)
    e = math.e
    assert p[0] == pytest.approx(e / (e + 1), rel=1e-15)
    assert p[1] == pytest.approx(1 / (e + 1), rel=1e-14)
    assert out[0] == pytest.approx(2 * e / (e + 1), rel=1e-15)
    assert out[1] == pytest.approx(4 / (e + 1), rel=1e-14)


def test_attention_probs_sum_to_one_and_scale():
    rng = np.random.default_rng(6)
    K = _bits(rng.standard_normal((33, 16)) * 3)
    V = _bits(rng.standard_normal((33, 16)))
    q = rng.standard_normal(16) * 3
    out, p = orc.attention_head(q, K, V)
    assert p.sum() == pytest.approx(1.0, abs=1e-14)
    Kd = np.array([[orc.bf16_to_double(int(b)) for b in r] for r in K])
    s = Kd @ q / 4.0  # 1/sqrt(16)
    ref = np.exp(s - s.max())
    assert np.allclose(p, ref / ref.sum(), rtol=1e-12, atol=0)


# ---- SwiGLU / argmax -------------------------------------------------------

def test_silu_values():
    assert orc.silu(0.0) == 0.0
    assert orc.silu(1.0) == pytest.approx(0.7310585786300049, rel=1e-15)
    assert orc.silu(-1.0) == pytest.approx(-0.2689414213699951, rel=1e-15)
    assert orc.silu(40.0) == pytest.approx(40.0, rel=1e-15)
    assert abs(orc.silu(-40.0)) < 1e-15


def test_argmax_first_occurrence():
    assert orc.argmax([1.0, 3.0, 2.0, 3.0]) == 1
    assert orc.argmax([-5.0]) == 0
    assert orc.argmax([0.0, -0.0, 0.0]) == 0
