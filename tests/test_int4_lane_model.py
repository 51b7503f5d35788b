"""The integer arithmetic of the int4 GEMV, modelled in numpy on one packed
row, against the oracle's matrix-vector product on the same quantised
activations.  It checks the bit-level steps the kernel takes before they run
on a device: the XOR that turns 4-bit two's-complement codes into code + 8,
the masks that split a 32-bit word into even and odd codes, the order of the
int16 activation pairs fed to the two-way dot products, the bias of
8 x the activation sum, and the group-scale index of each 16-byte vector.
Nothing here is shared with the CUDA source; the model restates its steps."""
import numpy as np
import pytest

import oracle as orc
import synth_inputs as si


def _dp2a(a_pair, b_word, hi):
    """int16 pair (lo, hi halves of a) times unsigned bytes 0, 1 or 2, 3 of b."""
    def s16(u):
        return u - 0x10000 if u >= 0x8000 else u
    x0 = s16(a_pair & 0xFFFF)
    x1 = s16((a_pair >> 16) & 0xFFFF)
    sh = 16 if hi else 0
    b0 = (b_word >> sh) & 0xFF
    b1 = (b_word >> (sh + 8)) & 0xFF
    return x0 * b0 + x1 * b1


def _pair(a, b):
    return (int(a) & 0xFFFF) | ((int(b) & 0xFFFF) << 16)


def lane_model_row(packed_row, scales_row, xq, K):
    """sum over the row's 16-byte code vectors of group_scale(v) *
    (sum of dp2a terms - 8 * sum(xq of the vector)), as the kernel does."""
    total = 0.0
    for v in range(K // 32):
        vec = packed_row[16 * v:16 * v + 16]
        words = [int.from_bytes(bytes(vec[4 * q:4 * q + 4]), "little") for q in range(4)]
        xv = xq[32 * v:32 * v + 32]
        s = 0
        for q, wd in enumerate(words):
            t = wd ^ 0x88888888
            lo = t & 0x0F0F0F0F
            hi = (t >> 4) & 0x0F0F0F0F
            e = xv[8 * q:8 * q + 8]
            s += _dp2a(_pair(e[0], e[2]), lo, False)
            s += _dp2a(_pair(e[4], e[6]), lo, True)
            s += _dp2a(_pair(e[1], e[3]), hi, False)
            s += _dp2a(_pair(e[5], e[7]), hi, True)
        s -= 8 * int(np.sum(xv.astype(np.int64)))
        total += float(np.float16(scales_row.view(np.float16)[v >> 2])) * s
    return total


@pytest.mark.parametrize("K", [64, 192, 576, 2048])
def test_lane_model_equals_oracle_matvec(K):
    cfg = si.get_config("tiny").with_(quant="w4a16", hidden=K, ffn=192, n_heads=4,
                                      n_kv_heads=2, head_dim=K // 4)
    w = si.make_model(cfg, seed=5)
    W = orc.to_numpy_bits(w["wq"][0])      # packed [rows, K / 2]
    S = orc.to_numpy_bits(w["sq"][0])      # fp16 bits [rows, groups]
    rng = np.random.default_rng(K)
    xq = rng.integers(-32767, 32768, size=K).astype(np.int64)
    ref = orc.matvec(W, xq.astype(np.float64), scale_bits=S)
    for r in range(min(8, W.shape[0])):
        got = lane_model_row(W[r], S[r], xq, K)
        assert abs(got - ref[r]) <= 1e-9 * max(1.0, abs(ref[r])), (r, got, ref[r])


def test_lane_model_extreme_codes():
    """Every code value -8 .. 7 against the largest int16 activations: the
    int32 sum of one vector stays exact and the bias removes the offset."""
    K = 32
    codes = np.tile(np.arange(-8, 8), 2)
    nib = codes & 0xF
    packed = (nib[0::2] | (nib[1::2] << 4)).astype(np.uint8)
    scales = np.array([0x3C00], dtype=np.uint16)  # 1.0
    for xv in (np.full(K, 32767), np.full(K, -32767), np.arange(K) * 1000 - 16000):
        xq = np.asarray(xv, dtype=np.int64)
        want = int(np.dot(codes, xq))
        assert lane_model_row(packed, scales, xq, K) == want
        assert abs(want) < 2 ** 31
