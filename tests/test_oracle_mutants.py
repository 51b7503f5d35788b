"""Plants plausible mistakes in copies of the oracle's C source and checks that
the pin battery (tests/test_oracle_pins.py, tests/test_oracle_brute.py)
catches every one: a dropped term, a wrong sign or index, a swapped operand.

The mutants are compiled into temporary libraries on the CPU; the committed
oracle is untouched.
"""
import os
import tempfile

import pytest

import oracle as orc
from oracle import build as orc_build
import test_oracle_brute as tb
import test_oracle_pins as tp

# (name, [(original text, mutated text), ...])
MUTANTS = [
    ("rope_sign", [("v[i] = x0 * c - x1 * s;", "v[i] = x0 * c + x1 * s;")]),
    ("rope_freq", [("pow(theta, -2.0 * i / head_dim)", "pow(theta, -1.0 * i / head_dim)")]),
    ("rope_interleaved_pairs", [
        ("double x0 = v[i], x1 = v[i + half];", "double x0 = v[2 * i], x1 = v[2 * i + 1];"),
        ("v[i] = x0 * c - x1 * s;\n        v[i + half] = x1 * c + x0 * s;",
         "v[2 * i] = x0 * c - x1 * s;\n        v[2 * i + 1] = x1 * c + x0 * s;")]),
    ("rope_k_skipped", [("orc_rope(k + (size_t)g * hd, hd, pos, c->rope_theta);", ";")]),
    ("rmsnorm_gain_dropped", [("out[i] = orc_bf16_to_double(g[i]) * (x[i] * inv);",
                               "out[i] = (x[i] * inv);")]),
    ("rmsnorm_eps_dropped", [("sqrt(ss / n + eps)", "sqrt(ss / n)")]),
    ("rmsnorm_sum_not_mean", [("sqrt(ss / n + eps)", "sqrt(ss + eps)")]),
    ("ffn_norm_uses_attn_gain", [("orc_rmsnorm(x, w->ffn_norm[l]", "orc_rmsnorm(x, w->attn_norm[l]")]),
    ("final_norm_skipped", [("orc_rmsnorm(x, w->final_norm, h, c->rms_eps, u);",
                             "memcpy(u, x, sizeof(double) * h);")]),
    ("attn_scale_dropped", [("double scale = 1.0 / sqrt((double)head_dim);", "double scale = 1.0;")]),
    ("attn_excludes_current", [("orc_attention_head(q + (size_t)hh * hd, Kc, Vc, pos + 1, hd,",
                                "orc_attention_head(q + (size_t)hh * hd, Kc, Vc, pos > 0 ? pos : 1, hd,")]),
    ("gqa_interleaved_map", [("int32_t g = hh / group;", "int32_t g = hh % nkv;")]),
    ("residual_dropped_attn", [("x[i] += o[i];", "x[i] = o[i];")]),
    ("residual_dropped_ffn", [("x[i] += dn[i];", "x[i] = dn[i];")]),
    ("silu_is_sigmoid", [("return z / (1.0 + exp(-z));", "return 1.0 / (1.0 + exp(-z));")]),
    ("swiglu_swapped", [("a[j] = orc_silu(gt[j]) * up[j];", "a[j] = orc_silu(up[j]) * gt[j];")]),
    ("int8_scale_dropped", [("y[j] = orc_fp16_to_double(scale[j]) * acc;", "y[j] = acc;")]),
    ("int4_nibbles_swapped", [("int nib = (row[k >> 1] >> ((k & 1) * 4)) & 0xF;",
                               "int nib = (row[k >> 1] >> ((~k & 1) * 4)) & 0xF;")]),
    ("int4_unsigned_codes", [("return nib >= 8 ? nib - 16 : nib;", "return nib;")]),
    ("int4_offset_binary", [("return nib >= 8 ? nib - 16 : nib;", "return nib - 8;")]),
    ("int4_group_of_64", [("sj[k / ORC_INT4_GROUP]", "sj[k / 64]")]),
    ("int4_row_stride_bytes", [("(const uint8_t *)W + (size_t)j * (cols / 2);",
                                "(const uint8_t *)W + (size_t)j * cols;")]),
    ("matvec_transposed", [("acc += orc_bf16_to_double(w[k]) * x[k];",
                            "acc += orc_bf16_to_double(((const uint16_t *)W)[(size_t)k * rows + j]) * x[k];")]),
    ("embed_row_index", [("w->embed[(size_t)token * h + i]", "w->embed[(size_t)token + i]")]),
    ("kv_round_truncates", [("double q = nearbyint(ldexp(v, -step));", "double q = trunc(ldexp(v, -step));")]),
    ("fp16_bias", [("v = ldexp((double)(m + 1024), e - 25);", "v = ldexp((double)(m + 1024), e - 24);")]),
    ("argmax_last_tie", [("if (v[i] > v[best])", "if (v[i] >= v[best])")]),
    ("v_cache_gets_k", [("Vc[(size_t)pos * hd + t] = orc_double_to_bf16(v[(size_t)g * hd + t]);",
                         "Vc[(size_t)pos * hd + t] = orc_double_to_bf16(k[(size_t)g * hd + t]);")]),
]

# cheap op-level pins first, whole-step comparisons last
BATTERY = [getattr(tp, n) for n in dir(tp) if n.startswith("test_")] + [
    tb.test_tiny_full_sequence_12_positions,
    tb.test_tiny_tied_head,
    tb.test_tiny_w8a16,
    tb.test_tiny_w4a16,
    tb.test_gqa_head_to_group_mapping_at_pos0,
]


def _caught(lib) -> str:
    saved = orc._LIB
    orc._LIB = lib
    try:
        for t in BATTERY:
            try:
                t()
            except (AssertionError, ValueError, FloatingPointError) as e:
                return t.__name__
        return ""
    finally:
        orc._LIB = saved


@pytest.mark.parametrize("name,edits", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(name, edits):
    src = open(orc_build.SRC).read()
    for old, new in edits:
        assert src.count(old) == 1, f"mutation site for {name} not found once"
        src = src.replace(old, new)
    with tempfile.TemporaryDirectory() as d:
        c_path = os.path.join(d, "mutant.c")
        open(c_path, "w").write(src)
        so = os.path.join(d, "libmutant.so")
        saved_src = orc_build.SRC
        try:
            orc_build.SRC = c_path
            orc_build.build(out=so, force=True)
        finally:
            orc_build.SRC = saved_src
        lib = orc.load(so)
        assert _caught(lib), f"mutant {name} passed every pin"
