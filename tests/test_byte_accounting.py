"""Pins of the byte accounting the roofline uses: the streamed-bytes count
equals the tensors the input generator makes, and the int8-scope reading
(the tied LM head stays bf16) reproduces the pages' published byte ratio."""
import os

import pytest

import synth_inputs as si


def _golden(name):
    vals = {}
    with open(os.path.join(os.path.dirname(__file__), "golden", name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                k, v = line.split(None, 1)
                vals[k] = v
    return vals


def test_int8_byte_ratio_matches_published():
    """The int8 scope reading (tied head stays bf16) reproduces the pages'
    0.61x byte ratio; an int8 tied head would give ~0.50."""
    g = _golden("int8_byte_ratio.txt")
    cfg = si.get_config(g["model"])
    ratio = (si.streamed_weight_bytes(cfg.with_(quant="w8a16"))
             / si.streamed_weight_bytes(cfg.with_(quant="bf16")))
    assert abs(ratio - float(g["ratio"])) <= float(g["abs_tolerance"]), ratio


def test_int4_byte_ratio_matches_published():
    """The W4A16 reading (symmetric int4, one fp16 scale per 128 inputs of a
    row, tied head in bf16) against the pages' 2.42x weight-traffic cut; one
    scale per row (2.44x) or per 64 inputs (2.38x) falls outside."""
    g = _golden("int4_byte_ratio.txt")
    cfg = si.get_config(g["model"])
    ratio = (si.streamed_weight_bytes(cfg.with_(quant="bf16"))
             / si.streamed_weight_bytes(cfg.with_(quant="w4a16")))
    assert abs(ratio - float(g["ratio"])) <= float(g["abs_tolerance"]), ratio


@pytest.mark.parametrize("tied", [False, True])
@pytest.mark.parametrize("quant", ["bf16", "w8a16", "w4a16"])
def test_byte_accounting_matches_generated_tensors(tied, quant):
    """model_bytes / streamed_weight_bytes count exactly the tensors that
    make_model produces (so the byte ratio above is about real weights)."""
    cfg = si.get_config("tiny").with_(tied=tied, quant=quant)
    m = si.make_model(cfg)
    layer_keys = ("wq", "wk", "wv", "wo", "wgate", "wup", "wdown")
    nb = lambda t: t.numel() * t.element_size()
    linear = sum(nb(t) for k in layer_keys for t in m[k])
    scales = sum(nb(t) for k in layer_keys if m["s" + k[1:]] for t in m["s" + k[1:]])
    if m["lm_head_scale"] is not None:
        scales += nb(m["lm_head_scale"])
    head = nb(m["embed"]) if tied else nb(m["lm_head"])
    norms = nb(m["final_norm"]) + sum(nb(t) for t in m["attn_norm"] + m["ffn_norm"])
    row = m["embed"].shape[1] * m["embed"].element_size()
    assert si.streamed_weight_bytes(cfg) == linear + scales + head + norms + row
