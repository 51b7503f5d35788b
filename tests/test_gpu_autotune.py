"""Schedule-knob search: candidates are lowered and validated by amk_create,
gated on the default schedule's logits, timed, and the fastest kept
(README "Two autoresearch loops": lower -> validate -> check -> measure ->
keep or revert)."""
import pytest
import torch

import persistent_megakernel_decode_cta_b200 as amk
from persistent_megakernel_decode_cta_b200 import autotune, build
import synth_inputs as si
from parity_helpers import Pair, compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built(cuda_ok):
    build.build()


def test_tune_keeps_fastest_passing_schedule():
    cfg = si.get_config("tinyllama")
    w = si.make_model(cfg, device="cuda")
    kv = si.make_kv_fill(cfg, 64, device="cuda")
    space = {"ring_stages": [2, 3], "ffn_fused": [1, 2], "stage_bytes": [65536, 1000]}
    best, rows = autotune.tune(cfg, w, ctx=64, kv=kv, space=space, steps=5)
    assert len(rows) == 1 + 8
    bad = [r for r in rows if r["knobs"].get("stage_bytes") == 1000]
    assert bad and all(r["status"] == "rejected: AMK_ERR_INVALID_ARG" for r in bad)
    ok = [r for r in rows if r["status"] == "ok"]
    assert len(ok) == 1 + 4  # the default and the four valid candidates pass the gate
    fastest = min(ok, key=lambda r: r["us"])
    for k, v in fastest["knobs"].items():
        assert getattr(best, k) == v
    # every schedule that passed the gate, the chosen one included, against
    # the fp64 oracle on the same bytes (the gate itself compares with the
    # default schedule, since the product has no oracle)
    for r in ok:
        pair = Pair(cfg, options=amk.default_options(**r["knobs"]), weights=w)
        pair.fill_kv(64)
        g, am, ref, ref_am = pair.step(7, 64)
        compare(cfg, g, am, ref, ref_am, what=f"tuned knobs {r['knobs']}")
        del pair
    pair = Pair(cfg, options=best, weights=w)
    pair.fill_kv(64)
    g, am, ref, ref_am = pair.step(7, 64)
    compare(cfg, g, am, ref, ref_am, what="chosen options")
    del pair
    torch.cuda.empty_cache()
