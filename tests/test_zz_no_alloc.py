"""amk_decode_step_noalloc: the decode step for callers that may not allocate
device memory (a plugin whose host framework owns every device byte through
its own allocator, or a loop that cannot afford cudaMalloc's implicit
synchronisation).  The caller brings the weights, the KV cache and the
logits buffer; the step's scratch is the library's fixed static array.

The tests call it through the C ABI several times in a row (positions 0, 1,
... so that each call reads the KV rows the earlier ones wrote) and check
logits, greedy token and KV cache against the allocating entry point
amk_decode_step, within the parity tolerance the other GPU tests use, and
the logits against the fp64 oracle directly.  The "_fused" SmolLM2 cases
run the fused FFN level (options ffn_fused = 2, with the level counters),
whose Wdown tiles come through tensor maps kept in the static array (bf16
and int8 maps); the others run the default schedule (separate FFN levels,
flagged waits).  Two fused models with different weights alternate on the
array.  This file is collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as orc
import persistent_megakernel_decode_cta_b200 as amk
from persistent_megakernel_decode_cta_b200 import abi, build
import synth_inputs as si
from parity_helpers import compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built(cuda_ok):
    build.build()


def _weights_struct(cfg, w):
    """amk_weights for torch tensors; returns the struct and its keep-alive list."""
    s = abi.Weights()
    keep = []
    s.embed = w["embed"].data_ptr()
    s.final_norm = w["final_norm"].data_ptr()
    s.lm_head = w["lm_head"].data_ptr() if w["lm_head"] is not None else None
    s.lm_head_scale = (w["lm_head_scale"].data_ptr()
                       if w.get("lm_head_scale") is not None else None)
    for name in amk.Decoder._PER_LAYER:
        lst = w.get(name)
        if lst is None:
            continue
        arr = (ctypes.c_void_p * cfg.n_layers)(*[t.data_ptr() for t in lst])
        keep.append(arr)
        setattr(s, name, ctypes.cast(arr, abi.c_vpp))
    return s, keep


def _config(name):
    """(config, options) of a test case name."""
    opts = None
    if name.endswith("_fused"):
        name = name[:-len("_fused")]
        opts = amk.default_options(ffn_fused=2)
    if name == "tiny_w8":
        return si.get_config("tiny").with_(quant="w8a16", name="tiny_w8"), opts
    if name == "smol135_w8":
        return si.get_config("smol135").with_(quant="w8a16", name="smol135_w8"), opts
    return si.get_config(name), opts


class NoAlloc:
    """A caller of amk_decode_step_noalloc: its own KV cache and logits."""

    def __init__(self, cfg, w, options=None):
        self.cfg = cfg
        sms = torch.cuda.get_device_properties(0).multi_processor_count
        self.plan = amk.Plan(cfg, sms, options)
        if options is not None and options.ffn_fused == 2:
            assert self.plan.stats().ffn_fused == 1
        self.ws, self.keep = _weights_struct(cfg, w)
        self.kv = torch.zeros((cfg.n_layers, 2, cfg.n_kv_heads, cfg.max_ctx, cfg.head_dim),
                              dtype=torch.bfloat16, device="cuda")
        self.out = torch.empty(cfg.vocab, dtype=torch.float32, device="cuda")

    def step(self, token, pos):
        am = ctypes.c_int32(-1)
        lib = abi.lib()
        rc = lib.amk_decode_step_noalloc(
            self.plan._p, ctypes.byref(self.ws), self.kv.data_ptr(), int(token), int(pos),
            self.out.data_ptr(), ctypes.byref(am),
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert rc == 0, lib.amk_last_error().decode()
        return self.out.double().cpu().numpy(), am.value

    def close(self):
        self.plan.close()


@pytest.mark.parametrize("name", ["tiny", "tiny_w8", "smol135", "smol135_fused",
                                  "smol135_w8_fused"])
def test_noalloc_matches_allocating_entry_point(name):
    cfg, opts = _config(name)
    w = si.make_model(cfg, device="cuda")
    n = 4
    toks = si.make_prompt(cfg, n)
    tol = (2e-2 if cfg.quant == "w8a16" else 1e-2)

    # reference: the allocating entry point
    dec = amk.Decoder(cfg, w, opts)
    ref_logits, ref_tok = [], []
    lg = torch.empty(cfg.vocab, dtype=torch.float32, device="cuda")
    for pos, t in enumerate(toks):
        ref_tok.append(dec.step(t, pos, logits=lg))
        ref_logits.append(lg.clone())
    ref_kv = [torch.stack(dec.kv(l))[:, :, :n].clone() for l in range(cfg.n_layers)]
    dec.close()

    # the no-allocation entry point: caller-owned KV cache and logits
    na = NoAlloc(cfg, w, opts)
    for pos, t in enumerate(toks):
        g, am = na.step(t, pos)
        r = ref_logits[pos].double().cpu().numpy()
        assert np.abs(g - r).max() <= tol * np.abs(r).max()
        assert am == ref_tok[pos]
    for l in range(cfg.n_layers):
        got = na.kv[l, :, :, :n].float()
        assert torch.allclose(got, ref_kv[l].float(), rtol=2 ** -7, atol=1e-6)
    na.close()


@pytest.mark.parametrize("name", ["tiny", "smol135", "smol135_fused", "smol135_w8_fused"])
def test_noalloc_matches_oracle(name):
    """The no-allocation step against the fp64 oracle on the same bytes,
    element by element, at positions 0..3 (the fused cases run the FFN level
    through the tensor maps in the static array)."""
    cfg, opts = _config(name)
    w = si.make_model(cfg, device="cuda")
    ref = orc.OracleModel(cfg, w)
    na = NoAlloc(cfg, w, opts)
    for pos, t in enumerate(si.make_prompt(cfg, 4)):
        g, am = na.step(t, pos)
        r, r_am, _ = ref.step(t, pos)
        compare(cfg, g, am, r, r_am, what=f"{name} noalloc pos {pos}")
    na.close()


def test_noalloc_two_models_alternate():
    """Two SmolLM2-shaped models with different weights take turns on the
    one static array: every call re-writes the Wdown tensor maps there, and
    each model's logits must still be its own."""
    cfg = si.get_config("smol135")
    opts = amk.default_options(ffn_fused=2)
    ws = [si.make_model(cfg, seed=s, device="cuda") for s in (0, 7)]
    refs = []
    for w in ws:
        dec = amk.Decoder(cfg, w, opts)
        lg = torch.empty(cfg.vocab, dtype=torch.float32, device="cuda")
        out = []
        for pos, t in enumerate(si.make_prompt(cfg, 3)):
            dec.step(t, pos, logits=lg)
            out.append(lg.double().cpu().numpy())
        dec.close()
        refs.append(out)
    nas = [NoAlloc(cfg, w, opts) for w in ws]
    for pos, t in enumerate(si.make_prompt(cfg, 3)):
        for i in (0, 1):
            g, _ = nas[i].step(t, pos)
            r = refs[i][pos]
            assert np.abs(g - r).max() <= 1e-2 * np.abs(r).max(), f"model {i} pos {pos}"
            other = refs[1 - i][pos]
            assert np.abs(g - other).max() > 1e-2 * np.abs(other).max()
    for na in nas:
        na.close()


def test_noalloc_refuses_a_capturing_stream():
    """Under stream capture the call returns AMK_ERR_UNSUPPORTED and enqueues
    nothing (its uploads read host stack memory)."""
    cfg = si.get_config("tiny")
    w = si.make_model(cfg, device="cuda")
    na = NoAlloc(cfg, w)
    na.step(1, 0)  # the first call on the device (set-up) comes before any capture
    s = torch.cuda.Stream()
    lib = abi.lib()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    rc = None
    with torch.cuda.stream(s):
        g.capture_begin()
        try:
            rc = lib.amk_decode_step_noalloc(na.plan._p, ctypes.byref(na.ws), na.kv.data_ptr(),
                                             1, 1, na.out.data_ptr(), None,
                                             ctypes.c_void_p(s.cuda_stream))
            na.out.add_(0.0)  # something for the graph to hold
        finally:
            g.capture_end()
    torch.cuda.current_stream().wait_stream(s)
    assert rc == abi.ERR["AMK_ERR_UNSUPPORTED"]
    assert b"capturing" in lib.amk_last_error()
    del g
    # the handle-free step still works afterwards
    na.step(2, 1)
    na.close()


def test_noalloc_position0_schedule_only_at_position0():
    """The position-0 schedule has no attention level: with pos > 0 the call
    is refused instead of skipping attention over the cache."""
    cfg = si.get_config("tiny")
    w = si.make_model(cfg, device="cuda")
    na = NoAlloc(cfg, w)
    p0 = na.plan.pos0()
    assert p0 is not None
    lib = abi.lib()
    rc = lib.amk_decode_step_noalloc(p0._p, ctypes.byref(na.ws), na.kv.data_ptr(), 1, 1,
                                     na.out.data_ptr(), None, None)
    assert rc == abi.ERR["AMK_ERR_INVALID_ARG"]
    am = ctypes.c_int32(-1)
    rc = lib.amk_decode_step_noalloc(p0._p, ctypes.byref(na.ws), na.kv.data_ptr(), 1, 0,
                                     na.out.data_ptr(), ctypes.byref(am), None)
    assert rc == 0, lib.amk_last_error().decode()
    na.close()


def test_noalloc_rejects_models_beyond_the_static_scratch():
    """A model whose scratch does not fit the static array is refused before
    any GPU work (the pointers below are valid but never read)."""
    big = si.get_config("llama7b").with_(n_layers=120, name="big")  # ~23 MB of scratch
    plan = amk.Plan(big, 148)
    dummy = torch.empty(64, dtype=torch.uint8, device="cuda")
    ptrs = (ctypes.c_void_p * big.n_layers)(*([dummy.data_ptr()] * big.n_layers))
    ws = abi.Weights()
    for f in ("embed", "final_norm", "lm_head"):
        setattr(ws, f, dummy.data_ptr())
    for name in ("attn_norm", "ffn_norm", "wq", "wk", "wv", "wo", "wgate", "wup", "wdown"):
        setattr(ws, name, ctypes.cast(ptrs, abi.c_vpp))
    lib = abi.lib()
    rc = lib.amk_decode_step_noalloc(plan._p, ctypes.byref(ws), dummy.data_ptr(), 0, 0,
                                     dummy.data_ptr(), None, None)
    assert rc == abi.ERR["AMK_ERR_UNSUPPORTED"]
    assert b"static array" in lib.amk_last_error()
    plan.close()
